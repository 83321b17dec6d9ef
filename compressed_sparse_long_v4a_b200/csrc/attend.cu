// attend.cu -- CSA / HCA attention over compressed entries plus the window,
// CUDA-core split-K flash-decoding path (any dtype, d in {64,128,256,512}).
//
// For every query (b, j) at position t and head h: one joint softmax, scale
// 1/sqrt(d), over the candidate rows -- the selected entries (CSA) or every
// visible entry (HCA) followed by the raw window tokens (t-W, t] -- with the
// same row serving as key and value ("DeepSeek-V4: Million-Token Context via
// Hybrid Compressed Attention", CSA "Core attention with shared KV MQA";
// "1M Context != Lossless Long Memory", sections 5 and 6).
//
// The candidate list of a query is cut into n_splits contiguous ranges; one
// block per (split, query, head group) keeps an online softmax (running max
// in the log2 domain, running sum, fp32 output slice in registers) and writes
// a partial (m, l, o) that attend_combine_kernel merges.  With one split the
// block writes the normalised output directly.  A thread owns 32 consecutive
// elements of d for one head; the P = d/32 threads of a head are adjacent
// lanes and reduce the dot product with shuffles.  Rows are staged in shared
// memory as fp32; each lane walks its 8 float4 chunks in an order rotated by
// its lane-in-head, so the 8 lanes of a quarter-warp hit distinct banks.
#include "common.cuh"
#include "internal.h"

namespace v4a {
namespace {

constexpr int kRows = 8;          // rows staged per tile
constexpr int kBlockThreads = 128;
constexpr int kEpt = 32;          // elements of d owned by one thread
constexpr float kLog2e = 1.4426950408889634f;

struct SplitPlan {
    int n_splits;
    int heads_per_block;
    int head_groups;
    int threads;
};

template <typename T, int P>
__global__ void __launch_bounds__(kBlockThreads, 1) attend_split_kernel(AttendArgs a, SplitPlan plan, float* part_ml,
                                                                     float* part_o) {
    griddep_wait();  // everything before this kernel on the stream has finished
    griddep_launch_dependents();
    __shared__ __align__(16) float rows_s[kRows * kEpt * P];
    __shared__ int valid_s[kRows];
    __shared__ float lg_s[kBlockThreads * kRows];  // per head-in-block logits of the tile
    const int d = kEpt * P;
    const int split = blockIdx.x;
    const int row = blockIdx.y;  // b * n_q + j
    const int b = row / a.n_q, j = row % a.n_q;
    const long long t = a.ctx_len - a.n_q + j;
    long long nvis = n_visible(t, a.m);
    if (nvis > a.n_ent) nvis = a.n_ent;
    const long long n_sel = a.idx ? (long long)a.k : nvis;
    long long win_lo = t - a.window + 1;
    if (win_lo < 0) win_lo = 0;
    const long long n_win = a.window > 0 ? t - win_lo + 1 : 0;
    const long long n_cand = n_sel + n_win;
    const long long chunk = (n_cand + plan.n_splits - 1) / plan.n_splits;
    const long long c0 = (long long)split * chunk;
    long long c1 = c0 + chunk;
    if (c1 > n_cand) c1 = n_cand;

    const int hl = threadIdx.x / P, part = threadIdx.x % P;
    const int h = blockIdx.z * plan.heads_per_block + hl;
    const bool active = hl < plan.heads_per_block && h < a.heads;
    const float scale_log2 = kLog2e / sqrtf((float)d);

    // query slice, stored in the lane's rotated chunk order
    float q[kEpt], o[kEpt];
    {
        const long long qoff = (((long long)row * a.heads + (active ? h : 0)) * d) + part * kEpt;
#pragma unroll
        for (int i = 0; i < kEpt / 4; ++i) {
            const int ch = (i + part) & (kEpt / 4 - 1);
            float f[8];
            if constexpr (sizeof(T) == 2) {
                const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(a.q) + qoff + ch * 4;
                uint2 v = *reinterpret_cast<const uint2*>(qp);
                f[0] = __uint_as_float(v.x << 16);
                f[1] = __uint_as_float(v.x & 0xffff0000u);
                f[2] = __uint_as_float(v.y << 16);
                f[3] = __uint_as_float(v.y & 0xffff0000u);
            } else {
                float4 v = *reinterpret_cast<const float4*>(static_cast<const float*>(a.q) + qoff + ch * 4);
                f[0] = v.x;
                f[1] = v.y;
                f[2] = v.z;
                f[3] = v.w;
            }
            q[4 * i + 0] = f[0];
            q[4 * i + 1] = f[1];
            q[4 * i + 2] = f[2];
            q[4 * i + 3] = f[3];
            o[4 * i + 0] = o[4 * i + 1] = o[4 * i + 2] = o[4 * i + 3] = 0.f;
        }
    }
    float m_run = -INFINITY, l_run = 0.f;

    const int units_per_row = d / 8;
    for (long long base = c0; base < c1; base += kRows) {
        // stage up to kRows candidate rows as fp32
#pragma unroll 1
        for (int u = threadIdx.x; u < kRows * units_per_row; u += blockDim.x) {
            const int r = u / units_per_row, c8 = u % units_per_row;
            const long long c = base + r;
            const T* src = nullptr;
            bool ok = c < c1;
            if (ok) {
                if (c < n_sel) {
                    long long s = c;
                    if (a.idx) {
                        s = a.idx[(long long)row * a.k + c];
                        if (s == -1) {
                            ok = false;
                        } else if (s < 0 || s >= nvis) {
                            ok = false;
                            if (c8 == 0 && a.dev_status) atomicExch(a.dev_status, (int)V4A_ERR_DEVICE_FAULT);
                        }
                    }
                    if (ok) {
                        long long er = (long long)b * a.n_ent + s;
                        if (a.bt) {
                            const long long blk = a.bt[(long long)b * a.bt_stride + s / a.epb];
                            er = blk * a.epb + s % a.epb;
                            if (blk < 0 || er >= a.pool_rows) {  // a block id outside the pool
                                ok = false;
                                if (c8 == 0 && a.dev_status) atomicExch(a.dev_status, (int)V4A_ERR_DEVICE_FAULT);
                            }
                        }
                        if (ok) src = static_cast<const T*>(a.entries) + er * d;
                    }
                } else {
                    const long long p = win_lo + (c - n_sel);
                    const long long tr = a.ring_rows > 0 ? (long long)b * a.ring_rows + p % a.ring_rows
                                                         : (long long)b * a.l_tok + (p - a.tok_pos0);
                    src = static_cast<const T*>(a.token_kv) + tr * d;
                }
            }
            float f[8];
            if (ok) {
                Vec8<T>::load_nc(src + c8 * 8, f);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = 0.f;
            }
            Vec8<float>::store(rows_s + r * d + c8 * 8, f);
            if (c8 == 0) valid_s[r] = ok ? 1 : 0;
        }
        __syncthreads();

        // logits of the staged rows (log2 domain), one row at a time
        float mt = -INFINITY;
#pragma unroll 1
        for (int r = 0; r < kRows; ++r) {
            const float* rp = rows_s + r * d + part * kEpt;
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < kEpt / 4; ++i) {
                const float4 v = *reinterpret_cast<const float4*>(rp + ((i + part) & (kEpt / 4 - 1)) * 4);
                acc = fmaf(q[4 * i + 0], v.x, acc);
                acc = fmaf(q[4 * i + 1], v.y, acc);
                acc = fmaf(q[4 * i + 2], v.z, acc);
                acc = fmaf(q[4 * i + 3], v.w, acc);
            }
            acc = group_sum<P>(acc);
            const float lgv = valid_s[r] ? acc * scale_log2 : -INFINITY;
            mt = fmaxf(mt, lgv);
            if (part == 0) lg_s[hl * kRows + r] = lgv;
        }
        __syncwarp();
        const float m_new = fmaxf(m_run, mt);
        if (m_new != -INFINITY) {
            const float alpha = exp2f(m_run - m_new);
            l_run *= alpha;
#pragma unroll
            for (int e = 0; e < kEpt; ++e) o[e] *= alpha;
#pragma unroll 1
            for (int r = 0; r < kRows; ++r) {
                const float p = exp2f(lg_s[hl * kRows + r] - m_new);
                l_run += p;
                const float* rp = rows_s + r * d + part * kEpt;
#pragma unroll
                for (int i = 0; i < kEpt / 4; ++i) {
                    const float4 v = *reinterpret_cast<const float4*>(rp + ((i + part) & (kEpt / 4 - 1)) * 4);
                    o[4 * i + 0] = fmaf(p, v.x, o[4 * i + 0]);
                    o[4 * i + 1] = fmaf(p, v.y, o[4 * i + 1]);
                    o[4 * i + 2] = fmaf(p, v.z, o[4 * i + 2]);
                    o[4 * i + 3] = fmaf(p, v.w, o[4 * i + 3]);
                }
            }
            m_run = m_new;
        }
        __syncthreads();
    }
    if (!active) return;

    if (plan.n_splits == 1 && a.sink == nullptr && a.rope_dims == 0) {  // no combine pass: write the output
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        float* op = a.out + (((long long)row * a.heads + h) * d) + part * kEpt;
#pragma unroll
        for (int i = 0; i < kEpt / 4; ++i) {
            const int ch = (i + part) & (kEpt / 4 - 1);
            *reinterpret_cast<float4*>(op + ch * 4) =
                make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
        }
        return;
    }
    const long long pidx = ((long long)row * plan.n_splits + split) * a.heads + h;
    if (part == 0) {
        part_ml[2 * pidx] = m_run;
        part_ml[2 * pidx + 1] = l_run;
    }
    float* op = part_o + pidx * d + part * kEpt;
#pragma unroll
    for (int i = 0; i < kEpt / 4; ++i) {
        const int ch = (i + part) & (kEpt / 4 - 1);
        *reinterpret_cast<float4*>(op + ch * 4) = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
    }
}

// grid (rows, heads); each thread merges 4 consecutive output elements
__global__ void attend_combine_kernel(const float* part_ml, const float* part_o, int n_splits, AttendArgs a) {
    griddep_wait();  // everything before this kernel on the stream has finished
    griddep_launch_dependents();
    const int row = blockIdx.x, h = blockIdx.y;
    const int heads = a.heads, d = a.d;
    float* out = a.out;
    const long long t = a.ctx_len - a.n_q + (row % a.n_q);  // the query position (output RoPE)
    float mmax = -INFINITY;
    for (int s = 0; s < n_splits; ++s)
        mmax = fmaxf(mmax, part_ml[2 * (((long long)row * n_splits + s) * heads + h)]);
    float* op = out + ((long long)row * heads + h) * d;
    for (int e = threadIdx.x * 4; e < d; e += blockDim.x * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float l = 0.f;
        if (mmax != -INFINITY) {
            for (int s = 0; s < n_splits; ++s) {
                const long long pidx = ((long long)row * n_splits + s) * heads + h;
                const float ms = part_ml[2 * pidx];
                if (ms == -INFINITY) continue;
                const float wgt = exp2f(ms - mmax);
                l += wgt * part_ml[2 * pidx + 1];
                const float4 v = *reinterpret_cast<const float4*>(part_o + pidx * d + e);
                acc.x = fmaf(wgt, v.x, acc.x);
                acc.y = fmaf(wgt, v.y, acc.y);
                acc.z = fmaf(wgt, v.z, acc.z);
                acc.w = fmaf(wgt, v.w, acc.w);
            }
        }
        if (a.sink && mmax != -INFINITY) l += exp2f(a.sink[h] * kLog2e - mmax);  // the sink's share
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float v[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
        if (a.rope_dims > 0) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {  // dims (e + 2j, e + 2j + 1) are one RoPE pair
                const int dim = e + 2 * j;
                if (dim >= d - a.rope_dims) {
                    float s, c;
                    rope_sincos(t, (dim - (d - a.rope_dims)) >> 1, a.rope_dims, a.rope_base, &s, &c);
                    const float x = v[2 * j], y = v[2 * j + 1];
                    v[2 * j] = fmaf(x, c, -y * s);
                    v[2 * j + 1] = fmaf(x, s, y * c);
                }
            }
        }
        *reinterpret_cast<float4*>(op + e) = make_float4(v[0], v[1], v[2], v[3]);
    }
}

SplitPlan plan_for(const AttendArgs& a) {
    SplitPlan p;
    const int P = a.d / kEpt;
    p.heads_per_block = kBlockThreads / P;
    if (p.heads_per_block > a.heads) p.heads_per_block = a.heads;
    p.head_groups = (a.heads + p.heads_per_block - 1) / p.heads_per_block;
    p.threads = kBlockThreads;
    const long long rows = (long long)a.batch * a.n_q;
    const long long n_cand = (a.idx ? (long long)a.k : a.n_ent) + a.window;
    long long want = (2LL * kNumSMs + rows * p.head_groups - 1) / (rows * p.head_groups);
    long long cap = (n_cand + 31) / 32;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    if (want > 4096) want = 4096;
    p.n_splits = (int)want;
    return p;
}

template <typename T, int P>
cudaError_t launch_t(const AttendArgs& a, const SplitPlan& plan, float* ml, float* po, cudaStream_t stream) {
    dim3 grid(plan.n_splits, a.batch * a.n_q, plan.head_groups);
    cudaError_t le = launch_pdl(attend_split_kernel<T, P>, grid, dim3(plan.threads), 0, stream, a, plan, ml, po);
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dtype(const AttendArgs& a, const SplitPlan& plan, float* ml, float* po, cudaStream_t stream) {
    switch (a.d) {
    case 64: return launch_t<T, 2>(a, plan, ml, po, stream);
    case 128: return launch_t<T, 4>(a, plan, ml, po, stream);
    case 256: return launch_t<T, 8>(a, plan, ml, po, stream);
    default: return launch_t<T, 16>(a, plan, ml, po, stream);
    }
}

}  // namespace

static size_t core_workspace_bytes(const AttendArgs& a) {
    SplitPlan p = plan_for(a);
    size_t rows = (size_t)a.batch * a.n_q;
    size_t n = rows * p.n_splits * a.heads;
    size_t ml = ((n * 2 * sizeof(float)) + 255) / 256 * 256;
    return ml + n * a.d * sizeof(float);
}

size_t attend_workspace_bytes(const AttendArgs& a) {
    size_t w = core_workspace_bytes(a);
    if (attend_tc_shape_ok(a)) {
        size_t t = attend_tc_workspace_bytes(a);
        if (t > w) w = t;
    }
    return w;
}

cudaError_t launch_attend(const AttendArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (a.batch == 0) return cudaSuccess;
    if (ws_bytes < attend_workspace_bytes(a)) return cudaErrorInvalidValue;
    if (attend_tc_available(a)) return launch_attend_tc(a, ws, ws_bytes, stream);
    SplitPlan plan = plan_for(a);
    size_t rows = (size_t)a.batch * a.n_q;
    size_t n = rows * plan.n_splits * a.heads;
    float* ml = static_cast<float*>(ws);
    float* po = reinterpret_cast<float*>(static_cast<char*>(ws) + ((n * 2 * sizeof(float)) + 255) / 256 * 256);
    cudaError_t e = a.dtype == V4A_BF16 ? launch_dtype<__nv_bfloat16>(a, plan, ml, po, stream)
                                        : launch_dtype<float>(a, plan, ml, po, stream);
    if (e != cudaSuccess || (plan.n_splits == 1 && a.sink == nullptr && a.rope_dims == 0)) return e;
    e = launch_pdl(attend_combine_kernel, dim3((unsigned)rows, a.heads), dim3(a.d / 4 < 128 ? a.d / 4 : 128), 0,
                   stream, (const float*)ml, (const float*)po, plan.n_splits, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace v4a
