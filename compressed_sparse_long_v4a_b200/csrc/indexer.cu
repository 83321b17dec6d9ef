// indexer.cu -- Lightning-Indexer scores and the top-k select.
//
// Score ("How V4 makes a million-token context actually affordable",
// Lightning-Indexer section): I(t,s) = scale_s * sum_j w_j * ReLU(q_j . k_s),
// one key per entry shared by every indexer head.  Only entries visible to the
// query (m*(s+1) <= t+1) get a score.
//
// CUDA-core path, any (heads_i <= 64, d_i % 8 == 0) and key format: one thread
// per entry streams the entry's key with 16-byte loads (fp8 keys: 8 bytes at a
// time, widened exactly to fp32) and accumulates every head's dot product in
// registers against the query held in shared memory (broadcast reads).
//
// Select: per query row, an exact radix select over order-preserving 32-bit
// keys of the fp32 scores (four 8-bit digits, most significant first) finds
// the k-th largest key T and how many entries equal to T are still needed;
// an ordered block-wide compaction then writes the winners in ascending entry
// order, taking ties at T from the lowest entries first.
#include "common.cuh"
#include "internal.h"

namespace v4a {
namespace {

constexpr int kScoreThreads = 256;

template <int KFMT>
__device__ __forceinline__ void load_key8(const void* k, long long off, float f[8]) {
    if constexpr (KFMT == V4A_F32) {
        Vec8<float>::load_nc(static_cast<const float*>(k) + off, f);
    } else if constexpr (KFMT == V4A_BF16) {
        Vec8<__nv_bfloat16>::load_nc(static_cast<const __nv_bfloat16*>(k) + off, f);
    } else {
        uint2 v = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(k) + off));
        unpack_e4m3x8(v, f);
    }
}

// grid: (ceil(N / 256), B * n_q); q of the block's query staged in shared memory
template <int HMAX, int KFMT>
__global__ void __launch_bounds__(kScoreThreads) index_score_kernel(IndexArgs a, float* scores) {
    extern __shared__ float smem[];
    float* q_s = smem;                         // [HI][DI]
    float* w_s = smem + a.heads_i * a.d_i;     // [HI]
    const int row = blockIdx.y;                // b * n_q + j
    const int b = row / a.n_q, j = row % a.n_q;
    const long long t = a.ctx_len - a.n_q + j;
    long long nvis = n_visible(t, a.m);
    if (nvis > a.n_ent) nvis = a.n_ent;

    const int qn = a.heads_i * a.d_i;
    if (a.q_dtype == V4A_BF16) {
        const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(a.q) + (long long)row * qn;
        for (int i = threadIdx.x; i < qn; i += blockDim.x) q_s[i] = __bfloat162float(qp[i]);
    } else {
        const float* qp = static_cast<const float*>(a.q) + (long long)row * qn;
        for (int i = threadIdx.x; i < qn; i += blockDim.x) q_s[i] = qp[i];
    }
    for (int i = threadIdx.x; i < a.heads_i; i += blockDim.x) w_s[i] = a.w[(long long)row * a.heads_i + i];
    __syncthreads();

    const long long s = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= a.n_ent) return;
    float* out = scores + (long long)row * a.n_ent + s;
    if (s >= nvis) {
        *out = -INFINITY;
        return;
    }
    float acc[HMAX];
#pragma unroll
    for (int h = 0; h < HMAX; ++h) acc[h] = 0.f;
    const long long koff = ((long long)b * a.n_ent + s) * a.d_i;
    for (int c = 0; c < a.d_i; c += 8) {
        float kv[8];
        load_key8<KFMT>(a.k, koff + c, kv);
#pragma unroll
        for (int h = 0; h < HMAX; ++h) {
            if (h < a.heads_i) {
                const float4 q0 = *reinterpret_cast<const float4*>(q_s + h * a.d_i + c);
                const float4 q1 = *reinterpret_cast<const float4*>(q_s + h * a.d_i + c + 4);
                float r = acc[h];
                r = fmaf(q0.x, kv[0], r);
                r = fmaf(q0.y, kv[1], r);
                r = fmaf(q0.z, kv[2], r);
                r = fmaf(q0.w, kv[3], r);
                r = fmaf(q1.x, kv[4], r);
                r = fmaf(q1.y, kv[5], r);
                r = fmaf(q1.z, kv[6], r);
                r = fmaf(q1.w, kv[7], r);
                acc[h] = r;
            }
        }
    }
    float sc = 0.f;
#pragma unroll
    for (int h = 0; h < HMAX; ++h)
        if (h < a.heads_i) sc = fmaf(w_s[h], fmaxf(acc[h], 0.f), sc);
    if (a.kscale) sc *= a.kscale[(long long)b * a.n_ent + s];
    *out = sc + 0.0f;  // -0 -> +0
}

// ---------------------------------------------------------------------
// select
// ---------------------------------------------------------------------
constexpr int kSelThreads = 1024;

// exclusive block scan of one int per thread; returns the block total in *total
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_buf, int* total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_buf[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int wv = lane < (int)(blockDim.x >> 5) ? warp_buf[lane] : 0;
        int xs = wv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, xs, o);
            if (lane >= o) xs += y;
        }
        warp_buf[lane] = xs - wv;  // exclusive prefix of warp totals
        if (lane == 31) warp_buf[32] = xs;
    }
    __syncthreads();
    int r = warp_buf[wid] + x - v;
    *total = warp_buf[32];
    __syncthreads();
    return r;
}

// one block per query row; scores[row][N] with -inf beyond N_vis
__global__ void __launch_bounds__(kSelThreads) topk_select_kernel(const float* scores, IndexArgs a, int k,
                                                                   int32_t* idx_out, float* score_out) {
    __shared__ unsigned int hist[256];
    __shared__ int warp_buf[33];
    __shared__ unsigned int sh_digit, sh_above;
    const int row = blockIdx.x;
    const int j = row % a.n_q;
    const long long t = a.ctx_len - a.n_q + j;
    long long nvis = n_visible(t, a.m);
    if (nvis > a.n_ent) nvis = a.n_ent;
    const float* sc = scores + (long long)row * a.n_ent;
    int32_t* io = idx_out + (long long)row * k;
    float* so = score_out ? score_out + (long long)row * k : nullptr;

    uint32_t prefix = 0, mask = 0;
    long long need = k;  // how many entries with key == prefix (so far) are still wanted
    const bool all = nvis <= k;
    if (!all) {
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
            __syncthreads();
            for (long long s = threadIdx.x; s < nvis; s += blockDim.x) {
                uint32_t key = float_to_ordered(sc[s]);
                if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                unsigned int above = 0;
                int dgt = 255;
                for (; dgt > 0; --dgt) {
                    if (above + hist[dgt] >= (unsigned int)need) break;
                    above += hist[dgt];
                }
                sh_digit = (unsigned int)dgt;
                sh_above = above;
            }
            __syncthreads();
            prefix |= sh_digit << shift;
            mask |= 255u << shift;
            need -= sh_above;
            __syncthreads();
        }
    }
    // ordered compaction: key > prefix, or key == prefix among the first `need` such entries
    int out_base = 0, eq_base = 0;
    for (long long base = 0; base < nvis; base += blockDim.x) {
        long long s = base + threadIdx.x;
        bool in = s < nvis;
        float v = in ? sc[s] : 0.f;
        uint32_t key = in ? float_to_ordered(v) : 0u;
        int gt = (in && (all || key > prefix)) ? 1 : 0;
        int eq = (in && !all && key == prefix) ? 1 : 0;
        int eq_total;
        int eq_rank = eq_base + block_exclusive_scan(eq, warp_buf, &eq_total);
        int sel = gt | (eq && eq_rank < need ? 1 : 0);
        int sel_total;
        int pos = out_base + block_exclusive_scan(sel, warp_buf, &sel_total);
        if (sel && pos < k) {
            io[pos] = (int32_t)s;
            if (so) so[pos] = v;
        }
        out_base += sel_total;
        eq_base += eq_total;
    }
    for (int p = out_base + threadIdx.x; p < k; p += blockDim.x) {
        io[p] = -1;
        if (so) so[p] = -INFINITY;
    }
}

template <int HMAX>
cudaError_t launch_scores_h(const IndexArgs& a, float* scores, cudaStream_t stream) {
    long long nblk = (a.n_ent + kScoreThreads - 1) / kScoreThreads;
    dim3 grid((unsigned)nblk, (unsigned)(a.batch * a.n_q));
    size_t smem = sizeof(float) * (size_t)(a.heads_i * a.d_i + a.heads_i);
    switch (a.k_dtype) {
    case V4A_F32: {
        auto kern = index_score_kernel<HMAX, V4A_F32>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<grid, kScoreThreads, smem, stream>>>(a, scores);
        break;
    }
    case V4A_BF16: {
        auto kern = index_score_kernel<HMAX, V4A_BF16>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<grid, kScoreThreads, smem, stream>>>(a, scores);
        break;
    }
    default: {
        auto kern = index_score_kernel<HMAX, V4A_FP8E4M3>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<grid, kScoreThreads, smem, stream>>>(a, scores);
        break;
    }
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_index_scores(const IndexArgs& a, float* scores, cudaStream_t stream) {
    if (a.batch == 0 || a.n_ent == 0) return cudaSuccess;
    if (a.heads_i <= 4) return launch_scores_h<4>(a, scores, stream);
    if (a.heads_i <= 8) return launch_scores_h<8>(a, scores, stream);
    if (a.heads_i <= 16) return launch_scores_h<16>(a, scores, stream);
    if (a.heads_i <= 32) return launch_scores_h<32>(a, scores, stream);
    return launch_scores_h<64>(a, scores, stream);
}

size_t topk_workspace_bytes(const IndexArgs& a, int k) {
    (void)k;
    size_t n = (size_t)a.batch * (size_t)a.n_q * (size_t)(a.n_ent > 0 ? a.n_ent : 1);
    return ((n * sizeof(float) + 255) / 256) * 256;
}

cudaError_t launch_topk(const IndexArgs& a, int k, int32_t* idx_out, float* score_out, void* ws, size_t ws_bytes,
                        cudaStream_t stream) {
    if (a.batch == 0) return cudaSuccess;
    if (ws_bytes < topk_workspace_bytes(a, k)) return cudaErrorInvalidValue;
    float* scores = static_cast<float*>(ws);
    if (a.n_ent > 0) {
        cudaError_t e = launch_index_scores(a, scores, stream);
        if (e != cudaSuccess) return e;
    }
    topk_select_kernel<<<a.batch * a.n_q, kSelThreads, 0, stream>>>(scores, a, k, idx_out, score_out);
    return cudaGetLastError();
}

}  // namespace v4a
