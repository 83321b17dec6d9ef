// compress.cu -- chunk compression of token rows into compressed entries.
//
// "DeepSeek-V4 的暗线之一：分层记忆比输入框更关键" (blog.xieydd.top), section 3:
// an entry is the per-channel softmax (over the chunk's m tokens, from the gate
// logits Z) weighted sum of the content rows C.  One launch compresses both the
// K=V stream and, optionally, the indexer-key stream of the same chunks.
// The dual-series form ("DeepSeek-V4: Million-Token Context via Hybrid
// Compressed Attention", CSA, "Dual-series KV compression") adds series b's
// rows of the previous block to the same per-channel softmax.
//
// Mapping: S adjacent lanes (S = the largest power of two <= min(m, 32); 1
// for FP8 and MXFP4 output) own 8 consecutive channels of one entry; each takes every
// S-th token of the chunk with 16-byte vector loads (two for fp32), four
// tokens per round with all loads issued first, keeping a running max /
// denominator / numerator per channel in registers.  The S partial states are
// merged with shuffles: common max, one rescale per lane, then sums.  For FP8
// output the lanes of one entry are consecutive lanes of one warp, so the
// entry's amax is found with warp shuffles too; for MXFP4 output (OCP MX,
// the FP4 indexer keys) each block of 32 channels is 4 consecutive lanes.
// Long chunks of one unquantised stream (the HCA chunk) go to
// compress_wide_kernel instead, whose warp loads are coalesced across channels.
#include "common.cuh"
#include "internal.h"

namespace v4a {
namespace {

constexpr int kMaxRingStreams = 8;

struct StreamDesc {
    const void* x;
    const void* gate;
    const void* xb;     // dual series: series b over the range (null: single series)
    const void* gateb;
    const void* pxb;    // series b over the block before the range (null: none)
    const void* pgateb;
    long long xb_bs, gateb_bs, prev_bs;
    void* out;
    float* out_scale;
    uint8_t* out_exp;      // MXFP4 output: block exponents
    long long exp_bs;
    int channels, groups;  // groups = channels / 8
    int split;             // S: lanes sharing one (entry, channel group)
    int in_dtype, out_dtype;
    long long x_bs, gate_bs, out_bs, scale_bs;
    // paged output: entry first + s of sequence b goes to pool row bt[b*bt_stride + (first+s)/epb]*epb +
    // (first+s)%epb (null: the sequence's own rows)
    const int32_t* bt;
    int bt_stride, epb;
    long long first, n_blocks;  // a block id outside [0, n_blocks): the entry is not written
};

// This lane's share of one (entry, 8-channel group): tokens sub, sub + S, ... of the chunk, in
// rounds of kU tokens whose loads are all issued first; per round one max, one rescale of the
// running state and one exp per element.
template <typename T>
__device__ __forceinline__ void compress_span(const StreamDesc& d, const T* xp, const T* zp, int m, int sub,
                                              float mx[8], float den[8], float num[8]) {
    constexpr int kU = 4;
    for (int i0 = sub; i0 < m; i0 += kU * d.split) {
        float xv[kU][8], zv[kU][8];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int i = i0 + u * d.split;
            if (i < m) {
                Vec8<T>::load_nc(xp + (long long)i * d.channels, xv[u]);
                Vec8<T>::load_nc(zp + (long long)i * d.channels, zv[u]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    xv[u][e] = 0.f;
                    zv[u][e] = -INFINITY;
                }
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float nm = mx[e];
#pragma unroll
            for (int u = 0; u < kU; ++u) nm = fmaxf(nm, zv[u][e]);
            const float a = mx[e] == -INFINITY ? 0.f : expf(mx[e] - nm);  // rescale of the running state
            float dn = den[e] * a, nu = num[e] * a;
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const float p = zv[u][e] == -INFINITY ? 0.f : expf(zv[u][e] - nm);
                dn += p;
                nu = fmaf(p, xv[u][e], nu);
            }
            den[e] = dn;
            num[e] = nu;
            mx[e] = nm;
        }
    }
}

__global__ void __launch_bounds__(256) compress_kernel(StreamDesc s0, StreamDesc s1, int batch, long long n_ent,
                                                       int m) {
    griddep_wait();  // everything before this kernel on the stream has finished
    griddep_launch_dependents();
    const StreamDesc& d = blockIdx.y == 0 ? s0 : s1;
    const long long per_entry = (long long)d.groups * d.split;
    long long total = (long long)batch * n_ent * per_entry;
    long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    bool active = g < total;
    long long gg = active ? g : 0;
    const int sub = (int)(gg % d.split);
    int b = (int)(gg / (n_ent * per_entry));
    long long rem = (gg % (n_ent * per_entry)) / d.split;
    long long s = rem / d.groups;
    int grp = (int)(rem % d.groups);

    float mx[8], den[8], num[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        mx[e] = -INFINITY;
        den[e] = 0.f;
        num[e] = 0.f;
    }
    if (active) {
        // series a (or the single series) over block s; series b over block s-1 of the range, or the
        // block before the range
        const long long off = s * m * d.channels + grp * 8;
        const size_t es = d.in_dtype == V4A_BF16 ? 2 : 4;
        const char* xa = static_cast<const char*>(d.x) + ((long long)b * d.x_bs + off) * es;
        const char* za = static_cast<const char*>(d.gate) + ((long long)b * d.gate_bs + off) * es;
        const char* xb = nullptr;
        const char* zb = nullptr;
        if (d.xb && s >= 1) {
            xb = static_cast<const char*>(d.xb) + ((long long)b * d.xb_bs + off - (long long)m * d.channels) * es;
            zb = static_cast<const char*>(d.gateb) + ((long long)b * d.gateb_bs + off - (long long)m * d.channels) * es;
        } else if (d.xb && d.pxb) {
            xb = static_cast<const char*>(d.pxb) + ((long long)b * d.prev_bs + grp * 8) * es;
            zb = static_cast<const char*>(d.pgateb) + ((long long)b * d.prev_bs + grp * 8) * es;
        }
        if (d.in_dtype == V4A_BF16) {
            compress_span(d, reinterpret_cast<const __nv_bfloat16*>(xa), reinterpret_cast<const __nv_bfloat16*>(za),
                          m, sub, mx, den, num);
            if (xb)
                compress_span(d, reinterpret_cast<const __nv_bfloat16*>(xb),
                              reinterpret_cast<const __nv_bfloat16*>(zb), m, sub, mx, den, num);
        } else {
            compress_span(d, reinterpret_cast<const float*>(xa), reinterpret_cast<const float*>(za), m, sub, mx,
                          den, num);
            if (xb)
                compress_span(d, reinterpret_cast<const float*>(xb), reinterpret_cast<const float*>(zb), m, sub, mx,
                              den, num);
        }
    }
    // merge the S lanes' partial states (S adjacent lanes, S a power of two): the common max,
    // one rescale per lane, then plain sums
    if (d.split > 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float gm = mx[e];
            for (int o = d.split / 2; o > 0; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
            const float a = mx[e] == -INFINITY ? 0.f : expf(mx[e] - gm);
            float dn = den[e] * a, nu = num[e] * a;
            for (int o = d.split / 2; o > 0; o >>= 1) {
                dn += __shfl_xor_sync(0xffffffffu, dn, o);
                nu += __shfl_xor_sync(0xffffffffu, nu, o);
            }
            den[e] = dn;
            num[e] = nu;
        }
    }
    float out[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = active ? num[e] / den[e] : 0.f;
    if (sub != 0) return;
    // output row (in entries of `channels` elements) and its block-scale slot
    long long orow, srow;
    if (d.bt) {
        const long long es = d.first + s;
        const long long blk = d.bt[(long long)b * d.bt_stride + es / d.epb];
        if (blk < 0 || blk >= d.n_blocks) active = false;  // nowhere to write it (shuffles are done)
        orow = blk * d.epb + es % d.epb;
        srow = orow;
    } else {
        orow = -1;
        srow = (long long)b * d.scale_bs + s;
    }
    const long long obase = d.bt ? orow * d.channels : (long long)b * d.out_bs + s * d.channels;

    if (d.out_dtype == V4A_FP8E4M3) {
        // per-entry amax over the entry's `groups` consecutive lanes (a power of two <= 32)
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(out[e]));
        for (int o = d.groups / 2; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (!active) return;
        float scale = a > 0.f ? a / 448.0f : 1.0f;
        uint8_t* op = static_cast<uint8_t*>(d.out) + obase + grp * 8;
        uint32_t lo = (uint32_t)pack_e4m3x2(out[0] / scale, out[1] / scale) |
                      ((uint32_t)pack_e4m3x2(out[2] / scale, out[3] / scale) << 16);
        uint32_t hi = (uint32_t)pack_e4m3x2(out[4] / scale, out[5] / scale) |
                      ((uint32_t)pack_e4m3x2(out[6] / scale, out[7] / scale) << 16);
        *reinterpret_cast<uint2*>(op) = make_uint2(lo, hi);
        if (grp == 0) d.out_scale[srow] = scale;
        return;
    }
    if (d.out_dtype == V4A_MXFP4) {
        // blocks of 32 channels = 4 consecutive lanes (groups is a multiple of 4)
        int x;
        const uint32_t w = mx_quantize8(out, &x);
        if (!active) return;
        uint8_t* op = static_cast<uint8_t*>(d.out) + (obase + grp * 8) / 2;
        *reinterpret_cast<uint32_t*>(op) = w;
        const long long xb = d.bt ? orow * (d.channels / 32) : (long long)b * d.exp_bs + s * (d.channels / 32);
        if ((grp & 3) == 0) d.out_exp[xb + grp / 4] = (uint8_t)(x + 127);
        return;
    }
    if (!active) return;
    if (d.out_dtype == V4A_BF16) {
        __nv_bfloat16* op = static_cast<__nv_bfloat16*>(d.out) + obase + grp * 8;
        Vec8<__nv_bfloat16>::store(op, out);
    } else {
        float* op = static_cast<float*>(d.out) + obase + grp * 8;
        Vec8<float>::store(op, out);
    }
}

// Long chunks (m >= 32: the HCA chunk of 128 tokens) of one stream with bf16 / fp32 output: a block
// per (entry, 16 channel groups = 128 channels), kWideThreads threads.  Lane l of warp w owns channel
// group 16 blockIdx.y + l % 16 and token slot 2 w + l / 16, i.e. tokens slot, slot + 32, ... of the
// chunk (compress_span with a stride of 32), so each warp load reads 256 contiguous bytes of two
// adjacent token rows.  The two slots of a group within a warp merge with one shuffle, the 16 warps'
// states through shared memory, and 128 threads (group x channel) finish.  (The lanes-per-entry
// mapping of compress_kernel has each warp load touch 32 token rows, 16 bytes each.)
constexpr int kWideGroups = 16;
constexpr int kWideThreads = 512;

__global__ void __launch_bounds__(kWideThreads) compress_wide_kernel(StreamDesc d, long long n_ent, int m) {
    griddep_wait();  // everything before this kernel on the stream has finished
    griddep_launch_dependents();
    __shared__ float s_st[kWideThreads / 32][kWideGroups][25];  // (max, den, num) x 8 channels, padded
    __shared__ __align__(16) float s_out[kWideGroups][8];
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = (int)(blockIdx.x / n_ent);
    const long long s = blockIdx.x - (long long)b * n_ent;
    const int gl = lane & 15, grp = blockIdx.y * kWideGroups + gl;
    const int slot = 2 * w + (lane >> 4);
    float mx[8], den[8], num[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        mx[e] = -INFINITY;
        den[e] = 0.f;
        num[e] = 0.f;
    }
    if (grp < d.groups) {
        StreamDesc dd = d;
        dd.split = 32;  // token stride of compress_span
        const long long off = s * m * d.channels + grp * 8;
        if (d.in_dtype == V4A_BF16) {
            compress_span(dd, static_cast<const __nv_bfloat16*>(d.x) + (long long)b * d.x_bs + off,
                          static_cast<const __nv_bfloat16*>(d.gate) + (long long)b * d.gate_bs + off, m, slot, mx,
                          den, num);
        } else {
            compress_span(dd, static_cast<const float*>(d.x) + (long long)b * d.x_bs + off,
                          static_cast<const float*>(d.gate) + (long long)b * d.gate_bs + off, m, slot, mx, den, num);
        }
    }
    // lanes l and l ^ 16: the same group, two token slots
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float gm = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 16));
        const float a = mx[e] == -INFINITY ? 0.f : expf(mx[e] - gm);
        float dn = den[e] * a, nu = num[e] * a;
        dn += __shfl_xor_sync(0xffffffffu, dn, 16);
        nu += __shfl_xor_sync(0xffffffffu, nu, 16);
        mx[e] = gm;
        den[e] = dn;
        num[e] = nu;
    }
    if (lane < 16) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            s_st[w][gl][3 * e] = mx[e];
            s_st[w][gl][3 * e + 1] = den[e];
            s_st[w][gl][3 * e + 2] = num[e];
        }
    }
    __syncthreads();
    if (threadIdx.x < kWideGroups * 8) {
        const int gi = threadIdx.x >> 3, ch = threadIdx.x & 7;
        float gm = -INFINITY;
#pragma unroll 4
        for (int v = 0; v < kWideThreads / 32; ++v) gm = fmaxf(gm, s_st[v][gi][3 * ch]);
        float dn = 0.f, nu = 0.f;
#pragma unroll 4
        for (int v = 0; v < kWideThreads / 32; ++v) {
            const float mv = s_st[v][gi][3 * ch];
            const float a = mv == -INFINITY ? 0.f : expf(mv - gm);
            dn = fmaf(s_st[v][gi][3 * ch + 1], a, dn);
            nu = fmaf(s_st[v][gi][3 * ch + 2], a, nu);
        }
        s_out[gi][ch] = nu / dn;
    }
    __syncthreads();
    if (threadIdx.x >= kWideGroups) return;
    const int og = blockIdx.y * kWideGroups + threadIdx.x;
    if (og >= d.groups) return;
    long long obase;
    if (d.bt) {
        const long long es = d.first + s;
        const long long blk = d.bt[(long long)b * d.bt_stride + es / d.epb];
        if (blk < 0 || blk >= d.n_blocks) return;  // nowhere to write it
        obase = (blk * d.epb + es % d.epb) * d.channels;
    } else {
        obase = (long long)b * d.out_bs + s * d.channels;
    }
    float out[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = s_out[threadIdx.x][e];
    if (d.out_dtype == V4A_BF16) Vec8<__nv_bfloat16>::store(static_cast<__nv_bfloat16*>(d.out) + obase + og * 8, out);
    else Vec8<float>::store(static_cast<float*>(d.out) + obase + og * 8, out);
}

// quantised outputs need every lane of an entry's block (or entry) to hold a finished value
bool quantised(int dt) { return dt == V4A_FP8E4M3 || dt == V4A_MXFP4; }

// one stream, unquantised, chunks of at least 32 tokens: compress_wide_kernel (a block per entry: the
// entries of a launch must fit the grid's x dimension)
bool wide(const StreamDesc& s0, bool two_streams, int batch, long long n_ent, int m) {
    return !two_streams && m >= 32 && !quantised(s0.out_dtype) && s0.xb == nullptr &&
           (long long)batch * n_ent <= 0x7fffffffLL;
}
cudaError_t launch_wide(const StreamDesc& s0, int batch, long long n_ent, int m, cudaStream_t stream) {
    const dim3 grid((unsigned)((long long)batch * n_ent), (unsigned)((s0.groups + kWideGroups - 1) / kWideGroups));
    const cudaError_t e = launch_pdl(compress_wide_kernel, grid, dim3(kWideThreads), 0, stream, s0, n_ent, m);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// MXFP4 quantisation of rows: one thread per 8 elements, 4 lanes per 32-element block
template <typename T>
__global__ void __launch_bounds__(256) quantize_mxfp4_kernel(const T* x, long long rows, int cols, uint8_t* codes,
                                                             uint8_t* exps) {
    griddep_wait();  // everything before this kernel on the stream has finished
    griddep_launch_dependents();
    const int groups = cols / 8;
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const bool active = g < rows * groups;
    const long long row = active ? g / groups : 0;
    const int grp = active ? (int)(g - row * groups) : 0;
    float v[8];
    if (active) {
        Vec8<T>::load_nc(x + row * cols + grp * 8, v);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    int xe;
    const uint32_t w = mx_quantize8(v, &xe);
    if (!active) return;
    *reinterpret_cast<uint32_t*>(codes + row * (cols / 2) + grp * 4) = w;
    if ((grp & 3) == 0) exps[row * (cols / 32) + grp / 4] = (uint8_t)(xe + 127);
}

StreamDesc describe(const v4a_compress_io* io) {
    StreamDesc d;
    d.x = io->x;
    d.gate = io->gate;
    d.xb = d.gateb = d.pxb = d.pgateb = nullptr;
    d.xb_bs = d.gateb_bs = d.prev_bs = 0;
    d.out = io->out;
    d.out_scale = io->out_scale;
    d.out_exp = io->out_exp;
    d.exp_bs = io->exp_batch_stride;
    d.channels = io->channels;
    d.groups = io->channels / 8;
    d.split = 1;
    d.in_dtype = io->in_dtype;
    d.out_dtype = io->out_dtype;
    d.x_bs = io->x_batch_stride;
    d.gate_bs = io->gate_batch_stride;
    d.out_bs = io->out_batch_stride;
    d.scale_bs = io->scale_batch_stride;
    d.bt = nullptr;
    d.bt_stride = d.epb = 0;
    d.first = d.n_blocks = 0;
    return d;
}

// one 16-byte chunk per thread: the new row of each stream into its ring slot pos % ring_rows
struct RingArgs {
    v4a_ring_io io[kMaxRingStreams];
    int n, batch;
    long long pos;
    int chunks[kMaxRingStreams];  // 16-byte chunks per row of each stream
};

__global__ void __launch_bounds__(256) ring_append_kernel(RingArgs r) {
    griddep_wait();  // everything before this kernel on the stream has finished
    griddep_launch_dependents();
    int g = blockIdx.x * blockDim.x + threadIdx.x;
    for (int i = 0; i < r.n; ++i) {
        const int per = r.batch * r.chunks[i];
        if (g < per) {
            const v4a_ring_io& io = r.io[i];
            const int b = g / r.chunks[i], c = g - b * r.chunks[i];
            const size_t es = io.dtype == V4A_F32 ? 4 : io.dtype == V4A_BF16 ? 2 : 1;
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const char*>(io.src) +
                                                              (size_t)b * io.src_batch_stride * es) + c;
            uint4* dst = reinterpret_cast<uint4*>(static_cast<char*>(io.ring) +
                                                  ((size_t)b * io.ring_rows + (size_t)(r.pos % io.ring_rows)) *
                                                      io.channels * es) + c;
            *dst = __ldg(src);
            return;
        }
        g -= per;
    }
}

}  // namespace

cudaError_t launch_compress(const v4a_compress_io* kv, const v4a_compress_io* idx, int batch, long long n_tok,
                            int m, cudaStream_t stream) {
    long long n_ent = n_tok / m;
    if (batch == 0 || n_ent == 0) return cudaSuccess;
    StreamDesc s0 = describe(kv);
    StreamDesc s1 = idx ? describe(idx) : s0;
    if (wide(s0, idx != nullptr, batch, n_ent, m)) return launch_wide(s0, batch, n_ent, m, stream);
    // lanes per (entry, channel group): up to a warp, to spread long chunks; 1 for FP8 output
    // (its per-entry amax runs over the entry's consecutive lanes)
    int split = 1;
    while (split < 32 && split * 2 <= m) split *= 2;
    if (!quantised(s0.out_dtype)) s0.split = split;
    if (!quantised(s1.out_dtype)) s1.split = split;
    long long w0 = (long long)s0.groups * s0.split, w1 = (long long)s1.groups * s1.split;
    long long total = (long long)batch * n_ent * (w0 > w1 ? w0 : w1);
    const int threads = 256;
    dim3 grid((unsigned)((total + threads - 1) / threads), idx ? 2 : 1);
    const cudaError_t e = launch_pdl(compress_kernel, grid, dim3(threads), 0, stream, s0, s1, batch, n_ent, m);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_quantize_mxfp4(const void* x, v4a_dtype dt, long long rows, int cols, uint8_t* codes,
                                  uint8_t* exps, cudaStream_t stream) {
    const long long total = rows * (cols / 8);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    const unsigned blocks = (unsigned)((total + threads - 1) / threads);
    const cudaError_t e =
        dt == V4A_BF16 ? launch_pdl(quantize_mxfp4_kernel<__nv_bfloat16>, dim3(blocks), dim3(threads), 0, stream,
                                    static_cast<const __nv_bfloat16*>(x), rows, cols, codes, exps)
                       : launch_pdl(quantize_mxfp4_kernel<float>, dim3(blocks), dim3(threads), 0, stream,
                                    static_cast<const float*>(x), rows, cols, codes, exps);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_compress_paged(const v4a_compress_io* kv, const v4a_compress_io* idx, int batch, long long n_tok,
                                  int m, long long first_entry, const int32_t* bt, int bt_stride, int epb,
                                  long long n_blocks, cudaStream_t stream) {
    long long n_ent = n_tok / m;
    if (batch == 0 || n_ent == 0) return cudaSuccess;
    StreamDesc s0 = describe(kv);
    StreamDesc s1 = idx ? describe(idx) : s0;
    for (StreamDesc* d : {&s0, &s1}) {
        d->bt = bt;
        d->bt_stride = bt_stride;
        d->epb = epb;
        d->first = first_entry;
        d->n_blocks = n_blocks;
    }
    if (wide(s0, idx != nullptr, batch, n_ent, m)) return launch_wide(s0, batch, n_ent, m, stream);
    int split = 1;
    while (split < 32 && split * 2 <= m) split *= 2;
    if (!quantised(s0.out_dtype)) s0.split = split;
    if (!quantised(s1.out_dtype)) s1.split = split;
    long long w0 = (long long)s0.groups * s0.split, w1 = (long long)s1.groups * s1.split;
    long long total = (long long)batch * n_ent * (w0 > w1 ? w0 : w1);
    const int threads = 256;
    dim3 grid((unsigned)((total + threads - 1) / threads), idx ? 2 : 1);
    const cudaError_t e = launch_pdl(compress_kernel, grid, dim3(threads), 0, stream, s0, s1, batch, n_ent, m);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_ring_append(const v4a_ring_io* io, int n, int batch, long long pos, cudaStream_t stream) {
    if (n == 0 || batch == 0) return cudaSuccess;
    RingArgs r;
    r.n = n;
    r.batch = batch;
    r.pos = pos;
    long long total = 0;
    for (int i = 0; i < n; ++i) {
        r.io[i] = io[i];
        const size_t es = io[i].dtype == V4A_F32 ? 4 : io[i].dtype == V4A_BF16 ? 2 : 1;
        r.chunks[i] = (int)((size_t)io[i].channels * es / 16);
        total += (long long)batch * r.chunks[i];
    }
    const int threads = 256;
    const cudaError_t e =
        launch_pdl(ring_append_kernel, dim3((unsigned)((total + threads - 1) / threads)), dim3(threads), 0, stream, r);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_compress_dual(const v4a_compress_io* a, const v4a_series_b* b, int batch, long long n_tok, int m,
                                 cudaStream_t stream) {
    long long n_ent = n_tok / m;
    if (batch == 0 || n_ent == 0) return cudaSuccess;
    StreamDesc s0 = describe(a);
    s0.xb = b->x;
    s0.gateb = b->gate;
    s0.pxb = b->prev_x;
    s0.pgateb = b->prev_gate;
    s0.xb_bs = b->x_batch_stride;
    s0.gateb_bs = b->gate_batch_stride;
    s0.prev_bs = b->prev_batch_stride;
    int split = 1;
    while (split < 32 && split * 2 <= m) split *= 2;
    if (!quantised(s0.out_dtype)) s0.split = split;
    const long long total = (long long)batch * n_ent * s0.groups * s0.split;
    const int threads = 256;
    dim3 grid((unsigned)((total + threads - 1) / threads), 1);
    const cudaError_t e = launch_pdl(compress_kernel, grid, dim3(threads), 0, stream, s0, s0, batch, n_ent, m);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace v4a
