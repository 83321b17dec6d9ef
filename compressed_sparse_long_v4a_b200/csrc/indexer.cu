// indexer.cu -- Lightning-Indexer scores and the top-k select.
//
// Score ("How V4 makes a million-token context actually affordable",
// Lightning-Indexer section): I(t,s) = scale_s * sum_j w_j * ReLU(q_j . k_s),
// one key per entry shared by every indexer head.  Only entries visible to the
// query (m*(s+1) <= t+1) get a score.
//
// CUDA-core path, any (heads_i <= 64, d_i % 8 == 0) and key format: one thread
// per entry streams the entry's key with 16-byte loads (fp8 keys: 8 bytes at a
// time, MXFP4 keys 4 bytes, widened exactly to fp32) and accumulates every
// head's dot product in registers against the query held in shared memory
// (broadcast reads; for MXFP4 keys the query is quantised to MXFP4 first).
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

// 8 key elements starting at element `off` of the key array (decoded exactly to fp32)
template <int KFMT>
__device__ __forceinline__ void load_key8(const IndexArgs& a, long long off, float f[8]) {
    if constexpr (KFMT == V4A_F32) {
        Vec8<float>::load_nc(static_cast<const float*>(a.k) + off, f);
    } else if constexpr (KFMT == V4A_BF16) {
        Vec8<__nv_bfloat16>::load_nc(static_cast<const __nv_bfloat16*>(a.k) + off, f);
    } else if constexpr (KFMT == V4A_FP8E4M3) {
        uint2 v = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(a.k) + off));
        unpack_e4m3x8(v, f);
    } else {  // MXFP4: 4 bytes of codes and their block's exponent
        const uint32_t cw = __ldg(reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(a.k) + off / 2));
        const float sc = e8m0_value(__ldg(a.kexp + off / 32));
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = e2m1_value((cw >> (4 * i)) & 0xfu) * sc;
    }
}

// grid: (ceil(N / 256), B * n_q); q of the block's query staged in shared memory
template <int HMAX, int KFMT>
__global__ void __launch_bounds__(kScoreThreads) index_score_kernel(IndexArgs a, float* scores) {
    griddep_wait();  // everything before this kernel on the stream has finished
    griddep_launch_dependents();
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
    if constexpr (KFMT == V4A_MXFP4) {
        // FP4 dot products: the query of every head is quantised to MXFP4 (blocks of 32 along d_i)
        // and replaced by its decoded values
        __syncthreads();
        for (int i = threadIdx.x; i < qn / 32; i += blockDim.x) {
            float* p = q_s + 32 * i;
            float am = 0.f;
            for (int j = 0; j < 32; ++j) am = fmaxf(am, fabsf(p[j]));
            const int x = mx_block_exp(am);
            const float inv = pow2i(-x), sc = e8m0_value((uint32_t)(x + 127));
            for (int j = 0; j < 32; ++j) p[j] = e2m1_value(e2m1_code(p[j] * inv)) * sc;
        }
    }
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
    long long krow = (long long)b * a.n_ent + s;
    if (a.bt) {
        const long long blk = a.bt[(long long)b * a.bt_stride + s / a.epb];
        krow = (blk >= 0 && blk * a.epb < a.pool_rows) ? blk * a.epb + s % a.epb : -1;  // -1: outside the pool
    }
    if (krow < 0) {  // reads as a key of zeros
        *out = 0.0f;
        return;
    }
    const long long koff = krow * a.d_i;
    for (int c = 0; c < a.d_i; c += 8) {
        float kv[8];
        load_key8<KFMT>(a, koff + c, kv);
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
    if (a.kscale) sc *= a.kscale[krow];
    *out = sc + 0.0f;  // -0 -> +0
}

// ---------------------------------------------------------------------
// select
// ---------------------------------------------------------------------

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

// sum of v over the threads with a larger index (the block total in *total)
__device__ __forceinline__ int block_exclusive_scan_rev(int v, int* warp_buf, int* total) {
    // scan in reversed thread order by scanning the mirrored value
    const int n = blockDim.x;
    __shared__ int mirror[1024];
    mirror[n - 1 - threadIdx.x] = v;
    __syncthreads();
    const int mv = mirror[threadIdx.x];
    __syncthreads();
    const int ex = block_exclusive_scan(mv, warp_buf, total);
    mirror[threadIdx.x] = ex;
    __syncthreads();
    const int r = mirror[n - 1 - threadIdx.x];
    __syncthreads();
    return r;
}

// The digit d of a histogram (bins 0..nbins-1, nbins <= blockDim.x) at which
// the count of keys in bins above d stays below `rem` while bins >= d reach it;
// *above = count above d.  One bin per thread, block-wide suffix scan.
__device__ void find_digit(const unsigned int* h, int nbins, long long rem, int* digit, long long* above) {
    __shared__ int s_dgt;
    __shared__ long long s_above;
    __shared__ int warp_buf[33];
    const int c = threadIdx.x < nbins ? (int)h[threadIdx.x] : 0;
    int tot;
    const int hi_sum = block_exclusive_scan_rev(c, warp_buf, &tot);  // keys in bins above this thread's
    if (threadIdx.x == 0) {
        s_dgt = 0;
        s_above = 0;
    }
    __syncthreads();
    if (threadIdx.x < nbins && hi_sum < rem && (long long)hi_sum + c >= rem) {
        s_dgt = threadIdx.x;
        s_above = hi_sum;
    }
    __syncthreads();
    *digit = s_dgt;
    *above = s_above;
    __syncthreads();
}

// Exact radix select of one row (scores[0..nvis), -inf never selected): the
// min(k, nvis) largest, ties to the lower entry, written in ascending entry
// order and padded with -1.  Called by a whole block (any size of at least 256 threads).
__device__ void select_row_radix(const float* sc, long long nvis, int k, int32_t* io, float* so) {
    __shared__ unsigned int hist[256];
    __shared__ int warp_buf[33];
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
            int dgt;
            long long above;
            find_digit(hist, 256, need, &dgt, &above);
            prefix |= (uint32_t)dgt << shift;
            mask |= 255u << shift;
            need -= above;
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

__device__ __forceinline__ long long row_nvis(const IndexArgs& a, int row) {
    const long long t = a.ctx_len - a.n_q + (row % a.n_q);
    long long nvis = n_visible(t, a.m);
    return nvis > a.n_ent ? a.n_ent : nvis;
}


// ---------------------------------------------------------------------
// select for few query rows: histogram threshold, then one kernel whose
// blocks each compact one chunk of a row and whose last block per row
// finishes that row
// ---------------------------------------------------------------------
constexpr int kHistBins = 4096;  // top 12 bits of the ordered key (built by the score kernels)
constexpr int kFastThreads = 512;
constexpr int kFastPer = 8;                              // consecutive scores per thread per step
constexpr int kFastStep = kFastThreads * kFastPer;       // 4096 scores per block step
constexpr int kMaxFastRows = 256;
constexpr int kMaxFastParts = 512;
constexpr int kCandCap = 7168;   // candidates the finishing block holds in shared memory (two blocks fit an SM)
constexpr size_t kFastSmem = (size_t)kCandCap * 8 + 2 * 4096 * sizeof(int32_t);
constexpr int kMaxK = 4096;      // largest k the API takes
constexpr int kSelCap = 4096;    // threshold-bin candidates of a row the few-rows select holds
constexpr size_t kSelSmem = (size_t)kSelCap * 8 + 2 * kMaxK * sizeof(int32_t);


// Block-wide bin search: thread t owns bins [P t, P t + P) with counts c[] (in registers).
// Finds the bin d where the keys in bins above d number fewer than `rem` while bins >= d hold at
// least `rem`; *above = keys above d; d = -1 when all bins together hold fewer than `rem`.
// Per-thread sums go to shared memory, warp 0 locates the owning thread (each lane sums a run of
// threads, read with a conflict-free swizzle, then a suffix scan over lanes), and the owner scans
// its own P bins.  Every thread of the block gets the answer.
template <int P>
__device__ void block_find_bin(const int (&c)[P], long long rem, int* digit, long long* above, long long* total) {
    __shared__ int psum[1024];
    __shared__ int s_t, s_d;
    __shared__ long long s_tab, s_tot, s_ab;
    int sum = 0;
#pragma unroll
    for (int i = 0; i < P; ++i) sum += c[i];
    psum[threadIdx.x] = sum;
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x, nt = blockDim.x, per = (nt + 31) / 32;
        long long local = 0;
        for (int j = 0; j < per; ++j) {
            const int idx = lane * per + ((j + lane / 2) % per);
            if (idx < nt) local += psum[idx];
        }
        long long incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_down_sync(0xffffffffu, incl, o);
            if (lane + o < 32) incl += y;
        }
        const long long higher = incl - local;  // keys in threads owned by higher lanes
        int tsel = -1;
        long long tab = 0;
        if (higher < rem && incl >= rem) {
            long long run = higher;
            for (int j = per - 1; j >= 0; --j) {
                const int idx = lane * per + j;
                const long long v = idx < nt ? psum[idx] : 0;
                if (run + v >= rem) {
                    tsel = idx;
                    tab = run;
                    break;
                }
                run += v;
            }
        }
        const unsigned who = __ballot_sync(0xffffffffu, tsel >= 0);
        const int src = who ? __ffs(who) - 1 : 0;
        tsel = __shfl_sync(0xffffffffu, tsel, src);
        tab = __shfl_sync(0xffffffffu, tab, src);
        const long long tot = __shfl_sync(0xffffffffu, incl, 0);
        if (lane == 0) {
            s_t = who ? tsel : -1;
            s_tab = tab;
            s_tot = tot;
            if (!who) {
                s_d = -1;
                s_ab = 0;
            }
        }
    }
    __syncthreads();
    if ((int)threadIdx.x == s_t) {
        long long run = s_tab;
        for (int i = P - 1; i >= 0; --i) {
            if (run + c[i] >= rem) {
                s_d = P * (int)threadIdx.x + i;
                s_ab = run;
                break;
            }
            run += c[i];
        }
    }
    __syncthreads();
    *digit = s_d;
    *above = s_ab;
    *total = s_tot;
    __syncthreads();  // the shared words may be reused by the next call
}

// The bin holding the k-th largest key: its index, and how many keys lie in higher bins.
// Every thread of the block gets the answer; `all` when at most k keys exist.  blockDim.x must
// be kHistBins / 8 (each thread owns 8 bins).
__device__ void threshold_bin(const uint32_t* hist_row, int k, int* bin, int* above, bool* all) {
    const uint4* h4 = reinterpret_cast<const uint4*>(hist_row) + 2 * threadIdx.x;
    const uint4 u = __ldcg(h4), v = __ldcg(h4 + 1);
    const int c[8] = {(int)u.x, (int)u.y, (int)u.z, (int)u.w, (int)v.x, (int)v.y, (int)v.z, (int)v.w};
    int d;
    long long ab, tot;
    block_find_bin<8>(c, k, &d, &ab, &tot);
    *bin = d;
    *above = (int)ab;
    *all = tot <= k;
}

// The digit of a 1024-bin shared histogram, found by warp 0 in two levels (32 bins per lane read
// with a conflict-free rotation, suffix scan over lanes; then the owning lane's 32 bins, one per
// lane, scanned again) and broadcast to the block.
__device__ void find_digit_1024(const unsigned int* h, long long rem, int* digit, long long* above) {
    __shared__ int s_dgt;
    __shared__ long long s_above;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        long long local = 0;
#pragma unroll 8
        for (int j = 0; j < 32; ++j) local += h[32 * lane + ((j + lane) & 31)];
        long long incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_down_sync(0xffffffffu, incl, o);
            if (lane + o < 32) incl += y;
        }
        const long long higher = incl - local;
        const unsigned who = __ballot_sync(0xffffffffu, higher < rem && incl >= rem);
        const int L = who ? __ffs(who) - 1 : 0;
        const long long hL = __shfl_sync(0xffffffffu, higher, L);
        const long long v = h[32 * L + lane];
        long long incl2 = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_down_sync(0xffffffffu, incl2, o);
            if (lane + o < 32) incl2 += y;
        }
        const long long higher2 = hL + incl2 - v;
        const unsigned who2 = __ballot_sync(0xffffffffu, higher2 < rem && higher2 + v >= rem);
        const int j = who2 ? __ffs(who2) - 1 : 0;
        const long long ab = __shfl_sync(0xffffffffu, higher2, j);
        if (lane == 0) {
            s_dgt = who ? 32 * L + j : 0;
            s_above = who ? ab : 0;
        }
    }
    __syncthreads();
    *digit = s_dgt;
    *above = s_above;
    __syncthreads();
}

// first position in sorted v[0..n) holding a value >= x
__device__ __forceinline__ int lower_bound(const int32_t* v, int n, int32_t x) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (v[mid] < x) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

// The row's answer from the parts' compacted lists: every definite entry (key in a bin above the
// threshold bin) plus the best `need` candidates (keys in the threshold bin), ties to the lower
// entry, in ascending entry order, padded with -1.  Whole block; the parts' writes are visible.
// The row's answer from its definite entries defs[0..D) and candidates (cidx, ckey)[0..C) in
// shared memory, both in ascending entry order: every definite entry plus the best `need` candidates
// (radix select over the low 20 key bits, whose top 12 are equal; ties to the lower entry), merged
// in ascending order into io (and so), padded with -1.  Whole block of kFastThreads threads.
__device__ void finish_lists(const float* sc, int k, int D, int C, int32_t* defs, int32_t* cidx, uint32_t* ckey,
                             int32_t* sels, int32_t* io, float* so) {
    __shared__ unsigned int h1[1024];
    __shared__ int warp_buf[33];
    const int need = (D + C) < k ? C : k - D;  // candidates to take
    __syncthreads();
    // radix select of the need-th largest candidate key over its low 20 bits (the top 12 are equal)
    uint32_t prefix = C > 0 ? (ckey[0] & 0xfff00000u) : 0u, mask = 0xfff00000u;
    int rem = need;
    if (need > 0 && need < C) {
        for (int shift = 10; shift >= 0; shift -= 10) {
            for (int i = threadIdx.x; i < 1024; i += blockDim.x) h1[i] = 0;
            __syncthreads();
            for (int i = threadIdx.x; i < C; i += blockDim.x)
                if ((ckey[i] & mask) == prefix) atomicAdd(&h1[(ckey[i] >> shift) & 1023u], 1u);
            __syncthreads();
            int dgt;
            long long above;
            find_digit_1024(h1, rem, &dgt, &above);
            prefix |= (uint32_t)dgt << shift;
            rem -= (int)above;
            mask |= 1023u << shift;
        }
    }
    // mark: key > prefix, or key == prefix among the first `rem` such (in entry order).  Thread t
    // takes candidates [t*per, t*per + per) into registers; two block scans give the equal-key ranks
    // and the output positions; the compacted keys go back into ckey after everyone has read.
    const bool take_all = need >= C;
    constexpr int kMaxPer = kCandCap / kFastThreads;
    const int per = (C + (int)blockDim.x - 1) / (int)blockDim.x;
    const int i0 = threadIdx.x * per;
    uint32_t mk[kMaxPer];
    int32_t mi[kMaxPer];
    int n_eq = 0;
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {
        const int i = i0 + j;
        const bool in = j < per && i < C;
        mk[j] = in ? ckey[i] : 0u;
        mi[j] = in ? cidx[i] : -1;
        n_eq += (in && !take_all && mk[j] == prefix) ? 1 : 0;
    }
    int eq_tot;
    int eq_rank = block_exclusive_scan(n_eq, warp_buf, &eq_tot);
    uint32_t selmask = 0;
    int n_sel = 0;
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {
        const bool in = mi[j] >= 0;
        const bool gt = in && (take_all || mk[j] > prefix);
        const bool eq = in && !take_all && mk[j] == prefix;
        const bool sel = gt || (eq && eq_rank < rem);
        eq_rank += eq ? 1 : 0;
        if (sel) {
            selmask |= 1u << j;
            ++n_sel;
        }
    }
    int out;
    int pos = block_exclusive_scan(n_sel, warp_buf, &out);  // ends with a barrier: all reads are done
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j)
        if (selmask & (1u << j)) {
            sels[pos] = mi[j];
            ckey[pos] = mk[j];
            ++pos;
        }
    __syncthreads();
    const int total = D + out;
    // merge the two ascending lists into the output
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
        const int32_t x = defs[i];
        const int pos = i + lower_bound(sels, out, x);
        io[pos] = x;
        if (so) so[pos] = sc[x];
    }
    for (int j = threadIdx.x; j < out; j += blockDim.x) {
        const int32_t y = sels[j];
        const int pos = j + lower_bound(defs, D, y);
        io[pos] = y;
        if (so) so[pos] = ordered_to_float(ckey[j]);
    }
    for (int p = total + threadIdx.x; p < k; p += blockDim.x) {
        io[p] = -1;
        if (so) so[p] = -INFINITY;
    }
}


// Bitonic sort of v[0 .. n2) ascending in shared memory (n2 a power of two; padded with 0x7fffffff).
// Whole block.
__device__ void bitonic_sort(int32_t* v, int n2) {
    for (int size = 2; size <= n2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < (n2 >> 1); i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
                const int32_t x = v[lo], y = v[hi];
                if ((x > y) == ((lo & size) == 0)) {
                    v[lo] = y;
                    v[hi] = x;
                }
            }
            __syncthreads();
        }
    }
}

__device__ __forceinline__ int pow2_at_least(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

// ---------------------------------------------------------------------
// select for few query rows: kFastThreads-thread blocks, `parts` per row
// ---------------------------------------------------------------------
// Block (row, p) finds the threshold bin (the 12-bit bin of the row's k-th largest key, from the
// histogram the scoring kernel built) and compacts entries [p chunk, (p+1) chunk) of the row into the
// row's two lists in global memory: definite entries (keys in higher bins; fewer than k in the row)
// and candidates (keys in the threshold bin, with their keys), reserving its span of both with one
// 64-bit atomic per step.  The last block of the row to finish (an atomic ticket; nothing waits)
// finishes the row: a radix select over the candidates' low 20 key bits picks the best `need`
// (ties to the lower entries), and the chosen entries are marked in a bitmap over the row whose
// prefix counts give each its place in the ascending output (rows longer than the bitmap sort the
// chosen entries instead).  Loops are kept rolled: these blocks run briefly, and on B200 a short
// kernel's time went largely to fetching its instructions (a step streams more than L2 holds), at
// about 120 cycles per element for an unrolled 32-element loop.
constexpr int kBitmapWords = kSelCap * 2;  // the candidate arrays, reused: rows of up to 262,144 entries

__device__ void finish_row(const float* sc, long long nvis, int k, int D, int C, const int32_t* def_row,
                           const int32_t* cidx_row, const uint32_t* ckey_row, int32_t* io, float* so, uint8_t* dsm) {
    uint32_t* ckey = reinterpret_cast<uint32_t*>(dsm);          // [kSelCap]
    int32_t* cidx = reinterpret_cast<int32_t*>(ckey + kSelCap);  // [kSelCap]
    int32_t* sel = cidx + kSelCap;                               // [kMaxK]: the answer
    int32_t* eqv = sel + kMaxK;                                  // [kMaxK]: candidates equal to the threshold key
    uint32_t* bits = ckey;                                       // [kBitmapWords] once the candidates are used
    __shared__ unsigned int h1[1024];
    __shared__ int s_ngt, s_neq, warp_buf[33];
    if (C > kSelCap || D > k) {
        // more candidates than the finish holds (e.g. huge blocks of equal scores): exact select over the row
        select_row_radix(sc, nvis, k, io, so);
        return;
    }
    // the lists, four loads in flight per thread
#pragma unroll 1
    for (int i0 = threadIdx.x; i0 < C; i0 += 4 * kFastThreads) {
        uint32_t kk[4];
        int32_t ii[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * kFastThreads;
            kk[u] = i < C ? __ldcg(ckey_row + i) : 0u;
            ii[u] = i < C ? __ldcg(cidx_row + i) : 0;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * kFastThreads;
            if (i < C) {
                ckey[i] = kk[u];
                cidx[i] = ii[u];
            }
        }
    }
#pragma unroll 1
    for (int i0 = threadIdx.x; i0 < D; i0 += 4 * kFastThreads) {
        int32_t dd[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) dd[u] = i0 + u * kFastThreads < D ? __ldcg(def_row + i0 + u * kFastThreads) : 0;
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (i0 + u * kFastThreads < D) sel[i0 + u * kFastThreads] = dd[u];
    }
    if (threadIdx.x == 0) {
        s_ngt = D;
        s_neq = 0;
    }
    const int need = (D + C) <= k ? C : k - D;  // candidates to take
    const bool take_all = need >= C;
    __syncthreads();
    // radix select of the need-th largest candidate key over its low 20 bits (the top 12 are equal)
    uint32_t prefix = C > 0 ? (ckey[0] & 0xfff00000u) : 0u, mask = 0xfff00000u;
    int rem = need;
    if (!take_all) {
#pragma unroll 1
        for (int shift = 10; shift >= 0; shift -= 10) {
            for (int i = threadIdx.x; i < 1024; i += blockDim.x) h1[i] = 0;
            __syncthreads();
#pragma unroll 1
            for (int i = threadIdx.x; i < C; i += blockDim.x)
                if ((ckey[i] & mask) == prefix) atomicAdd(&h1[(ckey[i] >> shift) & 1023u], 1u);
            __syncthreads();
            int dgt;
            long long above;
            find_digit_1024(h1, rem, &dgt, &above);
            prefix |= (uint32_t)dgt << shift;
            rem -= (int)above;
            mask |= 1023u << shift;
        }
    }
    // candidates above the threshold key join the answer; those equal to it are collected (rem of them
    // are taken, the lowest entries)
#pragma unroll 1
    for (int i0 = 0; i0 < C; i0 += blockDim.x) {  // warp-uniform trip count (ballots below)
        const int i = i0 + threadIdx.x;
        const uint32_t key = i < C ? ckey[i] : 0u;
        const bool gt = i < C && (take_all || key > prefix);
        const bool eq = i < C && !take_all && key == prefix;
        const unsigned mg = __ballot_sync(0xffffffffu, gt), me = __ballot_sync(0xffffffffu, eq);
        const int lane = threadIdx.x & 31;
        int bg = 0, be = 0;
        if (lane == 0) {
            bg = mg ? atomicAdd(&s_ngt, __popc(mg)) : 0;
            be = me ? atomicAdd(&s_neq, __popc(me)) : 0;
        }
        bg = __shfl_sync(0xffffffffu, bg, 0);
        be = __shfl_sync(0xffffffffu, be, 0);
        const unsigned below = (1u << lane) - 1u;
        if (gt) sel[bg + __popc(mg & below)] = cidx[i];
        if (eq && be + __popc(me & below) < kMaxK) eqv[be + __popc(me & below)] = cidx[i];
    }
    __syncthreads();
    const int ngt = s_ngt, neq = s_neq;
    if (!take_all && rem > 0) {
        if (neq > kMaxK) {  // (at most k - D tied keys are wanted; a larger tie goes the exact way)
            select_row_radix(sc, nvis, k, io, so);
            return;
        }
        if (rem < neq) {  // the lowest entries among the tied candidates
            const int n2 = pow2_at_least(neq);
            for (int i = neq + threadIdx.x; i < n2; i += blockDim.x) eqv[i] = 0x7fffffff;
            __syncthreads();
            bitonic_sort(eqv, n2);
        }
        for (int i = threadIdx.x; i < rem; i += blockDim.x) sel[ngt + i] = eqv[i];
    }
    const int total = ngt + (take_all ? 0 : rem);
    __syncthreads();
    const int words = (int)((nvis + 31) >> 5);
    if (words <= kBitmapWords) {
        // bitmap over the row; thread t owns words [16 t, 16 t + 16) (kBitmapWords = 16 x kFastThreads), held
        // in registers from four 16-byte loads, and its set bits go out in order after those of lower threads
        static_assert(kBitmapWords == 16 * kFastThreads, "bitmap words per thread");
        uint4* b4 = reinterpret_cast<uint4*>(bits);
        for (int i = threadIdx.x; i < kBitmapWords / 4; i += blockDim.x) b4[i] = make_uint4(0u, 0u, 0u, 0u);
        __syncthreads();
        for (int i = threadIdx.x; i < total; i += blockDim.x) atomicOr(&bits[sel[i] >> 5], 1u << (sel[i] & 31));
        __syncthreads();
        uint32_t wv[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 x = b4[4 * threadIdx.x + q];
            wv[4 * q] = x.x;
            wv[4 * q + 1] = x.y;
            wv[4 * q + 2] = x.z;
            wv[4 * q + 3] = x.w;
        }
        int cnt = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) cnt += __popc(wv[j]);
        int tot;
        int pos = block_exclusive_scan(cnt, warp_buf, &tot);
#pragma unroll
        for (int j = 0; j < 16; ++j) {  // unrolled: wv stays in registers
            uint32_t b = wv[j];
            while (b) {
                io[pos++] = (int32_t)((16 * (int)threadIdx.x + j) * 32 + __ffs(b) - 1);
                b &= b - 1;
            }
        }
    } else {
        const int n2 = pow2_at_least(total < 2 ? 2 : total);
        for (int i = total + threadIdx.x; i < n2; i += blockDim.x) sel[i] = 0x7fffffff;
        __syncthreads();
        bitonic_sort(sel, n2);
        for (int p = threadIdx.x; p < total; p += blockDim.x) io[p] = sel[p];
    }
    for (int p = total + threadIdx.x; p < k; p += blockDim.x) io[p] = -1;
    if (so) {
        __syncthreads();  // io is written (by this block; read back below)
#pragma unroll 1
        for (int p = threadIdx.x; p < k; p += blockDim.x) {
            const int32_t x = __ldcg(io + p);
            so[p] = x >= 0 ? __ldcg(sc + x) : -INFINITY;
        }
    }
}

// grid rows * parts, kFastThreads threads (see above).  ctr: per row one 64-bit word (definite entries
// in its low half, candidates in its high half) and one finished-parts count, all starting at zero.
__global__ void __launch_bounds__(kFastThreads) topk_fast_kernel(const float* scores, const uint32_t* hist, IndexArgs a,
                                                                 int k, int parts, long long chunk, int32_t* def_buf,
                                                                 int32_t* cidx_buf, uint32_t* ckey_buf,
                                                                 unsigned long long* ctr, int32_t* idx_out,
                                                                 float* score_out) {
    griddep_wait();  // everything before this kernel on the stream has finished
    griddep_launch_dependents();
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ int warp_buf[33];
    __shared__ int s_last;
    __shared__ unsigned long long s_base;
    const int row = blockIdx.x / parts, p = blockIdx.x % parts;
    const long long nvis = row_nvis(a, row);
    int tbin, above;
    bool all;
    threshold_bin(hist + (long long)row * kHistBins, k, &tbin, &above, &all);
    const float* sc = scores + (long long)row * a.n_ent;
    const long long lo = (long long)p * chunk;
    long long hi = lo + chunk;
    if (hi > nvis) hi = nvis;
    int32_t* dout = def_buf + (long long)row * k;
    int32_t* ciout = cidx_buf + (long long)row * kSelCap;
    uint32_t* ckout = ckey_buf + (long long)row * kSelCap;
    unsigned long long* rc = ctr + 2LL * row;
    const bool vec = (reinterpret_cast<uintptr_t>(sc) & 15) == 0;
#pragma unroll 1
    for (long long base = lo; base < hi; base += kFastStep) {
        // this thread's kFastPer consecutive scores (16-byte loads when the row is 16-byte aligned)
        const long long s0 = base + (long long)threadIdx.x * kFastPer;
        float v[kFastPer];
        if (vec && s0 + kFastPer <= hi) {
            const float4 x0 = __ldcg(reinterpret_cast<const float4*>(sc + s0));
            const float4 x1 = __ldcg(reinterpret_cast<const float4*>(sc + s0) + 1);
            v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
            v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
        } else {
#pragma unroll
            for (int i = 0; i < kFastPer; ++i) v[i] = s0 + i < hi ? __ldcg(sc + s0 + i) : 0.f;
        }
        int nd = 0, nc = 0;
#pragma unroll
        for (int i = 0; i < kFastPer; ++i) {
            const int bin = (int)(float_to_ordered(v[i]) >> 20);
            const bool in = s0 + i < hi;
            nd += (in && (all || bin > tbin)) ? 1 : 0;
            nc += (in && !all && bin == tbin) ? 1 : 0;
        }
        int tot;
        const int packed = block_exclusive_scan(nd | (nc << 16), warp_buf, &tot);
        if (threadIdx.x == 0)
            s_base = atomicAdd(rc, (unsigned long long)(tot & 0xffff) | ((unsigned long long)(tot >> 16) << 32));
        __syncthreads();
        int od = (int)(s_base & 0xffffffffu) + (packed & 0xffff), oc = (int)(s_base >> 32) + (packed >> 16);
#pragma unroll 1
        for (int i = 0; i < kFastPer; ++i) {
            const uint32_t key = float_to_ordered(v[i]);
            const int bin = (int)(key >> 20);
            const bool in = s0 + i < hi;
            if (in && (all || bin > tbin)) {
                if (od < k) dout[od] = (int32_t)(s0 + i);  // fewer than k entries lie above the threshold bin
                ++od;
            }
            if (in && !all && bin == tbin) {
                if (oc < kSelCap) {
                    ciout[oc] = (int32_t)(s0 + i);
                    ckout[oc] = key;
                }
                ++oc;
            }
        }
        __syncthreads();  // s_base is read before the next step overwrites it
    }
    __threadfence();  // this block's list entries are visible before it is counted
    __syncthreads();
    if (threadIdx.x == 0)
        s_last = atomicAdd(reinterpret_cast<unsigned int*>(rc + 1), 1u) == (unsigned)(parts - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const unsigned long long dc = __ldcg(rc);
    finish_row(sc, nvis, k, (int)(dc & 0xffffffffu), (int)(dc >> 32), dout, ciout, ckout,
               idx_out + (long long)row * k, score_out ? score_out + (long long)row * k : nullptr, dsm);
}

// Many query rows (prefill): one block (kFastThreads) per row.  Pass 1 builds the histogram of
// the row's keys' top 12 bits in shared memory (warp-aggregated atomics), the threshold bin
// follows, pass 2 compacts the definite entries and the threshold bin's candidates into shared
// memory in entry order, and finish_lists selects and merges.  A row whose threshold bin holds
// more than kCandCap candidates falls back to the exact radix select over the row.
__global__ void __launch_bounds__(kFastThreads) topk_rows_kernel(const float* scores, IndexArgs a, int k,
                                                                 int32_t* idx_out, float* score_out) {
    griddep_wait();  // everything before this kernel on the stream has finished
    griddep_launch_dependents();
    extern __shared__ __align__(16) uint8_t dsm[];
    uint32_t* ckey = reinterpret_cast<uint32_t*>(dsm);           // [kCandCap]
    int32_t* cidx = reinterpret_cast<int32_t*>(ckey + kCandCap);  // [kCandCap]
    int32_t* defs = cidx + kCandCap;                              // [4096]
    int32_t* sels = defs + 4096;                                  // [4096]; the histogram before that
    uint32_t* hist = reinterpret_cast<uint32_t*>(sels);
    __shared__ int warp_buf[33];
    const int row = blockIdx.x;
    const long long nvis = row_nvis(a, row);
    const float* sc = scores + (long long)row * a.n_ent;
    int32_t* io = idx_out + (long long)row * k;
    float* so = score_out ? score_out + (long long)row * k : nullptr;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    // kFastPer consecutive scores per thread per step, all loaded before any is counted; lanes of a
    // warp that hit the same bin add once
    for (long long base = 0; base < nvis; base += kFastStep) {
        const long long s0 = base + (long long)threadIdx.x * kFastPer;
        uint32_t bins[kFastPer];
#pragma unroll
        for (int i = 0; i < kFastPer; ++i) bins[i] = s0 + i < nvis ? float_to_ordered(sc[s0 + i]) >> 20 : 0xffffffffu;
#pragma unroll
        for (int i = 0; i < kFastPer; ++i) {
            const unsigned peers = __match_any_sync(0xffffffffu, bins[i]);
            if (bins[i] != 0xffffffffu && (threadIdx.x & 31) == (unsigned)(__ffs(peers) - 1))
                atomicAdd(&hist[bins[i]], (uint32_t)__popc(peers));
        }
    }
    __syncthreads();
    int tbin;
    bool all;
    {
        int c[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j] = (int)hist[8 * threadIdx.x + j];
        int d;
        long long ab, tot;
        block_find_bin<8>(c, k, &d, &ab, &tot);
        tbin = d;
        all = tot <= k;
    }
    int n_def = 0, n_cand = 0;
    for (long long base = 0; base < nvis; base += kFastStep) {
        const long long s0 = base + (long long)threadIdx.x * kFastPer;
        uint32_t keys[kFastPer];
        int nd = 0, nc = 0;
#pragma unroll
        for (int i = 0; i < kFastPer; ++i) {
            const long long s = s0 + i;
            keys[i] = s < nvis ? float_to_ordered(sc[s]) : 0u;
            const int bin = (int)(keys[i] >> 20);
            nd += (s < nvis && (all || bin > tbin)) ? 1 : 0;
            nc += (s < nvis && !all && bin == tbin) ? 1 : 0;
        }
        int tot;
        const int packed = block_exclusive_scan(nd | (nc << 16), warp_buf, &tot);
        int od = n_def + (packed & 0xffff), oc = n_cand + (packed >> 16);
#pragma unroll
        for (int i = 0; i < kFastPer; ++i) {
            const long long s = s0 + i;
            const int bin = (int)(keys[i] >> 20);
            if (s < nvis && (all || bin > tbin)) {
                if (od < 4096) defs[od] = (int32_t)s;
                ++od;
            }
            if (s < nvis && !all && bin == tbin) {
                if (oc < kCandCap) {
                    cidx[oc] = (int32_t)s;
                    ckey[oc] = keys[i];
                }
                ++oc;
            }
        }
        n_def += tot & 0xffff;
        n_cand += tot >> 16;
    }
    __syncthreads();
    if (n_cand > kCandCap || n_def > 4096) {
        select_row_radix(sc, nvis, k, io, so);
        return;
    }
    finish_lists(sc, k, n_def, n_cand, defs, cidx, ckey, sels, io, so);
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
        const cudaError_t le = launch_pdl(kern, grid, dim3(kScoreThreads), smem, stream, a, scores);
        if (le != cudaSuccess) return le;
        break;
    }
    case V4A_BF16: {
        auto kern = index_score_kernel<HMAX, V4A_BF16>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        const cudaError_t le = launch_pdl(kern, grid, dim3(kScoreThreads), smem, stream, a, scores);
        if (le != cudaSuccess) return le;
        break;
    }
    case V4A_MXFP4: {
        auto kern = index_score_kernel<HMAX, V4A_MXFP4>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        const cudaError_t le = launch_pdl(kern, grid, dim3(kScoreThreads), smem, stream, a, scores);
        if (le != cudaSuccess) return le;
        break;
    }
    default: {
        auto kern = index_score_kernel<HMAX, V4A_FP8E4M3>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        const cudaError_t le = launch_pdl(kern, grid, dim3(kScoreThreads), smem, stream, a, scores);
        if (le != cudaSuccess) return le;
        break;
    }
    }
    return cudaGetLastError();
}


// How the select is done for a shape: few query rows take the histogram /
// multi-block scan / final path; many rows take one radix-select block per row.
struct TopkPlan {
    bool fast;
    int parts;
    long long chunk;
    size_t off_hist, off_def, off_cidx, off_ckey, total;
};

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

static TopkPlan topk_plan(const IndexArgs& a, int k) {
    TopkPlan p = {};
    const long long rows = (long long)a.batch * a.n_q;
    const long long n = a.n_ent > 0 ? a.n_ent : 1;
    size_t off = align256((size_t)rows * n * sizeof(float));  // scores
    p.fast = rows >= 1 && rows <= kMaxFastRows;
    if (!p.fast) {
        p.total = off;
        return p;
    }
    if (k < 1) k = 1;
    // parts of kFastStep scores (more per part only if a row would need more than kMaxFastParts)
    long long parts = (n + kFastStep - 1) / kFastStep;
    if (parts > kMaxFastParts) parts = kMaxFastParts;
    if (parts < 1) parts = 1;
    p.parts = (int)parts;
    p.chunk = ((n + parts - 1) / parts + kFastStep - 1) / kFastStep * kFastStep;
    // histograms, then per row a 64-bit list counter and a finished-parts counter: zeroed together
    p.off_hist = off;
    off = align256(off + (size_t)rows * (kHistBins * sizeof(uint32_t) + 2 * sizeof(unsigned long long)));
    p.off_def = off;
    off = align256(off + (size_t)rows * k * sizeof(int32_t));
    p.off_cidx = off;
    off = align256(off + (size_t)rows * kSelCap * sizeof(int32_t));
    p.off_ckey = off;
    off = align256(off + (size_t)rows * kSelCap * sizeof(uint32_t));
    p.total = off;
    return p;
}

// histogram of the order-preserving keys' top 12 bits, for the CUDA-core score path
__global__ void score_hist_kernel(const float* scores, IndexArgs a, uint32_t* hist) {
    griddep_wait();  // everything before this kernel on the stream has finished
    griddep_launch_dependents();
    const int row = blockIdx.y;
    const long long nvis = row_nvis(a, row);
    for (long long s = (long long)blockIdx.x * blockDim.x + threadIdx.x; s < nvis; s += (long long)gridDim.x * blockDim.x)
        atomicAdd(&hist[(long long)row * kHistBins + (float_to_ordered(scores[(long long)row * a.n_ent + s]) >> 20)], 1u);
}

}  // namespace

cudaError_t launch_index_scores(const IndexArgs& a, float* scores, cudaStream_t stream) {
    if (a.batch == 0 || a.n_ent == 0) return cudaSuccess;
    if (index_tc_available(a)) return launch_index_scores_tc(a, scores, nullptr, a.dev_status, stream);
    if (a.heads_i <= 4) return launch_scores_h<4>(a, scores, stream);
    if (a.heads_i <= 8) return launch_scores_h<8>(a, scores, stream);
    if (a.heads_i <= 16) return launch_scores_h<16>(a, scores, stream);
    if (a.heads_i <= 32) return launch_scores_h<32>(a, scores, stream);
    return launch_scores_h<64>(a, scores, stream);
}

size_t topk_workspace_bytes(const IndexArgs& a, int k) { return topk_plan(a, k).total; }

cudaError_t launch_topk(const IndexArgs& a, int k, int32_t* idx_out, float* score_out, void* ws, size_t ws_bytes,
                        cudaStream_t stream) {
    if (a.batch == 0) return cudaSuccess;
    const TopkPlan p = topk_plan(a, k);
    if (ws_bytes < p.total) return cudaErrorInvalidValue;
    char* base = static_cast<char*>(ws);
    float* scores = reinterpret_cast<float*>(base);
    const int rows = a.batch * a.n_q;
    cudaError_t e;
    if (!p.fast || a.n_ent == 0) {
        if (a.n_ent > 0) {
            e = launch_index_scores(a, scores, stream);
            if (e != cudaSuccess) return e;
        }
        e = cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFastSmem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(topk_rows_kernel, dim3(rows), dim3(kFastThreads), kFastSmem, stream, (const float*)scores, a, k,
                       idx_out, score_out);
        return e != cudaSuccess ? e : cudaGetLastError();
    }
    uint32_t* hist = reinterpret_cast<uint32_t*>(base + p.off_hist);
    unsigned long long* ctr = reinterpret_cast<unsigned long long*>(hist + (size_t)rows * kHistBins);
    int32_t* def_buf = reinterpret_cast<int32_t*>(base + p.off_def);
    int32_t* cidx = reinterpret_cast<int32_t*>(base + p.off_cidx);
    uint32_t* ckey = reinterpret_cast<uint32_t*>(base + p.off_ckey);
    e = launch_zero_words(hist, (long long)rows * (kHistBins + 4), stream);
    if (e != cudaSuccess) return e;
    if (index_tc_available(a)) {
        e = launch_index_scores_tc(a, scores, hist, a.dev_status, stream);
    } else {
        e = launch_index_scores(a, scores, stream);
        if (e == cudaSuccess) {
            e = launch_pdl(score_hist_kernel, dim3(64, rows), dim3(256), 0, stream, (const float*)scores, a, hist);
            if (e == cudaSuccess) e = cudaGetLastError();
        }
    }
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(topk_fast_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSelSmem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(topk_fast_kernel, dim3(rows * p.parts), dim3(kFastThreads), kSelSmem, stream, (const float*)scores,
                   (const uint32_t*)hist, a, k, p.parts, p.chunk, def_buf, cidx, ckey, ctr, idx_out, score_out);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace v4a
