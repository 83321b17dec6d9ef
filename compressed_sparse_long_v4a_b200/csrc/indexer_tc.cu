// indexer_tc.cu -- tensor-core Lightning-Indexer scores for d_I = 128 keys
// (bf16, FP8 e4m3 with one fp32 scale per entry, or MXFP4) and up to 32 heads.
//
// I(t,s) = scale_s * sum_j w_j * ReLU(q_j . k_s)   ("How V4 makes a
// million-token context actually affordable", Lightning-Indexer section).
//
// Per tile of 256 entries of one query row, D[256 entries x N] = K B^T on
// tcgen05 (two M=128 halves, K=128), then the epilogue (one thread per pair
// of entries r, r+128; TMEM lane = r) forms the scores, writes them as fp32
// and counts them in a 4096-bin histogram of the order-preserving key's top
// 12 bits (the select step starts from that histogram).  Tiles of 256
// entries make 32 KB FP8 stages: a 128 KB ring of such stages streams HBM
// at about 7 TB/s on B200, while 16 KB stages stay near 5.5 TB/s.
//  * bf16 keys: kind::f16, B = q (N = heads, bf16), 8 MMAs of K=16.
//  * FP8 keys: kind::f8f6f4 straight from the TMA tile, 4 MMAs of K=32.  B
//    holds q split exactly into e4m3 pieces, four columns per head: with q
//    scaled per head by 2^s so that its largest magnitude lies in [128, 256),
//    an element x with |x| >= 1/4 is hi + lo (hi = nearest e4m3 of x, lo =
//    x - hi, both exact in e4m3), and a smaller one is (hi' + lo') * 2^-10
//    from x * 2^10 the same way (exact down to 2^-20 of the head's maximum).
//    q_j . k = (D_hi + D_lo) + (D_hi' + D_lo') * 2^-10, times 2^-s (folded
//    into the head weight).  These MMAs accumulate in f32 at least as
//    precisely as a sequential f32 sum (measured on B200), so the score keeps
//    f32 accuracy without widening the keys.
// Several queries of one sequence (prefill) are scored together: the B operand
// then holds G queries' heads (N = G x heads for bf16 keys, G x 4 x heads for
// FP8), so every key tile is read once per G queries and each MMA does G
// times the work.
//  * MXFP4 keys (and the query quantised to MXFP4 per head): see the section
//    "MXFP4 keys and queries" below.
// Warp 0 loads key tiles into a shared-memory ring (4 x 32 KB for FP8, 2 x 64
// KB for bf16), warp 1 (all lanes, one elected lane issuing) issues the MMAs, warps 2-5 stage each row's B
// operand, warps 6-13 run the epilogue: two warps per TMEM sub-partition, one
// per half of the tile, so each scheduler has two to switch between while one
// waits on tensor memory.  Per-entry scales are fetched 8 tiles ahead (HBM
// latency under load spans several tiles).  CTAs take contiguous ranges of the
// flat (query row, tile) sequence; a run of one row's tiles inside a CTA's
// range is a segment, with its own B buffer and histogram (both
// double-buffered).  Every wait is bounded.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace v4a {
namespace {

constexpr int kDI = 128;                 // indexer dim handled here
constexpr int kTileK = 256;              // entries per tile (two M=128 halves)
constexpr int kHalf = 128;
constexpr int kRingBytes = 131072;       // key-tile ring
constexpr int kMaxStages = 8;
constexpr int kThreads = 448;              // producer, MMA, 4 staging / converter warps, 8 epilogue warps
constexpr int kEpiFirst = 192;             // first epilogue thread (warp 6)
constexpr int kEpiThreads = 256;           // warps 6-9 score half 0 of a tile, warps 10-13 half 1
constexpr int kXAhead = 8;                 // tiles of per-entry scale words each epilogue thread fetches ahead
constexpr int kXSlots = kXAhead + 1;
constexpr int kHistBins = 4096;          // top 12 bits of the ordered score key
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxDStages = 4;
constexpr int kQBufBytes = 16384;        // B operand of one segment: up to 128 rows of 128 B
constexpr int kMinEpb = 32;                // paged keys on this path: blocks of at least 32 entries
constexpr int kMxXAhead = 3;               // MXFP4: 512-entry tiles of block exponents each staging thread fetches ahead
constexpr int kMxXSlots = kMxXAhead + 1;

template <bool FP8> struct Ring {
    static constexpr int kStageBytes = FP8 ? kTileK * kDI : kTileK * kDI * 2;
    static constexpr int kStages = kRingBytes / kStageBytes;
};
// accumulators: N columns per half (4 pieces per head for FP8, for each of G queries), two halves
// per tile
template <bool FP8, int NP, int G> struct Acc {
    static constexpr int kNq = FP8 ? 4 * NP : NP;  // columns of one query
    static constexpr int kN = kNq * G;
    static constexpr uint32_t kCols = 2 * kN;                                          // per tile
    static constexpr int kStages = (int)(kTmemCols / kCols) < kMaxDStages ? (int)(kTmemCols / kCols) : kMaxDStages;
    static_assert(kN <= 128 && kN * 128 * (FP8 ? 1 : 2) <= 16384, "B operand exceeds its buffer");
};

struct __align__(1024) IdxSmem {
    uint8_t ring[kRingBytes];                 // bf16: [2 slabs][128][128 B] per stage; fp8: [128][128 B]
    uint8_t q[2][kQBufBytes];                 // B operand per segment buffer
    float wq[2][128];                         // head weights of the G queries (times 2^-s for FP8)
    uint32_t hist[2][kHistBins];
    union {
        uint32_t xring[kXSlots][kEpiThreads];  // FP8: per-entry scales, per epilogue thread
        uint32_t mx_xring[kMxXSlots][16][128]; // MXFP4: block-exponent words, per staging thread
    };
    uint64_t k_full[kMaxStages], k_empty[kMaxStages], d_full[kMaxDStages], d_free[kMaxDStages], q_full[2], q_free[2],
        sf_full[2], sf_free[2], ep_sync, drain;
    int abort_flag;
    uint32_t tmem_base;
};

static_assert(sizeof(IdxSmem) + 1024 <= 232448, "shared memory beyond the 227 KB a block can have");

struct IdxTcArgs {
    const __nv_bfloat16* q;  // [rows][HI][128] bf16
    const float* w;          // [rows][HI]
    const float* kscale;     // [B][N] (FP8) or null
    const uint8_t* kexp;     // [B][N][4] MXFP4 block exponents or null
    const int32_t* bt;       // paged keys: block table [B][bt_stride], epb entries per block; null = contiguous
    int bt_stride, epb, epb_shift;  // epb = 1 << epb_shift (this path takes power-of-two blocks)
    long long n_blocks;      // blocks in the pools; an id outside [0, n_blocks) reads as zero keys
    float* scores;           // [rows][N]
    uint32_t* hist;          // [rows][4096]
    int* err;                // device fault word (may be null)
    long long n_ent, ctx_len, total_tiles;
    int rows, n_q, m, heads_i, tiles_per_row, grid;
    int ngroups;  // query groups per sequence: ceil(n_q / G)
};

__device__ __forceinline__ void idx_fault(IdxSmem& sm, const IdxTcArgs& a) {
    sm.abort_flag = 1;
    if (a.err) atomicExch(a.err, (int)V4A_ERR_DEVICE_FAULT);
}
__device__ __forceinline__ bool aborted(IdxSmem& sm) { return *reinterpret_cast<volatile int*>(&sm.abort_flag) != 0; }

// bounded wait taken by a whole warp: true only if every lane saw the phase complete
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
    return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity));
}
__device__ __forceinline__ bool warp_aborted(const IdxSmem& sm) {
    return __any_sync(0xffffffffu, *reinterpret_cast<const volatile int*>(&sm.abort_flag) != 0);
}

__device__ __forceinline__ long long irange(int c, const IdxTcArgs& a) { return (long long)c * a.total_tiles / a.grid; }

// walks (query group, tile) in flat order: group `grp` = queries q0 .. q0 + G - 1 of sequence bat
struct ICursor {
    int grp, ti, q0, bat, G;
    __device__ ICursor(long long f, const IdxTcArgs& a, int g) : G(g) {
        grp = (int)(f / a.tiles_per_row);
        ti = (int)(f - (long long)grp * a.tiles_per_row);
        bat = grp / a.ngroups;
        q0 = (grp - bat * a.ngroups) * G;
    }
    __device__ __forceinline__ void next(const IdxTcArgs& a) {
        if (++ti == a.tiles_per_row) {
            ti = 0;
            ++grp;
            q0 += G;
            if (q0 >= a.n_q) {
                q0 = 0;
                ++bat;
            }
        }
    }
};

__device__ __forceinline__ long long nvis_of(int qj, const IdxTcArgs& a) {
    const long long t = a.ctx_len - a.n_q + qj;
    const long long nv = n_visible(t, a.m);
    return nv > a.n_ent ? a.n_ent : nv;
}

// pool row of entry e (< n_ent) of sequence bat through the block table, or -1 for a block id outside
// the pool (pool rows fit in 31 bits on this path)
__device__ __forceinline__ int paged_row(const IdxTcArgs& a, int bat, int e) {
    const int blk = a.bt[(long long)bat * a.bt_stride + (e >> a.epb_shift)];
    return (blk >= 0 && blk < a.n_blocks) ? (blk << a.epb_shift) + (e & (a.epb - 1)) : -1;
}
// first pool row of the block holding entries e .. e+epb-1, or -epb (a box the TMA fills with zeros)
// past the last entry or for a block id outside the pool (reported)
__device__ __forceinline__ int block_row(const IdxTcArgs& a, int bat, long long e) {
    if (e >= a.n_ent) return -a.epb;
    const int blk = a.bt[(long long)bat * a.bt_stride + (int)(e >> a.epb_shift)];
    if (blk >= 0 && blk < a.n_blocks) return blk << a.epb_shift;
    if (a.err) atomicExch(a.err, (int)V4A_ERR_DEVICE_FAULT);
    return -a.epb;
}

// the first pool rows of the nb blocks of a tile that starts at entry e0 (paged keys), loaded together so
// their latencies overlap; the producer fetches them one tile ahead
template <int kMaxB>
__device__ __forceinline__ void fetch_block_rows(const IdxTcArgs& a, int bat, long long e0, int nb, int (&rows)[kMaxB]) {
#pragma unroll
    for (int j = 0; j < kMaxB; ++j)
        if (j < nb) rows[j] = block_row(a, bat, e0 + (long long)j * a.epb);
}

// Lane 0 of warp 0, before the grid dependency wait: an L2 prefetch of this CTA's first `tiles` key
// tiles of `rows` entries (boxes of the key tensor map, `xboxes` 64-column boxes across for bf16 keys)
// and of their per-entry words (FP8 scales or MXFP4 exponents, `wbytes` bytes per entry), so that the
// first loads' DRAM and address-translation latency overlaps the previous kernel's tail.  A prefetch
// only warms L2, the point of coherence: a key the previous kernel is still writing (the newest entry)
// is read afresh by the load after the wait.  Contiguous keys only.
__device__ void prefetch_first_tiles(const IdxTcArgs& a, const CUtensorMap* kmap, long long f0, long long f1,
                                     int rows, int boxes, int xboxes, int tiles, const void* words, int wbytes) {
    ICursor cur(f0, a, 1);
    for (int j = 0; j < tiles && f0 + j < f1; ++j, cur.next(a)) {
        const long long e0 = (long long)cur.ti * rows;
        const int y = (int)((long long)cur.bat * a.n_ent + e0);
        for (int bx = 0; bx < boxes; ++bx)
            for (int x = 0; x < xboxes; ++x) tc::tma_prefetch_2d(kmap, 64 * x, y + bx * (rows / boxes));
        if (words && (reinterpret_cast<uintptr_t>(words) & 15) == 0) {
            // the tile's words, trimmed to 16-byte boundaries (the bulk prefetch's alignment rule); the base
            // being 16-byte aligned keeps the trimmed range inside the array
            long long ne = a.n_ent - e0;
            if (ne > rows) ne = rows;
            const uintptr_t lo = reinterpret_cast<uintptr_t>(words) + ((long long)cur.bat * a.n_ent + e0) * wbytes;
            const uintptr_t b0 = (lo + 15) & ~(uintptr_t)15, b1 = (lo + ne * wbytes) & ~(uintptr_t)15;
            if (b1 > b0) tc::prefetch_l2(reinterpret_cast<const void*>(b0), (uint32_t)(b1 - b0));
        }
    }
}

template <bool FP8, int G>
__device__ void idx_producer(IdxSmem& sm, const IdxTcArgs& a, const CUtensorMap* kmap, long long f0, long long f1) {
    constexpr int kSt = Ring<FP8>::kStages, kBytes = Ring<FP8>::kStageBytes;
    constexpr int kMaxB = kTileK / kMinEpb;  // blocks per tile at the smallest block
    ICursor cur(f0, a, G);
    const long long n = f1 - f0;
    const int nb = a.bt ? kTileK / a.epb : 0;
    int rows[kMaxB], next_rows[kMaxB];
    // key tiles: read once per call unless several query groups of a sequence share them
    const uint64_t pol = tc::l2_stream_policy(a.ngroups);
    if (a.bt && n > 0) fetch_block_rows<kMaxB>(a, cur.bat, (long long)cur.ti * kTileK, nb, next_rows);
    for (long long jt = 0; jt < n; ++jt, cur.next(a)) {
        if (a.bt) {
#pragma unroll
            for (int j = 0; j < kMaxB; ++j) rows[j] = next_rows[j];
            if (jt + 1 < n) {  // the next tile's block rows, a tile ahead
                ICursor nx = cur;
                nx.next(a);
                fetch_block_rows<kMaxB>(a, nx.bat, (long long)nx.ti * kTileK, nb, next_rows);
            }
        }
        if (aborted(sm)) break;
        const int st = (int)(jt % kSt);
        if (jt >= kSt && !tc::mbar_wait(&sm.k_empty[st], (uint32_t)((jt / kSt) - 1) & 1)) { idx_fault(sm, a); break; }
        const int y = (int)((long long)cur.bat * a.n_ent + (long long)cur.ti * kTileK);
        uint8_t* dst = sm.ring + st * kBytes;
        tc::mbar_arrive_expect_tx(&sm.k_full[st], kBytes);
        if (a.bt) {
            // paged keys: one box of epb rows per block of the tile
#pragma unroll
            for (int j = 0; j < kMaxB; ++j) {
                if (j >= nb) break;
                tc::tma_load_2d_hint(dst + j * a.epb * 128, kmap, 0, rows[j], &sm.k_full[st], pol);
                if (!FP8) tc::tma_load_2d_hint(dst + kTileK * 128 + j * a.epb * 128, kmap, 64, rows[j], &sm.k_full[st], pol);
            }
        } else {
            tc::tma_load_2d_hint(dst, kmap, 0, y, &sm.k_full[st], pol);
            if (!FP8) tc::tma_load_2d_hint(dst + kTileK * 128, kmap, 64, y, &sm.k_full[st], pol);  // second 64-column slab
        }
    }
    // no copy may still be in flight when the CTA exits
    for (long long jt = n - kSt; jt < n; ++jt)
        if (jt >= 0) tc::mbar_wait(&sm.k_full[jt % kSt], (uint32_t)(jt / kSt) & 1);
}

template <bool FP8, int NP, int G>
__device__ void idx_mma(IdxSmem& sm, const IdxTcArgs& a, uint32_t tmem, long long f0, long long f1) {
    constexpr int kSt = Ring<FP8>::kStages, kBytes = Ring<FP8>::kStageBytes;
    constexpr int kDS = Acc<FP8, NP, G>::kStages, kN = Acc<FP8, NP, G>::kN;
    constexpr uint32_t kQSlab = kN * 128;  // bf16: bytes per K-slab of q
    constexpr uint32_t idesc = FP8 ? tc::idesc_e4m3(128, kN) : tc::idesc_f16(128, kN, 0, 0, 1);
    bool ok = true;
    int seg = 0, b = 0;
    uint64_t qd = 0;
    ICursor cur(f0, a, G);
    for (long long f = f0; f < f1; ++f, cur.next(a)) {
        if (warp_aborted(sm)) { ok = false; break; }
        const int jt = (int)(f - f0), st = jt % kSt, sd = jt % kDS;
        if (f == f0 || cur.ti == 0) {
            b = seg & 1;
            if (!warp_wait(&sm.q_full[b], (seg >> 1) & 1)) { ok = false; break; }
            qd = tc::sw128_desc(tc::smem_u32(sm.q[b]), 16, 1024);
            ++seg;
        }
        const bool seg_end = (f == f1 - 1) || (cur.ti == a.tiles_per_row - 1);
        if (!warp_wait(&sm.k_full[st], (jt / kSt) & 1)) { ok = false; break; }
        if (jt >= kDS && !warp_wait(&sm.d_free[sd], ((jt / kDS) - 1) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t stage = tc::smem_u32(sm.ring + st * kBytes);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const uint32_t d = tmem + Acc<FP8, NP, G>::kCols * sd + kN * hf;
            // rows 128 hf .. 128 hf + 127 of every 128-byte slab of the tile
            const uint64_t kd = tc::sw128_desc(stage + hf * kHalf * 128, 16, 1024);
            if (FP8) {
                // K = 32 e4m3 per MMA: 32 bytes along the 128-byte rows of both operands
#pragma unroll
                for (int kk = 0; kk < kDI / 32; ++kk)
                    tc::mma_f8f6f4(d, kd + (uint64_t)((kk * 32) >> 4), qd + (uint64_t)((kk * 32) >> 4), idesc,
                                   kk ? 1u : 0u);
            } else {
#pragma unroll
                for (int kk = 0; kk < kDI / 16; ++kk) {
                    const uint64_t ad = kd + ((((kk >> 2) * (kTileK * 128)) + (kk & 3) * 32) >> 4);
                    const uint64_t bd = qd + ((((kk >> 2) * kQSlab) + (kk & 3) * 32) >> 4);
                    tc::mma_f16(d, ad, bd, idesc, kk ? 1u : 0u);
                }
            }
        }
        tc::mma_commit(&sm.k_empty[st]);
        tc::mma_commit(&sm.d_full[sd]);
        if (seg_end) tc::mma_commit(&sm.q_free[b]);
    }
    if (!ok) idx_fault(sm, a);
    tc::mma_commit(&sm.drain);
    tc::mbar_wait(&sm.drain, 0);
}

__device__ __forceinline__ uint32_t e4m3_rn(float x) {
    return (uint32_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float e4m3_value(uint32_t c) {
    return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3)));
}

// B operand of one query group into buffer b (K-major, 128-byte swizzle, 128-byte rows) and the
// head weights; ct = 0..127.  Virtual head vh = g NP + h is head h of query q0 + g (zero past the
// last query or head).  bf16 keys: q itself (two K-slabs of G NP rows).  FP8 keys: rows
// g 4 NP + p NP + h hold piece p of that head (p = hi, lo, hi', lo'), one e4m3 per element.
template <bool FP8, int NP, int G>
__device__ void stage_query(IdxSmem& sm, const IdxTcArgs& a, int bat, int q0, int b, int ct) {
    constexpr int kN = Acc<FP8, NP, G>::kN;
    // warp w handles virtual heads w, w+4, ...; lane owns 4 of the 128 elements
    const int warp = ct >> 5, lane = ct & 31;
    const int k = lane * 4;
    for (int vh = warp; vh < G * NP; vh += 4) {
        const int g = vh / NP, h = vh - g * NP, qj = q0 + g;
        const bool live = qj < a.n_q && h < a.heads_i;
        const long long row = (long long)bat * a.n_q + qj;
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        if (live) {
            const __nv_bfloat16* qp = a.q + (row * a.heads_i + h) * kDI + k;
            const uint2 raw = *reinterpret_cast<const uint2*>(qp);
            v[0] = __uint_as_float(raw.x << 16);
            v[1] = __uint_as_float(raw.x & 0xffff0000u);
            v[2] = __uint_as_float(raw.y << 16);
            v[3] = __uint_as_float(raw.y & 0xffff0000u);
        }
        float wq = live ? a.w[row * a.heads_i + h] : 0.f;
        if (FP8) {
            float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            int e = 0;
            if (amax > 0.f) frexpf(amax, &e);       // amax = f * 2^e, f in [0.5, 1)
            const int sh = amax > 0.f ? 8 - e : 0;  // amax * 2^sh in [128, 256)
            wq = ldexpf(wq, -sh);
            uint32_t pc[4] = {0u, 0u, 0u, 0u};      // pieces hi, lo, hi', lo': 4 codes each
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float x = ldexpf(v[i], sh);
                const bool big = fabsf(x) >= 0.25f;
                const float y = big ? x : x * 1024.0f;
                const uint32_t hi = e4m3_rn(y);
                const uint32_t lo = e4m3_rn(y - e4m3_value(hi));
                pc[big ? 0 : 2] |= hi << (8 * i);
                pc[big ? 1 : 3] |= lo << (8 * i);
            }
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const int n = g * 4 * NP + p * NP + h;
                uint8_t* dst = sm.q[b] + (n >> 3) * 1024 + (n & 7) * 128 + ((((k >> 4) ^ (n & 7))) << 4) + (k & 15);
                *reinterpret_cast<uint32_t*>(dst) = pc[p];
            }
        } else {
            __nv_bfloat162 b0 = __floats2bfloat162_rn(v[0], v[1]), b1 = __floats2bfloat162_rn(v[2], v[3]);
            // element k of virtual head vh: K-slab k/64, 16-byte chunk (k%64)/8, 8-byte half
            uint8_t* slab = sm.q[b] + (k >> 6) * (kN * 128);
            uint8_t* dst = slab + (vh >> 3) * 1024 + (vh & 7) * 128 + ((((k & 63) >> 3) ^ (vh & 7)) << 4) + ((k & 7) ? 8 : 0);
            *reinterpret_cast<uint2*>(dst) =
                make_uint2(*reinterpret_cast<uint32_t*>(&b0), *reinterpret_cast<uint32_t*>(&b1));
        }
        if (lane == 0) sm.wq[b][vh] = wq;
    }
}

// warps 2-5: per segment, stage the query group's B operand
template <bool FP8, int NP, int G>
__device__ void idx_stage(IdxSmem& sm, const IdxTcArgs& a, long long f0, long long f1) {
    const int ct = threadIdx.x - 64;
    bool ok = true;
    int seg = 0;
    ICursor cur(f0, a, G);
    for (long long f = f0; f < f1; ++f, cur.next(a)) {
        if (f != f0 && cur.ti != 0) continue;
        if (warp_aborted(sm)) { ok = false; break; }
        const int b = seg & 1;
        if (seg >= 2 && !warp_wait(&sm.q_free[b], ((seg >> 1) - 1) & 1)) { ok = false; break; }
        stage_query<FP8, NP, G>(sm, a, cur.bat, cur.q0, b, ct);
        tc::fence_proxy_async();
        tc::mbar_arrive(&sm.q_full[b]);
        ++seg;
    }
    if (!ok) idx_fault(sm, a);
}

// q_j . k of the 128 entries' row of D (this thread's TMEM lane), for every head
template <bool FP8, int NP>
__device__ __forceinline__ float score_of(uint32_t taddr, const float* wq) {
    float acc = 0.f;
    if (!FP8) {
        uint32_t dv[NP];
        if constexpr (NP == 16) tc::tmem_ld_x16(taddr, dv);
        else tc::tmem_ld_x32(taddr, dv);
        tc::tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < NP; ++h) acc = fmaf(wq[h], fmaxf(__uint_as_float(dv[h]), 0.f), acc);
    } else if (NP == 16) {
        uint32_t r[64];  // columns: hi | lo | hi' | lo', 16 heads each
        tc::tmem_ld_x64(taddr, r);
        tc::tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            const float d1 = __uint_as_float(r[h]) + __uint_as_float(r[16 + h]);
            const float d2 = __uint_as_float(r[32 + h]) + __uint_as_float(r[48 + h]);
            acc = fmaf(wq[h], fmaxf(fmaf(d2, 0x1p-10f, d1), 0.f), acc);
        }
    } else {
        // 16 heads at a time: pieces hi | lo | hi' | lo' of heads 16 hg .. 16 hg + 15
#pragma unroll
        for (int hg = 0; hg < 2; ++hg) {
            uint32_t p4[4][16];
#pragma unroll
            for (int p = 0; p < 4; ++p) tc::tmem_ld_x16(taddr + 32 * p + 16 * hg, p4[p]);
            tc::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float d1 = __uint_as_float(p4[0][i]) + __uint_as_float(p4[1][i]);
                const float d2 = __uint_as_float(p4[2][i]) + __uint_as_float(p4[3][i]);
                acc = fmaf(wq[16 * hg + i], fmaxf(fmaf(d2, 0x1p-10f, d1), 0.f), acc);
            }
        }
    }
    return acc;
}

// This epilogue thread's per-entry scale word (FP8 scale, MXFP4 exponents) for every tile of its
// range, fetched kXAhead tiles ahead with 4-byte cp.async into a ring of shared memory only this
// thread touches: HBM latency under load (2-4 us) is several tiles long, so a load issued one tile
// ahead would stall the epilogue.  One commit group per tile, so wait_group<kXAhead> leaves the
// current tile's word landed.
struct XPrefetch {
    ICursor cur;
    long long f, f0, f1;
    const uint32_t* src;  // [B][N] words
    int et, hf, r;
    __device__ XPrefetch(long long f0_, long long f1_, const IdxTcArgs& a, int G, const uint32_t* src_, int et_,
                         int hf_, int r_)
        : cur(f0_, a, G), f(f0_), f0(f0_), f1(f1_), src(src_), et(et_), hf(hf_), r(r_) {}
    __device__ __forceinline__ void issue(IdxSmem& sm, const IdxTcArgs& a) {
        if (f < f1) {
            const long long e = (long long)cur.ti * kTileK + kHalf * hf + r;
            if (e < a.n_ent) {
                const long long kr = a.bt ? (long long)paged_row(a, cur.bat, (int)e) : (long long)cur.bat * a.n_ent + e;
                if (kr >= 0) tc::cp_async_4(&sm.xring[(int)((f - f0) % kXSlots)][et], src + kr);
            }
            cur.next(a);
            ++f;
        }
        tc::cp_async_commit();
    }
    __device__ __forceinline__ void start(IdxSmem& sm, const IdxTcArgs& a) {
        for (int i = 0; i < kXAhead; ++i) issue(sm, a);
    }
    // the word of tile jt (local index), once its copy has landed; issues the copy kXAhead tiles on
    __device__ __forceinline__ uint32_t take(IdxSmem& sm, const IdxTcArgs& a, int jt) {
        issue(sm, a);
        tc::cp_async_wait<kXAhead>();
        return sm.xring[jt % kXSlots][et];
    }
};

// warps 6-13: per tile the scores of entry 128 hf + r (r = this thread's TMEM lane, hf = which four
// warps) for each query of the group, their histogram counts (single queries only) and stores
template <bool FP8, int NP, int G>
__device__ void idx_epilogue(IdxSmem& sm, const IdxTcArgs& a, uint32_t tmem, long long f0, long long f1) {
    constexpr int kDS = Acc<FP8, NP, G>::kStages, kN = Acc<FP8, NP, G>::kN, kNq = Acc<FP8, NP, G>::kNq;
    const int et = threadIdx.x - kEpiFirst;
    const int hf = et >> 7;
    const int sub = (threadIdx.x >> 5) & 3;
    const int r = 32 * sub + (threadIdx.x & 31);
    const uint32_t lane_addr = (uint32_t)(32 * sub) << 16;
    bool ok = true;
    int seg = 0, b = 0, nsync = 0;
    int nv[G];            // visible entries of each query of the group (0 past the last query)
    float* srow0 = nullptr;  // the group's first score row; query g's is g rows further
#pragma unroll
    for (int g = 0; g < G; ++g) nv[g] = 0;
    ICursor cur(f0, a, G);
    XPrefetch xp(f0, f1, a, G, reinterpret_cast<const uint32_t*>(a.kscale), et, hf, r);
    if (FP8) xp.start(sm, a);
    for (long long f = f0; f < f1; ++f) {
        if (warp_aborted(sm)) { ok = false; break; }
        const int jt = (int)(f - f0), sd = jt % kDS;
        if (f == f0 || cur.ti == 0) {
            b = seg & 1;
            if (!warp_wait(&sm.q_full[b], (seg >> 1) & 1)) { ok = false; break; }
            ++seg;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const int qj = cur.q0 + g;
                nv[g] = qj < a.n_q ? (int)nvis_of(qj, a) : 0;
            }
            srow0 = a.scores + ((long long)cur.bat * a.n_q + cur.q0) * a.n_ent;
        }
        const bool seg_end = (f == f1 - 1) || (cur.ti == a.tiles_per_row - 1);
        const int ti = cur.ti, q0t = cur.q0, row = cur.bat * a.n_q + cur.q0;  // row: the group's first query
        cur.next(a);
        if (!warp_wait(&sm.d_full[sd], (jt / kDS) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        float acc[G];
#pragma unroll
        for (int g = 0; g < G; ++g)
            acc[g] = score_of<FP8, NP>(tmem + lane_addr + Acc<FP8, NP, G>::kCols * sd + kN * hf + kNq * g,
                                       sm.wq[b] + NP * g);
        tc::tc_fence_before();
        tc::mbar_arrive(&sm.d_free[sd]);
        const float sc_e = FP8 ? __uint_as_float(xp.take(sm, a, jt)) : 1.f;
        const long long e = (long long)ti * kTileK + kHalf * hf + r;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            if (q0t + g >= a.n_q || e >= a.n_ent) continue;  // past the last query of the sequence / entry
            float sc = -INFINITY;
            if (e < nv[g]) {
                float v = acc[g];
                if (FP8) v *= sc_e;
                sc = v + 0.0f;
                if (G == 1 && a.hist) atomicAdd(&sm.hist[b][float_to_ordered(sc) >> 20], 1u);
            }
            srow0[(long long)g * a.n_ent + e] = sc;
        }
        if (seg_end) {
            tc::mbar_arrive(&sm.q_free[b]);  // done with wq[b]
            if (G == 1 && a.hist) {
                // every epilogue thread has counted this segment's scores (bounded, unlike a named barrier)
                tc::mbar_arrive(&sm.ep_sync);
                if (!warp_wait(&sm.ep_sync, nsync++ & 1)) { ok = false; break; }
                uint32_t* gh = a.hist + (long long)row * kHistBins;
                for (int i = et; i < kHistBins; i += kEpiThreads) {
                    const uint32_t v = sm.hist[b][i];
                    if (v) {
                        atomicAdd(gh + i, v);
                        sm.hist[b][i] = 0;
                    }
                }
            }
        }
    }
    tc::cp_async_wait<0>();  // no copy into shared memory may be in flight at exit
    if (!ok) idx_fault(sm, a);
}

template <bool FP8, int NP, int G>
__global__ void __launch_bounds__(kThreads, 1) index_score_tc_kernel(const __grid_constant__ CUtensorMap kmap, IdxTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    IdxSmem& sm = *reinterpret_cast<IdxSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long f0 = irange(blockIdx.x, a), f1 = irange(blockIdx.x + 1, a);
    if (threadIdx.x == 0) {
        for (int i = 0; i < Ring<FP8>::kStages; ++i) {
            tc::mbar_init(&sm.k_full[i], 1);
            tc::mbar_init(&sm.k_empty[i], 1);
        }
        for (int i = 0; i < Acc<FP8, NP, G>::kStages; ++i) {
            tc::mbar_init(&sm.d_full[i], 1);
            tc::mbar_init(&sm.d_free[i], kEpiThreads);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&sm.q_full[i], 128);
            tc::mbar_init(&sm.q_free[i], 1 + kEpiThreads);  // the MMAs' commit + every epilogue thread
        }
        tc::mbar_init(&sm.ep_sync, kEpiThreads);
        tc::mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        tc::fence_barrier_init();
    }
    for (int i = threadIdx.x; i < 2 * kHistBins; i += kThreads) (&sm.hist[0][0])[i] = 0;
    if (FP8)  // rows of the B buffers past 4 NP are never read, but keep them defined
        for (int i = threadIdx.x; i < 2 * kQBufBytes / 4; i += kThreads) reinterpret_cast<uint32_t*>(sm.q)[i] = 0;
    if (warp == 1) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (threadIdx.x == 0 && !a.bt && G == 1)
        prefetch_first_tiles(a, &kmap, f0, f1, kTileK, 1, FP8 ? 1 : 2, Ring<FP8>::kStages + 2, a.kscale, 4);
    griddep_wait();  // the prologue above touched only shared and tensor memory (and prefetched into L2)
    griddep_launch_dependents();
    const uint32_t tmem = sm.tmem_base;
    if (warp == 0) {
        if (lane == 0) idx_producer<FP8, G>(sm, a, &kmap, f0, f1);
    } else if (warp == 1) {
        idx_mma<FP8, NP, G>(sm, a, tmem, f0, f1);  // the whole warp (one elected lane issues)
    } else if (warp < 6) {
        idx_stage<FP8, NP, G>(sm, a, f0, f1);
    } else {
        idx_epilogue<FP8, NP, G>(sm, a, tmem, f0, f1);
    }
    __syncwarp();
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------
// MXFP4 keys and queries: FP4 dot products on the block-scaled tensor cores
// ---------------------------------------------------------------------
// Key rows are 64 bytes of packed e2m1 codes; their 4 E8M0 block exponents
// live in a separate array, one 32-bit word per entry whose byte j scales
// elements 32j .. 32j+31.  A tile is 512 entries: two TMA boxes of 256 rows
// (64-byte swizzle) fill one 32 KB stage, and the stage IS the MMA's A
// operand: tcgen05 kind::mxf4 (block32) reads packed e2m1 from shared memory
// and applies one E8M0 scale per 32 K-elements from tensor memory, so a tile
// is 8 MMAs (4 quarters of 128 rows x K = 2 x 64) with f32 accumulation, and
// one set of waits and commits.  The scale words need no repacking: row m of
// a 128-row quarter reads the word at lane m % 32 (of every sub-partition),
// column m / 32, bytes 0-1 for K 0..63 and bytes 2-3 for K 64..127.  Warps
// 2-5 (one per sub-partition) write each tile's words there with
// tcgen05.st, from a ring of 4-byte cp.async copies fetched kMxXAhead tiles
// ahead; per query they also quantise q to MXFP4 (the B operand, same
// layout) and write its scale words.  The epilogue is the bf16-key one: each
// accumulator column is already q_h . k_s with both block scales applied.

constexpr int kMxTile = 512;                              // entries per tile
constexpr int kMxQuarterBytes = kHalf * 64;               // 128 rows of packed codes
constexpr int kMxStageBytes = kMxTile * 64;               // one tile per 32 KB stage
constexpr int kMxStages = kRingBytes / kMxStageBytes;     // 4
constexpr uint32_t kMxSfaCol = 256;                       // two A-scale slots of 16 columns
constexpr uint32_t kMxSfbCol = 320;                       // two B-scale columns (query buffers), 16 apart
template <int NP> struct MxAcc {
    static constexpr uint32_t kCols = 4 * NP;             // per tile: 4 quarters x NP heads
    static constexpr int kStages = (int)(kMxSfaCol / kCols) < kMaxDStages ? (int)(kMxSfaCol / kCols) : kMaxDStages;
    static_assert(kStages >= 2, "accumulators");
};
static_assert(kMxStages <= kMaxStages, "ring stages");

__device__ void mx_producer(IdxSmem& sm, const IdxTcArgs& a, const CUtensorMap* kmap, long long f0, long long f1) {
    constexpr int kMaxB = kMxTile / kMinEpb;  // blocks per tile at the smallest block
    ICursor cur(f0, a, 1);
    const long long n = f1 - f0;
    const int nb = a.bt ? kMxTile / a.epb : 0;
    int rows[kMaxB], next_rows[kMaxB];
    // key tiles: read once per call unless several query groups of a sequence share them
    const uint64_t pol = tc::l2_stream_policy(a.ngroups);
    if (a.bt && n > 0) fetch_block_rows<kMaxB>(a, cur.bat, (long long)cur.ti * kMxTile, nb, next_rows);
    for (long long jt = 0; jt < n; ++jt, cur.next(a)) {
        if (a.bt) {
#pragma unroll
            for (int j = 0; j < kMaxB; ++j) rows[j] = next_rows[j];
            if (jt + 1 < n) {  // the next tile's block rows, a tile ahead
                ICursor nx = cur;
                nx.next(a);
                fetch_block_rows<kMaxB>(a, nx.bat, (long long)nx.ti * kMxTile, nb, next_rows);
            }
        }
        if (aborted(sm)) break;
        const int st = (int)(jt % kMxStages);
        if (jt >= kMxStages && !tc::mbar_wait(&sm.k_empty[st], (uint32_t)((jt / kMxStages) - 1) & 1)) {
            idx_fault(sm, a);
            break;
        }
        const int y = (int)((long long)cur.bat * a.n_ent + (long long)cur.ti * kMxTile);
        tc::mbar_arrive_expect_tx(&sm.k_full[st], (uint32_t)kMxStageBytes);
        if (a.bt) {
            // paged keys: one box of epb rows per block of the tile
#pragma unroll
            for (int j = 0; j < kMaxB; ++j) {
                if (j >= nb) break;
                tc::tma_load_2d_hint(sm.ring + st * kMxStageBytes + j * a.epb * 64, kmap, 0, rows[j], &sm.k_full[st], pol);
            }
        } else {
            // boxes of 256 rows; rows past the tensor's end are filled with zeros (and still counted)
            tc::tma_load_2d_hint(sm.ring + st * kMxStageBytes, kmap, 0, y, &sm.k_full[st], pol);
            tc::tma_load_2d_hint(sm.ring + st * kMxStageBytes + kMxStageBytes / 2, kmap, 0, y + 256, &sm.k_full[st], pol);
        }
    }
    // no copy may still be in flight when the CTA exits
    for (long long jt = n - kMxStages; jt < n; ++jt)
        if (jt >= 0) tc::mbar_wait(&sm.k_full[jt % kMxStages], (uint32_t)(jt / kMxStages) & 1);
}

template <int NP>
__device__ void mx_mma(IdxSmem& sm, const IdxTcArgs& a, uint32_t tmem, long long f0, long long f1) {
    using Acc = MxAcc<NP>;
    constexpr int kDS = Acc::kStages;
    // descriptors: the ring's first stage and both query buffers; every operand is a fixed offset
    // from one of them (start addresses count 16-byte units in the low 14 bits; no carry here)
    const uint64_t ring_desc = tc::sw64_desc(tc::smem_u32(sm.ring));
    const uint64_t q_desc0 = tc::sw64_desc(tc::smem_u32(sm.q[0])), q_desc1 = tc::sw64_desc(tc::smem_u32(sm.q[1]));
    constexpr uint32_t id0 = tc::idesc_mxf4(128, NP, 0, 0), id1 = tc::idesc_mxf4(128, NP, 2, 2);
    bool ok = true;
    int seg = 0, b = 0;
    ICursor cur(f0, a, 1);
    for (long long f = f0; f < f1; ++f, cur.next(a)) {
        if (warp_aborted(sm)) { ok = false; break; }
        const int jt = (int)(f - f0);
        const int st = jt % kMxStages, slot = jt & 1, sd = jt % kDS;
        if (f == f0 || cur.ti == 0) {
            b = seg & 1;
            if (!warp_wait(&sm.q_full[b], (seg >> 1) & 1)) { ok = false; break; }
            ++seg;
        }
        const bool seg_end = (f == f1 - 1) || (cur.ti == a.tiles_per_row - 1);
        if (!warp_wait(&sm.k_full[st], (uint32_t)(jt / kMxStages) & 1)) { ok = false; break; }
        if (!warp_wait(&sm.sf_full[slot], (uint32_t)(jt >> 1) & 1)) { ok = false; break; }
        if (jt >= kDS && !warp_wait(&sm.d_free[sd], (uint32_t)((jt / kDS) - 1) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        const uint64_t a0 = ring_desc + (uint64_t)((st * kMxStageBytes) >> 4), b0 = b ? q_desc1 : q_desc0;
        const uint32_t d0 = tmem + Acc::kCols * sd, sfa = tmem + kMxSfaCol + 16 * slot, sfb = tmem + kMxSfbCol + 16 * b;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            tc::mma_mxf4(d0 + NP * qq, a0 + (uint64_t)((qq * kMxQuarterBytes) >> 4), b0, id0, sfa + 4 * qq, sfb, 0u);
            tc::mma_mxf4(d0 + NP * qq, a0 + (uint64_t)((qq * kMxQuarterBytes + 32) >> 4), b0 + 2, id1,
                         (sfa + 4 * qq) | (2u << 30), sfb | (2u << 30), 1u);
        }
        tc::mma_commit(&sm.k_empty[st]);
        tc::mma_commit(&sm.sf_free[slot]);
        tc::mma_commit(&sm.d_full[sd]);
        if (seg_end) tc::mma_commit(&sm.q_free[b]);
    }
    if (!ok) idx_fault(sm, a);
    tc::mma_commit(&sm.drain);
    tc::mbar_wait(&sm.drain, 0);
}

// Query of one segment: its B operand (NP rows of 64 bytes of packed e2m1, 64-byte swizzle), its
// scale words in tensor memory and the head weights.  A half-warp quantises one head, lane l
// elements 8l .. 8l+7; then every lane h (< NP) of every staging warp writes head h's 4 block
// exponents to its sub-partition's copy of the B scales.
template <int NP>
__device__ void stage_query_mx(IdxSmem& sm, const IdxTcArgs& a, uint32_t tmem, int bat, int qj, int b, int ct) {
    const int warp = ct >> 5, lane = ct & 31, l = lane & 15;
    const long long row = (long long)bat * a.n_q + qj;
    for (int h = 2 * warp + (lane >> 4); h < NP; h += 8) {  // NP is a multiple of 8: whole warps iterate
        const bool live = h < a.heads_i;
        float v[8];
        if (live) {
            Vec8<__nv_bfloat16>::load_nc(a.q + (row * a.heads_i + h) * kDI + 8 * l, v);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.f;
        }
        int x;
        const uint32_t cw = mx_quantize8(v, &x);  // lanes 4k .. 4k+3 of the half-warp share block k
        const int j = 4 * l;                       // byte of the row
        *reinterpret_cast<uint32_t*>(sm.q[b] + h * 64 + ((((j >> 4) ^ ((h >> 1) & 3))) << 4) + (j & 15)) = cw;
        if (l == 0) sm.wq[b][h] = live ? a.w[row * a.heads_i + h] : 0.f;
    }
    // B scale words: lane h of this warp's sub-partition, column kMxSfbCol + 16 b
    uint32_t word = 0x7f7f7f7fu;  // 2^0 for rows past the last head (their codes are 0)
    if (lane < NP && lane < a.heads_i) {
        const __nv_bfloat16* qp = a.q + (row * a.heads_i + lane) * kDI;
        word = 0;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            float am = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v[8];
                Vec8<__nv_bfloat16>::load_nc(qp + 32 * blk + 8 * c, v);
#pragma unroll
                for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[i]));
            }
            word |= (uint32_t)(mx_block_exp(am) + 127) << (8 * blk);
        }
    }
    const int sub = (threadIdx.x >> 5) & 3;
    tc::tmem_st_x1(tmem + ((uint32_t)(32 * sub) << 16) + kMxSfbCol + 16 * b, word);
    tc::tmem_st_wait();
}

// warps 2-5: per segment the query (B operand and scales); per tile the keys' scale words (A
// scales) in tensor memory: thread (sub-partition p, lane t) writes, in its sub-partition, column
// 16 slot + 4 q + c the word of entry 128 q + 32 c + t (quarter q, c < 4)
template <int NP>
__device__ void mx_stage(IdxSmem& sm, const IdxTcArgs& a, uint32_t tmem, long long f0, long long f1) {
    const int ct = threadIdx.x - 64;
    const int lane = threadIdx.x & 31;
    const int sub = (threadIdx.x >> 5) & 3;
    const uint32_t lane_addr = (uint32_t)(32 * sub) << 16;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(a.kexp);
    bool ok = true;
    int seg = 0;
    // block-exponent words fetched kMxXAhead tiles ahead (one commit group per tile)
    ICursor pre(f0, a, 1);
    long long fp = f0;
    auto prefetch = [&]() {
        if (fp < f1) {
            const int xs = (int)((fp - f0) % kMxXSlots);
            const long long e0 = (long long)pre.ti * kMxTile + lane;
            if (!a.bt) {
                const uint32_t* sp = src + (long long)pre.bat * a.n_ent + e0;
#pragma unroll
                for (int w = 0; w < 16; ++w)  // word w: quarter w / 4, column w % 4
                    if (e0 + 32 * w < a.n_ent) tc::cp_async_4(&sm.mx_xring[xs][w][ct], sp + 32 * w);
            } else {
#pragma unroll
                for (int w = 0; w < 16; ++w) {
                    const long long e = e0 + 32 * w;
                    const int kr = e < a.n_ent ? paged_row(a, pre.bat, (int)e) : -1;
                    if (kr >= 0) tc::cp_async_4(&sm.mx_xring[xs][w][ct], src + kr);
                }
            }
            pre.next(a);
            ++fp;
        }
        tc::cp_async_commit();
    };
    for (int i = 0; i < kMxXAhead; ++i) prefetch();
    ICursor cur(f0, a, 1);
    for (long long f = f0; f < f1; ++f, cur.next(a)) {
        if (warp_aborted(sm)) { ok = false; break; }
        const int jt = (int)(f - f0);
        if (f == f0 || cur.ti == 0) {
            const int b = seg & 1;
            if (seg >= 2 && !warp_wait(&sm.q_free[b], ((seg >> 1) - 1) & 1)) { ok = false; break; }
            stage_query_mx<NP>(sm, a, tmem, cur.bat, cur.q0, b, ct);
            tc::fence_proxy_async();
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.q_full[b]);
            ++seg;
        }
        prefetch();  // tile f + kMxXAhead
        const int slot = jt & 1;
        if (jt >= 2 && !warp_wait(&sm.sf_free[slot], (uint32_t)((jt >> 1) - 1) & 1)) { ok = false; break; }
        tc::cp_async_wait<kMxXAhead>();
        const int xs = jt % kMxXSlots;
        uint32_t wv[16];
#pragma unroll
        for (int w = 0; w < 16; ++w) wv[w] = sm.mx_xring[xs][w][ct];
        tc::tc_fence_after();
        tc::tmem_st_x16(tmem + lane_addr + kMxSfaCol + 16 * slot, wv);
        tc::tmem_st_wait();
        tc::tc_fence_before();
        tc::mbar_arrive(&sm.sf_full[slot]);
    }
    tc::cp_async_wait<0>();  // no copy into shared memory may be in flight at exit
    if (!ok) idx_fault(sm, a);
}

// warps 6-13: the scores of entries 128 q + r of each tile (q = g, g + 2 for warp group g),
// histogram counts and stores
template <int NP>
__device__ void mx_epilogue(IdxSmem& sm, const IdxTcArgs& a, uint32_t tmem, long long f0, long long f1) {
    using Acc = MxAcc<NP>;
    constexpr int kDS = Acc::kStages;
    const int et = threadIdx.x - kEpiFirst;
    const int g = et >> 7;
    const int sub = (threadIdx.x >> 5) & 3;
    const int r = 32 * sub + (threadIdx.x & 31);
    const uint32_t lane_addr = (uint32_t)(32 * sub) << 16;
    bool ok = true;
    int seg = 0, b = 0, nsync = 0;
    long long nv = 0;
    float* srow = nullptr;
    ICursor cur(f0, a, 1);
    for (long long f = f0; f < f1; ++f) {
        if (warp_aborted(sm)) { ok = false; break; }
        const int jt = (int)(f - f0), sd = jt % kDS;
        if (f == f0 || cur.ti == 0) {
            b = seg & 1;
            if (!warp_wait(&sm.q_full[b], (seg >> 1) & 1)) { ok = false; break; }
            ++seg;
            nv = nvis_of(cur.q0, a);
            srow = a.scores + ((long long)cur.bat * a.n_q + cur.q0) * a.n_ent;
        }
        const bool seg_end = (f == f1 - 1) || (cur.ti == a.tiles_per_row - 1);
        const int ti = cur.ti, row = cur.bat * a.n_q + cur.q0;
        cur.next(a);
        if (!warp_wait(&sm.d_full[sd], (jt / kDS) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        float acc[2];
#pragma unroll
        for (int i = 0; i < 2; ++i)
            acc[i] = score_of<false, NP>(tmem + lane_addr + Acc::kCols * sd + NP * (g + 2 * i), sm.wq[b]);
        tc::tc_fence_before();
        tc::mbar_arrive(&sm.d_free[sd]);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const long long e = (long long)ti * kMxTile + kHalf * (g + 2 * i) + r;
            if (e < a.n_ent) {
                float sc = -INFINITY;
                if (e < nv) {
                    sc = acc[i] + 0.0f;
                    if (a.hist) atomicAdd(&sm.hist[b][float_to_ordered(sc) >> 20], 1u);
                }
                srow[e] = sc;
            }
        }
        if (seg_end) {
            tc::mbar_arrive(&sm.q_free[b]);  // done with wq[b]
            if (a.hist) {
                tc::mbar_arrive(&sm.ep_sync);
                if (!warp_wait(&sm.ep_sync, nsync++ & 1)) { ok = false; break; }
                uint32_t* gh = a.hist + (long long)row * kHistBins;
                for (int i = et; i < kHistBins; i += kEpiThreads) {
                    const uint32_t v = sm.hist[b][i];
                    if (v) {
                        atomicAdd(gh + i, v);
                        sm.hist[b][i] = 0;
                    }
                }
            }
        }
    }
    if (!ok) idx_fault(sm, a);
}

template <int NP>
__global__ void __launch_bounds__(kThreads, 1) index_score_mx_kernel(const __grid_constant__ CUtensorMap kmap, IdxTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    IdxSmem& sm = *reinterpret_cast<IdxSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long f0 = irange(blockIdx.x, a), f1 = irange(blockIdx.x + 1, a);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kMxStages; ++i) {
            tc::mbar_init(&sm.k_full[i], 1);
            tc::mbar_init(&sm.k_empty[i], 1);
        }
        for (int i = 0; i < MxAcc<NP>::kStages; ++i) {
            tc::mbar_init(&sm.d_full[i], 1);
            tc::mbar_init(&sm.d_free[i], kEpiThreads);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&sm.q_full[i], 128);
            tc::mbar_init(&sm.q_free[i], 1 + kEpiThreads);
            tc::mbar_init(&sm.sf_full[i], 128);
            tc::mbar_init(&sm.sf_free[i], 1);
        }
        tc::mbar_init(&sm.ep_sync, kEpiThreads);
        tc::mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        tc::fence_barrier_init();
    }
    for (int i = threadIdx.x; i < 2 * kHistBins; i += kThreads) (&sm.hist[0][0])[i] = 0;
    for (int i = threadIdx.x; i < 2 * kQBufBytes / 4; i += kThreads) reinterpret_cast<uint32_t*>(sm.q)[i] = 0;
    if (warp == 1) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (threadIdx.x == 0 && !a.bt) prefetch_first_tiles(a, &kmap, f0, f1, kMxTile, 2, 1, kMxStages + 2, a.kexp, 4);
    griddep_wait();  // the prologue above touched only shared and tensor memory (and prefetched into L2)
    griddep_launch_dependents();
    const uint32_t tmem = sm.tmem_base;
    if (warp == 0) {
        if (lane == 0) mx_producer(sm, a, &kmap, f0, f1);
    } else if (warp == 1) {
        mx_mma<NP>(sm, a, tmem, f0, f1);  // the whole warp (one elected lane issues)
    } else if (warp < 6) {
        mx_stage<NP>(sm, a, tmem, f0, f1);
    } else {
        mx_epilogue<NP>(sm, a, tmem, f0, f1);
    }
    __syncwarp();
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 idx_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// MXFP4 keys: one query row per segment (no multi-query grouping); tiles of 256 entries
cudaError_t launch_index_scores_mx(const IndexArgs& a, float* scores, uint32_t* hist, int* err, cudaStream_t stream,
                                   PFN_cuTensorMapEncodeTiled_v12000 fn) {
    CUtensorMap kmap;
    cuuint64_t dims[2] = {64, (cuuint64_t)(a.bt ? a.pool_rows : (long long)a.batch * a.n_ent)};
    cuuint64_t strides[1] = {64};
    cuuint32_t box[2] = {64u, (cuuint32_t)(a.bt ? a.epb : kTileK)};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a.k), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    IdxTcArgs t;
    t.q = static_cast<const __nv_bfloat16*>(a.q);
    t.w = a.w;
    t.kscale = nullptr;
    t.kexp = a.kexp;
    t.bt = a.bt;
    t.bt_stride = a.bt_stride;
    t.epb = a.epb;
    t.epb_shift = a.epb > 0 ? __builtin_ctz((unsigned)a.epb) : 0;
    t.n_blocks = a.epb > 0 ? a.pool_rows / a.epb : 0;
    t.scores = scores;
    t.hist = hist;
    t.err = err;
    t.n_ent = a.n_ent;
    t.ctx_len = a.ctx_len;
    t.rows = a.batch * a.n_q;
    t.n_q = a.n_q;
    t.m = a.m;
    t.heads_i = a.heads_i;
    t.ngroups = a.n_q;
    long long nv_max = n_visible(a.ctx_len - 1, a.m);
    if (nv_max > a.n_ent) nv_max = a.n_ent;
    t.tiles_per_row = (int)((nv_max + kMxTile - 1) / kMxTile);
    t.total_tiles = (long long)a.batch * t.ngroups * t.tiles_per_row;
    if (t.total_tiles == 0) return cudaSuccess;
    t.grid = (int)(t.total_tiles < kNumSMs ? t.total_tiles : kNumSMs);
    const size_t smem = sizeof(IdxSmem) + 1024;
    auto go = [&](auto kernel) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) e = launch_pdl(kernel, dim3(t.grid), dim3(kThreads), smem, stream, kmap, t);
        return e;
    };
    cudaError_t e = a.heads_i <= 16 ? go(index_score_mx_kernel<16>) : go(index_score_mx_kernel<32>);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

bool index_tc_shape_ok(const IndexArgs& a) {
    // paged keys: blocks of kMinEpb .. 256 entries (a power of two), so a tile is whole blocks
    const bool paged_ok =
        !a.bt || (a.epb >= kMinEpb && a.epb <= 256 && (a.epb & (a.epb - 1)) == 0 && a.pool_rows < (1LL << 31));
    return a.d_i == kDI && a.heads_i <= 32 && a.q_dtype == V4A_BF16 &&
           (a.k_dtype == V4A_BF16 || a.k_dtype == V4A_FP8E4M3 || (a.k_dtype == V4A_MXFP4 && a.kexp)) &&
           a.n_ent >= 1 && (long long)a.batch * a.n_ent < (1LL << 31) && paged_ok;
}

bool index_tc_available(const IndexArgs& a) { return index_tc_shape_ok(a) && idx_encode_fn() != nullptr; }

cudaError_t launch_index_scores_tc(const IndexArgs& a, float* scores, uint32_t* hist, int* err, cudaStream_t stream) {
    auto fn = idx_encode_fn();
    if (!fn) return cudaErrorNotSupported;
    if (a.k_dtype == V4A_MXFP4) return launch_index_scores_mx(a, scores, hist, err, stream, fn);
    const bool fp8 = a.k_dtype == V4A_FP8E4M3;
    CUtensorMap kmap;
    cuuint64_t dims[2] = {(cuuint64_t)kDI, (cuuint64_t)(a.bt ? a.pool_rows : (long long)a.batch * a.n_ent)};
    cuuint64_t strides[1] = {(cuuint64_t)kDI * (fp8 ? 1 : 2)};
    cuuint32_t box[2] = {fp8 ? 128u : 64u, (cuuint32_t)(a.bt ? a.epb : kTileK)};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&kmap, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.k),
           dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    IdxTcArgs t;
    t.q = static_cast<const __nv_bfloat16*>(a.q);
    t.w = a.w;
    t.kscale = a.kscale;
    t.kexp = nullptr;
    t.bt = a.bt;
    t.bt_stride = a.bt_stride;
    t.epb = a.epb;
    t.epb_shift = a.epb > 0 ? __builtin_ctz((unsigned)a.epb) : 0;
    t.n_blocks = a.epb > 0 ? a.pool_rows / a.epb : 0;
    t.scores = scores;
    t.hist = hist;
    t.err = err;
    t.n_ent = a.n_ent;
    t.ctx_len = a.ctx_len;
    t.rows = a.batch * a.n_q;
    t.n_q = a.n_q;
    t.m = a.m;
    t.heads_i = a.heads_i;
    // queries scored together: several per key tile when there are many queries and no histogram
    const bool narrow = a.heads_i <= 16;
    int G = 1;
    if (a.n_q > 1 && hist == nullptr) G = fp8 ? (narrow ? 2 : 1) : (narrow ? 4 : 2);
    t.ngroups = (a.n_q + G - 1) / G;
    // tiles up to the last entry any query of the row block can see
    long long nv_max = n_visible(a.ctx_len - 1, a.m);
    if (nv_max > a.n_ent) nv_max = a.n_ent;
    t.tiles_per_row = (int)((nv_max + kTileK - 1) / kTileK);
    t.total_tiles = (long long)a.batch * t.ngroups * t.tiles_per_row;
    if (t.total_tiles == 0) return cudaSuccess;
    t.grid = (int)(t.total_tiles < kNumSMs ? t.total_tiles : kNumSMs);
    const size_t smem = sizeof(IdxSmem) + 1024;
    auto go = [&](auto kernel) {
        cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err == cudaSuccess) err = launch_pdl(kernel, dim3(t.grid), dim3(kThreads), smem, stream, kmap, t);
        return err;
    };
    cudaError_t e;
    if (fp8) {
        if (narrow) e = G == 2 ? go(index_score_tc_kernel<true, 16, 2>) : go(index_score_tc_kernel<true, 16, 1>);
        else e = go(index_score_tc_kernel<true, 32, 1>);
    } else {
        if (narrow) e = G == 4 ? go(index_score_tc_kernel<false, 16, 4>) : go(index_score_tc_kernel<false, 16, 1>);
        else e = G == 2 ? go(index_score_tc_kernel<false, 32, 2>) : go(index_score_tc_kernel<false, 32, 1>);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace v4a
