// indexer_tc.cu -- tensor-core Lightning-Indexer scores for d_I = 128 keys
// (bf16, or FP8 e4m3 with one fp32 scale per entry) and up to 32 heads.
//
// I(t,s) = scale_s * sum_j w_j * ReLU(q_j . k_s)   ("How V4 makes a
// million-token context actually affordable", Lightning-Indexer section).
//
// Per tile of 128 entries of one query row: D[128 entries x N heads] = K Q^T
// on tcgen05 (M=128, N=16 or 32, K=128 in 8 steps of 16), then the epilogue
// (one thread per entry, TMEM lane = entry) forms the score, writes it as
// fp32 and counts it in a 4096-bin histogram of its order-preserving key's
// top 12 bits (the select step starts from that histogram).
//  * bf16 keys: the key tile (TMA, 128-byte swizzle) is the MMA's A operand
//    in shared memory; q is B (bf16).
//  * FP8 keys: the tile is widened in registers, exactly, to f16
//    (e4m3 -> f16 is exact) and stored to TMEM, where it is the MMA's A
//    operand; q is B in f16, each head scaled by a power of two so that its
//    largest element lies in [2^13, 2^14) (exact for every bf16 value within
//    2^-30 of it; the head weight carries the inverse power of two).
// Warp 0 loads key tiles into a shared-memory ring (8 x 16 KB for FP8, 4 x 32 KB
// for bf16), warp 1 issues the MMAs, warps 2-5 stage each row's q and (FP8)
// widen key tiles into TMEM, warps 6-9 run the epilogue; widening of tile j,
// the MMAs of tile j-1 and the epilogue of tile j-2 overlap.  CTAs take
// contiguous ranges of the flat (query row, tile) sequence; a run of one
// row's tiles inside a CTA's range is a segment, with its own q buffer and
// histogram (both double-buffered).  Every wait is bounded.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace v4a {
namespace {

constexpr int kDI = 128;                 // indexer dim handled here
constexpr int kTileK = 128;              // entries per tile
constexpr int kRingBytes = 131072;       // key-tile ring
constexpr int kMaxStages = 8;
constexpr int kThreads = 320;
constexpr int kHistBins = 4096;          // top 12 bits of the ordered score key
constexpr int kAStages = 2;              // FP8: widened key tiles in TMEM
constexpr int kDStages = 4;              // accumulators in TMEM
constexpr uint32_t kColA = 0;            // 2 x 64 columns
constexpr uint32_t kColD = 128;          // 4 x 32 columns
constexpr uint32_t kTmemCols = 256;

template <bool FP8> struct Ring {
    static constexpr int kStageBytes = FP8 ? kTileK * kDI : kTileK * kDI * 2;
    static constexpr int kStages = kRingBytes / kStageBytes;
};

struct __align__(1024) IdxSmem {
    uint8_t ring[kRingBytes];                 // bf16: [2 slabs][128][128 B] per stage; fp8: [128][128 B]
    uint8_t q[2][2 * 32 * 128];               // B operand per segment buffer: 2 K-slabs of [N heads][128 B]
    float wq[2][32];                          // head weights (times 2^-s for FP8)
    uint32_t hist[2][kHistBins];
    uint64_t k_full[kMaxStages], k_empty[kMaxStages], a_full[kAStages], a_free[kAStages], d_full[kDStages],
        d_free[kDStages], q_full[2], q_free[2], ep_sync, drain;
    int abort_flag;
    uint32_t tmem_base;
};

struct IdxTcArgs {
    const __nv_bfloat16* q;  // [rows][HI][128] bf16
    const float* w;          // [rows][HI]
    const float* kscale;     // [B][N] (FP8) or null
    float* scores;           // [rows][N]
    uint32_t* hist;          // [rows][4096]
    int* err;                // device fault word (may be null)
    long long n_ent, ctx_len, total_tiles;
    int rows, n_q, m, heads_i, tiles_per_row, grid;
};

__device__ __forceinline__ void idx_fault(IdxSmem& sm, const IdxTcArgs& a) {
    sm.abort_flag = 1;
    if (a.err) atomicExch(a.err, (int)V4A_ERR_DEVICE_FAULT);
}

// bounded wait taken by a whole warp: true only if every lane saw the phase complete
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
    return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity));
}
__device__ __forceinline__ bool warp_aborted(const IdxSmem& sm) {
    return __any_sync(0xffffffffu, *reinterpret_cast<const volatile int*>(&sm.abort_flag) != 0);
}

__device__ __forceinline__ long long irange(int c, const IdxTcArgs& a) { return (long long)c * a.total_tiles / a.grid; }

// walks (row, tile) in flat order; rq = row % n_q and bat = row / n_q kept incrementally
struct ICursor {
    int row, ti, rq, bat;
    __device__ ICursor(long long f, const IdxTcArgs& a) {
        row = (int)(f / a.tiles_per_row);
        ti = (int)(f - (long long)row * a.tiles_per_row);
        bat = row / a.n_q;
        rq = row - bat * a.n_q;
    }
    __device__ __forceinline__ void next(const IdxTcArgs& a) {
        if (++ti == a.tiles_per_row) {
            ti = 0;
            ++row;
            if (++rq == a.n_q) {
                rq = 0;
                ++bat;
            }
        }
    }
};

__device__ __forceinline__ long long nvis_of(const ICursor& c, const IdxTcArgs& a) {
    const long long t = a.ctx_len - a.n_q + c.rq;
    const long long nv = n_visible(t, a.m);
    return nv > a.n_ent ? a.n_ent : nv;
}

template <bool FP8>
__device__ void idx_producer(IdxSmem& sm, const IdxTcArgs& a, const CUtensorMap* kmap, long long f0, long long f1) {
    constexpr int kSt = Ring<FP8>::kStages, kBytes = Ring<FP8>::kStageBytes;
    ICursor cur(f0, a);
    const long long n = f1 - f0;
    for (long long jt = 0; jt < n; ++jt, cur.next(a)) {
        if (*reinterpret_cast<volatile int*>(&sm.abort_flag)) break;
        const int st = (int)(jt % kSt);
        if (jt >= kSt && !tc::mbar_wait(&sm.k_empty[st], (uint32_t)((jt / kSt) - 1) & 1)) { idx_fault(sm, a); break; }
        const int y = (int)((long long)cur.bat * a.n_ent + (long long)cur.ti * kTileK);
        uint8_t* dst = sm.ring + st * kBytes;
        tc::mbar_arrive_expect_tx(&sm.k_full[st], kBytes);
        tc::tma_load_2d(dst, kmap, 0, y, &sm.k_full[st]);
        if (!FP8) tc::tma_load_2d(dst + kTileK * 128, kmap, 64, y, &sm.k_full[st]);
    }
    // no copy may still be in flight when the CTA exits
    for (long long jt = n - kSt; jt < n; ++jt)
        if (jt >= 0) tc::mbar_wait(&sm.k_full[jt % kSt], (uint32_t)(jt / kSt) & 1);
}

template <bool FP8, int NP>
__device__ void idx_mma(IdxSmem& sm, const IdxTcArgs& a, uint32_t tmem, long long f0, long long f1) {
    constexpr int kSt = Ring<FP8>::kStages, kBytes = Ring<FP8>::kStageBytes;
    constexpr uint32_t kQSlab = NP * 128;  // bytes per K-slab of q
    constexpr uint32_t idesc = tc::idesc_f16(128, NP, 0, 0, FP8 ? 0 : 1);
    bool ok = true;
    int seg = 0, b = 0;
    uint64_t qd = 0;
    ICursor cur(f0, a);
    for (long long f = f0; f < f1; ++f, cur.next(a)) {
        if (*reinterpret_cast<volatile int*>(&sm.abort_flag)) { ok = false; break; }
        const int jt = (int)(f - f0), s = jt & 1, st = jt % kSt, sd = jt & 3;
        if (f == f0 || cur.ti == 0) {
            b = seg & 1;
            if (!tc::mbar_wait(&sm.q_full[b], (seg >> 1) & 1)) { ok = false; break; }
            qd = tc::sw128_desc(tc::smem_u32(sm.q[b]), 16, 1024);
            ++seg;
        }
        const bool seg_end = (f == f1 - 1) || (cur.ti == a.tiles_per_row - 1);
        if (FP8) {
            if (!tc::mbar_wait(&sm.a_full[s], (jt >> 1) & 1)) { ok = false; break; }
        } else {
            if (!tc::mbar_wait(&sm.k_full[st], (jt / kSt) & 1)) { ok = false; break; }
        }
        if (jt >= kDStages && !tc::mbar_wait(&sm.d_free[sd], ((jt >> 2) - 1) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t d = tmem + kColD + 32 * sd;
        if (FP8) {
            const uint32_t at = tmem + kColA + 64 * s;
#pragma unroll
            for (int kk = 0; kk < kDI / 16; ++kk) {
                const uint64_t bd = qd + ((((kk >> 2) * kQSlab) + (kk & 3) * 32) >> 4);
                asm volatile(
                    "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                    " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
                    "r"(at + 8 * kk), "l"(bd), "r"(idesc), "r"(kk ? 1u : 0u)
                    : "memory");
            }
            tc::mma_commit(&sm.a_free[s]);
        } else {
            const uint64_t kd = tc::sw128_desc(tc::smem_u32(sm.ring + st * kBytes), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < kDI / 16; ++kk) {
                const uint64_t ad = kd + ((((kk >> 2) * (kTileK * 128)) + (kk & 3) * 32) >> 4);
                const uint64_t bd = qd + ((((kk >> 2) * kQSlab) + (kk & 3) * 32) >> 4);
                tc::mma_f16(d, ad, bd, idesc, kk ? 1u : 0u);
            }
            tc::mma_commit(&sm.k_empty[st]);
        }
        tc::mma_commit(&sm.d_full[sd]);
        if (seg_end) tc::mma_commit(&sm.q_free[b]);
    }
    if (!ok) idx_fault(sm, a);
    tc::mma_commit(&sm.drain);
    tc::mbar_wait(&sm.drain, 0);
}

// q of one row into buffer b in the B-operand layout (K-major, 128-byte
// swizzle, NP head rows per K-slab), and the head weights; ct = 0..127
template <bool FP8, int NP>
__device__ void stage_query(IdxSmem& sm, const IdxTcArgs& a, int row, int b, int ct) {
    // warp w handles heads w, w+4, ...; lane owns 4 of the 128 elements
    const int warp = ct >> 5, lane = ct & 31;
    for (int h = warp; h < NP; h += 4) {
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        if (h < a.heads_i) {
            const __nv_bfloat16* qp = a.q + ((long long)row * a.heads_i + h) * kDI + lane * 4;
            const uint2 raw = *reinterpret_cast<const uint2*>(qp);
            v[0] = __uint_as_float(raw.x << 16);
            v[1] = __uint_as_float(raw.x & 0xffff0000u);
            v[2] = __uint_as_float(raw.y << 16);
            v[3] = __uint_as_float(raw.y & 0xffff0000u);
        }
        float wq = h < a.heads_i ? a.w[(long long)row * a.heads_i + h] : 0.f;
        uint32_t packed[2];
        if (FP8) {
            float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            int e = 0;
            if (amax > 0.f) frexpf(amax, &e);  // amax = f * 2^e, f in [0.5, 1)
            const int sh = amax > 0.f ? 14 - e : 0;  // amax * 2^sh in [2^13, 2^14)
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = ldexpf(v[i], sh);
            wq = ldexpf(wq, -sh);
            __half2 h0 = __floats2half2_rn(v[0], v[1]), h1 = __floats2half2_rn(v[2], v[3]);
            packed[0] = *reinterpret_cast<uint32_t*>(&h0);
            packed[1] = *reinterpret_cast<uint32_t*>(&h1);
        } else {
            __nv_bfloat162 b0 = __floats2bfloat162_rn(v[0], v[1]), b1 = __floats2bfloat162_rn(v[2], v[3]);
            packed[0] = *reinterpret_cast<uint32_t*>(&b0);
            packed[1] = *reinterpret_cast<uint32_t*>(&b1);
        }
        // element k = 4*lane .. 4*lane+3 of head h: K-slab k/64, 16-byte chunk (k%64)/8, 8-byte half
        const int k = lane * 4;
        uint8_t* slab = sm.q[b] + (k >> 6) * (NP * 128);
        uint8_t* dst = slab + (h >> 3) * 1024 + (h & 7) * 128 + ((((k & 63) >> 3) ^ (h & 7)) << 4) + ((k & 7) ? 8 : 0);
        *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
        if (lane == 0) sm.wq[b][h] = wq;
    }
}

// warps 2-5: per segment stage q; per tile (FP8) widen the key tile to f16 in TMEM
template <bool FP8, int NP>
__device__ void idx_convert(IdxSmem& sm, const IdxTcArgs& a, uint32_t tmem, long long f0, long long f1) {
    constexpr int kSt = Ring<FP8>::kStages, kBytes = Ring<FP8>::kStageBytes;
    const int ct = threadIdx.x - 64;
    const int sub = (threadIdx.x >> 5) & 3;
    const int r = 32 * sub + (threadIdx.x & 31);  // TMEM lane = entry row of the tile
    const uint32_t lane_addr = (uint32_t)(32 * sub) << 16;
    bool ok = true;
    int seg = 0;
    ICursor cur(f0, a);
    for (long long f = f0; f < f1; ++f, cur.next(a)) {
        if (warp_aborted(sm)) { ok = false; break; }
        const int jt = (int)(f - f0);
        if (f == f0 || cur.ti == 0) {
            const int b = seg & 1;
            if (seg >= 2 && !warp_wait(&sm.q_free[b], ((seg >> 1) - 1) & 1)) { ok = false; break; }
            stage_query<FP8, NP>(sm, a, cur.row, b, ct);
            tc::fence_proxy_async();
            tc::mbar_arrive(&sm.q_full[b]);
            ++seg;
        }
        if (FP8) {
            const int s = jt & 1, st = jt % kSt;
            if (!warp_wait(&sm.k_full[st], (jt / kSt) & 1)) { ok = false; break; }
            if (jt >= kAStages && !warp_wait(&sm.a_free[s], ((jt >> 1) - 1) & 1)) { ok = false; break; }
            tc::tc_fence_after();
            const uint8_t* kr = sm.ring + st * kBytes + r * 128;
            uint32_t cv[64];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 raw = *reinterpret_cast<const uint4*>(kr + ((c ^ (r & 7)) << 4));
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w4[i] & 0xffffu), __NV_E4M3);
                    __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w4[i] >> 16), __NV_E4M3);
                    cv[8 * c + 2 * i] = *reinterpret_cast<uint32_t*>(&lo);
                    cv[8 * c + 2 * i + 1] = *reinterpret_cast<uint32_t*>(&hi);
                }
            }
            tc::mbar_arrive(&sm.k_empty[st]);  // the smem tile has been read
            tc::tmem_st_x64(tmem + lane_addr + kColA + 64 * s, cv);
            tc::tmem_st_wait();
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.a_full[s]);
        }
    }
    if (!ok) idx_fault(sm, a);
}

// warps 6-9: per tile the score of one entry per thread, its histogram count and store
template <bool FP8, int NP>
__device__ void idx_epilogue(IdxSmem& sm, const IdxTcArgs& a, uint32_t tmem, long long f0, long long f1) {
    const int et = threadIdx.x - 192;
    const int sub = (threadIdx.x >> 5) & 3;
    const int r = 32 * sub + (threadIdx.x & 31);  // TMEM lane = entry row of the tile
    const uint32_t lane_addr = (uint32_t)(32 * sub) << 16;
    bool ok = true;
    int seg = 0, b = 0, nsync = 0;
    long long nv = 0;
    float* srow = nullptr;
    ICursor cur(f0, a);
    // scale of the current tile's entry, loaded one tile ahead
    auto scale_of = [&](const ICursor& c) -> float {
        const long long e = (long long)c.ti * kTileK + r;
        return e < a.n_ent ? __ldg(a.kscale + (long long)c.bat * a.n_ent + e) : 1.f;
    };
    float sc_cur = FP8 ? scale_of(cur) : 1.f;
    for (long long f = f0; f < f1; ++f) {
        if (warp_aborted(sm)) { ok = false; break; }
        const int jt = (int)(f - f0), sd = jt & 3;
        if (f == f0 || cur.ti == 0) {
            b = seg & 1;
            if (!warp_wait(&sm.q_full[b], (seg >> 1) & 1)) { ok = false; break; }
            ++seg;
            nv = nvis_of(cur, a);
            srow = a.scores + (long long)cur.row * a.n_ent;
        }
        const bool seg_end = (f == f1 - 1) || (cur.ti == a.tiles_per_row - 1);
        const int ti = cur.ti, row = cur.row;
        cur.next(a);
        float sc_next = 1.f;
        if (FP8 && f + 1 < f1) sc_next = scale_of(cur);
        if (!warp_wait(&sm.d_full[sd], (jt >> 2) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        uint32_t dv[NP];
        if constexpr (NP == 16) tc::tmem_ld_x16(tmem + lane_addr + kColD + 32 * sd, dv);
        else tc::tmem_ld_x32(tmem + lane_addr + kColD + 32 * sd, dv);
        tc::tmem_ld_wait();
        tc::tc_fence_before();
        tc::mbar_arrive(&sm.d_free[sd]);
        const long long e = (long long)ti * kTileK + r;
        if (e < a.n_ent) {
            float sc = -INFINITY;
            if (e < nv) {
                float acc = 0.f;
#pragma unroll
                for (int h = 0; h < NP; ++h) acc = fmaf(sm.wq[b][h], fmaxf(__uint_as_float(dv[h]), 0.f), acc);
                if (FP8) acc *= sc_cur;
                sc = acc + 0.0f;
                if (a.hist) atomicAdd(&sm.hist[b][float_to_ordered(sc) >> 20], 1u);
            }
            srow[e] = sc;
        }
        sc_cur = sc_next;
        if (seg_end) {
            tc::mbar_arrive(&sm.q_free[b]);  // done with wq[b]
            // every epilogue thread has counted this segment's scores (bounded, unlike a named barrier)
            tc::mbar_arrive(&sm.ep_sync);
            if (!warp_wait(&sm.ep_sync, nsync++ & 1)) { ok = false; break; }
            if (a.hist) {
                uint32_t* g = a.hist + (long long)row * kHistBins;
                for (int i = et; i < kHistBins; i += 128) {
                    const uint32_t v = sm.hist[b][i];
                    if (v) {
                        atomicAdd(g + i, v);
                        sm.hist[b][i] = 0;
                    }
                }
            }
        }
    }
    if (!ok) idx_fault(sm, a);
}

template <bool FP8, int NP>
__global__ void __launch_bounds__(kThreads, 1) index_score_tc_kernel(const __grid_constant__ CUtensorMap kmap, IdxTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    IdxSmem& sm = *reinterpret_cast<IdxSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long f0 = irange(blockIdx.x, a), f1 = irange(blockIdx.x + 1, a);
    if (threadIdx.x == 0) {
        for (int i = 0; i < Ring<FP8>::kStages; ++i) {
            tc::mbar_init(&sm.k_full[i], 1);
            tc::mbar_init(&sm.k_empty[i], FP8 ? 128 : 1);
        }
        for (int i = 0; i < kAStages; ++i) {
            tc::mbar_init(&sm.a_full[i], 128);
            tc::mbar_init(&sm.a_free[i], 1);
        }
        for (int i = 0; i < kDStages; ++i) {
            tc::mbar_init(&sm.d_full[i], 1);
            tc::mbar_init(&sm.d_free[i], 128);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&sm.q_full[i], 128);
            tc::mbar_init(&sm.q_free[i], 1 + 128);  // the MMAs' commit + every epilogue thread
        }
        tc::mbar_init(&sm.ep_sync, 128);
        tc::mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        tc::fence_barrier_init();
    }
    for (int i = threadIdx.x; i < 2 * kHistBins; i += kThreads) (&sm.hist[0][0])[i] = 0;
    if (warp == 1) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    if (warp == 0) {
        if (lane == 0) idx_producer<FP8>(sm, a, &kmap, f0, f1);
    } else if (warp == 1) {
        if (lane == 0) idx_mma<FP8, NP>(sm, a, tmem, f0, f1);
    } else if (warp < 6) {
        idx_convert<FP8, NP>(sm, a, tmem, f0, f1);
    } else {
        idx_epilogue<FP8, NP>(sm, a, tmem, f0, f1);
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

}  // namespace

bool index_tc_shape_ok(const IndexArgs& a) {
    return a.d_i == kDI && a.heads_i <= 32 && a.q_dtype == V4A_BF16 &&
           (a.k_dtype == V4A_BF16 || a.k_dtype == V4A_FP8E4M3) && a.n_ent >= 1 &&
           (long long)a.batch * a.n_ent < (1LL << 31);
}

bool index_tc_available(const IndexArgs& a) { return index_tc_shape_ok(a) && idx_encode_fn() != nullptr; }

cudaError_t launch_index_scores_tc(const IndexArgs& a, float* scores, uint32_t* hist, int* err, cudaStream_t stream) {
    auto fn = idx_encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const bool fp8 = a.k_dtype == V4A_FP8E4M3;
    CUtensorMap kmap;
    cuuint64_t dims[2] = {(cuuint64_t)kDI, (cuuint64_t)((long long)a.batch * a.n_ent)};
    cuuint64_t strides[1] = {(cuuint64_t)kDI * (fp8 ? 1 : 2)};
    cuuint32_t box[2] = {fp8 ? 128u : 64u, (cuuint32_t)kTileK};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&kmap, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.k),
           dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    IdxTcArgs t;
    t.q = static_cast<const __nv_bfloat16*>(a.q);
    t.w = a.w;
    t.kscale = a.kscale;
    t.scores = scores;
    t.hist = hist;
    t.err = err;
    t.n_ent = a.n_ent;
    t.ctx_len = a.ctx_len;
    t.rows = a.batch * a.n_q;
    t.n_q = a.n_q;
    t.m = a.m;
    t.heads_i = a.heads_i;
    // tiles up to the last entry any query of the row block can see
    long long nv_max = n_visible(a.ctx_len - 1, a.m);
    if (nv_max > a.n_ent) nv_max = a.n_ent;
    t.tiles_per_row = (int)((nv_max + kTileK - 1) / kTileK);
    t.total_tiles = (long long)t.rows * t.tiles_per_row;
    if (t.total_tiles == 0) return cudaSuccess;
    t.grid = (int)(t.total_tiles < kNumSMs ? t.total_tiles : kNumSMs);
    const size_t smem = sizeof(IdxSmem) + 1024;
    auto go = [&](auto kernel) {
        cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err == cudaSuccess) kernel<<<t.grid, kThreads, smem, stream>>>(kmap, t);
        return err;
    };
    const bool narrow = a.heads_i <= 16;
    cudaError_t e = fp8 ? (narrow ? go(index_score_tc_kernel<true, 16>) : go(index_score_tc_kernel<true, 32>))
                        : (narrow ? go(index_score_tc_kernel<false, 16>) : go(index_score_tc_kernel<false, 32>));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace v4a
