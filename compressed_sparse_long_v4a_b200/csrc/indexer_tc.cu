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
// Warp 0 loads key tiles into a 4-stage ring, warp 1 issues the MMAs, warps
// 2-5 convert (FP8) and run the epilogue.  CTAs take contiguous ranges of the
// flat (query row, tile) sequence.  Every wait is bounded.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace v4a {
namespace {

constexpr int kDI = 128;                 // indexer dim handled here
constexpr int kTileK = 128;              // entries per tile
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kHistBins = 4096;          // top 12 bits of the ordered score key
constexpr uint32_t kColA = 0;            // FP8: converted key tiles, 2 x 64 columns
constexpr uint32_t kColD = 128;          // D: 2 x 32 columns
constexpr uint32_t kTmemCols = 256;

struct __align__(1024) IdxSmem {
    uint8_t keys[kStages][kTileK * kDI * 2];  // bf16: 2 slabs of [128][128 B]; fp8: [128][128 B]
    uint8_t q[2][32 * 128];                   // B operand: 2 K-slabs of [32 heads][128 B]
    float wq[32];                             // head weights (times 2^-s for FP8)
    uint32_t hist[kHistBins];
    uint64_t k_full[kStages], k_empty[kStages], a_full[2], d_full[2], d_free[2], q_ready, q_free, drain;
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
    int rows, n_q, m, heads_i, n_pad, tiles_per_row, grid;
};

__device__ __forceinline__ void idx_fault(IdxSmem& sm, const IdxTcArgs& a) {
    sm.abort_flag = 1;
    if (a.err) atomicExch(a.err, (int)V4A_ERR_DEVICE_FAULT);
}

__device__ __forceinline__ long long irange(int c, const IdxTcArgs& a) { return (long long)c * a.total_tiles / a.grid; }

struct ICursor {
    int row, ti;
    __device__ ICursor(long long f, int tpr) : row((int)(f / tpr)), ti((int)(f % tpr)) {}
    __device__ void next(int tpr) {
        if (++ti == tpr) {
            ti = 0;
            ++row;
        }
    }
};

__device__ __forceinline__ long long nvis_of(int row, const IdxTcArgs& a) {
    const long long t = a.ctx_len - a.n_q + (row % a.n_q);
    long long nv = n_visible(t, a.m);
    return nv > a.n_ent ? a.n_ent : nv;
}

// idesc: M=128, N = n_pad, A and B both f16 (FP8 path) or both bf16
__device__ __forceinline__ uint32_t idx_idesc(int n_pad, bool fp8) { return tc::idesc_f16(128, n_pad, 0, 0, fp8 ? 0 : 1); }

template <bool FP8>
__device__ void idx_producer(IdxSmem& sm, const IdxTcArgs& a, const CUtensorMap* kmap, long long f0, long long f1) {
    const int lane = threadIdx.x & 31;
    ICursor cur(f0, a.tiles_per_row);
    for (long long f = f0; f < f1; ++f, cur.next(a.tiles_per_row)) {
        if (sm.abort_flag) break;
        const int jt = (int)(f - f0), st = jt % kStages;
        if (jt >= kStages && !tc::mbar_wait(&sm.k_empty[st], ((jt / kStages) - 1) & 1)) { idx_fault(sm, a); break; }
        if (lane == 0) {
            const int b = cur.row / a.n_q;
            const int y = (int)((long long)b * a.n_ent + (long long)cur.ti * kTileK);
            if (FP8) {
                tc::mbar_arrive_expect_tx(&sm.k_full[st], kTileK * kDI);
                tc::tma_load_2d(sm.keys[st], kmap, 0, y, &sm.k_full[st]);
            } else {
                tc::mbar_arrive_expect_tx(&sm.k_full[st], kTileK * kDI * 2);
                tc::tma_load_2d(sm.keys[st], kmap, 0, y, &sm.k_full[st]);
                tc::tma_load_2d(sm.keys[st] + kTileK * 128, kmap, 64, y, &sm.k_full[st]);
            }
        }
    }
    const long long n = f1 - f0;
    for (long long jt = n - kStages; jt < n; ++jt)
        if (jt >= 0) tc::mbar_wait(&sm.k_full[jt % kStages], (jt / kStages) & 1);
}

template <bool FP8>
__device__ void idx_mma(IdxSmem& sm, const IdxTcArgs& a, uint32_t tmem, long long f0, long long f1) {
    bool ok = true;
    int seg = 0;
    const uint32_t idesc = idx_idesc(a.n_pad, FP8);
    const uint64_t qd = tc::sw128_desc(tc::smem_u32(sm.q[0]), 16, 1024);
    const uint32_t qslab = (uint32_t)a.n_pad * 128;  // bytes per K-slab of q
    ICursor cur(f0, a.tiles_per_row);
    for (long long f = f0; f < f1; ++f, cur.next(a.tiles_per_row)) {
        if (sm.abort_flag) { ok = false; break; }
        const int jt = (int)(f - f0), s = jt & 1, st = jt % kStages;
        const bool seg_start = (f == f0) || (cur.ti == 0);
        const bool seg_end = (f == f1 - 1) || (cur.ti == a.tiles_per_row - 1);
        if (seg_start) {
            if (!tc::mbar_wait(&sm.q_ready, seg & 1)) { ok = false; break; }
            ++seg;
        }
        if (FP8) {
            if (!tc::mbar_wait(&sm.a_full[s], (jt >> 1) & 1)) { ok = false; break; }
        } else {
            if (!tc::mbar_wait(&sm.k_full[st], (jt / kStages) & 1)) { ok = false; break; }
            if (jt >= 2 && !tc::mbar_wait(&sm.d_free[s], ((jt >> 1) - 1) & 1)) { ok = false; break; }
        }
        tc::tc_fence_after();
        const uint32_t d = tmem + kColD + 32 * s;
        if (FP8) {
            const uint32_t at = tmem + kColA + 64 * s;
#pragma unroll
            for (int kk = 0; kk < kDI / 16; ++kk) {
                const uint64_t bd = qd + ((((kk >> 2) * qslab) + (kk & 3) * 32) >> 4);
                asm volatile(
                    "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                    " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
                    "r"(at + 8 * kk), "l"(bd), "r"(idesc), "r"(kk ? 1u : 0u)
                    : "memory");
            }
        } else {
            const uint64_t kd = tc::sw128_desc(tc::smem_u32(sm.keys[st]), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < kDI / 16; ++kk) {
                const uint64_t ad = kd + ((((kk >> 2) * (kTileK * 128)) + (kk & 3) * 32) >> 4);
                const uint64_t bd = qd + ((((kk >> 2) * qslab) + (kk & 3) * 32) >> 4);
                tc::mma_f16(d, ad, bd, idesc, kk ? 1u : 0u);
            }
            tc::mma_commit(&sm.k_empty[st]);
        }
        tc::mma_commit(&sm.d_full[s]);
        if (seg_end) tc::mma_commit(&sm.q_free);
    }
    if (!ok) idx_fault(sm, a);
    tc::mma_commit(&sm.drain);
    tc::mbar_wait(&sm.drain, 0);
}

// q of `row` into the B-operand layout (K-major, 128-byte swizzle), and the head weights
template <bool FP8>
__device__ void stage_query(IdxSmem& sm, const IdxTcArgs& a, int row) {
    const int t = threadIdx.x - 64;  // 0..127
    // one warp per head group: warp w handles heads w, w+4, ...; lane owns 4 of the 128 elements
    const int warp = t >> 5, lane = t & 31;
    for (int h = warp; h < a.n_pad; h += 4) {
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
        uint8_t* slab = sm.q[0] + (k >> 6) * (a.n_pad * 128);
        uint8_t* dst = slab + (h >> 3) * 1024 + (h & 7) * 128 + ((((k & 63) >> 3) ^ (h & 7)) << 4) + ((k & 7) ? 8 : 0);
        *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
        if (lane == 0) sm.wq[h] = wq;
    }
}

template <bool FP8>
__device__ void idx_epilogue(IdxSmem& sm, const IdxTcArgs& a, uint32_t tmem, long long f0, long long f1) {
    const int t = threadIdx.x - 64;                 // entry within the tile
    const int sub = (threadIdx.x >> 5) & 3;
    const int r = 32 * sub + (threadIdx.x & 31);    // TMEM lane = entry row of the tile
    const uint32_t lane_addr = (uint32_t)(32 * sub) << 16;
    bool ok = true;
    int seg = 0;
    long long nvis = 0;
    ICursor cur(f0, a.tiles_per_row);
    // pending epilogue (tile j-1), with its entry's scale loaded ahead
    int p_row = -1, p_ti = 0, p_jt = -1;
    float p_scale = 1.f;
    auto epilogue = [&](int jt, int row, int ti) -> bool {
        const int s = jt & 1;
        if (!tc::mbar_wait(&sm.d_full[s], (jt >> 1) & 1)) return false;
        tc::tc_fence_after();
        uint32_t dv[32];
        tc::tmem_ld_x32(tmem + lane_addr + kColD + 32 * s, dv);
        tc::tmem_ld_wait();
        if (!FP8) {
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.d_free[s]);
        }
        const long long e = (long long)ti * kTileK + r;
        const long long nv = nvis_of(row, a);
        if (e < a.n_ent) {
            float sc = -INFINITY;
            if (e < nv) {
                float acc = 0.f;
#pragma unroll
                for (int h = 0; h < 32; ++h)
                    if (h < a.heads_i) acc = fmaf(sm.wq[h], fmaxf(__uint_as_float(dv[h]), 0.f), acc);
                if (FP8) acc *= p_scale;
                sc = acc + 0.0f;
                if (a.hist) atomicAdd(&sm.hist[float_to_ordered(sc) >> 20], 1u);
            }
            a.scores[(long long)row * a.n_ent + e] = sc;
        }
        return true;
    };
    for (long long f = f0; f < f1; ++f, cur.next(a.tiles_per_row)) {
        if (sm.abort_flag) { ok = false; break; }
        const int jt = (int)(f - f0), s = jt & 1, st = jt % kStages;
        const bool seg_start = (f == f0) || (cur.ti == 0);
        const bool seg_end = (f == f1 - 1) || (cur.ti == a.tiles_per_row - 1);
        if (seg_start) {
            // finish the previous row: its last tile's epilogue, then flush its histogram
            if (p_jt >= 0) {
                if (!epilogue(p_jt, p_row, p_ti)) { ok = false; break; }
                p_jt = -1;
                tc::named_barrier(1, 128);
                if (a.hist)
                    for (int i = t; i < kHistBins; i += 128)
                        if (sm.hist[i]) atomicAdd(&a.hist[(long long)p_row * kHistBins + i], sm.hist[i]);
            }
            // the MMAs of the previous row no longer read q
            if (seg > 0 && !tc::mbar_wait(&sm.q_free, (seg - 1) & 1)) { ok = false; break; }
            tc::named_barrier(1, 128);
            for (int i = t; i < kHistBins; i += 128) sm.hist[i] = 0;
            stage_query<FP8>(sm, a, cur.row);
            tc::fence_proxy_async();
            tc::mbar_arrive(&sm.q_ready);
            ++seg;
            nvis = nvis_of(cur.row, a);
        }
        if (FP8) {
            // widen this thread's entry (row r of the tile) to f16 into TMEM
            if (!tc::mbar_wait(&sm.k_full[st], (jt / kStages) & 1)) { ok = false; break; }
            const uint8_t* kr = sm.keys[st] + r * 128;
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
        // this tile's scale, used by its epilogue one iteration later
        float scale_next = 1.f;
        if (FP8) {
            const long long e = (long long)cur.ti * kTileK + r;
            if (e < a.n_ent) scale_next = __ldg(a.kscale + (long long)(cur.row / a.n_q) * a.n_ent + e);
        }
        // epilogue of the previous tile overlaps this tile's MMA
        if (p_jt >= 0 && !epilogue(p_jt, p_row, p_ti)) { ok = false; break; }
        p_jt = jt;
        p_row = cur.row;
        p_ti = cur.ti;
        p_scale = scale_next;
        (void)seg_end;
    }
    if (ok && p_jt >= 0) {
        ok = epilogue(p_jt, p_row, p_ti);
        tc::named_barrier(1, 128);
        if (ok && a.hist)
            for (int i = t; i < kHistBins; i += 128)
                if (sm.hist[i]) atomicAdd(&a.hist[(long long)p_row * kHistBins + i], sm.hist[i]);
    }
    if (!ok) idx_fault(sm, a);
    (void)nvis;
}

template <bool FP8>
__global__ void __launch_bounds__(kThreads, 1) index_score_tc_kernel(const __grid_constant__ CUtensorMap kmap, IdxTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    IdxSmem& sm = *reinterpret_cast<IdxSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const long long f0 = irange(blockIdx.x, a), f1 = irange(blockIdx.x + 1, a);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            tc::mbar_init(&sm.k_full[i], 1);
            tc::mbar_init(&sm.k_empty[i], FP8 ? 128 : 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&sm.a_full[i], 128);
            tc::mbar_init(&sm.d_full[i], 1);
            tc::mbar_init(&sm.d_free[i], 128);
        }
        tc::mbar_init(&sm.q_ready, 128);
        tc::mbar_init(&sm.q_free, 1);
        tc::mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    if (warp == 0) {
        idx_producer<FP8>(sm, a, &kmap, f0, f1);
    } else if (warp == 1) {
        if ((threadIdx.x & 31) == 0) idx_mma<FP8>(sm, a, tmem, f0, f1);
        __syncwarp();
    } else {
        idx_epilogue<FP8>(sm, a, tmem, f0, f1);
    }
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
    t.n_pad = a.heads_i <= 16 ? 16 : 32;
    // tiles up to the last entry any query of the row block can see
    long long nv_max = n_visible(a.ctx_len - 1, a.m);
    if (nv_max > a.n_ent) nv_max = a.n_ent;
    t.tiles_per_row = (int)((nv_max + kTileK - 1) / kTileK);
    t.total_tiles = (long long)t.rows * t.tiles_per_row;
    if (t.total_tiles == 0) return cudaSuccess;
    t.grid = (int)(t.total_tiles < kNumSMs ? t.total_tiles : kNumSMs);
    const size_t smem = sizeof(IdxSmem) + 1024;
    cudaError_t e;
    if (fp8) {
        e = cudaFuncSetAttribute(index_score_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) index_score_tc_kernel<true><<<t.grid, kThreads, smem, stream>>>(kmap, t);
    } else {
        e = cudaFuncSetAttribute(index_score_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) index_score_tc_kernel<false><<<t.grid, kThreads, smem, stream>>>(kmap, t);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace v4a
