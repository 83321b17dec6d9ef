// attend_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) CSA and HCA attention
// for the 64-head, d = 512, bf16 shape of DeepSeek-V4's compressed layers.
//
// What it computes is the joint softmax of attend.cu: for query (b, j) at
// position t and head h, softmax_r(q_h . v_r / sqrt(d)) over the candidate
// rows (selected or all visible compressed entries, then the window tokens
// (t-W, t]), times the same rows ("DeepSeek-V4: Million-Token Context via
// Hybrid Compressed Attention", CSA "Core attention with shared KV MQA").
//
// Shape of the work.  One query has 64 heads sharing every K=V row, so per
// tile of T candidate rows (T = 64, or 48 for long rows: see Tiles):
//   S  = Q K^T      tcgen05 M=64 (heads) x N=T (rows) x K=512, Q and K in smem
//   P  = softmax(S) (online, two threads per head)
//   O^T += V^T P^T  tcgen05 M=128 (d chunk) x N=64 (heads) x K=T (rows),
//                   four d chunks, V^T read MN-major from the same smem tile
// One warp issues the MMAs (an elected lane per instruction, descriptors in
// uniform registers); the issue rate, not the tensor pipe, bounds small MMAs,
// so tiles are as wide as shared memory allows next to the 64 KB query.
// The accumulator O^T (512 x 64 fp32) and two S buffers live in TMEM.
//
// Work split: the candidate tiles of all queries form one flat sequence that
// is cut into `grid` contiguous ranges, one per CTA (one CTA per SM).  A CTA
// whose range covers a query's tiles completely writes that query's output;
// a query cut between CTAs gets one partial (m, l, O) per piece, merged by
// attend_tc_combine.  Per CTA: warp 0 loads into a ring of 2 or 3 stages -- one
// TMA box per tile for contiguous rows and per query, or, with warp 6 (G = 2),
// cp.async gathers of selected, paged or ring rows, 32 rows per warp -- warp 1
// (all lanes; one elected lane) issues the MMAs, warps 2-5 run the softmax and
// the output.  Every wait is bounded; on a time-out the CTA records a device
// fault, poisons its outputs with NaN and winds down.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace v4a {
namespace {

constexpr int kD = 512;
constexpr int kH = 64;
constexpr uint32_t kSCols = 64;                  // TMEM columns between the two S buffers
constexpr int kSlabs = kD / 64;                  // 64-element (128 B) column slabs
constexpr uint32_t kQBytes = kSlabs * kH * 128;  // 64 KB
constexpr uint32_t kPBytes = kH * 128;           // 64 heads x up to 64 rows bf16
constexpr uint32_t kColO = 0;                    // O^T: 4 chunks of 64 columns
constexpr uint32_t kColS = 256;                  // S: 2 buffers of 64 columns
constexpr uint32_t kTmemCols = 512;
// Warps: 0 (and 6, when two warps gather) loads, 1 issues the MMAs, 2-5 run the softmax and the output.
template <int G>
constexpr int threads_for() { return 32 * (5 + G); }
constexpr float kRescaleSlack = 8.0f;  // keep a stale running max until the true one exceeds it by 2^8
// Piece layout: a piece (partial O of a query split between CTAs) holds O[h][d] for 64 heads x 512
// dims as float4 groups of four heads: the group of heads 4i .. 4i+3 at dim d is float4 number
// ((d / 32) * 16 + i) * 32 + d % 32.  This is the order the epilogue's threads hold O^T in (thread
// = TMEM lane = dim, its registers = heads), so each warp store is 512 contiguous bytes, and the
// combine reads it back in the same 512-byte runs.  (Stored d-major, [d][64 heads], a warp store
// touched 32 cache lines and a 128 KB piece took ~9,900 cycles to write on B200.)

constexpr uint32_t kIdescPV = tc::idesc_f16(128, 64, 1, 0);

// Tile shapes.  A tile is T candidate rows; its 8 column slabs of T x 128 bytes sit in one of C::kStages
// stages beside the 64 KB query.  T = 64 with two stages keeps one tile load in flight while a tile is
// processed and spends the fewest MMA instructions per row; T = 48 fits a third stage, so two loads
// are in flight, at a third more QK instructions per row.  Long rows (HCA: thousands of entries per
// query, streamed) take 48; short ones (CSA selections, prefill rows) take 64 (measured on B200: HCA
// attention at 1M context 81 -> 77 us with 48; the prefill chunk's attention 1.72 -> 2.10 ms with 48).
template <int T>
struct Tiles {
    static_assert(T == 48 || T == 64, "tile rows");
    static constexpr int kTile = T;
    static constexpr int kStages = T == 64 ? 2 : 3;
    static constexpr uint64_t kTileMask = T == 64 ? ~0ull : ((1ull << T) - 1ull);
    static constexpr uint32_t kSlabBytes = T * 128;
    static constexpr uint32_t kTileBytes = kSlabs * kSlabBytes;
    static constexpr uint32_t kIdescQK = tc::idesc_f16(64, T, 0, 0);
    static constexpr int kHalfRows = T / 2;          // S values per softmax thread
    static constexpr int kHiRows = T / 2 - 16;       // ... of which from the second 16x32bx2 load
};

template <int T>
struct __align__(1024) Smem {
    using C = Tiles<T>;
    uint8_t q[kQBytes];
    uint8_t kv[C::kStages][C::kTileBytes];
    uint8_t p[2][kPBytes];
    uint64_t kv_full[C::kStages], kv_empty[C::kStages], s_full[2], p_full[2], p_free[2];
    uint64_t q_full, q_empty, drain;
    uint64_t mask[C::kStages];
    float alpha[2][kH], inv_l[kH];  // alpha / rescale_tag by tile parity; 1 / l of a whole row's heads
    int rescale_tag[2];
    int abort_flag;
    uint32_t tmem_base;
};

struct TcArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* entries;
    const __nv_bfloat16* token_kv;
    const int32_t* idx;  // CSA selections, or null for HCA
    float* out;
    float* part_ml;      // [2*grid][64][2]
    float* part_o;       // [2*grid] pieces of 64 x 512 floats (piece layout above)
    int* dev_status;
    long long n_ent, l_tok, tok_pos0, ctx_len, total_tiles;
    int rows, n_q, m, k, window;
    int e_tiles, w_tiles, tpr, grid;
    float scale_log2;
    const float* sink;  // [64] sink logits, or null
    int rope_dims;      // output dims rotated at minus the query position (0: none)
    float rope_base;
    const int32_t* bt;  // paged entries: block table [B][bt_stride] (epb entries per block), or null
    int bt_stride, epb;
    long long n_blocks;
    int ring_rows;      // > 0: window rows come from a ring [B][ring_rows][512] (position p in row p % ring_rows)
    int comb_pieces;    // bound on the pieces of one query (attend_tc_combine's shared memory)
    // bounded-wait limits (polls of an mbarrier; cycles without progress for the MMA warp) and the
    // fault-injection switch of the test hook (v4a_test_attend_fault): a CTA withholds its tile
    // `withhold` (local index; -1: never), issuing no copy and no arrival for it
    uint32_t wait_polls;
    long long stall_cycles;
    int withhold;
};

// tiles whose rows the producer gathers with cp.async (CSA selections, paged entries, ring windows)
__device__ __forceinline__ bool tile_gathered(const TcArgs& a, int ti) {
    return ti < a.e_tiles ? (a.idx != nullptr || a.bt != nullptr) : a.ring_rows > 0;
}
// row of visible entry s of sequence b; null for a block id outside the pool
__device__ __forceinline__ const __nv_bfloat16* entry_row(const TcArgs& a, int b, long long s) {
    if (a.bt) {
        const long long blk = a.bt[(long long)b * a.bt_stride + s / a.epb];
        if (blk < 0 || blk >= a.n_blocks) return nullptr;
        return a.entries + (blk * a.epb + s % a.epb) * kD;
    }
    return a.entries + ((long long)b * a.n_ent + s) * kD;
}

__device__ __forceinline__ long long range_start(int c, const TcArgs& a) {
    return (long long)c * a.total_tiles / a.grid;
}

struct RowInfo {
    int b;
    long long t, nvis;
};

// walks the flat tile sequence f0, f0+1, ... keeping (row, tile-in-row) without divisions
struct Cursor {
    int row, ti;
    __device__ Cursor(long long f, int tpr) : row((int)(f / tpr)), ti((int)(f % tpr)) {}
    __device__ void next(int tpr) {
        if (++ti == tpr) {
            ti = 0;
            ++row;
        }
    }
};

__device__ __forceinline__ RowInfo row_info(int row, const TcArgs& a) {
    RowInfo r;
    r.b = row / a.n_q;
    const int j = row % a.n_q;
    r.t = a.ctx_len - a.n_q + j;
    r.nvis = n_visible(r.t, a.m);
    if (r.nvis > a.n_ent) r.nvis = a.n_ent;
    return r;
}

template <int T>
__device__ __forceinline__ void fault(Smem<T>& sm, const TcArgs& a) {
    sm.abort_flag = 1;
    if (a.dev_status) atomicExch(a.dev_status, (int)V4A_ERR_DEVICE_FAULT);
}

// ---------------------------------------------------------------------
// warp 0: loads
// ---------------------------------------------------------------------
// The rows of a gathered tile are worked out in two steps, so the index (or block-table) loads of the
// next tiles are in flight while this tile's copies are issued: fetch_rows issues them, resolve_rows
// turns what they returned into row pointers.  RowInfo is the query row's, taken once per query row.
// With G loading warps, warp `part` owns rows 32 (h2 + part) + lane, h2 < 2 / G, of every tile: one
// warp owns rows lane and lane + 32, two warps own 32 rows each.
struct RowFetch {
    long long v[2];  // CSA: the selection (-1: none); paged HCA: the block id; ring: unused
    bool gath;       // the tile is gathered (false: loaded as a contiguous box)
};

template <int T, int G>
__device__ __forceinline__ RowFetch fetch_rows(const TcArgs& a, const RowInfo& ri, int row, int ti, int lane, int part) {
    using C = Tiles<T>;
    RowFetch f;
    f.gath = tile_gathered(a, ti);
    f.v[0] = f.v[1] = -1;
    if (!f.gath || ti >= a.e_tiles) return f;
#pragma unroll
    for (int h2 = 0; h2 < 2 / G; ++h2) {
        const int r = lane + 32 * (h2 + part);
        const long long c = (long long)ti * C::kTile + r;
        if (r >= C::kTile) continue;
        if (a.idx) {
            if (c < a.k) f.v[h2] = a.idx[(long long)row * a.k + c];
        } else if (c < ri.nvis) {  // HCA over a paged pool: entries c0 .. c0 + T - 1 through the block table
            f.v[h2] = a.bt[(long long)ri.b * a.bt_stride + c / a.epb];
        }
    }
    return f;
}

// Row pointers (src) and participation (ok) of this lane's rows of a gathered tile from fetch_rows'
// values.  Bad selections and block ids are reported; an excluded row still gets finite data (this
// query's head-0 row of q).
template <int T, int G>
__device__ __forceinline__ void resolve_rows(const TcArgs& a, const RowInfo& ri, int row, int ti, int lane, int part,
                                             const RowFetch& f, const __nv_bfloat16* (&src)[2], bool (&ok)[2]) {
    using C = Tiles<T>;
    const __nv_bfloat16* fallback = a.q + (long long)row * kH * kD;
#pragma unroll
    for (int h2 = 0; h2 < 2 / G; ++h2) {
        const int r = lane + 32 * (h2 + part);
        const __nv_bfloat16* er = nullptr;
        bool bad = false;
        if (r < C::kTile) {
            if (ti < a.e_tiles) {
                if (a.idx) {
                    const long long sidx = f.v[h2];
                    if (sidx >= 0 && sidx < ri.nvis) {
                        er = entry_row(a, ri.b, sidx);
                        bad = er == nullptr;  // a block id outside the pool
                    } else {
                        bad = sidx != -1;  // neither a selection nor the -1 filler
                    }
                } else {
                    const long long s = (long long)ti * C::kTile + r;
                    if (s < ri.nvis) {
                        const long long blk = f.v[h2];
                        if (blk >= 0 && blk < a.n_blocks) er = a.entries + (blk * a.epb + s % a.epb) * kD;
                        else bad = true;
                    }
                }
            } else {
                // window tokens p0 .. p0 + T - 1 from the ring (they may wrap around its end)
                const long long wi = ti - a.e_tiles;
                const long long p = ri.t - a.window + 1 + wi * C::kTile + r;
                if (wi * C::kTile + r < a.window && p >= 0)
                    er = a.token_kv + ((long long)ri.b * a.ring_rows + p % a.ring_rows) * kD;
            }
        }
        if (bad && a.dev_status) atomicExch(a.dev_status, (int)V4A_ERR_DEVICE_FAULT);
        ok[h2] = er != nullptr;
        src[h2] = ok[h2] ? er : fallback;
    }
}

// cp.async this warp's rows of a tile (src / ok from resolve_rows) into the 128-byte-swizzled stage,
// eight lanes per row: lane l copies 16-byte chunk l % 8 of every slab of rows 4 i + l / 8, so each warp
// copy is four whole 128-byte lines and each row pointer is shuffled once for eight copies.  Returns the
// warp's rows' bits of the tile's row mask.
template <int T, int G>
__device__ __forceinline__ uint64_t gather_tile(uint8_t* dst, const __nv_bfloat16* const (&src)[2], const bool (&ok)[2],
                                                int lane, int part, uint64_t policy) {
    using C = Tiles<T>;
    uint64_t mask = 0;
#pragma unroll
    for (int h2 = 0; h2 < 2 / G; ++h2) mask |= (uint64_t)__ballot_sync(0xffffffffu, ok[h2]) << (32 * (h2 + part));
    const int rl = lane >> 3, k = lane & 7;
    const int i0 = 8 * part, i1 = (8 * (part + 2 / G) < C::kTile / 4) ? 8 * (part + 2 / G) : C::kTile / 4;
#pragma unroll 4
    for (int i = i0; i < i1; ++i) {
        const int r = 4 * i + rl;
        // row r is lane r % 32's row number r / 32 - part (i is the same in every lane)
        const unsigned long long pr =
            __shfl_sync(0xffffffffu, (unsigned long long)((i >> 3) == part ? src[0] : src[1]), r & 31);
        const __nv_bfloat16* rs = (const __nv_bfloat16*)pr + k * 8;
        uint8_t* d = dst + r * 128 + ((k ^ (r & 7)) << 4);
#pragma unroll
        for (int c = 0; c < kSlabs; ++c) tc::cp_async_16_hint(d + c * C::kSlabBytes, rs + c * 64, policy);
    }
    return mask;
}

// Warp 0 lane 0, before the grid dependency wait: the query of the CTA's first segment and an L2
// prefetch of its first contiguous (TMA-loaded) entry tiles.  Both only read.  No kernel of this library
// writes attention queries, and a kernel before this one on the stream that is not programmatically
// launched has completed before this one starts, so the query is complete; the prefetch only warms L2,
// the point of coherence, so an entry still being written is read afresh by the load after the wait.
template <int T>
__device__ void early_loads(Smem<T>& sm, const TcArgs& a, const CUtensorMap* ent_map, const CUtensorMap* q_map,
                            long long f0, long long f1) {
    using C = Tiles<T>;
    const Cursor cur(f0, a.tpr);
    tc::mbar_arrive_expect_tx(&sm.q_full, kQBytes);
    tc::tma_load_3d(sm.q, q_map, 0, cur.row * kH, 0, &sm.q_full);
    if (a.idx || a.bt) return;
    const RowInfo ri = row_info(cur.row, a);
    for (int j = 0; j < C::kStages && f0 + j < f1 && cur.ti + j < a.e_tiles; ++j) {
        const int y = (int)((long long)ri.b * a.n_ent + (long long)(cur.ti + j) * C::kTile);
        tc::tma_prefetch_3d(ent_map, 0, y, 0);
    }
}

// Loading warp `part` of G.  Part 0 also loads the queries and the contiguous tiles; with two loading
// warps each gathers its 32 rows of a gathered tile and writes its half of the row mask.
template <int T, int G>
__device__ void producer(Smem<T>& sm, const TcArgs& a, const CUtensorMap* ent_map, const CUtensorMap* tok_map,
                         const CUtensorMap* q_map, long long f0, long long f1, int part) {
    using C = Tiles<T>;
    const int lane = threadIdx.x & 31;
    int seg = 0;
    Cursor cur(f0, a.tpr);
    // candidate rows: read once per call in decode, shared by the queries of a chunk in prefill
    const uint64_t stream_policy = tc::l2_stream_policy(a.n_q);
    int last_load[C::kStages];  // the last tile whose copies went into each stage (-1: none)
    for (int i = 0; i < C::kStages; ++i) last_load[i] = -1;
    // The rows of gathered tiles are fetched two tiles ahead (their index / block-table loads queue behind
    // a whole tile's copies) and resolved into row pointers once the current tile's copies are issued.
    // c1, c2: the next two tiles; ri, ri1, ri2: their query rows' info.
    Cursor c1 = cur, c2 = cur;
    c1.next(a.tpr);
    c2.next(a.tpr);
    c2.next(a.tpr);
    RowInfo ri = {0, 0, 0}, ri1 = {0, 0, 0};
    RowFetch fn1 = {{-1, -1}, false};
    bool gath = false;  // the current tile is gathered
    const __nv_bfloat16* src[2] = {a.q, a.q};
    bool ok[2] = {false, false};
    if (f0 < f1) {
        ri = row_info(cur.row, a);
        const RowFetch fc = fetch_rows<T, G>(a, ri, cur.row, cur.ti, lane, part);
        if (f0 + 1 < f1) {
            ri1 = c1.row != cur.row ? row_info(c1.row, a) : ri;
            fn1 = fetch_rows<T, G>(a, ri1, c1.row, c1.ti, lane, part);
        }
        gath = fc.gath;
        if (gath) resolve_rows<T, G>(a, ri, cur.row, cur.ti, lane, part, fc, src, ok);
    }
    for (long long f = f0; f < f1; ++f) {
        if (sm.abort_flag) break;
        const int jt = (int)(f - f0), st = jt % C::kStages;
        const int row = cur.row, ti = cur.ti;
        const bool seg_start = (f == f0) || (ti == 0);
        RowInfo ri2 = ri1;
        RowFetch fn2 = {{-1, -1}, false};
        if (f + 2 < f1) {
            if (c2.row != c1.row) ri2 = row_info(c2.row, a);
            fn2 = fetch_rows<T, G>(a, ri2, c2.row, c2.ti, lane, part);
        }
        if (jt >= C::kStages && !tc::mbar_wait(&sm.kv_empty[st], ((jt / C::kStages) - 1) & 1, a.wait_polls)) { fault(sm, a); break; }
        uint8_t* dst = sm.kv[st];
        if (jt != a.withhold) {  // test hook: the withheld stage never fills (no copy, no arrival)
            last_load[st] = jt;
            uint64_t mask = 0;
            if (gath) {
                mask = gather_tile<T, G>(dst, src, ok, lane, part, stream_policy);
                if (lane == 0) {
                    if (G == 1) sm.mask[st] = mask;
                    else reinterpret_cast<uint32_t*>(&sm.mask[st])[part] = (uint32_t)(mask >> (32 * part));
                    if (part == 0) tc::mbar_arrive_expect_tx(&sm.kv_full[st], 0);
                    else tc::mbar_arrive(&sm.kv_full[st]);
                }
            } else if (part > 0) {
                if (lane == 0) tc::mbar_arrive(&sm.kv_full[st]);  // part 0 loads a contiguous tile alone
            } else if (ti < a.e_tiles) {
                // HCA: rows c0 .. c0+T-1 of this sequence's entries are contiguous
                const long long c0 = (long long)ti * C::kTile;
                const long long nv = ri.nvis - c0;
                mask = nv >= C::kTile ? C::kTileMask : (nv <= 0 ? 0ull : ((1ull << nv) - 1ull));
                if (lane == 0) {
                    sm.mask[st] = mask;
                    tc::mbar_arrive_expect_tx(&sm.kv_full[st], C::kTileBytes);
                    const int y = (int)((long long)ri.b * a.n_ent + c0);
                    tc::tma_load_3d_hint(dst, ent_map, 0, y, 0, &sm.kv_full[st], stream_policy);
                }
            } else {
                // window tokens p0 .. p0+T-1 (contiguous rows of token_kv)
                const long long wi = ti - a.e_tiles;
                const long long p0 = ri.t - a.window + 1 + wi * C::kTile;
                for (int r = 0; r < C::kTile; ++r) {
                    const long long p = p0 + r;
                    if (wi * C::kTile + r < a.window && p >= 0) mask |= 1ull << r;
                }
                if (lane == 0) {
                    sm.mask[st] = mask;
                    tc::mbar_arrive_expect_tx(&sm.kv_full[st], C::kTileBytes);
                    const int y = (int)((long long)ri.b * a.l_tok + (p0 - a.tok_pos0));
                    tc::tma_load_3d_hint(dst, tok_map, 0, y, 0, &sm.kv_full[st], stream_policy);
                }
            }
            tc::cp_async_arrive_noinc(&sm.kv_full[st]);  // 32 lanes: after their cp.async copies (if any) land
        }
        // a new query's rows are on their way; its query replaces the last one's once that one's last QK is done
        if (seg_start && part == 0) {
            if (seg > 0 && !tc::mbar_wait(&sm.q_empty, (seg - 1) & 1, a.wait_polls)) { fault(sm, a); break; }
            if (lane == 0 && seg > 0) {  // the first segment's query was requested before the dependency wait
                tc::mbar_arrive_expect_tx(&sm.q_full, kQBytes);
                tc::tma_load_3d(sm.q, q_map, 0, row * kH, 0, &sm.q_full);
            }
            ++seg;
        }
        gath = fn1.gath;
        if (f + 1 < f1 && gath) resolve_rows<T, G>(a, ri1, c1.row, c1.ti, lane, part, fn1, src, ok);
        ri = ri1;
        ri1 = ri2;
        fn1 = fn2;
        cur = c1;
        c1 = c2;
        c2.next(a.tpr);
    }
    // make sure nothing this warp started is still in flight before the CTA retires (also after an abort
    // or a withheld stage: the last copies issued into each stage)
    for (int st = 0; st < C::kStages; ++st)
        if (last_load[st] >= 0) tc::mbar_wait(&sm.kv_full[st], (last_load[st] / C::kStages) & 1, a.wait_polls);
    // ... nor a query load (the first segment's was issued before the loop)
    const int q_loads = seg > 0 ? seg : (f0 < f1 ? 1 : 0);
    if (part == 0 && q_loads > 0) tc::mbar_wait(&sm.q_full, (q_loads - 1) & 1, a.wait_polls);
}

// ---------------------------------------------------------------------
// warp 1: MMA issue (one thread)
// ---------------------------------------------------------------------
// descriptor + byte offset (the start-address field counts 16-byte units)
__device__ __forceinline__ uint64_t dadd(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// O^T += V^T P^T for tile jp (its P is in shared memory)
template <int T>
__device__ void issue_pv(Smem<T>& sm, uint32_t tmem, int jp, bool first_in_seg) {
    using C = Tiles<T>;
    const int sp = jp & 1, st = jp % C::kStages;
    tc::tc_fence_after();
    // A = V^T (M = 128 d of slabs 2cc, 2cc+1; K = 16 rows), MN-major; B = P^T, K-major rows of P
    const uint64_t a0 = tc::sw128_desc(tc::smem_u32(sm.kv[st]), C::kSlabBytes, 1024);
    const uint64_t b0 = tc::sw128_desc(tc::smem_u32(sm.p[sp]), 16, 1024);
#pragma unroll
    for (int kk = 0; kk < C::kTile / 16; ++kk) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
            tc::mma_f16(tmem + kColO + 64 * cc, dadd(a0, (2 * cc) * C::kSlabBytes + kk * 2048), dadd(b0, kk * 32),
                        kIdescPV, (!first_in_seg || kk > 0) ? 1u : 0u);
    }
    tc::mma_commit(&sm.kv_empty[st]);
    tc::mma_commit(&sm.p_free[sp]);
}

// S = Q K^T for tile jq (its rows are in shared memory)
template <int T>
__device__ void issue_qk(Smem<T>& sm, uint32_t tmem, int jq, bool gathered, uint64_t q0) {
    using C = Tiles<T>;
    const int s = jq & 1, st = jq % C::kStages;
    if (gathered) tc::fence_proxy_async();  // rows gathered with cp.async become visible to the tensor core
    tc::tc_fence_after();
    const uint64_t k0 = tc::sw128_desc(tc::smem_u32(sm.kv[st]), 16, 1024);
    const uint32_t d_s = tmem + kColS + kSCols * s;
#pragma unroll
    for (int c = 0; c < kSlabs; ++c) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            tc::mma_f16(d_s, dadd(q0, c * kH * 128 + kk * 32), dadd(k0, c * C::kSlabBytes + kk * 32), C::kIdescQK,
                        (c | kk) ? 1u : 0u);
    }
    tc::mma_commit(&sm.s_full[s]);
}

// No CTA-wide progress for this many cycles (about a second) counts as a fault.
constexpr long long kStallCycles = 1LL << 31;

// Warp 1, all 32 lanes (one elected lane issues each MMA and commit; every decision below is taken
// on lane 0's view, so the warp stays converged).  The two MMA groups of every tile are issued in
// whatever order their inputs become ready: PV(j) as soon as the softmax has written P(j) (which frees
// tile j's stage for the next load early), QK(j) as soon as tile j has landed and S buffer j&1 is free
// (PV(j-2) issued).
template <int T>
__device__ void mma_issuer(Smem<T>& sm, const TcArgs& a, uint32_t tmem, long long f0, long long f1) {
    using C = Tiles<T>;
    const long long n = f1 - f0;
    const uint64_t q0 = tc::sw128_desc(tc::smem_u32(sm.q), 16, 1024);
    long long jq = 0, jp = 0;
    int segq = 0;
    bool ok = true;
    Cursor cq(f0, a.tpr), cp(f0, a.tpr);
    long long t_last = clock64();
    while (jp < n) {
        if (__shfl_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&sm.abort_flag), 0)) { ok = false; break; }
        bool progressed = false;
        if (jp < jq && tc::mbar_test_warp(&sm.p_full[jp & 1], (uint32_t)(jp >> 1) & 1)) {
            issue_pv(sm, tmem, (int)jp, jp == 0 || cp.ti == 0);
            ++jp;
            cp.next(a.tpr);
            progressed = true;
        } else if (jq < n && jp >= jq - 1) {
            const bool qseg = jq == 0 || cq.ti == 0;
            if (tc::mbar_test_warp(&sm.kv_full[jq % C::kStages], (uint32_t)(jq / C::kStages) & 1) &&
                (!qseg || tc::mbar_test_warp(&sm.q_full, segq & 1))) {
                issue_qk<T>(sm, tmem, (int)jq, tile_gathered(a, cq.ti), q0);
                if (jq == n - 1 || cq.ti == a.tpr - 1) tc::mma_commit(&sm.q_empty);  // last QK of this query
                if (qseg) ++segq;
                ++jq;
                cq.next(a.tpr);
                progressed = true;
            }
        }
        if (progressed) {
            t_last = clock64();
        } else if (__shfl_sync(0xffffffffu, (int)(clock64() - t_last > a.stall_cycles), 0)) {
            ok = false;
            break;
        }
    }
    if (!ok) fault(sm, a);
    // every MMA issued has completed before the CTA frees TMEM
    tc::mma_commit(&sm.drain);
    tc::mbar_wait(&sm.drain, 0);
}

// ---------------------------------------------------------------------
// warps 2-5: softmax, rescale, output
// ---------------------------------------------------------------------
template <int T>
__device__ void softmax_warps(Smem<T>& sm, const TcArgs& a, uint32_t tmem, long long f0, long long f1, int cta) {
    using C = Tiles<T>;
    const int sub = (threadIdx.x >> 5) & 3;  // TMEM sub-partition this warp may access
    const int lane = threadIdx.x & 31;
    // M = 64: head 16*sub + (lane & 15) lives in TMEM lane 32*sub + (lane & 15); lanes 0-15 take the
    // first 32 columns of each tile, lanes 16-31 the last 32
    const int half = lane >> 4;
    const int h = 16 * sub + (lane & 15);
    const uint32_t lane_addr = (uint32_t)(32 * sub) << 16;
    float m_run = -INFINITY, l_run = 0.f;  // l_run: this thread's half of the row sum
    bool ok = true;
    Cursor cur(f0, a.tpr);
    const int first_row = cur.row;
    for (long long f = f0; f < f1; ++f, cur.next(a.tpr)) {
        if (sm.abort_flag) { ok = false; break; }
        const int jt = (int)(f - f0), s = jt & 1, st = jt % C::kStages;
        const int row = cur.row, ti = cur.ti;
        const bool seg_start = (f == f0) || (ti == 0);
        const bool seg_end = (f == f1 - 1) || (ti == a.tpr - 1);
        if (seg_start) {
            m_run = -INFINITY;
            l_run = 0.f;
        }
        if (!tc::mbar_wait(&sm.kv_full[st], (jt / C::kStages) & 1, a.wait_polls)) { ok = false; break; }
        // this thread's kHalfRows rows of the tile: 16 from S columns [0, 32) (rows 16 half .. 16 half + 15)
        // and kHiRows from columns [32, T) (rows 32 + kHiRows half ..), the two halves of each 16x32bx2 load
        constexpr int kNR = C::kHalfRows, kHi = C::kHiRows;
        const uint64_t tmask = sm.mask[st];
        const uint32_t mask = (uint32_t)((tmask >> (16 * half)) & 0xffffu) |
                              ((uint32_t)((tmask >> (32 + kHi * half)) & ((1ull << kHi) - 1ull)) << 16);
        if (!tc::mbar_wait(&sm.s_full[s], (jt >> 1) & 1, a.wait_polls)) { ok = false; break; }
        tc::tc_fence_after();
        uint32_t r[kNR];
        tc::tmem_ld_16x32bx2_x16(tmem + lane_addr + kColS + kSCols * s, r);
        if constexpr (kHi == 16) tc::tmem_ld_16x32bx2_x16(tmem + lane_addr + kColS + kSCols * s + 32, r + 16);
        else tc::tmem_ld_16x32bx2_x8(tmem + lane_addr + kColS + kSCols * s + 32, r + 16);
        tc::tmem_ld_wait();
        float alpha = 1.f;
        bool rescale = false;
        uint32_t pk[kNR / 2];  // bf16 pairs of this thread's probabilities
        {
            // independent partial maxima / sums keep the dependent chains short
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < kNR; ++i) {
                const float x = ((mask >> i) & 1) ? __uint_as_float(r[i]) * a.scale_log2 : -INFINITY;
                r[i] = __float_as_uint(x);
                mx4[i & 3] = fmaxf(mx4[i & 3], x);
            }
            float mt = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));  // both halves of the row
            if (mt > m_run + kRescaleSlack) {
                if (m_run != -INFINITY) {
                    alpha = exp2f(m_run - mt);
                    rescale = true;
                    l_run *= alpha;
                }
                m_run = mt;
            }
            const float msub = m_run == -INFINITY ? 0.f : m_run;  // all-masked so far: every x is -inf
            float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < kNR / 2; ++i) {
                const float p0 = exp2f(__uint_as_float(r[2 * i]) - msub);
                const float p1 = exp2f(__uint_as_float(r[2 * i + 1]) - msub);
                const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                ls4[i & 3] += __low2float(pb) + __high2float(pb);
                pk[i] = *reinterpret_cast<const uint32_t*>(&pb);
            }
            l_run += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
            if (half == 0) {
                sm.alpha[s][h] = alpha;
                if (rescale) sm.rescale_tag[s] = jt + 1;
            }
        }
        // the P buffer of this parity is free once PV two tiles back is done
        if (jt >= 2 && !tc::mbar_wait(&sm.p_free[s], ((jt >> 1) - 1) & 1, a.wait_polls)) { ok = false; break; }
        tc::named_barrier(1, 128);
        if (sm.rescale_tag[s] == jt + 1) {
            // O^T (lanes = d, columns = heads) was accumulated with the old maxima
            if (!tc::mbar_wait(&sm.p_free[(jt - 1) & 1], ((jt - 1) >> 1) & 1, a.wait_polls)) { ok = false; break; }
            tc::tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t o[64];
                tc::tmem_ld_x64(tmem + lane_addr + kColO + 64 * cc, o);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 64; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * sm.alpha[s][i]);
                tc::tmem_st_x64(tmem + lane_addr + kColO + 64 * cc, o);
            }
            tc::tmem_st_wait();
        }
        {
            // head h's row of P: the tile's probabilities as one 128 B swizzled row (the first 2 T bytes
            // used); this thread writes the 16-byte chunks of its rows: 8-row chunks 2 half, 2 half + 1 (rows
            // 16 half ..) and then 4 + (kHi / 8) half .. (rows 32 + kHi half ..)
            uint8_t* prow = sm.p[s] + (h >> 3) * 1024 + (h & 7) * 128;
#pragma unroll
            for (int u = 0; u < kNR / 8; ++u) {
                const int chunk = u < 2 ? 2 * half + u : 4 + (kHi / 8) * half + (u - 2);
                *reinterpret_cast<uint4*>(prow + ((chunk ^ (h & 7)) << 4)) =
                    make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
            }
        }
        tc::fence_proxy_async();
        tc::tc_fence_before();
        tc::mbar_arrive(&sm.p_full[s]);

        if (seg_end) {
            if (!tc::mbar_wait(&sm.p_free[s], (jt >> 1) & 1, a.wait_polls)) { ok = false; break; }
            tc::tc_fence_after();
            const float l_row = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
            const long long rs = (long long)row * a.tpr;
            const bool whole = (rs >= f0) && (rs + a.tpr <= f1);
            if (half == 0 && whole) {
                // a whole row is normalised here: the sink joins its denominator (a split row's in the combine)
                const float l = l_row + ((a.sink && m_run != -INFINITY)
                                             ? exp2f(a.sink[h] * 1.4426950408889634f - m_run) : 0.f);
                sm.inv_l[h] = l > 0.f ? 1.f / l : 0.f;  // an empty row stays zero
            }
            tc::named_barrier(1, 128);
            // a piece of a split query: slot 2c for the CTA's first query, 2c+1 for its last
            const int slot = 2 * cta + (row == first_row ? 0 : 1);
            float* dst;
            if (whole) {
                dst = a.out + (long long)row * kH * kD;
            } else {
                dst = a.part_o + (long long)slot * kH * kD;
                if (half == 0) {
                    a.part_ml[((long long)slot * kH + h) * 2] = m_run;
                    a.part_ml[((long long)slot * kH + h) * 2 + 1] = l_row;
                }
            }
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t o[64];
                tc::tmem_ld_x64(tmem + lane_addr + kColO + 64 * cc, o);
                tc::tmem_ld_wait();
                const int d = 128 * cc + 32 * sub + lane;
                if (whole) {
                    // output RoPE: dims d and d ^ 1 are a pair held by neighbouring lanes
                    const bool rot = a.rope_dims > 0;
                    float rs_ = 0.f, rc_ = 1.f;
                    if (rot && d >= kD - a.rope_dims)
                        rope_sincos(a.ctx_len - a.n_q + (row % a.n_q), (d - (kD - a.rope_dims)) >> 1, a.rope_dims,
                                    a.rope_base, &rs_, &rc_);
#pragma unroll
                    for (int i = 0; i < kH; ++i) {
                        float v = __uint_as_float(o[i]) * sm.inv_l[i];
                        if (rot) {
                            const float p = __shfl_xor_sync(0xffffffffu, v, 1);
                            if (d >= kD - a.rope_dims) v = rope_apply(d, v, p, rs_, rc_);
                        }
                        o[i] = __float_as_uint(v);
                    }
                    // out[row][h][d]: lanes 4q .. 4q+3 exchange their 4 x 4 blocks (heads 4g .. 4g+3 at dims
                    // d - j .. d - j + 3, j = lane % 4) in two xor steps, so that lane 4q + j holds head 4g + j
                    // at those 4 dims: one 16-byte store per head group instead of four 4-byte ones
                    const int j = lane & 3;
#pragma unroll
                    for (int g = 0; g < kH / 4; ++g) {
                        float x[4] = {__uint_as_float(o[4 * g]), __uint_as_float(o[4 * g + 1]),
                                      __uint_as_float(o[4 * g + 2]), __uint_as_float(o[4 * g + 3])};
#pragma unroll
                        for (int msk = 1; msk <= 2; msk <<= 1) {
                            const bool hi = (j & msk) != 0;
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                if (k & msk) continue;
                                const float send = hi ? x[k] : x[k + msk];
                                const float recv = __shfl_xor_sync(0xffffffffu, send, msk);
                                if (hi) x[k] = recv;
                                else x[k + msk] = recv;
                            }
                        }
                        // streaming store: the output is not read again here, so it should not push the
                        // entries that other queries gather out of L2
                        __stcs(reinterpret_cast<float4*>(dst + (4 * g + j) * kD + (d - j)), make_float4(x[0], x[1], x[2], x[3]));
                    }
                } else {
                    // a piece is stored in the order the threads hold it (piece layout): one warp store
                    // writes 512 contiguous bytes, heads 4i .. 4i+3 of this warp's 32 dims
                    float4* pd = reinterpret_cast<float4*>(dst) + (long long)(4 * cc + sub) * (16 * 32) + lane;
#pragma unroll
                    for (int i = 0; i < kH / 4; ++i)
                        pd[32 * i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                                 __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
                }
            }
            tc::tc_fence_before();
            tc::named_barrier(1, 128);
        }
    }
    if (!ok || sm.abort_flag) {
        fault(sm, a);
        // poison every output this CTA contributes to
        const int r0 = (int)(f0 / a.tpr), r1 = f1 > f0 ? (int)((f1 - 1) / a.tpr) : r0 - 1;
        const int t = threadIdx.x - 64;
        for (int rr = r0; rr <= r1; ++rr)
            for (int i = t; i < kH * kD; i += 128) a.out[(long long)rr * kH * kD + i] = NAN;
        for (int i = t; i < 2 * kH * 2; i += 128) a.part_ml[(long long)2 * cta * kH * 2 + i] = NAN;
    }
}

template <int T, int G>
__global__ void __launch_bounds__(threads_for<G>(), 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap ent_map, const __grid_constant__ CUtensorMap tok_map,
                     const __grid_constant__ CUtensorMap q_map, TcArgs a) {
    using C = Tiles<T>;
    extern __shared__ uint8_t smem_raw[];
    Smem<T>& sm = *reinterpret_cast<Smem<T>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int cta = blockIdx.x;
    const long long f0 = range_start(cta, a), f1 = range_start(cta + 1, a);

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            tc::mbar_init(&sm.kv_full[i], 33 * G);  // per loading warp: lane 0's arrival + 32 cp.async arrivals
            tc::mbar_init(&sm.kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&sm.s_full[i], 1);
            tc::mbar_init(&sm.p_full[i], 128);
            tc::mbar_init(&sm.p_free[i], 1);
        }
        tc::mbar_init(&sm.q_full, 1);
        tc::mbar_init(&sm.q_empty, 1);
        tc::mbar_init(&sm.drain, 1);
        sm.rescale_tag[0] = sm.rescale_tag[1] = 0;
        sm.abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (warp == 0 && (threadIdx.x & 31) == 0 && f0 < f1) early_loads(sm, a, &ent_map, &q_map, f0, f1);
    griddep_wait();  // the prologue above touched only shared and tensor memory (and read the query)
    // No early griddep_launch_dependents here: the next kernel (the combine, or the next call) is let
    // in as this grid's CTAs exit, so its blocks spread over every SM instead of packing onto the first
    // SMs to free up (measured on B200: the 32-query combine ran 1.8 us faster, the step 2 us faster).
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0 || warp == 6) {
        producer<T, G>(sm, a, &ent_map, &tok_map, &q_map, f0, f1, warp == 0 ? 0 : 1);
    } else if (warp == 1) {
        mma_issuer(sm, a, tmem, f0, f1);
    } else {
        softmax_warps(sm, a, tmem, f0, f1, cta);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// Merge the partials of queries whose tiles were split between CTAs.
// grid (rows, 16 groups of 32 dims), 256 threads, a.comb_pieces * 64 floats of dynamic shared memory
// (at least the pieces of any query).  The per-head weights exp2(m_piece - m_max) come first, from
// four groups of 64 threads each taking every fourth piece.  Then warp w sums heads 4w .. 4w+3 and
// 4w+32 .. 4w+35 of the block's 32 dims (lane = dim) over the pieces: per piece two float4 loads, each
// warp-wide load one 512-byte run of the piece (piece layout), up to kU pieces in flight.  The sums
// are scaled by 1 / l and written to out[row][h][d], 32 consecutive dims (128 bytes) per warp store.
// KU: pieces whose loads are in flight together.  8 for a few queries with many pieces each (CSA decode:
// up to 18), 4 for many queries with few pieces (fewer registers, more blocks resident).
template <int KU>
__global__ void __launch_bounds__(256) attend_tc_combine(TcArgs a) {
    griddep_wait();  // everything before this kernel on the stream has finished
    griddep_launch_dependents();
    constexpr int kU = KU;
    const int row = blockIdx.x, dg = blockIdx.y;
    const long long rs = (long long)row * a.tpr, re = rs + a.tpr - 1;
    // CTA holding flat tile f: the largest c with range_start(c) <= f
    auto cta_of = [&](long long f) { return (int)(((f + 1) * a.grid - 1) / a.total_tiles); };
    const int c0 = cta_of(rs), c1 = cta_of(re);
    if (c0 == c1) return;  // written directly by its only CTA
    // the first CTA's piece is its first query only if the query starts its range; every later CTA's
    // range starts inside this query, so the piece is that CTA's first (slot 2c)
    const int n = c1 - c0 + 1;
    if (n > a.comb_pieces) {  // the host's bound on pieces per query does not hold
        if (threadIdx.x == 0 && a.dev_status) atomicExch(a.dev_status, (int)V4A_ERR_DEVICE_FAULT);
        return;
    }
    extern __shared__ __align__(16) float s_w[];  // [n][64]: weight of piece i for head h
    __shared__ int s_slot[kNumSMs + kU];
    __shared__ float s_red[4][kH];
    __shared__ __align__(16) float s_inv[kH];
    const int t = threadIdx.x, g = t >> 6, h = t & (kH - 1);
    for (int i = t; i < n; i += blockDim.x)
        s_slot[i] = 2 * (c0 + i) + ((i == 0 && range_start(c0, a) < rs) ? 1 : 0);
    __syncthreads();
    // per head: the largest piece max, then the weights and the total l; NaN anywhere poisons the head
    const float2* ml = reinterpret_cast<const float2*>(a.part_ml);  // [slot][64] of (m, l)
    bool bad = false;
    float mg = -INFINITY;
#pragma unroll 4
    for (int i = g; i < n; i += 4) {
        const float m = ml[(long long)s_slot[i] * kH + h].x;
        bad |= isnan(m);
        mg = fmaxf(mg, m);
    }
    s_red[g][h] = bad ? NAN : mg;
    __syncthreads();
    float mmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float x = s_red[j][h];
        bad |= isnan(x);
        mmax = fmaxf(mmax, x);
    }
    float lg = 0.f;
#pragma unroll 4
    for (int i = g; i < n; i += 4) {
        const float2 p = ml[(long long)s_slot[i] * kH + h];
        bad |= isnan(p.y);
        const float wgt = (p.x != -INFINITY && mmax != -INFINITY) ? exp2f(p.x - mmax) : 0.f;
        s_w[i * kH + h] = wgt;
        lg += wgt * p.y;
    }
    __syncthreads();  // every group has read s_red
    s_red[g][h] = bad ? NAN : lg;
    __syncthreads();
    if (t < kH) {
        float l = (s_red[0][h] + s_red[1][h]) + (s_red[2][h] + s_red[3][h]);
        if (a.sink && mmax != -INFINITY) l += exp2f(a.sink[h] * 1.4426950408889634f - mmax);  // the sink's share
        s_inv[h] = isnan(l) ? NAN : (l > 0.f ? 1.f / l : 0.f);  // an empty row stays zero
    }
    __syncthreads();  // s_w and s_inv are written
    // thread (warp w, lane): dim 32 dg + lane, head quads w and w + 8 (a piece of weight 0 holds finite
    // values: it adds 0)
    const int w = t >> 5, lane = t & 31, d = 32 * dg + lane;
    const float4* src = reinterpret_cast<const float4*>(a.part_o) + (long long)dg * (16 * 32) + lane;
    float4 acc[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
    for (int i0 = 0; i0 < n; i0 += kU) {
        float4 v[kU][2];
#pragma unroll
        for (int u = 0; u < kU; ++u)
#pragma unroll
            for (int r = 0; r < 2; ++r)
                v[u][r] = i0 + u < n ? __ldcg(src + (long long)s_slot[i0 + u] * (kH * kD / 4) + 32 * (w + 8 * r))
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (i0 + u >= n) break;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const float4 wt = *reinterpret_cast<const float4*>(s_w + (i0 + u) * kH + 4 * (w + 8 * r));
                acc[r].x = fmaf(wt.x, v[u][r].x, acc[r].x);
                acc[r].y = fmaf(wt.y, v[u][r].y, acc[r].y);
                acc[r].z = fmaf(wt.z, v[u][r].z, acc[r].z);
                acc[r].w = fmaf(wt.w, v[u][r].w, acc[r].w);
            }
        }
    }
    // out[row][h][d] (output RoPE: the pair partner of d is d ^ 1, the neighbouring lane)
    const bool rot = a.rope_dims > 0 && d >= kD - a.rope_dims;
    float rs_ = 0.f, rc_ = 1.f;
    if (rot)
        rope_sincos(a.ctx_len - a.n_q + (row % a.n_q), (d - (kD - a.rope_dims)) >> 1, a.rope_dims, a.rope_base, &rs_,
                    &rc_);
    float* orow = a.out + (long long)row * kH * kD + d;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int h0 = 4 * (w + 8 * r);
        const float4 inv = *reinterpret_cast<const float4*>(s_inv + h0);  // NaN for a poisoned head
        const float vals[4] = {acc[r].x * inv.x, acc[r].y * inv.y, acc[r].z * inv.z, acc[r].w * inv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float vv = vals[j];
            const float pp = __shfl_xor_sync(0xffffffffu, vv, 1);
            if (rot) vv = rope_apply(d, vv, pp, rs_, rc_);
            orow[(long long)(h0 + j) * kD] = vv;
        }
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// [rows][512] bf16 viewed as (64 columns, rows, 8 slabs of 64 columns): the row stride is 1 KB and the
// slab stride 128 bytes, so every address the view reaches lies inside the [rows][512] array.  One box of
// 64 columns x box_rows rows x 8 slabs lands in shared memory as 8 slabs of box_rows 128-byte rows, the
// tile layout (128-byte swizzle), in one TMA instruction.
bool make_map(CUtensorMap* map, const void* base, long long rows, int box_rows) {
    auto fn = encode_fn();
    if (!fn || rows < 1) return false;
    cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)kSlabs};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, 128};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)kSlabs};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct TcPlan {
    int tile;  // rows per tile: 48 for rows of more than 2,048 candidates, else 64 (see Tiles)
    int e_tiles, w_tiles, tpr, grid;
    long long total;
};

TcPlan tc_plan(const AttendArgs& a) {
    TcPlan p;
    const long long n_sel_max = a.idx ? (long long)a.k : (a.ctx_len / a.m < a.n_ent ? a.ctx_len / a.m : a.n_ent);
    p.tile = n_sel_max > 2048 ? 48 : 64;
    p.e_tiles = (int)((n_sel_max + p.tile - 1) / p.tile);
    p.w_tiles = (a.window + p.tile - 1) / p.tile;
    p.tpr = p.e_tiles + p.w_tiles;
    p.total = (long long)a.batch * a.n_q * p.tpr;
    p.grid = (int)(p.total < kNumSMs ? p.total : kNumSMs);
    return p;
}

}  // namespace

AttendFaultTest g_test_fault = {-1, 0, 0};

bool attend_tc_shape_ok(const AttendArgs& a) {
    if (a.dtype != V4A_BF16 || a.d != kD || a.heads != kH) return false;
    TcPlan p = tc_plan(a);
    if (p.tpr < 1 || p.grid < 1) return false;
    if ((long long)a.batch * a.n_ent >= (1LL << 31) || (long long)a.batch * a.l_tok >= (1LL << 31)) return false;
    if (a.bt && a.pool_rows >= (1LL << 31)) return false;
    if ((long long)a.batch * a.n_q * kH >= (1LL << 31)) return false;
    return true;
}

bool attend_tc_available(const AttendArgs& a) { return attend_tc_shape_ok(a) && encode_fn() != nullptr; }

size_t attend_tc_workspace_bytes(const AttendArgs& a) {
    TcPlan p = tc_plan(a);
    size_t slots = 2 * (size_t)p.grid;
    size_t ml = (slots * kH * 2 * sizeof(float) + 255) / 256 * 256;
    return ml + slots * kH * kD * sizeof(float);
}

cudaError_t launch_attend_tc(const AttendArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (ws_bytes < attend_tc_workspace_bytes(a)) return cudaErrorInvalidValue;
    TcPlan p = tc_plan(a);
    CUtensorMap ent_map, tok_map, q_map;
    const long long ent_rows = a.bt ? a.pool_rows : (long long)a.batch * a.n_ent;
    const long long tok_rows = (long long)a.batch * (a.ring_rows > 0 ? a.ring_rows : a.l_tok);
    const void* tok = a.token_kv ? a.token_kv : a.q;  // a window of 0 never reads it
    if (!make_map(&tok_map, tok, a.token_kv ? tok_rows : (long long)a.batch * a.n_q * kH, p.tile))
        return cudaErrorInvalidValue;
    if (ent_rows > 0) {
        if (!make_map(&ent_map, a.entries, ent_rows, p.tile)) return cudaErrorInvalidValue;
    } else {
        ent_map = tok_map;  // no entry tiles exist
    }
    if (!make_map(&q_map, a.q, (long long)a.batch * a.n_q * kH, kH)) return cudaErrorInvalidValue;

    TcArgs t;
    t.q = static_cast<const __nv_bfloat16*>(a.q);
    t.entries = static_cast<const __nv_bfloat16*>(a.entries);
    t.token_kv = static_cast<const __nv_bfloat16*>(tok);
    t.idx = a.idx;
    t.out = a.out;
    const size_t slots = 2 * (size_t)p.grid;
    t.part_ml = static_cast<float*>(ws);
    t.part_o = reinterpret_cast<float*>(static_cast<char*>(ws) + (slots * kH * 2 * sizeof(float) + 255) / 256 * 256);
    t.dev_status = a.dev_status;
    t.n_ent = a.n_ent;
    t.l_tok = a.l_tok;
    t.tok_pos0 = a.tok_pos0;
    t.ctx_len = a.ctx_len;
    t.total_tiles = p.total;
    t.rows = a.batch * a.n_q;
    t.n_q = a.n_q;
    t.m = a.m;
    t.k = a.idx ? a.k : 0;
    t.window = a.window;
    t.e_tiles = p.e_tiles;
    t.w_tiles = p.w_tiles;
    t.tpr = p.tpr;
    t.grid = p.grid;
    t.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
    t.sink = a.sink;
    t.rope_dims = a.rope_dims;
    t.rope_base = a.rope_base;
    t.wait_polls = g_test_fault.withhold >= 0 ? g_test_fault.wait_polls : tc::kWaitPolls;
    t.stall_cycles = g_test_fault.withhold >= 0 ? g_test_fault.stall_cycles : kStallCycles;
    t.withhold = g_test_fault.withhold;
    t.bt = a.bt;
    t.bt_stride = a.bt_stride;
    t.epb = a.epb;
    t.n_blocks = a.epb > 0 ? a.pool_rows / a.epb : 0;
    t.ring_rows = a.ring_rows;
    {
        // CTA c covers flat tiles [c T / G, (c+1) T / G), at least floor(T / G) of them, so a query's tpr
        // tiles meet at most ceil(tpr / floor(T / G)) + 1 CTAs
        const long long per = p.total / p.grid;
        const long long bound = (p.tpr + per - 1) / per + 1;
        t.comb_pieces = (int)(bound < p.grid ? bound : p.grid);
    }

    auto go = [&](auto kernel, size_t smem, int threads) {
        cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err == cudaSuccess)
            err = launch_pdl(kernel, dim3(p.grid), dim3(threads), smem, stream, ent_map, tok_map, q_map, t);
        return err == cudaSuccess ? cudaGetLastError() : err;
    };
    static_assert(sizeof(Smem<48>) + 1024 <= 232448 && sizeof(Smem<64>) + 1024 <= 232448, "shared memory");
    // tiles gathered row by row get a second loading warp
    const bool gathered = a.idx != nullptr || a.bt != nullptr || a.ring_rows > 0;
    cudaError_t e;
    if (p.tile == 48)
        e = gathered ? go(attend_tc_kernel<48, 2>, sizeof(Smem<48>) + 1024, threads_for<2>())
                     : go(attend_tc_kernel<48, 1>, sizeof(Smem<48>) + 1024, threads_for<1>());
    else
        e = gathered ? go(attend_tc_kernel<64, 2>, sizeof(Smem<64>) + 1024, threads_for<2>())
                     : go(attend_tc_kernel<64, 1>, sizeof(Smem<64>) + 1024, threads_for<1>());
    if (e != cudaSuccess) return e;
    if (p.grid > 1) {
        const size_t csm = (size_t)t.comb_pieces * kH * sizeof(float);
        e = t.comb_pieces > 8 ? launch_pdl(attend_tc_combine<8>, dim3(t.rows, kD / 32), dim3(256), csm, stream, t)
                              : launch_pdl(attend_tc_combine<4>, dim3(t.rows, kD / 32), dim3(256), csm, stream, t);
        if (e == cudaSuccess) e = cudaGetLastError();
    }
    return e;
}

}  // namespace v4a
