/*
 * v4a.h -- C ABI of libv4a.so: the compressed-attention step of DeepSeek-V4
 * (CSA = compressed sparse attention, HCA = heavily compressed attention,
 * plus the raw sliding window) as hand-written CUDA kernels for sm_100a.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers named in the argument lists are DEVICE pointers unless said
 *    otherwise.  The caller owns every buffer; the library never allocates,
 *    frees or synchronises.  Scratch memory ("workspace") is passed in; its
 *    size comes from v4a_workspace_size().
 *  - Every call only enqueues work on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) and returns V4A_OK once the work is enqueued.
 *    Argument errors are found on the host, before anything is enqueued, and
 *    return V4A_ERR_INVALID_ARG or V4A_ERR_UNSUPPORTED; v4a_last_error()
 *    then holds a one-line reason (per host thread).  A failed launch returns
 *    V4A_ERR_CUDA.  Kernels never trap: data-dependent faults (an index out of
 *    range) are skipped and reported through a device status word.
 *  - Layouts are dense and row-major, innermost dimension last.  Sizes are in
 *    elements unless they say bytes.
 *  - Positions.  A sequence's context holds ctx_len tokens (positions
 *    0 .. ctx_len-1).  The n_q query tokens are the LAST n_q positions,
 *    t = ctx_len - n_q + j for query j (decode: n_q = 1, t = ctx_len - 1).
 *  - Compressed entries.  With compression rate m, entry s summarises tokens
 *    [m*s, m*s + m) and every sequence holds N = floor(ctx_len / m) entries
 *    (only complete chunks are compressed).  Entry s is visible to query
 *    position t iff m*(s+1) <= t+1, i.e. N_vis(t) = floor((t+1)/m): a query
 *    never reads its own incomplete block ("1M Context != Lossless Long
 *    Memory", section 6.1).
 *  - Sliding window.  Query t also attends to the raw tokens (t-W, t],
 *    clipped at 0 (same page, section 6; W = n_win = 128 in V4).  Window rows
 *    come from a token_kv buffer [batch][l_tok][d] whose row r holds position
 *    tok_pos0 + r; it must cover every query's window.
 *  - K = V.  One compressed vector per entry (and one vector per window
 *    token) serves as key and value for every query head ("DeepSeek-V4:
 *    Million-Token Context via Hybrid Compressed Attention", CSA "Core
 *    attention with shared KV MQA").
 */
#ifndef V4A_H
#define V4A_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define V4A_API __attribute__((visibility("default")))
#else
#define V4A_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum v4a_status {
    V4A_OK = 0,
    V4A_ERR_INVALID_ARG = 1,  /* a pointer, size or layout the call cannot take */
    V4A_ERR_UNSUPPORTED = 2,  /* a valid combination this build has no kernel for */
    V4A_ERR_CUDA = 3,         /* the CUDA runtime refused a launch */
    V4A_ERR_DEVICE_FAULT = 4  /* written to a device status word: bad data found by a kernel */
} v4a_status;

typedef enum v4a_dtype {
    V4A_F32 = 0,      /* IEEE binary32 */
    V4A_BF16 = 1,     /* bfloat16 */
    V4A_FP8E4M3 = 2,  /* float8 e4m3 ("fn": no inf, max 448), with one fp32 scale per row */
    V4A_MXFP4 = 3     /* OCP Microscaling MXFP4: e2m1 codes (1 sign, 2 exponent bits with bias 1,
                         1 fraction bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6), two per byte with element 2i
                         in the low nibble of byte i, and one E8M0 exponent byte e per 32
                         consecutive elements of a row, scaling them by 2^(e-127) (e = 255 is NaN) */
} v4a_dtype;

/* Problem shape.  Fields an entry point does not use are ignored. */
typedef struct v4a_shape {
    int batch;          /* B: independent sequences */
    int n_q;            /* T: query tokens per sequence (the last T positions) */
    int heads;          /* H: attention query heads */
    int d;              /* K = V vector dimension */
    int m;              /* compression rate (4 for CSA, 128 for HCA) */
    int k;              /* top-k: entries selected per query (CSA) */
    int window;         /* W: sliding-window length (0 = no window) */
    long long ctx_len;  /* L: tokens in each sequence's context */
} v4a_shape;

/* ------------------------------------------------------------------ */
/* compression                                                          */
/* ------------------------------------------------------------------ */

/* One stream of token rows to compress.  Rows are `channels` wide; row 0 of
 * x and gate is the first token of the first chunk, row 0 of out the entry it
 * produces.  Each sequence's rows start *_batch_stride elements apart. */
typedef struct v4a_compress_io {
    const void* x;                /* content rows [batch][n_tok][channels], in_dtype */
    const void* gate;             /* gate logits, same shape, in_dtype */
    void* out;                    /* entries [batch][n_tok/m][channels], out_dtype */
    float* out_scale;             /* [batch][n_tok/m] per-entry scale; required iff out_dtype == FP8E4M3 */
    int channels;                 /* multiple of 8; <= 256 for FP8E4M3 output */
    v4a_dtype in_dtype;           /* F32 or BF16 */
    v4a_dtype out_dtype;          /* F32, BF16 or FP8E4M3 */
    long long x_batch_stride;     /* elements between sequences in x (>= n_tok*channels) */
    long long gate_batch_stride;  /* elements between sequences in gate */
    long long out_batch_stride;   /* elements between sequences in out (MXFP4: even; bytes = elements/2) */
    long long scale_batch_stride; /* floats between sequences in out_scale */
    uint8_t* out_exp;             /* [batch][n_tok/m][channels/32] E8M0 block exponents; required iff
                                     out_dtype == MXFP4 */
    long long exp_batch_stride;   /* bytes between sequences in out_exp */
} v4a_compress_io;

/* Chunk compression ("DeepSeek-V4 的暗线之一：分层记忆比输入框更关键",
 * section 3; "DeepSeek-V4: Million-Token Context ...", HCA "How it works"):
 * for every complete chunk s of m tokens and every channel c,
 *     out[s][c] = sum_{i<m} softmax_i(gate[m*s+i][c]) * x[m*s+i][c],
 * the softmax running over the chunk's tokens separately for each channel.
 * The same single-series rule serves m = 4 (CSA) and m' = 128 (HCA).
 * FP8E4M3 output stores, per entry, scale = amax/448 (1 for an all-zero
 * entry) in out_scale and each value as the nearest e4m3 code of
 * value/scale (ties to even, saturating).  MXFP4 output quantises each
 * block of 32 channels as v4a_quantize_mxfp4 does (channels a multiple of
 * 32; codes in out, exponents in out_exp).
 * kv: the K=V stream (required).  idx: the indexer-key stream compressed in
 * the same launch (may be NULL); it uses the same batch, n_tok and m.
 * n_tok: tokens per sequence; a trailing partial chunk is ignored.
 * Errors: V4A_ERR_INVALID_ARG for a NULL required pointer, m < 1, n_tok < 0,
 * channels not a multiple of 8, strides too small, misaligned pointers
 * (x/gate/out need 16-byte alignment); V4A_ERR_UNSUPPORTED for other dtype
 * combinations. */
V4A_API v4a_status v4a_compress(const v4a_compress_io* kv, const v4a_compress_io* idx, int batch, long long n_tok, int m,
                        void* stream);

/* Series b of the dual-series compressor: its rows over the same token range
 * as series a (the x / gate of the v4a_compress_io passed with it), and over
 * the m tokens just before that range. */
typedef struct v4a_series_b {
    const void* x;                 /* content rows [batch][n_tok][channels], series a's in_dtype */
    const void* gate;              /* gate logits, same shape and dtype */
    const void* prev_x;            /* rows of the block before the range [batch][m][channels], or NULL
                                      when the range starts the sequence */
    const void* prev_gate;         /* same shape; NULL exactly when prev_x is NULL */
    long long x_batch_stride;      /* elements between sequences in x (>= n_tok*channels) */
    long long gate_batch_stride;   /* elements between sequences in gate */
    long long prev_batch_stride;   /* elements between sequences in prev_x and prev_gate (>= m*channels) */
} v4a_series_b;

/* Dual-series chunk compression ("DeepSeek-V4: Million-Token Context via
 * Hybrid Compressed Attention", CSA, "Dual-series KV compression"): entry s
 * of the range mixes 2m token rows, the m of series a in block s and the m
 * of series b in block s-1, under one softmax per channel over their 2m
 * gate logits:
 *     out[s][c] = ( sum_{i<m} e^{Za[ms+i][c]} Xa[ms+i][c]
 *                 + sum_{i<m} e^{Zb[m(s-1)+i][c]} Xb[m(s-1)+i][c] ) / (same sums of e^Z),
 * with block -1 of the range read from b->prev_x / prev_gate, and left out
 * when those are NULL (the first entry of a sequence).
 * a: series a, the output and its dtype, exactly as for v4a_compress (out,
 * out_scale, FP8E4M3 rule).  b: series b.  n_tok: tokens per sequence in the
 * range, which starts at a chunk boundary; a trailing partial chunk is
 * ignored.  Errors: those of v4a_compress, plus V4A_ERR_INVALID_ARG for a
 * NULL b->x / b->gate, exactly one of prev_x / prev_gate NULL, strides too
 * small or misaligned series-b pointers (16 bytes). */
V4A_API v4a_status v4a_compress_dual(const v4a_compress_io* a, const v4a_series_b* b, int batch, long long n_tok,
                                     int m, void* stream);

/* ------------------------------------------------------------------ */
/* Lightning indexer and top-k                                          */
/* ------------------------------------------------------------------ */

/* MXFP4 quantisation (the OCP Microscaling v1.0 conversion; the FP4 indexer
 * keys of "1M Context != Lossless Long Memory", section 4.2 and footnote 3,
 * whose bit format the pages leave open).  Each row of x [rows][cols] (dtype
 * F32 or BF16, cols a multiple of 32) is cut into blocks of 32; a block with
 * largest magnitude amax gets X = max(floor(log2(amax)) - 2, -127) (-127 for
 * an all-zero block), exps[row][block] = X + 127, and element v the nearest
 * e2m1 code of v / 2^X (ties to the even code, magnitudes above 6 clamp to
 * 6, the sign bit kept even when the magnitude rounds to 0).
 * codes: [rows][cols/2] bytes; exps: [rows][cols/32] bytes.  Inputs are
 * taken to be finite.  Errors: V4A_ERR_INVALID_ARG for NULL pointers,
 * rows < 0, cols not a positive multiple of 32, x not 16-byte aligned or
 * codes not 4-byte aligned; V4A_ERR_UNSUPPORTED for another dtype. */
V4A_API v4a_status v4a_quantize_mxfp4(const void* x, v4a_dtype dtype, long long rows, int cols, uint8_t* codes,
                                      uint8_t* exps, void* stream);

/* Indexer scores ("How V4 makes a million-token context actually
 * affordable", Lightning-Indexer section):
 *     I(t,s) = scale[s] * sum_{j<heads_i} w[j] * ReLU(q_i[j] . k_i[s]),
 * for every entry s < N_vis(t); -inf for entries not yet visible.
 * q_i: [batch][n_q][heads_i][d_i] (q_dtype F32 or BF16);
 * w:   [batch][n_q][heads_i] fp32;
 * k_i: [batch][N][d_i], N = ctx_len/m (k_dtype F32, BF16 or FP8E4M3);
 * k_scale: [batch][N] fp32, required for FP8E4M3 keys, else NULL (= 1);
 * scores: [batch][n_q][N] fp32 output.
 * Uses shape->batch, n_q, m, ctx_len.  This entry point materialises every
 * score and exists for inspection and tests; v4a_topk never does. */
V4A_API v4a_status v4a_index_scores(const void* q_i, const float* w, const void* k_i, const float* k_scale, float* scores,
                            int heads_i, int d_i, v4a_dtype q_dtype, v4a_dtype k_dtype, const v4a_shape* shape,
                            void* stream);

/* Indexer + top-k select ("1M Context != Lossless Long Memory", section
 * 4.2: the query attends only to the k best-scoring entries).  For each
 * query, the min(k, N_vis) visible entries with the largest I(t,s), ties
 * going to the lower entry index, are written to idx_out [batch][n_q][k]
 * (int32) in ASCENDING entry order, padded with -1.  score_out (nullable)
 * [batch][n_q][k] receives each selected entry's fp32 score (-inf for
 * padding).  Arguments as v4a_index_scores; workspace of
 * v4a_workspace_size("topk", shape, heads_i, d_i) bytes.  Uses
 * shape->batch, n_q, m, k, ctx_len.  Errors: k < 1 or k > 4096. */
V4A_API v4a_status v4a_topk(const void* q_i, const float* w, const void* k_i, const float* k_scale, int32_t* idx_out,
                    float* score_out, int heads_i, int d_i, v4a_dtype q_dtype, v4a_dtype k_dtype, void* workspace,
                    size_t workspace_bytes, const v4a_shape* shape, void* stream);

/* Indexer scores and top-k with FP4 keys and FP4 dot products ("1M Context
 * != Lossless Long Memory", section 4.2: indexer KV in FP4, FP4 dot
 * products; "DeepSeek-V4: Million-Token Context ...", "Where It Breaks":
 * the FP4 QK indexer).  Keys are MXFP4: k_codes [batch][N][d_i/2] and
 * k_exp [batch][N][d_i/32] as v4a_quantize_mxfp4 writes them.  The query of
 * every indexer head (d_i values, F32 or BF16) is quantised to MXFP4 the same
 * way inside the call, and
 *     I(t,s) = sum_{j<heads_i} w[j] * ReLU(qhat_j . khat_s)
 * with qhat, khat the decoded MXFP4 values: the products of e2m1 codes are
 * exact, each 32-element block's partial sum is exact, and the blocks'
 * powers of two are applied in fp32.  There is no per-entry k_scale.
 * Otherwise arguments, results, workspace (v4a_workspace_size("topk", ...))
 * and errors are those of v4a_index_scores / v4a_topk; d_i must be a
 * multiple of 32, k_codes 16-byte and k_exp 4-byte aligned. */
V4A_API v4a_status v4a_index_scores_mxfp4(const void* q_i, const float* w, const uint8_t* k_codes,
                                          const uint8_t* k_exp, float* scores, int heads_i, int d_i,
                                          v4a_dtype q_dtype, const v4a_shape* shape, void* stream);
V4A_API v4a_status v4a_topk_mxfp4(const void* q_i, const float* w, const uint8_t* k_codes, const uint8_t* k_exp,
                                  int32_t* idx_out, float* score_out, int heads_i, int d_i, v4a_dtype q_dtype,
                                  void* workspace, size_t workspace_bytes, const v4a_shape* shape, void* stream);

/* The same operation as v4a_topk for callers that cannot allocate device
 * memory: a plug-in inside a host framework that owns every device
 * allocation, or a serving loop where allocating is not allowed.  (The pages
 * have no counterpart: this is an interface convenience, not part of the
 * method.)  Arguments, results and errors are those of v4a_topk, except that
 * there is no workspace argument: the scratch is a fixed 64 MiB array
 * compiled into the library, which every device that loads the library keeps
 * in its global memory until the process exits.  It bounds the problem size:
 * a shape whose v4a_workspace_size("topk", ...) exceeds 64 MiB (4 bytes per
 * score plus 16 KB per query row for the decode select, so some 16 million
 * scores per call; the 1M-context decode of 4 sequences has 1,048,576)
 * returns V4A_ERR_INVALID_ARG with both sizes in v4a_last_error().  A shape
 * that v4a_topk itself rejects gets v4a_topk's error.
 * The first call made with a given device current looks up the array's
 * device address (cudaGetSymbolAddress) and caches it; make that first call
 * outside any stream capture.  The cached address belongs to the device's
 * current context: after cudaDeviceReset on that device, do not call
 * v4a_topk_noalloc there again in the same process.  The call itself
 * allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 * routine.
 * Every call on a device uses the same array, and the array keeps whatever
 * the previous call left in it (each call writes every scratch byte before
 * reading it).  Calls whose work may overlap on the GPU -- on different
 * streams, or from several host threads without ordering -- race on the
 * array and must be serialised by the caller. */
V4A_API v4a_status v4a_topk_noalloc(const void* q_i, const float* w, const void* k_i, const float* k_scale,
                                    int32_t* idx_out, float* score_out, int heads_i, int d_i, v4a_dtype q_dtype,
                                    v4a_dtype k_dtype, const v4a_shape* shape, void* stream);

/* ------------------------------------------------------------------ */
/* attention                                                            */
/* ------------------------------------------------------------------ */

/* CSA attention: for every query (b, j) at position t and head h,
 *     out[h] = sum_r p_r * v_r,  p = softmax_r(q[h] . v_r / sqrt(d)),
 * one joint softmax over the candidate rows v_r = the selected entries
 * entries[idx[b][j][i]] (every idx >= 0; a value listed twice is two
 * candidates) and the window tokens (t-W, t].  The window may repeat tokens an entry already
 * summarises; both stay.  An empty candidate set yields zeros.
 * q: [batch][n_q][heads][d]; entries: [batch][N][d], N = ctx_len/m;
 * idx: [batch][n_q][k] int32, -1 = empty slot; token_kv: [batch][l_tok][d],
 * row r = position tok_pos0 + r; q/entries/token_kv share dtype (F32 or
 * BF16); out: [batch][n_q][heads][d] fp32.
 * dev_status (nullable, device int): set to V4A_OK by the call, and to
 * V4A_ERR_DEVICE_FAULT by the kernels if an idx entry is neither -1 nor a
 * visible entry; such slots are skipped.  Workspace:
 * v4a_workspace_size("csa_attend", shape, 0, 0) bytes.
 * Uses every shape field.  Errors: d not a multiple of 64 or > 512, a window
 * not covered by token_kv. */
V4A_API v4a_status v4a_csa_attend(const void* q, const void* entries, const int32_t* idx, const void* token_kv,
                          long long tok_pos0, long long l_tok, float* out, v4a_dtype dtype, void* workspace,
                          size_t workspace_bytes, int* dev_status, const v4a_shape* shape, void* stream);

/* HCA attention ("1M Context != Lossless Long Memory", section 5; "How V4
 * makes ...", CSA-vs-HCA table: no selection, dense over every entry): as
 * v4a_csa_attend with the candidate rows = every visible entry s < N_vis(t)
 * plus the window.  Uses shape->batch, n_q, heads, d, m, window, ctx_len;
 * workspace of v4a_workspace_size("hca_attend", shape, 0, 0) bytes. */
V4A_API v4a_status v4a_hca_attend(const void* q, const void* entries, const void* token_kv, long long tok_pos0,
                          long long l_tok, float* out, v4a_dtype dtype, void* workspace, size_t workspace_bytes,
                          const v4a_shape* shape, void* stream);

/* Options of the _ex attention calls ("1M Context != Lossless Long Memory",
 * sections 7 and 8).  A zeroed struct (or a NULL pointer) means neither. */
typedef struct v4a_attend_ext {
    const float* sink;   /* [heads] fp32 per-head sink logits z'_h, or NULL: each head's softmax
                            denominator gains e^{z'_h}, so its weights sum to less than 1 */
    int rope_dims;       /* R: 0, or an even number <= d: the output's last R dims are rotated by
                            RoPE at minus the query position t, pair k = dims (d-R+2k, d-R+2k+1)
                            turning by -t * rope_base^(-2k/R) */
    float rope_base;     /* RoPE frequency base (e.g. 10000); used when rope_dims > 0 */
} v4a_attend_ext;

/* v4a_csa_attend / v4a_hca_attend with the attention sink and the inverse
 * output RoPE of v4a_attend_ext (ext may be NULL: then identical to the
 * plain calls).  Errors as the plain calls, plus V4A_ERR_INVALID_ARG for an
 * odd or too large rope_dims or a rope_base <= 0 with rope_dims > 0. */
V4A_API v4a_status v4a_csa_attend_ex(const void* q, const void* entries, const int32_t* idx, const void* token_kv,
                                     long long tok_pos0, long long l_tok, float* out, v4a_dtype dtype,
                                     void* workspace, size_t workspace_bytes, int* dev_status,
                                     const v4a_attend_ext* ext, const v4a_shape* shape, void* stream);
V4A_API v4a_status v4a_hca_attend_ex(const void* q, const void* entries, const void* token_kv, long long tok_pos0,
                                     long long l_tok, float* out, v4a_dtype dtype, void* workspace,
                                     size_t workspace_bytes, const v4a_attend_ext* ext, const v4a_shape* shape,
                                     void* stream);

/* ------------------------------------------------------------------ */
/* heterogeneous KV cache: paged classical cache + token rings          */
/* ------------------------------------------------------------------ */

/* "DeepSeek-V4: Million-Token Context via Hybrid Compressed Attention",
 * "KV Cache Management" / "KV Cache Layout": the cache is split into a
 * classical cache of compressed entries (CSA / HCA), allocated in blocks that
 * each cover lcm(m, m') original tokens (128 in V4: 32 CSA entries with their
 * indexer keys, or 1 HCA entry), and a state cache pre-allocated per sequence
 * for the sliding window and the tokens of the still incomplete chunks.
 * Here the classical cache of a layer is a pool of n_blocks blocks: entries
 * (and keys, scales, exponents) are pools of n_blocks * epb rows, epb =
 * block_tokens / m, and entry s of sequence b is pool row
 *     block_table[b * bt_stride + s / epb] * epb + s % epb.
 * The state cache is a ring of ring_rows token rows per sequence for each
 * stream (K = V rows, gate logits, indexer rows): position p is row
 * p % ring_rows.  A decode step appends the new token to the rings
 * (v4a_ring_append), compresses a chunk into its block once its last token
 * has arrived (v4a_compress_paged, reading the chunk's rows from the rings),
 * and attends through the block table and the ring (the _paged calls).  All
 * sequences of a call are at the same position (ctx_len).
 * A block id outside [0, n_blocks) is a bad index: attention skips those
 * entries and reports V4A_ERR_DEVICE_FAULT in dev_status, the indexer scores
 * them as all-zero keys, compression does not write them. */
typedef struct v4a_paged {
    const int32_t* block_table;  /* [batch][bt_stride] block ids (device) */
    int bt_stride;               /* block-table entries per sequence (>= the blocks the context needs) */
    int block_tokens;            /* tokens per block, a multiple of m: lcm(m, m') = 128 in V4 */
    long long n_blocks;          /* blocks in the pools */
    int ring_rows;               /* rows of each sequence's token ring (attention calls; a multiple of m for
                                    compression), >= window + n_q - 1 */
} v4a_paged;

/* One stream of a ring append: the new token's row of each sequence. */
typedef struct v4a_ring_io {
    const void* src;             /* [batch] rows of `channels` elements, src_batch_stride elements apart */
    void* ring;                  /* [batch][ring_rows][channels] */
    int channels;                /* channels * element size a multiple of 16 bytes */
    int ring_rows;
    v4a_dtype dtype;             /* F32, BF16 (or FP8E4M3 / MXFP4 bytes copied as such) */
    long long src_batch_stride;  /* elements */
} v4a_ring_io;

/* Append the token at position pos to up to 8 rings in one launch: row b of
 * io[i].src goes to ring row pos % ring_rows of sequence b.  Pointers
 * 16-byte aligned.  Errors: V4A_ERR_INVALID_ARG for n_streams outside 0..8,
 * NULL or misaligned pointers, rows not a multiple of 16 bytes, pos < 0. */
V4A_API v4a_status v4a_ring_append(const v4a_ring_io* io, int n_streams, int batch, long long pos, void* stream);

/* v4a_compress whose entries go to paged pools: for each stream the chunk
 * rows are read as for v4a_compress (x / gate with their batch strides, e.g.
 * a slice of the rings), and entry first_entry + s of sequence b (s <
 * n_tok / m) is written to pool row block_table[b * bt_stride + e / epb] *
 * epb + e % epb, e = first_entry + s, epb = pg->block_tokens / m (out,
 * out_scale and out_exp are pools; their batch strides are ignored).
 * Errors: those of v4a_compress, plus V4A_ERR_INVALID_ARG for a NULL
 * block table, block_tokens not a multiple of m, n_blocks < 1 or entries
 * beyond bt_stride * epb. */
V4A_API v4a_status v4a_compress_paged(const v4a_compress_io* kv, const v4a_compress_io* idx, int batch, long long n_tok,
                                      int m, long long first_entry, const v4a_paged* pg, void* stream);

/* v4a_topk over paged keys: k_i (and k_scale for FP8E4M3) are pools of
 * n_blocks * epb rows addressed through pg's block table; everything else
 * as v4a_topk.  dev_status (nullable, device int) is set to V4A_OK and to
 * V4A_ERR_DEVICE_FAULT if a block id lies outside the pool. */
V4A_API v4a_status v4a_topk_paged(const void* q_i, const float* w, const void* k_i, const float* k_scale,
                                  int32_t* idx_out, float* score_out, int heads_i, int d_i, v4a_dtype q_dtype,
                                  v4a_dtype k_dtype, void* workspace, size_t workspace_bytes, int* dev_status,
                                  const v4a_paged* pg, const v4a_shape* shape, void* stream);
/* The same with MXFP4 keys (k_codes / k_exp pools, see v4a_topk_mxfp4). */
V4A_API v4a_status v4a_topk_mxfp4_paged(const void* q_i, const float* w, const uint8_t* k_codes, const uint8_t* k_exp,
                                        int32_t* idx_out, float* score_out, int heads_i, int d_i, v4a_dtype q_dtype,
                                        void* workspace, size_t workspace_bytes, int* dev_status,
                                        const v4a_paged* pg, const v4a_shape* shape, void* stream);

/* v4a_csa_attend_ex / v4a_hca_attend_ex over the heterogeneous cache:
 * entries is a pool addressed through pg's block table (epb =
 * block_tokens / m) and token_kv is the K = V ring ([batch][ring_rows][d],
 * position p in row p % ring_rows; pg->ring_rows >= window + n_q - 1).
 * Everything else (ext included) as the _ex calls. */
V4A_API v4a_status v4a_csa_attend_paged(const void* q, const void* entries, const int32_t* idx, const void* token_kv,
                                        float* out, v4a_dtype dtype, void* workspace, size_t workspace_bytes,
                                        int* dev_status, const v4a_attend_ext* ext, const v4a_paged* pg,
                                        const v4a_shape* shape, void* stream);
V4A_API v4a_status v4a_hca_attend_paged(const void* q, const void* entries, const void* token_kv, float* out,
                                        v4a_dtype dtype, void* workspace, size_t workspace_bytes, int* dev_status,
                                        const v4a_attend_ext* ext, const v4a_paged* pg, const v4a_shape* shape,
                                        void* stream);

/* ------------------------------------------------------------------ */
/* housekeeping                                                         */
/* ------------------------------------------------------------------ */

/* Bytes of device workspace an op needs for this shape: op is "topk",
 * "csa_attend" or "hca_attend" (0 for anything else).  heads_i/d_i are the
 * indexer's (used by "topk"). */
V4A_API size_t v4a_workspace_size(const char* op, const v4a_shape* shape, int heads_i, int d_i);

/* Static description of a status code. */
V4A_API const char* v4a_status_string(v4a_status status);

/* The reason for the last non-OK status returned on this host thread. */
V4A_API const char* v4a_last_error(void);

/* Library version: major*10000 + minor*100 + patch. */
V4A_API int v4a_version(void);

/* ------------------------------------------------------------------ */
/* test hook                                                            */
/* ------------------------------------------------------------------ */

/* Fault injection for tests of the bounded waits (not part of the method;
 * never needed in normal use).  With withhold_tile >= 0, every later launch
 * of the tensor-core attention kernel (the bf16, d = 512, 64-head path of
 * the CSA and HCA attention calls) makes each CTA skip the copies of its
 * local tile withhold_tile -- no copy is issued and no arrival made, so that
 * stage never fills -- and gives every wait of the kernel wait_polls polls
 * (each suspends for at most ~20 us) and the MMA warp ~2 ms without progress.
 * The waits then give up: the kernel records V4A_ERR_DEVICE_FAULT in the
 * call's dev_status, writes NaN to every output it contributes to, frees its
 * tensor memory and returns; nothing traps and nothing is left in flight.
 * withhold_tile = -1 restores normal launches.  Host-side global state: not
 * for concurrent use. */
V4A_API void v4a_test_attend_fault(int withhold_tile, int wait_polls);

#ifdef __cplusplus
}
#endif

#endif /* V4A_H */
