// internal.h -- host-side launchers behind the C ABI (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "v4a.h"

namespace v4a {

// Launch with programmatic stream serialization (see griddep_wait in common.cuh).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Record a one-line reason for v4a_last_error() and return st.
v4a_status report(v4a_status st, const char* fmt, ...);

// ---- v4a_api.cu -------------------------------------------------------
// Zero n 32-bit words with a kernel launched like every other kernel here, after the previous
// work on the stream (a memset node in its place would end the chain of overlapped launches).
cudaError_t launch_zero_words(uint32_t* p, long long n, cudaStream_t stream);

// ---- compress.cu ------------------------------------------------------
cudaError_t launch_compress(const v4a_compress_io* kv, const v4a_compress_io* idx, int batch, long long n_tok,
                            int m, cudaStream_t stream);
cudaError_t launch_compress_dual(const v4a_compress_io* a, const v4a_series_b* b, int batch, long long n_tok, int m,
                                 cudaStream_t stream);
cudaError_t launch_quantize_mxfp4(const void* x, v4a_dtype dt, long long rows, int cols, uint8_t* codes,
                                  uint8_t* exps, cudaStream_t stream);
// compression whose outputs go to a paged pool: entry first_entry + s of sequence b -> pool row
// bt[b*bt_stride + (first_entry+s)/epb]*epb + (first_entry+s)%epb (out_batch_stride ignored)
cudaError_t launch_compress_paged(const v4a_compress_io* kv, const v4a_compress_io* idx, int batch, long long n_tok,
                                  int m, long long first_entry, const int32_t* bt, int bt_stride, int epb,
                                  long long n_blocks, cudaStream_t stream);
cudaError_t launch_ring_append(const v4a_ring_io* io, int n, int batch, long long pos, cudaStream_t stream);

// ---- indexer.cu -------------------------------------------------------
struct IndexArgs {
    const void* q;        // [B][n_q][HI][DI]
    const float* w;       // [B][n_q][HI]
    const void* k;        // [B][N][DI]
    const float* kscale;  // [B][N] or null
    const uint8_t* kexp;  // [B][N][DI/32] MXFP4 block exponents (k_dtype MXFP4), else null
    // paged classical cache (as AttendArgs): keys, scales and exponents are pools of pool_rows rows; a
    // block id outside the pool reads as a block of zero keys
    const int32_t* bt;
    int bt_stride, epb;
    long long pool_rows;
    int* dev_status;  // nullable: V4A_ERR_DEVICE_FAULT for a block id outside the pool
    v4a_dtype q_dtype, k_dtype;
    int batch, n_q, m, heads_i, d_i;
    long long ctx_len, n_ent;
};

// every score (-inf where not visible) into scores[row][N], row = b*n_q + j
cudaError_t launch_index_scores(const IndexArgs& a, float* scores, cudaStream_t stream);

// ---- indexer_tc.cu (tcgen05 scores: d_i = 128, heads_i <= 32, bf16 q, bf16/fp8 keys) ----
bool index_tc_shape_ok(const IndexArgs& a);
bool index_tc_available(const IndexArgs& a);
// scores as launch_index_scores; hist (nullable) [rows][4096] += counts of the scores' ordered-key top 12 bits
cudaError_t launch_index_scores_tc(const IndexArgs& a, float* scores, uint32_t* hist, int* err, cudaStream_t stream);
size_t topk_workspace_bytes(const IndexArgs& a, int k);
cudaError_t launch_topk(const IndexArgs& a, int k, int32_t* idx_out, float* score_out, void* ws, size_t ws_bytes,
                        cudaStream_t stream);

// ---- attend.cu --------------------------------------------------------
struct AttendArgs {
    const void* q;         // [B][n_q][H][d]
    const void* entries;   // [B][N][d]
    const int32_t* idx;    // [B][n_q][k] (CSA) or null (HCA: every visible entry)
    const void* token_kv;  // [B][l_tok][d]
    long long tok_pos0, l_tok;
    float* out;            // [B][n_q][H][d]
    v4a_dtype dtype;
    int batch, n_q, heads, d, m, k, window;
    long long ctx_len, n_ent;
    int* dev_status;
    const float* sink;  // [heads] sink logits, or null
    int rope_dims;      // 0, or the output dims rotated at minus the query position
    float rope_base;
    // paged classical cache: entry s of sequence b is row bt[b*bt_stride + s/epb]*epb + s%epb of
    // `entries` (a pool of pool_rows rows); bt null = contiguous [B][N][d]
    const int32_t* bt;
    int bt_stride, epb;
    long long pool_rows;  // n_blocks * epb; a block id outside [0, n_blocks) is a bad index
    int ring_rows;  // > 0: token_kv is a ring [B][ring_rows][d] holding position p in row p % ring_rows
};

size_t attend_workspace_bytes(const AttendArgs& a);
cudaError_t launch_attend(const AttendArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream);

// ---- attend_tc.cu (tcgen05 path: bf16, d = 512, 64 heads) -------------
// Fault injection for the tensor-core attention's bounded waits (set by v4a_test_attend_fault only;
// withhold = -1 in normal use): every CTA withholds its local tile `withhold`, and the waits give up
// after wait_polls polls / stall_cycles cycles without progress.
struct AttendFaultTest {
    int withhold;
    uint32_t wait_polls;
    long long stall_cycles;
};
extern AttendFaultTest g_test_fault;

bool attend_tc_shape_ok(const AttendArgs& a);   // the shape this path takes
bool attend_tc_available(const AttendArgs& a);  // ... and the driver's tensor-map encoder is present
size_t attend_tc_workspace_bytes(const AttendArgs& a);
cudaError_t launch_attend_tc(const AttendArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream);

}  // namespace v4a
