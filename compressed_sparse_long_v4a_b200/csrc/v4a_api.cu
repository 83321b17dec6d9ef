// v4a_api.cu -- the exported C ABI: argument checks, then the launchers.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace v4a {
namespace {

// The previous kernel on the stream may still read or write these words: wait for it, then zero.
// The next kernel is let in only after the stores: letting it in at the start made its blocks wait,
// resident, through the whole of the kernel before this one (measured on B200: the select kernel
// before a status reset took 5-8 us longer while the attention blocks after it waited).
__global__ void __launch_bounds__(256) zero_words_kernel(uint32_t* p, long long n) {
    griddep_wait();
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        p[i] = 0u;
    griddep_launch_dependents();
}

}  // namespace

cudaError_t launch_zero_words(uint32_t* p, long long n, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    const long long want = (n + 255) / 256, cap = 8LL * kNumSMs;
    const cudaError_t e =
        launch_pdl(zero_words_kernel, dim3((unsigned)(want < cap ? want : cap)), dim3(256), 0, stream, p, n);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace v4a

namespace {

thread_local char g_last_error[512] = "";

v4a_status fail(v4a_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

v4a_status from_cuda(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return V4A_OK;
    return fail(V4A_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t dtype_size(v4a_dtype t) { return t == V4A_F32 ? 4 : t == V4A_BF16 ? 2 : 1; }

v4a_status check_compress_io(const v4a_compress_io* io, const char* name, long long n_tok, int m) {
    if (!io->x || !io->gate || !io->out) return fail(V4A_ERR_INVALID_ARG, "%s: x, gate and out are required", name);
    if (io->channels < 8 || io->channels % 8) return fail(V4A_ERR_INVALID_ARG, "%s: channels must be a multiple of 8", name);
    if (io->in_dtype != V4A_F32 && io->in_dtype != V4A_BF16)
        return fail(V4A_ERR_UNSUPPORTED, "%s: input dtype must be F32 or BF16", name);
    if (io->out_dtype != V4A_F32 && io->out_dtype != V4A_BF16 && io->out_dtype != V4A_FP8E4M3 &&
        io->out_dtype != V4A_MXFP4)
        return fail(V4A_ERR_UNSUPPORTED, "%s: unknown output dtype", name);
    if (io->out_dtype == V4A_MXFP4) {
        if (io->channels % 32) return fail(V4A_ERR_INVALID_ARG, "%s: MXFP4 output needs channels % 32 == 0", name);
        if (!io->out_exp) return fail(V4A_ERR_INVALID_ARG, "%s: MXFP4 output needs out_exp", name);
        const long long n_ent = n_tok / m;
        if (io->out_batch_stride < n_ent * io->channels || io->out_batch_stride % 8 ||
            io->exp_batch_stride < n_ent * (io->channels / 32))
            return fail(V4A_ERR_INVALID_ARG, "%s: MXFP4 out/out_exp batch stride too small or out stride not a multiple of 8",
                        name);
        if (!aligned(io->x, 16) || !aligned(io->gate, 16) || !aligned(io->out, 4) ||
            (io->x_batch_stride * dtype_size(io->in_dtype)) % 16 || (io->gate_batch_stride * dtype_size(io->in_dtype)) % 16)
            return fail(V4A_ERR_INVALID_ARG, "%s: x/gate (16 bytes) or out (4 bytes) misaligned", name);
        if (io->x_batch_stride < n_tok * io->channels || io->gate_batch_stride < n_tok * io->channels)
            return fail(V4A_ERR_INVALID_ARG, "%s: a batch stride is smaller than one sequence", name);
        return V4A_OK;
    }
    if (io->out_dtype == V4A_FP8E4M3) {
        int g = io->channels / 8;
        if (!io->out_scale) return fail(V4A_ERR_INVALID_ARG, "%s: FP8E4M3 output needs out_scale", name);
        if (g > 32 || (g & (g - 1))) return fail(V4A_ERR_UNSUPPORTED, "%s: FP8E4M3 output needs channels/8 a power of two <= 32", name);
        if (!aligned(io->out_scale, 4)) return fail(V4A_ERR_INVALID_ARG, "%s: out_scale misaligned", name);
    }
    long long n_ent = n_tok / m;
    if (io->x_batch_stride < n_tok * io->channels || io->gate_batch_stride < n_tok * io->channels ||
        io->out_batch_stride < n_ent * io->channels || (io->out_scale && io->scale_batch_stride < n_ent))
        return fail(V4A_ERR_INVALID_ARG, "%s: a batch stride is smaller than one sequence", name);
    size_t in_sz = dtype_size(io->in_dtype), out_sz = dtype_size(io->out_dtype);
    size_t out_al = out_sz == 1 ? 8 : 16;
    if (!aligned(io->x, 16) || !aligned(io->gate, 16) || !aligned(io->out, out_al) ||
        (io->x_batch_stride * in_sz) % 16 || (io->gate_batch_stride * in_sz) % 16 ||
        (io->out_batch_stride * out_sz) % out_al)
        return fail(V4A_ERR_INVALID_ARG, "%s: x/gate/out or their strides are not 16-byte aligned", name);
    return V4A_OK;
}

v4a_status check_shape_common(const v4a_shape* s) {
    if (!s) return fail(V4A_ERR_INVALID_ARG, "shape is NULL");
    if (s->batch < 0 || s->n_q < 1 || s->m < 1 || s->ctx_len < 1)
        return fail(V4A_ERR_INVALID_ARG, "need batch >= 0, n_q >= 1, m >= 1, ctx_len >= 1");
    if (s->n_q > s->ctx_len) return fail(V4A_ERR_INVALID_ARG, "n_q > ctx_len");
    if (s->ctx_len / s->m > 0x7fffffffLL) return fail(V4A_ERR_INVALID_ARG, "too many entries for int32 indices");
    if ((long long)s->batch * s->n_q > 65535) return fail(V4A_ERR_UNSUPPORTED, "batch * n_q must be <= 65535");
    return V4A_OK;
}

v4a_status index_args(const void* q_i, const float* w, const void* k_i, const float* k_scale, const uint8_t* k_exp,
                      int heads_i, int d_i, v4a_dtype q_dt, v4a_dtype k_dt, const v4a_shape* s, v4a::IndexArgs* a) {
    v4a_status st = check_shape_common(s);
    if (st != V4A_OK) return st;
    if (!q_i || !w || (!k_i && s->ctx_len / s->m > 0)) return fail(V4A_ERR_INVALID_ARG, "q_i, w and k_i are required");
    if (heads_i < 1 || heads_i > 64) return fail(V4A_ERR_UNSUPPORTED, "heads_i must be in 1..64");
    if (d_i < 8 || d_i % 8 || d_i > 1024) return fail(V4A_ERR_INVALID_ARG, "d_i must be a multiple of 8 (<= 1024)");
    if ((long long)heads_i * d_i > 32768) return fail(V4A_ERR_UNSUPPORTED, "heads_i * d_i must be <= 32768");
    if (q_dt != V4A_F32 && q_dt != V4A_BF16) return fail(V4A_ERR_UNSUPPORTED, "q_i dtype must be F32 or BF16");
    if (k_dt == V4A_MXFP4) {
        if (!k_exp && s->ctx_len / s->m > 0) return fail(V4A_ERR_INVALID_ARG, "MXFP4 keys need k_exp");
        if (d_i % 32) return fail(V4A_ERR_INVALID_ARG, "MXFP4 keys need d_i % 32 == 0");
        if (!aligned(k_exp, 4)) return fail(V4A_ERR_INVALID_ARG, "k_exp must be 4-byte aligned");
    } else if (k_dt != V4A_F32 && k_dt != V4A_BF16 && k_dt != V4A_FP8E4M3) {
        return fail(V4A_ERR_UNSUPPORTED, "k_i dtype must be F32, BF16 or FP8E4M3 (MXFP4 keys: the _mxfp4 calls)");
    }
    if (k_dt == V4A_FP8E4M3 && !k_scale) return fail(V4A_ERR_INVALID_ARG, "FP8E4M3 keys need k_scale");
    if (!aligned(k_i, 16) || !aligned(q_i, 16) || !aligned(w, 4))
        return fail(V4A_ERR_INVALID_ARG, "q_i/k_i must be 16-byte aligned");
    a->q = q_i;
    a->w = w;
    a->k = k_i;
    a->kscale = k_dt == V4A_MXFP4 ? nullptr : k_scale;
    a->kexp = k_dt == V4A_MXFP4 ? k_exp : nullptr;
    a->bt = nullptr;
    a->bt_stride = a->epb = 0;
    a->pool_rows = 0;
    a->dev_status = nullptr;
    a->q_dtype = q_dt;
    a->k_dtype = k_dt;
    a->batch = s->batch;
    a->n_q = s->n_q;
    a->m = s->m;
    a->heads_i = heads_i;
    a->d_i = d_i;
    a->ctx_len = s->ctx_len;
    a->n_ent = s->ctx_len / s->m;
    return V4A_OK;
}

v4a_status attend_args(const void* q, const void* entries, const int32_t* idx, const void* token_kv,
                       long long tok_pos0, long long l_tok, float* out, v4a_dtype dt, int* dev_status,
                       const v4a_shape* s, bool csa, v4a::AttendArgs* a) {
    v4a_status st = check_shape_common(s);
    if (st != V4A_OK) return st;
    if (!q || !out) return fail(V4A_ERR_INVALID_ARG, "q and out are required");
    if (!entries && s->ctx_len / s->m > 0) return fail(V4A_ERR_INVALID_ARG, "entries is required");
    if (csa && !idx) return fail(V4A_ERR_INVALID_ARG, "idx is required");
    if (csa && (s->k < 1 || s->k > 65536)) return fail(V4A_ERR_INVALID_ARG, "k must be in 1..65536");
    if (s->heads < 1) return fail(V4A_ERR_INVALID_ARG, "heads must be >= 1");
    if (s->d != 64 && s->d != 128 && s->d != 256 && s->d != 512)
        return fail(V4A_ERR_UNSUPPORTED, "d must be 64, 128, 256 or 512");
    if (s->window < 0) return fail(V4A_ERR_INVALID_ARG, "window must be >= 0");
    if (dt != V4A_F32 && dt != V4A_BF16) return fail(V4A_ERR_UNSUPPORTED, "dtype must be F32 or BF16");
    if (s->window > 0) {
        if (!token_kv) return fail(V4A_ERR_INVALID_ARG, "token_kv is required when window > 0");
        long long lo = s->ctx_len - s->n_q - s->window + 1;
        if (lo < 0) lo = 0;
        if (tok_pos0 > lo || tok_pos0 < 0 || tok_pos0 + l_tok < s->ctx_len)
            return fail(V4A_ERR_INVALID_ARG, "token_kv rows [%lld, %lld) do not cover the windows [%lld, %lld)",
                        tok_pos0, tok_pos0 + l_tok, lo, s->ctx_len);
    }
    if (!aligned(q, 16) || !aligned(entries, 16) || !aligned(token_kv, 16) || !aligned(out, 16) ||
        (idx && !aligned(idx, 4)))
        return fail(V4A_ERR_INVALID_ARG, "q/entries/token_kv/out must be 16-byte aligned");
    a->q = q;
    a->entries = entries;
    a->idx = csa ? idx : nullptr;
    a->token_kv = token_kv;
    a->tok_pos0 = tok_pos0;
    a->l_tok = l_tok;
    a->out = out;
    a->dtype = dt;
    a->batch = s->batch;
    a->n_q = s->n_q;
    a->heads = s->heads;
    a->d = s->d;
    a->m = s->m;
    a->k = csa ? s->k : 0;
    a->window = s->window;
    a->ctx_len = s->ctx_len;
    a->n_ent = s->ctx_len / s->m;
    a->dev_status = dev_status;
    a->bt = nullptr;
    a->bt_stride = a->epb = 0;
    a->pool_rows = 0;
    a->ring_rows = 0;
    return V4A_OK;
}

// checks a heterogeneous-cache descriptor for compression rate m and `entries` entries per sequence
v4a_status paged_check(const v4a_paged* pg, int m, long long entries, const char* what) {
    if (!pg || !pg->block_table) return fail(V4A_ERR_INVALID_ARG, "%s: a block table is required", what);
    if (!aligned(pg->block_table, 4)) return fail(V4A_ERR_INVALID_ARG, "%s: block_table misaligned", what);
    if (pg->block_tokens < m || pg->block_tokens % m)
        return fail(V4A_ERR_INVALID_ARG, "%s: block_tokens must be a positive multiple of m", what);
    if (pg->n_blocks < 1) return fail(V4A_ERR_INVALID_ARG, "%s: n_blocks must be >= 1", what);
    const long long epb = pg->block_tokens / m;
    if (pg->bt_stride < 0 || (long long)pg->bt_stride * epb < entries)
        return fail(V4A_ERR_INVALID_ARG, "%s: the block table holds %lld entries per sequence, %lld needed", what,
                    (long long)pg->bt_stride * epb, entries);
    if (pg->n_blocks * epb >= (1LL << 31)) return fail(V4A_ERR_UNSUPPORTED, "%s: pool too large", what);
    return V4A_OK;
}

}  // namespace

v4a_status v4a::report(v4a_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

static v4a_status topk_common(const v4a::IndexArgs& a, int32_t* idx_out, float* score_out, void* workspace,
                              size_t workspace_bytes, const v4a_shape* shape, void* stream, const char* what) {
    if (shape->k < 1 || shape->k > 4096) return fail(V4A_ERR_INVALID_ARG, "k must be in 1..4096");
    if (!idx_out) return fail(V4A_ERR_INVALID_ARG, "idx_out is required");
    size_t need = v4a::topk_workspace_bytes(a, shape->k);
    if (!workspace || workspace_bytes < need)
        return fail(V4A_ERR_INVALID_ARG, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (!aligned(workspace, 256)) return fail(V4A_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    return from_cuda(v4a::launch_topk(a, shape->k, idx_out, score_out, workspace, workspace_bytes,
                                      (cudaStream_t)stream),
                     what);
}

extern "C" {

v4a_status v4a_compress(const v4a_compress_io* kv, const v4a_compress_io* idx, int batch, long long n_tok, int m,
                        void* stream) {
    if (!kv) return fail(V4A_ERR_INVALID_ARG, "kv stream is NULL");
    if (batch < 0 || n_tok < 0 || m < 1) return fail(V4A_ERR_INVALID_ARG, "need batch >= 0, n_tok >= 0, m >= 1");
    if (batch == 0 || n_tok / m == 0) return V4A_OK;  // no complete chunk: nothing to write
    v4a_status st = check_compress_io(kv, "kv", n_tok, m);
    if (st != V4A_OK) return st;
    if (idx) {
        st = check_compress_io(idx, "idx", n_tok, m);
        if (st != V4A_OK) return st;
    }
    return from_cuda(v4a::launch_compress(kv, idx, batch, n_tok, m, (cudaStream_t)stream), "v4a_compress");
}

v4a_status v4a_compress_dual(const v4a_compress_io* a, const v4a_series_b* b, int batch, long long n_tok, int m,
                             void* stream) {
    if (!a || !b) return fail(V4A_ERR_INVALID_ARG, "v4a_compress_dual: series a and b are required");
    if (batch < 0 || n_tok < 0 || m < 1) return fail(V4A_ERR_INVALID_ARG, "need batch >= 0, n_tok >= 0, m >= 1");
    if (batch == 0 || n_tok / m == 0) return V4A_OK;  // no complete chunk: nothing to write
    v4a_status st = check_compress_io(a, "series a", n_tok, m);
    if (st != V4A_OK) return st;
    if (!b->x || !b->gate) return fail(V4A_ERR_INVALID_ARG, "series b: x and gate are required");
    if ((b->prev_x == nullptr) != (b->prev_gate == nullptr))
        return fail(V4A_ERR_INVALID_ARG, "series b: prev_x and prev_gate must both be given or both be NULL");
    const size_t in_sz = dtype_size(a->in_dtype);
    if (b->x_batch_stride < n_tok * a->channels || b->gate_batch_stride < n_tok * a->channels ||
        (b->prev_x && b->prev_batch_stride < (long long)m * a->channels))
        return fail(V4A_ERR_INVALID_ARG, "series b: a batch stride is smaller than one sequence");
    if (!aligned(b->x, 16) || !aligned(b->gate, 16) || (b->prev_x && (!aligned(b->prev_x, 16) || !aligned(b->prev_gate, 16))) ||
        (b->x_batch_stride * in_sz) % 16 || (b->gate_batch_stride * in_sz) % 16 ||
        (b->prev_x && (b->prev_batch_stride * in_sz) % 16))
        return fail(V4A_ERR_INVALID_ARG, "series b: pointers or strides are not 16-byte aligned");
    return from_cuda(v4a::launch_compress_dual(a, b, batch, n_tok, m, (cudaStream_t)stream), "v4a_compress_dual");
}

v4a_status v4a_index_scores(const void* q_i, const float* w, const void* k_i, const float* k_scale, float* scores,
                            int heads_i, int d_i, v4a_dtype q_dtype, v4a_dtype k_dtype, const v4a_shape* shape,
                            void* stream) {
    if (k_dtype == V4A_MXFP4) return fail(V4A_ERR_UNSUPPORTED, "MXFP4 keys: use v4a_index_scores_mxfp4");
    v4a::IndexArgs a;
    v4a_status st = index_args(q_i, w, k_i, k_scale, nullptr, heads_i, d_i, q_dtype, k_dtype, shape, &a);
    if (st != V4A_OK) return st;
    if (!scores && a.n_ent > 0) return fail(V4A_ERR_INVALID_ARG, "scores is required");
    return from_cuda(v4a::launch_index_scores(a, scores, (cudaStream_t)stream), "v4a_index_scores");
}

v4a_status v4a_index_scores_mxfp4(const void* q_i, const float* w, const uint8_t* k_codes, const uint8_t* k_exp,
                                  float* scores, int heads_i, int d_i, v4a_dtype q_dtype, const v4a_shape* shape,
                                  void* stream) {
    v4a::IndexArgs a;
    v4a_status st = index_args(q_i, w, k_codes, nullptr, k_exp, heads_i, d_i, q_dtype, V4A_MXFP4, shape, &a);
    if (st != V4A_OK) return st;
    if (!scores && a.n_ent > 0) return fail(V4A_ERR_INVALID_ARG, "scores is required");
    return from_cuda(v4a::launch_index_scores(a, scores, (cudaStream_t)stream), "v4a_index_scores_mxfp4");
}

v4a_status v4a_topk(const void* q_i, const float* w, const void* k_i, const float* k_scale, int32_t* idx_out,
                    float* score_out, int heads_i, int d_i, v4a_dtype q_dtype, v4a_dtype k_dtype, void* workspace,
                    size_t workspace_bytes, const v4a_shape* shape, void* stream) {
    if (k_dtype == V4A_MXFP4) return fail(V4A_ERR_UNSUPPORTED, "MXFP4 keys: use v4a_topk_mxfp4");
    v4a::IndexArgs a;
    v4a_status st = index_args(q_i, w, k_i, k_scale, nullptr, heads_i, d_i, q_dtype, k_dtype, shape, &a);
    if (st != V4A_OK) return st;
    return topk_common(a, idx_out, score_out, workspace, workspace_bytes, shape, stream, "v4a_topk");
}

v4a_status v4a_topk_mxfp4(const void* q_i, const float* w, const uint8_t* k_codes, const uint8_t* k_exp,
                          int32_t* idx_out, float* score_out, int heads_i, int d_i, v4a_dtype q_dtype,
                          void* workspace, size_t workspace_bytes, const v4a_shape* shape, void* stream) {
    v4a::IndexArgs a;
    v4a_status st = index_args(q_i, w, k_codes, nullptr, k_exp, heads_i, d_i, q_dtype, V4A_MXFP4, shape, &a);
    if (st != V4A_OK) return st;
    return topk_common(a, idx_out, score_out, workspace, workspace_bytes, shape, stream, "v4a_topk_mxfp4");
}


static v4a_status topk_paged_common(v4a::IndexArgs& a, int32_t* idx_out, float* score_out, void* workspace,
                                    size_t workspace_bytes, int* dev_status, const v4a_paged* pg,
                                    const v4a_shape* shape, void* stream, const char* what) {
    v4a_status st = paged_check(pg, shape->m, a.n_ent, what);
    if (st != V4A_OK) return st;
    if (dev_status && !aligned(dev_status, 4)) return fail(V4A_ERR_INVALID_ARG, "%s: dev_status misaligned", what);
    a.bt = pg->block_table;
    a.bt_stride = pg->bt_stride;
    a.epb = pg->block_tokens / shape->m;
    a.pool_rows = pg->n_blocks * a.epb;
    a.dev_status = dev_status;
    if (dev_status) {
        cudaError_t e = v4a::launch_zero_words(reinterpret_cast<uint32_t*>(dev_status), 1, (cudaStream_t)stream);
        if (e != cudaSuccess) return from_cuda(e, "dev_status reset");
    }
    return topk_common(a, idx_out, score_out, workspace, workspace_bytes, shape, stream, what);
}

v4a_status v4a_topk_paged(const void* q_i, const float* w, const void* k_i, const float* k_scale, int32_t* idx_out,
                          float* score_out, int heads_i, int d_i, v4a_dtype q_dtype, v4a_dtype k_dtype,
                          void* workspace, size_t workspace_bytes, int* dev_status, const v4a_paged* pg,
                          const v4a_shape* shape, void* stream) {
    if (k_dtype == V4A_MXFP4) return fail(V4A_ERR_UNSUPPORTED, "MXFP4 keys: use v4a_topk_mxfp4_paged");
    v4a::IndexArgs a;
    v4a_status st = index_args(q_i, w, k_i, k_scale, nullptr, heads_i, d_i, q_dtype, k_dtype, shape, &a);
    if (st != V4A_OK) return st;
    return topk_paged_common(a, idx_out, score_out, workspace, workspace_bytes, dev_status, pg, shape, stream,
                             "v4a_topk_paged");
}

v4a_status v4a_topk_mxfp4_paged(const void* q_i, const float* w, const uint8_t* k_codes, const uint8_t* k_exp,
                                int32_t* idx_out, float* score_out, int heads_i, int d_i, v4a_dtype q_dtype,
                                void* workspace, size_t workspace_bytes, int* dev_status, const v4a_paged* pg,
                                const v4a_shape* shape, void* stream) {
    v4a::IndexArgs a;
    v4a_status st = index_args(q_i, w, k_codes, nullptr, k_exp, heads_i, d_i, q_dtype, V4A_MXFP4, shape, &a);
    if (st != V4A_OK) return st;
    return topk_paged_common(a, idx_out, score_out, workspace, workspace_bytes, dev_status, pg, shape, stream,
                             "v4a_topk_mxfp4_paged");
}

v4a_status v4a_compress_paged(const v4a_compress_io* kv, const v4a_compress_io* idx, int batch, long long n_tok, int m,
                              long long first_entry, const v4a_paged* pg, void* stream) {
    if (!kv) return fail(V4A_ERR_INVALID_ARG, "kv stream is NULL");
    if (batch < 0 || n_tok < 0 || m < 1 || first_entry < 0)
        return fail(V4A_ERR_INVALID_ARG, "need batch >= 0, n_tok >= 0, m >= 1, first_entry >= 0");
    const long long n_ent = n_tok / m;
    if (batch == 0 || n_ent == 0) return V4A_OK;
    v4a_status st = paged_check(pg, m, first_entry + n_ent, "v4a_compress_paged");
    if (st != V4A_OK) return st;
    // the pools take the place of per-sequence outputs: check each stream as if its output rows were its own
    for (const v4a_compress_io* io : {kv, idx}) {
        if (!io) continue;
        v4a_compress_io c = *io;
        c.out_batch_stride = n_ent * c.channels;
        c.scale_batch_stride = n_ent;
        c.exp_batch_stride = n_ent * (c.channels / 32);
        st = check_compress_io(&c, io == kv ? "kv" : "idx", n_tok, m);
        if (st != V4A_OK) return st;
    }
    return from_cuda(v4a::launch_compress_paged(kv, idx, batch, n_tok, m, first_entry, pg->block_table, pg->bt_stride,
                                                pg->block_tokens / m, pg->n_blocks, (cudaStream_t)stream),
                     "v4a_compress_paged");
}

v4a_status v4a_ring_append(const v4a_ring_io* io, int n_streams, int batch, long long pos, void* stream) {
    if (n_streams < 0 || n_streams > 8) return fail(V4A_ERR_INVALID_ARG, "v4a_ring_append: 0 .. 8 streams");
    if (batch < 0 || pos < 0) return fail(V4A_ERR_INVALID_ARG, "v4a_ring_append: need batch >= 0, pos >= 0");
    if (n_streams == 0 || batch == 0) return V4A_OK;
    if (!io) return fail(V4A_ERR_INVALID_ARG, "v4a_ring_append: io is NULL");
    for (int i = 0; i < n_streams; ++i) {
        const v4a_ring_io& r = io[i];
        const size_t es = dtype_size(r.dtype);
        if (!r.src || !r.ring || r.channels < 1 || r.ring_rows < 1 || ((size_t)r.channels * es) % 16 ||
            !aligned(r.src, 16) || !aligned(r.ring, 16) || ((size_t)r.src_batch_stride * es) % 16 ||
            r.src_batch_stride < r.channels)
            return fail(V4A_ERR_INVALID_ARG, "v4a_ring_append: stream %d: pointers, sizes or strides", i);
    }
    return from_cuda(v4a::launch_ring_append(io, n_streams, batch, pos, (cudaStream_t)stream), "v4a_ring_append");
}

v4a_status v4a_quantize_mxfp4(const void* x, v4a_dtype dtype, long long rows, int cols, uint8_t* codes,
                              uint8_t* exps, void* stream) {
    if (rows < 0 || cols < 32 || cols % 32)
        return fail(V4A_ERR_INVALID_ARG, "v4a_quantize_mxfp4: need rows >= 0 and cols a positive multiple of 32");
    if (dtype != V4A_F32 && dtype != V4A_BF16) return fail(V4A_ERR_UNSUPPORTED, "v4a_quantize_mxfp4: dtype must be F32 or BF16");
    if (rows == 0) return V4A_OK;
    if (!x || !codes || !exps) return fail(V4A_ERR_INVALID_ARG, "v4a_quantize_mxfp4: x, codes and exps are required");
    if (!aligned(x, 16) || !aligned(codes, 4))
        return fail(V4A_ERR_INVALID_ARG, "v4a_quantize_mxfp4: x must be 16-byte and codes 4-byte aligned");
    return from_cuda(v4a::launch_quantize_mxfp4(x, dtype, rows, cols, codes, exps, (cudaStream_t)stream),
                     "v4a_quantize_mxfp4");
}

static v4a_status attend_common(const void* q, const void* entries, const int32_t* idx, const void* token_kv,
                                long long tok_pos0, long long l_tok, float* out, v4a_dtype dtype, void* workspace,
                                size_t workspace_bytes, int* dev_status, const v4a_attend_ext* ext,
                                const v4a_shape* shape, void* stream, bool csa, const v4a_paged* pg = nullptr) {
    v4a::AttendArgs a;
    v4a_status st = attend_args(q, entries, idx, token_kv, tok_pos0, l_tok, out, dtype, dev_status, shape, csa, &a);
    if (st != V4A_OK) return st;
    if (pg) {
        a.bt = pg->block_table;
        a.bt_stride = pg->bt_stride;
        a.epb = pg->block_tokens / shape->m;
        a.pool_rows = pg->n_blocks * a.epb;
        a.ring_rows = pg->ring_rows;
        a.l_tok = pg->ring_rows;
        a.tok_pos0 = 0;
    }
    a.sink = nullptr;
    a.rope_dims = 0;
    a.rope_base = 10000.f;
    if (ext) {
        if (ext->rope_dims < 0 || ext->rope_dims > a.d || (ext->rope_dims & 1))
            return fail(V4A_ERR_INVALID_ARG, "rope_dims must be even and in 0..d");
        if (ext->rope_dims > 0 && !(ext->rope_base > 0.f)) return fail(V4A_ERR_INVALID_ARG, "rope_base must be > 0");
        if (ext->sink && !aligned(ext->sink, 4)) return fail(V4A_ERR_INVALID_ARG, "sink must be 4-byte aligned");
        a.sink = ext->sink;
        a.rope_dims = ext->rope_dims;
        a.rope_base = ext->rope_base;
    }
    size_t need = v4a::attend_workspace_bytes(a);
    if (!workspace || workspace_bytes < need)
        return fail(V4A_ERR_INVALID_ARG, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (!aligned(workspace, 256)) return fail(V4A_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (dev_status) {
        cudaError_t e = v4a::launch_zero_words(reinterpret_cast<uint32_t*>(dev_status), 1, (cudaStream_t)stream);
        if (e != cudaSuccess) return from_cuda(e, "dev_status reset");
    }
    return from_cuda(v4a::launch_attend(a, workspace, workspace_bytes, (cudaStream_t)stream),
                     csa ? "v4a_csa_attend" : "v4a_hca_attend");
}

v4a_status v4a_csa_attend(const void* q, const void* entries, const int32_t* idx, const void* token_kv,
                          long long tok_pos0, long long l_tok, float* out, v4a_dtype dtype, void* workspace,
                          size_t workspace_bytes, int* dev_status, const v4a_shape* shape, void* stream) {
    return attend_common(q, entries, idx, token_kv, tok_pos0, l_tok, out, dtype, workspace, workspace_bytes,
                         dev_status, nullptr, shape, stream, true);
}

v4a_status v4a_csa_attend_ex(const void* q, const void* entries, const int32_t* idx, const void* token_kv,
                             long long tok_pos0, long long l_tok, float* out, v4a_dtype dtype, void* workspace,
                             size_t workspace_bytes, int* dev_status, const v4a_attend_ext* ext,
                             const v4a_shape* shape, void* stream) {
    return attend_common(q, entries, idx, token_kv, tok_pos0, l_tok, out, dtype, workspace, workspace_bytes,
                         dev_status, ext, shape, stream, true);
}

v4a_status v4a_hca_attend_ex(const void* q, const void* entries, const void* token_kv, long long tok_pos0,
                             long long l_tok, float* out, v4a_dtype dtype, void* workspace, size_t workspace_bytes,
                             const v4a_attend_ext* ext, const v4a_shape* shape, void* stream) {
    return attend_common(q, entries, nullptr, token_kv, tok_pos0, l_tok, out, dtype, workspace, workspace_bytes,
                         nullptr, ext, shape, stream, false);
}

v4a_status v4a_hca_attend(const void* q, const void* entries, const void* token_kv, long long tok_pos0,
                          long long l_tok, float* out, v4a_dtype dtype, void* workspace, size_t workspace_bytes,
                          const v4a_shape* shape, void* stream) {
    return attend_common(q, entries, nullptr, token_kv, tok_pos0, l_tok, out, dtype, workspace, workspace_bytes,
                         nullptr, nullptr, shape, stream, false);
}

static v4a_status attend_paged(const void* q, const void* entries, const int32_t* idx, const void* token_kv, float* out,
                               v4a_dtype dtype, void* workspace, size_t workspace_bytes, int* dev_status,
                               const v4a_attend_ext* ext, const v4a_paged* pg, const v4a_shape* shape, void* stream,
                               bool csa) {
    const char* what = csa ? "v4a_csa_attend_paged" : "v4a_hca_attend_paged";
    if (!shape) return fail(V4A_ERR_INVALID_ARG, "shape is NULL");
    v4a_status st = paged_check(pg, shape->m > 0 ? shape->m : 1, shape->m > 0 ? shape->ctx_len / shape->m : 0, what);
    if (st != V4A_OK) return st;
    if (shape->window > 0 && (pg->ring_rows < 1 || (long long)pg->ring_rows < (long long)shape->window + shape->n_q - 1))
        return fail(V4A_ERR_INVALID_ARG, "%s: the ring of %d rows cannot hold the window (%d + %d - 1)", what,
                    pg->ring_rows, shape->window, shape->n_q);
    return attend_common(q, entries, idx, token_kv, 0, shape->ctx_len, out, dtype, workspace, workspace_bytes,
                         dev_status, ext, shape, stream, csa, pg);
}

v4a_status v4a_csa_attend_paged(const void* q, const void* entries, const int32_t* idx, const void* token_kv, float* out,
                                v4a_dtype dtype, void* workspace, size_t workspace_bytes, int* dev_status,
                                const v4a_attend_ext* ext, const v4a_paged* pg, const v4a_shape* shape, void* stream) {
    return attend_paged(q, entries, idx, token_kv, out, dtype, workspace, workspace_bytes, dev_status, ext, pg, shape,
                        stream, true);
}

v4a_status v4a_hca_attend_paged(const void* q, const void* entries, const void* token_kv, float* out, v4a_dtype dtype,
                                void* workspace, size_t workspace_bytes, int* dev_status, const v4a_attend_ext* ext,
                                const v4a_paged* pg, const v4a_shape* shape, void* stream) {
    return attend_paged(q, entries, nullptr, token_kv, out, dtype, workspace, workspace_bytes, dev_status, ext, pg,
                        shape, stream, false);
}

size_t v4a_workspace_size(const char* op, const v4a_shape* shape, int heads_i, int d_i) {
    if (!op || !shape) return 0;
    if (strcmp(op, "topk") == 0) {
        v4a::IndexArgs a = {};
        a.batch = shape->batch;
        a.n_q = shape->n_q;
        a.m = shape->m > 0 ? shape->m : 1;
        a.heads_i = heads_i;
        a.d_i = d_i;
        a.ctx_len = shape->ctx_len;
        a.n_ent = shape->ctx_len / a.m;
        return v4a::topk_workspace_bytes(a, shape->k);
    }
    bool csa = strcmp(op, "csa_attend") == 0;
    if (csa || strcmp(op, "hca_attend") == 0) {
        v4a::AttendArgs a = {};
        a.batch = shape->batch;
        a.n_q = shape->n_q;
        a.heads = shape->heads > 0 ? shape->heads : 1;
        a.d = shape->d >= 64 ? shape->d : 64;
        a.m = shape->m > 0 ? shape->m : 1;
        a.k = csa ? shape->k : 0;
        a.window = shape->window;
        a.ctx_len = shape->ctx_len;
        a.n_ent = shape->ctx_len / a.m;
        a.idx = csa ? reinterpret_cast<const int32_t*>(1) : nullptr;
        a.dtype = V4A_BF16;  // no dtype argument: size for the larger (tensor-core) requirement
        return v4a::attend_workspace_bytes(a);
    }
    return 0;
}

const char* v4a_status_string(v4a_status st) {
    switch (st) {
    case V4A_OK: return "ok";
    case V4A_ERR_INVALID_ARG: return "invalid argument";
    case V4A_ERR_UNSUPPORTED: return "unsupported combination";
    case V4A_ERR_CUDA: return "CUDA error";
    case V4A_ERR_DEVICE_FAULT: return "device fault (bad data found by a kernel)";
    default: return "unknown status";
    }
}

const char* v4a_last_error(void) { return g_last_error; }

void v4a_test_attend_fault(int withhold_tile, int wait_polls) {
    v4a::g_test_fault.withhold = withhold_tile >= 0 ? withhold_tile : -1;
    v4a::g_test_fault.wait_polls = (uint32_t)(wait_polls > 0 ? wait_polls : 1);
    v4a::g_test_fault.stall_cycles = 1LL << 22;  // ~2 ms of no progress at 1.9 GHz
}

int v4a_version(void) { return 200; }

}  // extern "C"
