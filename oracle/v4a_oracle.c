/*
 * v4a_oracle.c -- plain, slow, obviously-correct CPU oracle for the hybrid
 * compressed-attention step of DeepSeek-V4 (CSA + HCA + sliding window).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library; it decodes every storage format itself from the
 * format's definition and accumulates everything in IEEE binary64.
 *
 * What each function follows (pages are cited by title and section):
 *  - v4ao_compress: "DeepSeek-V4 的暗线之一：分层记忆比输入框更关键"
 *    (blog.xieydd.top), section 3 "compressed KV entry 到底是什么" -- an entry
 *    is the sum over the chunk's tokens of per-channel softmax weights (from
 *    the gate logits Z) times the content vectors C; and "DeepSeek-V4:
 *    Million-Token Context via Hybrid Compressed Attention", section
 *    "Heavily Compressed Attention (HCA) / How it works" (single series, every
 *    m' consecutive tokens -> one entry, no overlap).  The same single-series
 *    rule is used for m = 4 and m' = 128.
 *  - v4ao_compress_dual: "DeepSeek-V4: Million-Token Context via Hybrid
 *    Compressed Attention", CSA, "Dual-series KV compression" -- entry i is a
 *    weighted sum of 2m tokens, the m of series a in block i and the m of
 *    series b in block i-1, with one softmax (per channel) over their 2m gate
 *    logits.
 *  - v4ao_index_scores: "How V4 makes a million-token context actually
 *    affordable" (deconstructedpapers.com), Lightning-Indexer section:
 *    I(t,s) = sum_j w_j * ReLU(q_j . k_s); the key k_s carries no head index.
 *    FP8 keys carry one positive fp32 scale per entry; the score is that scale
 *    times the sum over the stored (decoded) key values.
 *  - v4ao_topk: "1M Context != Lossless Long Memory", section 4.2 (the query
 *    attends only to the top-k entries by indexer score); ties go to the
 *    lower entry index; fewer visible entries than k selects them all.
 *  - v4ao_attend: "How V4 makes ..." attention refresher
 *    (softmax(q k^T / sqrt(d)) v) with K = V shared by all heads ("DeepSeek-V4:
 *    Million-Token Context ...", CSA "Core attention with shared KV MQA");
 *    candidates are the selected (CSA) or all visible (HCA) compressed entries
 *    plus the raw sliding-window tokens ("1M Context != ...", section 6), in
 *    ONE joint softmax.
 *  - Attention sink and output RoPE ("1M Context != Lossless Long Memory",
 *    sections 7 and 8): a per-head scalar z'_h joins the softmax denominator
 *    (read as the logit of an extra, empty candidate: the denominator gains
 *    e^{z'_h}); RoPE acts on the last R dims of the vectors, and the attention
 *    output of the query at position t is rotated at position -t.  RoPE pairs
 *    adjacent dims (2k, 2k+1) of those R with frequency base^(-2k/R).
 *  - Visibility: entry s covers tokens [m*s, m*s+m) and is visible to query
 *    position t iff m*(s+1) <= t+1 ("1M Context != ...", section 6.1: a query
 *    must not read its own, still incomplete, compressed block).
 *  - Window: tokens (t-W, t] clipped at 0 ("1M Context != ...", section 6.1,
 *    n_win = 128).  The window may overlap visible entries; both are kept.
 *  - FP4 indexer keys ("1M Context != Lossless Long Memory", section 4.2 and
 *    footnote 3: indexer KV in FP4, FP4 dot products; "DeepSeek-V4 ...",
 *    "Where It Breaks": FP4 QK indexer).  The pages name no bit format; the
 *    oracle reads it as the OCP Microscaling (MX v1.0) MXFP4 format: e2m1
 *    elements (1 sign, 2 exponent bits with bias 1, 1 fraction bit; values
 *    0, 0.5, 1, 1.5, 2, 3, 4, 6) in blocks of 32 sharing one power-of-two
 *    scale 2^X stored as an E8M0 byte X + 127.  A block is quantised with
 *    X = max(floor(log2(amax)) - 2, -127) (2 = the largest e2m1 exponent;
 *    X = -127 for an all-zero block) and element codes = nearest e2m1 of
 *    v / 2^X (ties to the even code, magnitudes above 6 clamp to 6, the sign
 *    kept even when the value rounds to zero).  "FP4 QK" is read as both
 *    operands in MXFP4: the query of each indexer head is quantised the same
 *    way (blocks of 32 along d_I), and the score is the definition above
 *    evaluated on the decoded values.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define OR_F32 0
#define OR_BF16 1
#define OR_E4M3 2
#define OR_F64 3 /* binary64 values (decoded MXFP4 operands) */

#define OR_OK 0
#define OR_ERR_ARG 1
#define OR_ERR_INDEX 4

/* ------------------------------------------------------------------ */
/* storage formats, decoded from their field definitions               */
/* ------------------------------------------------------------------ */

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double v4ao_bf16_decode(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 7) & 0xff;
    int f = h & 0x7f;
    double v;
    if (e == 0xff) {
        v = f ? NAN : INFINITY;
    } else if (e == 0) {
        v = ldexp((double)f, -126 - 7);               /* subnormal: 0.f * 2^-126 */
    } else {
        v = ldexp(1.0 + (double)f / 128.0, e - 127);
    }
    return s ? -v : v;
}

/* float8 e4m3 ("fn" variant): 1 sign, 4 exponent bits (bias 7), 3 fraction
 * bits; no infinities; S.1111.111 is NaN; largest finite magnitude 448. */
double v4ao_e4m3_decode(uint8_t c)
{
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 0xf;
    int f = c & 0x7;
    double v;
    if (e == 0xf && f == 0x7) return NAN;
    if (e == 0) v = ldexp((double)f, -6 - 3);           /* subnormal: 0.f * 2^-6 */
    else v = ldexp(1.0 + (double)f / 8.0, e - 7);
    return s ? -v : v;
}

/* Nearest e4m3 code, ties to the code with an even fraction, magnitudes
 * beyond 448 saturate to 448.  Found by searching the 127 finite
 * non-negative codes, whose values increase with the code. */
uint8_t v4ao_e4m3_encode(double v)
{
    if (isnan(v)) return 0x7f;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return sign | 0x7e;
    int lo = 0;                                        /* largest code with value <= a */
    for (int c = 0; c <= 0x7e; ++c) {
        if (v4ao_e4m3_decode((uint8_t)c) <= a) lo = c; else break;
    }
    int hi = lo < 0x7e ? lo + 1 : lo;
    double dl = a - v4ao_e4m3_decode((uint8_t)lo);
    double dh = v4ao_e4m3_decode((uint8_t)hi) - a;
    int pick;
    if (dl < dh) pick = lo;
    else if (dh < dl) pick = hi;
    else pick = (lo & 1) ? hi : lo;
    return sign | (uint8_t)pick;
}

/* Nearest bfloat16 of a binary64 value (ties to even), overflow to inf. */
uint16_t v4ao_bf16_encode(double v)
{
    if (isnan(v)) return 0x7fc0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);                                     /* a = f * 2^ex, f in [0.5,1) */
    int q = ex - 1 - 7;                                /* quantum of 8 significant bits */
    if (q < -126 - 7) q = -126 - 7;                    /* subnormal quantum */
    double r = nearbyint(ldexp(a, -q));                /* default mode: ties to even */
    double val = ldexp(r, q);
    /* largest finite bf16 is (2 - 2^-7) * 2^127 */
    if (val > ldexp(2.0 - ldexp(1.0, -7), 127)) return sign | 0x7f80;
    /* val is exactly representable in binary32; bf16 is its upper half */
    float fv = (float)val;
    uint32_t u;
    memcpy(&u, &fv, 4);
    return sign | (uint16_t)((u >> 16) & 0x7fff);
}

/* e2m1 (4 bits: sign, 2 exponent bits with bias 1, 1 fraction bit; no
 * infinities or NaN): exponent field 0 is subnormal, 0.f * 2^0. */
double v4ao_e2m1_decode(uint8_t c)
{
    int s = (c >> 3) & 1;
    int e = (c >> 1) & 3;
    int f = c & 1;
    double v = e == 0 ? 0.5 * f : ldexp(1.0 + 0.5 * f, e - 1);
    return s ? -v : v;
}

/* Nearest e2m1 code of v (ties to the code with an even fraction bit),
 * magnitudes above 6 clamp to 6; the sign bit is the sign of v, also when
 * the magnitude rounds to 0.  Found by searching the 8 non-negative codes,
 * whose values increase with the code. */
uint8_t v4ao_e2m1_encode(double v)
{
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    double a = fabs(v);
    if (a >= 6.0) return sign | 0x7;
    int lo = 0;                                        /* largest code with value <= a */
    for (int c = 0; c <= 7; ++c) {
        if (v4ao_e2m1_decode((uint8_t)c) <= a) lo = c; else break;
    }
    int hi = lo < 7 ? lo + 1 : lo;
    double dl = a - v4ao_e2m1_decode((uint8_t)lo);
    double dh = v4ao_e2m1_decode((uint8_t)hi) - a;
    int pick;
    if (dl < dh) pick = lo;
    else if (dh < dl) pick = hi;
    else pick = (lo & 1) ? hi : lo;
    return sign | (uint8_t)pick;
}

static double load_elem(const void* p, int dt, size_t i)
{
    switch (dt) {
    case OR_F32: return (double)((const float*)p)[i];
    case OR_BF16: return v4ao_bf16_decode(((const uint16_t*)p)[i]);
    case OR_E4M3: return v4ao_e4m3_decode(((const uint8_t*)p)[i]);
    case OR_F64: return ((const double*)p)[i];
    default: return NAN;
    }
}

/* ------------------------------------------------------------------ */
/* a tiny parallel-for over independent work items                     */
/* ------------------------------------------------------------------ */

static int g_threads = 0;

void v4ao_set_threads(int n) { g_threads = n; }

int v4ao_get_threads(void)
{
    if (g_threads > 0) return g_threads;
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

typedef void (*work_fn)(void* ctx, long long item);

typedef struct {
    work_fn fn;
    void* ctx;
    long long begin, end;
} span_t;

static void* run_span(void* arg)
{
    span_t* s = (span_t*)arg;
    for (long long i = s->begin; i < s->end; ++i) s->fn(s->ctx, i);
    return NULL;
}

static void parallel_for(long long n, work_fn fn, void* ctx)
{
    int t = v4ao_get_threads();
    if (t > n) t = (int)n;
    if (t <= 1) {
        for (long long i = 0; i < n; ++i) fn(ctx, i);
        return;
    }
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * t);
    span_t* sp = (span_t*)malloc(sizeof(span_t) * t);
    for (int k = 0; k < t; ++k) {
        sp[k].fn = fn;
        sp[k].ctx = ctx;
        sp[k].begin = n * k / t;
        sp[k].end = n * (k + 1) / t;
        pthread_create(&th[k], NULL, run_span, &sp[k]);
    }
    for (int k = 0; k < t; ++k) pthread_join(th[k], NULL);
    free(th);
    free(sp);
}

/* ------------------------------------------------------------------ */
/* visibility rule                                                     */
/* ------------------------------------------------------------------ */

/* number of compressed entries visible to query position t: those s with
 * m*(s+1) <= t+1 */
long long v4ao_n_visible(long long t, long long m) { return (t + 1) / m; }

/* ------------------------------------------------------------------ */
/* compression                                                          */
/* ------------------------------------------------------------------ */

typedef struct {
    const void* x;
    const void* z;
    int dt;
    long long n_tok, c, m, n_ent;
    double* out;
} compress_ctx;

static void compress_item(void* vctx, long long item)
{
    compress_ctx* k = (compress_ctx*)vctx;
    long long b = item / k->n_ent, s = item % k->n_ent;
    for (long long ch = 0; ch < k->c; ++ch) {
        /* softmax over the chunk's m tokens, separately for every channel */
        double zmax = -INFINITY;
        for (long long i = 0; i < k->m; ++i) {
            size_t at = (size_t)((b * k->n_tok + s * k->m + i) * k->c + ch);
            double z = load_elem(k->z, k->dt, at);
            if (z > zmax) zmax = z;
        }
        double den = 0.0, num = 0.0;
        for (long long i = 0; i < k->m; ++i) {
            size_t at = (size_t)((b * k->n_tok + s * k->m + i) * k->c + ch);
            double e = exp(load_elem(k->z, k->dt, at) - zmax);
            den += e;
            num += e * load_elem(k->x, k->dt, at);
        }
        k->out[(b * k->n_ent + s) * k->c + ch] = num / den;
    }
}

/* x, gate: [batch][n_tok][channels] in dtype dt (tokens of complete chunks
 * starting at a chunk boundary).  out: [batch][n_tok/m][channels] binary64. */
int v4ao_compress(const void* x, const void* gate, int dt, long long batch, long long n_tok,
                  long long channels, long long m, double* out)
{
    if (!x || !gate || !out || batch < 0 || n_tok < 0 || channels < 1 || m < 1) return OR_ERR_ARG;
    if (dt != OR_F32 && dt != OR_BF16) return OR_ERR_ARG;
    compress_ctx k = {x, gate, dt, n_tok, channels, m, n_tok / m, out};
    parallel_for(batch * k.n_ent, compress_item, &k);
    return OR_OK;
}

typedef struct {
    const void *xa, *za, *xb, *zb, *pxb, *pzb;
    int dt;
    long long n_tok, c, m, n_ent;
    double* out;
} compress_dual_ctx;

static void compress_dual_item(void* vctx, long long item)
{
    compress_dual_ctx* k = (compress_dual_ctx*)vctx;
    long long b = item / k->n_ent, s = item % k->n_ent;
    const int has_b = s >= 1 || (k->pxb && k->pzb);
    for (long long ch = 0; ch < k->c; ++ch) {
        /* the 2m logits: series a over block s, series b over block s-1 (from the
           previous block of the range, or from prev_* for block 0) */
        double zv[2][1024], xv[2][1024];
        for (long long i = 0; i < k->m; ++i) {
            size_t at = (size_t)((b * k->n_tok + s * k->m + i) * k->c + ch);
            zv[0][i] = load_elem(k->za, k->dt, at);
            xv[0][i] = load_elem(k->xa, k->dt, at);
            if (!has_b) continue;
            if (s >= 1) {
                size_t bt = (size_t)((b * k->n_tok + (s - 1) * k->m + i) * k->c + ch);
                zv[1][i] = load_elem(k->zb, k->dt, bt);
                xv[1][i] = load_elem(k->xb, k->dt, bt);
            } else {
                size_t bt = (size_t)((b * k->m + i) * k->c + ch);
                zv[1][i] = load_elem(k->pzb, k->dt, bt);
                xv[1][i] = load_elem(k->pxb, k->dt, bt);
            }
        }
        double zmax = -INFINITY;
        for (int ser = 0; ser < (has_b ? 2 : 1); ++ser)
            for (long long i = 0; i < k->m; ++i)
                if (zv[ser][i] > zmax) zmax = zv[ser][i];
        double den = 0.0, num = 0.0;
        for (int ser = 0; ser < (has_b ? 2 : 1); ++ser)
            for (long long i = 0; i < k->m; ++i) {
                double e = exp(zv[ser][i] - zmax);
                den += e;
                num += e * xv[ser][i];
            }
        k->out[(b * k->n_ent + s) * k->c + ch] = num / den;
    }
}

/* xa, za, xb, zb: [batch][n_tok][channels] (dtype dt), the two series over the
 * same token range starting at a block boundary; prev_xb, prev_zb: series b over
 * the block before the range, [batch][m][channels], or both NULL when the range
 * starts the sequence.  out: [batch][n_tok/m][channels] binary64.  m <= 1024. */
int v4ao_compress_dual(const void* xa, const void* za, const void* xb, const void* zb, const void* prev_xb,
                       const void* prev_zb, int dt, long long batch, long long n_tok, long long channels,
                       long long m, double* out)
{
    if (!xa || !za || !xb || !zb || !out || batch < 0 || n_tok < 0 || channels < 1 || m < 1 || m > 1024)
        return OR_ERR_ARG;
    if ((prev_xb == NULL) != (prev_zb == NULL)) return OR_ERR_ARG;
    if (dt != OR_F32 && dt != OR_BF16) return OR_ERR_ARG;
    compress_dual_ctx k = {xa, za, xb, zb, prev_xb, prev_zb, dt, n_tok, channels, m, n_tok / m, out};
    parallel_for(batch * k.n_ent, compress_dual_item, &k);
    return OR_OK;
}

/* Per-row e4m3 quantisation of binary64 values: scale = amax / 448 (1 when the
 * row is all zero), code = nearest e4m3 of value / scale. */
int v4ao_quantize_e4m3_rows(const double* v, long long rows, long long cols, uint8_t* codes,
                            double* scales)
{
    if (!v || !codes || !scales || rows < 0 || cols < 1) return OR_ERR_ARG;
    for (long long r = 0; r < rows; ++r) {
        double amax = 0.0;
        for (long long c = 0; c < cols; ++c) {
            double a = fabs(v[r * cols + c]);
            if (a > amax) amax = a;
        }
        double sc = amax > 0.0 ? amax / 448.0 : 1.0;
        scales[r] = sc;
        for (long long c = 0; c < cols; ++c) codes[r * cols + c] = v4ao_e4m3_encode(v[r * cols + c] / sc);
    }
    return OR_OK;
}

/* MXFP4 quantisation (OCP MX v1.0) of rows of binary64 values, cols a
 * multiple of 32: per block of 32, X = max(floor(log2(amax)) - 2, -127)
 * (-127 for an all-zero block), exps[block] = X + 127, element i's code =
 * nearest e2m1 of v_i / 2^X, two codes per byte (element 2i in the low
 * nibble of byte i). */
int v4ao_quantize_mxfp4(const double* v, long long rows, long long cols, uint8_t* codes, uint8_t* exps)
{
    if (!v || !codes || !exps || rows < 0 || cols < 32 || cols % 32) return OR_ERR_ARG;
    for (long long r = 0; r < rows; ++r) {
        for (long long b = 0; b < cols / 32; ++b) {
            const double* x = v + r * cols + b * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i)
                if (fabs(x[i]) > amax) amax = fabs(x[i]);
            int X = -127;
            if (amax > 0.0) {
                int e;
                frexp(amax, &e);                       /* amax = f * 2^e, f in [0.5, 1) */
                X = (e - 1) - 2;                       /* floor(log2(amax)) - 2 */
                if (X < -127) X = -127;
                if (X > 127) return OR_ERR_ARG;
            }
            exps[r * (cols / 32) + b] = (uint8_t)(X + 127);
            uint8_t* out = codes + r * (cols / 2) + b * 16;
            for (int i = 0; i < 32; i += 2) {
                uint8_t lo = v4ao_e2m1_encode(ldexp(x[i], -X));
                uint8_t hi = v4ao_e2m1_encode(ldexp(x[i + 1], -X));
                out[i / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
    return OR_OK;
}

/* MXFP4 rows -> binary64 values: element = e2m1 value * 2^(exp - 127). */
int v4ao_decode_mxfp4(const uint8_t* codes, const uint8_t* exps, long long rows, long long cols, double* out)
{
    if (!codes || !exps || !out || rows < 0 || cols < 32 || cols % 32) return OR_ERR_ARG;
    for (long long r = 0; r < rows; ++r)
        for (long long i = 0; i < cols; ++i) {
            uint8_t byte = codes[r * (cols / 2) + i / 2];
            uint8_t c = (i & 1) ? (byte >> 4) : (byte & 0xf);
            uint8_t xb = exps[r * (cols / 32) + i / 32];
            out[r * cols + i] = xb == 0xff ? NAN : ldexp(v4ao_e2m1_decode(c), (int)xb - 127);  /* 0xff: NaN */
        }
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* Lightning-Indexer scores                                            */
/* ------------------------------------------------------------------ */

typedef struct {
    const void* q;
    int q_dt;
    const float* w;
    const void* key;
    int k_dt;
    const float* scale;
    long long n_q, ctx_len, m, hi, di, n_ent;
    double* scores;
} index_ctx;

static void index_item(void* vctx, long long item)
{
    index_ctx* k = (index_ctx*)vctx;
    long long b = item / k->n_q, j = item % k->n_q;
    long long t = k->ctx_len - k->n_q + j;
    long long nvis = v4ao_n_visible(t, k->m);
    double* qd = (double*)malloc(sizeof(double) * k->hi * k->di);
    for (long long h = 0; h < k->hi; ++h)
        for (long long c = 0; c < k->di; ++c)
            qd[h * k->di + c] = load_elem(k->q, k->q_dt, (size_t)(((b * k->n_q + j) * k->hi + h) * k->di + c));
    double* kd = (double*)malloc(sizeof(double) * k->di);
    double* row = k->scores + (b * k->n_q + j) * k->n_ent;
    for (long long s = 0; s < k->n_ent; ++s) {
        if (s >= nvis) {
            row[s] = -INFINITY;
            continue;
        }
        for (long long c = 0; c < k->di; ++c)
            kd[c] = load_elem(k->key, k->k_dt, (size_t)((b * k->n_ent + s) * k->di + c));
        double acc = 0.0;
        for (long long h = 0; h < k->hi; ++h) {
            double dot = 0.0;
            for (long long c = 0; c < k->di; ++c) dot += qd[h * k->di + c] * kd[c];
            double wj = (double)k->w[(b * k->n_q + j) * k->hi + h];
            acc += wj * (dot > 0.0 ? dot : 0.0);
        }
        double sc = k->scale ? (double)k->scale[b * k->n_ent + s] : 1.0;
        row[s] = sc * acc;
    }
    free(kd);
    free(qd);
}

/* q: [batch][n_q][heads_i][d_i] (q_dt), w: [batch][n_q][heads_i] fp32,
 * key: [batch][ctx_len/m][d_i] (k_dt), scale: [batch][ctx_len/m] fp32 or NULL.
 * scores: [batch][n_q][ctx_len/m]; -inf where the entry is not visible. */
int v4ao_index_scores(const void* q, int q_dt, const float* w, const void* key, int k_dt,
                      const float* scale, long long batch, long long n_q, long long ctx_len, long long m,
                      long long heads_i, long long d_i, double* scores)
{
    if (!q || !w || !key || !scores || batch < 0 || n_q < 1 || m < 1 || heads_i < 1 || d_i < 1) return OR_ERR_ARG;
    if (n_q > ctx_len) return OR_ERR_ARG;
    if (q_dt != OR_F32 && q_dt != OR_BF16 && q_dt != OR_F64) return OR_ERR_ARG;
    if (k_dt != OR_F32 && k_dt != OR_BF16 && k_dt != OR_E4M3 && k_dt != OR_F64) return OR_ERR_ARG;
    index_ctx k = {q, q_dt, w, key, k_dt, scale, n_q, ctx_len, m, heads_i, d_i, ctx_len / m, scores};
    parallel_for(batch * n_q, index_item, &k);
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* top-k selection                                                      */
/* ------------------------------------------------------------------ */

typedef struct {
    double score;
    long long index;
} cand_t;

/* higher score first; equal scores: lower index first */
static int cand_cmp(const void* a, const void* b)
{
    const cand_t* x = (const cand_t*)a;
    const cand_t* y = (const cand_t*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->index > y->index) - (x->index < y->index);
}

static int ll_cmp(const void* a, const void* b)
{
    long long x = *(const long long*)a, y = *(const long long*)b;
    return (x > y) - (x < y);
}

/* For one row of n scores of which the first nvis are visible: the
 * min(k, nvis) best by (score desc, index asc), written in ascending index
 * order, padded with -1.  kth: the smallest selected score (-inf when fewer
 * than k entries are visible). */
int v4ao_select_row(const double* scores, long long nvis, long long k, int32_t* idx, double* sel_scores,
                    double* kth)
{
    if (!scores || !idx || nvis < 0 || k < 1) return OR_ERR_ARG;
    cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (nvis > 0 ? nvis : 1));
    for (long long s = 0; s < nvis; ++s) {
        c[s].score = scores[s];
        c[s].index = s;
    }
    qsort(c, (size_t)nvis, sizeof(cand_t), cand_cmp);
    long long take = nvis < k ? nvis : k;
    long long* chosen = (long long*)malloc(sizeof(long long) * (take > 0 ? take : 1));
    for (long long i = 0; i < take; ++i) chosen[i] = c[i].index;
    qsort(chosen, (size_t)take, sizeof(long long), ll_cmp);
    for (long long i = 0; i < k; ++i) {
        idx[i] = i < take ? (int32_t)chosen[i] : -1;
        if (sel_scores) sel_scores[i] = i < take ? scores[chosen[i]] : -INFINITY;
    }
    if (kth) *kth = (take == k) ? c[k - 1].score : -INFINITY;
    free(chosen);
    free(c);
    return OR_OK;
}

typedef struct {
    const double* scores;
    long long n_q, ctx_len, m, n_ent, k;
    int32_t* idx;
    double* sel;
    double* kth;
} topk_ctx;

static void topk_item(void* vctx, long long item)
{
    topk_ctx* c = (topk_ctx*)vctx;
    long long j = item % c->n_q;
    long long t = c->ctx_len - c->n_q + j;
    long long nvis = v4ao_n_visible(t, c->m);
    if (nvis > c->n_ent) nvis = c->n_ent;
    v4ao_select_row(c->scores + item * c->n_ent, nvis, c->k, c->idx + item * c->k,
                    c->sel ? c->sel + item * c->k : NULL, c->kth ? c->kth + item : NULL);
}

/* Indexer scores followed by the top-k select, per (sequence, query).
 * idx: [batch][n_q][k] int32; sel_scores (nullable): [batch][n_q][k];
 * kth (nullable): [batch][n_q]; scores_out (nullable): [batch][n_q][ctx_len/m]. */
int v4ao_topk(const void* q, int q_dt, const float* w, const void* key, int k_dt, const float* scale,
              long long batch, long long n_q, long long ctx_len, long long m, long long heads_i, long long d_i,
              long long k, int32_t* idx, double* sel_scores, double* kth, double* scores_out)
{
    if (k < 1 || !idx) return OR_ERR_ARG;
    long long n_ent = ctx_len / m;
    double* sc = scores_out;
    if (!sc) sc = (double*)malloc(sizeof(double) * (size_t)(batch * n_q * (n_ent > 0 ? n_ent : 1)));
    int st = v4ao_index_scores(q, q_dt, w, key, k_dt, scale, batch, n_q, ctx_len, m, heads_i, d_i, sc);
    if (st == OR_OK) {
        topk_ctx c = {sc, n_q, ctx_len, m, n_ent, k, idx, sel_scores, kth};
        parallel_for(batch * n_q, topk_item, &c);
    }
    if (!scores_out) free(sc);
    return st;
}

/* ------------------------------------------------------------------ */
/* attention over compressed entries + sliding window                  */
/* ------------------------------------------------------------------ */

typedef struct {
    const void* q;
    const void* ent;
    const int32_t* idx;
    long long k_sel;
    const void* tok;
    long long tok_pos0, l_tok;
    int dt;
    long long n_q, heads, d, m, window, ctx_len, n_ent, hgroup;
    double* out;
    int bad_index; /* set when an idx entry is out of range */
    const double* sink; /* per-head sink logits, or NULL */
    long long rope_dims;
    double rope_base;
} attend_ctx;

/* Candidate rows of query (b, j): pointers to element 0 of each row, as
 * (source, row) pairs.  Returns the count; *bad is set if an idx entry is
 * neither -1 nor a visible entry (such entries are skipped). */
static long long gather_candidates(const attend_ctx* a, long long b, long long j, size_t* rows, int* src,
                                   int* bad)
{
    long long t = a->ctx_len - a->n_q + j;
    long long nvis = v4ao_n_visible(t, a->m);
    if (nvis > a->n_ent) nvis = a->n_ent;
    long long n = 0;
    if (a->idx) {
        const int32_t* ix = a->idx + (b * a->n_q + j) * a->k_sel;
        for (long long i = 0; i < a->k_sel; ++i) {
            long long s = ix[i];
            if (s == -1) continue;
            if (s < 0 || s >= nvis) {
                *bad = 1;
                continue;
            }
            rows[n] = (size_t)(b * a->n_ent + s);
            src[n++] = 0;
        }
    } else {
        for (long long s = 0; s < nvis; ++s) {
            rows[n] = (size_t)(b * a->n_ent + s);
            src[n++] = 0;
        }
    }
    long long p0 = t - a->window + 1;
    if (p0 < 0) p0 = 0;
    for (long long p = p0; p <= t; ++p) {
        long long r = p - a->tok_pos0;
        if (r < 0 || r >= a->l_tok) {
            *bad = 1;
            continue;
        }
        rows[n] = (size_t)(b * a->l_tok + r);
        src[n++] = 1;
    }
    return n;
}

/* decode the n candidate rows into an [n][d] binary64 matrix */
static void decode_rows(const attend_ctx* a, const size_t* rows, const int* src, long long n, double* mat)
{
    for (long long i = 0; i < n; ++i) {
        const void* base = src[i] ? a->tok : a->ent;
        for (long long c = 0; c < a->d; ++c)
            mat[i * a->d + c] = load_elem(base, a->dt, rows[i] * (size_t)a->d + (size_t)c);
    }
}

/* softmax weights of one head over the n decoded candidate rows */
static void head_weights(const attend_ctx* a, long long b, long long j, long long h, const double* mat, long long n,
                         double* wts)
{
    long long d = a->d;
    double inv_sqrt_d = 1.0 / sqrt((double)d);
    size_t qoff = (size_t)(((b * a->n_q + j) * a->heads + h) * d);
    double* qd = (double*)malloc(sizeof(double) * d);
    for (long long c = 0; c < d; ++c) qd[c] = load_elem(a->q, a->dt, qoff + c);
    double mx = -INFINITY;
    for (long long i = 0; i < n; ++i) {
        double dot = 0.0;
        for (long long c = 0; c < d; ++c) dot += qd[c] * mat[i * d + c];
        wts[i] = dot * inv_sqrt_d;
        if (wts[i] > mx) mx = wts[i];
    }
    double den = 0.0;
    for (long long i = 0; i < n; ++i) {
        wts[i] = exp(wts[i] - mx);
        den += wts[i];
    }
    if (a->sink) den += exp(a->sink[h] - mx); /* the sink: in the denominator only */
    for (long long i = 0; i < n; ++i) wts[i] /= den;
    free(qd);
}

/* RoPE at position pos on the last rope_dims entries of x[0..d): pair k = (d - R + 2k,
 * d - R + 2k + 1) rotates by pos * base^(-2k/R). */
static void rope_rotate(double* x, long long d, long long rope_dims, double base, double pos)
{
    for (long long k = 0; k < rope_dims / 2; ++k) {
        double ang = pos * pow(base, -2.0 * (double)k / (double)rope_dims);
        double c = cos(ang), sn = sin(ang);
        double* p = x + (d - rope_dims) + 2 * k;
        double u = p[0], v = p[1];
        p[0] = u * c - v * sn;
        p[1] = u * sn + v * c;
    }
}

/* rows: [n][d] binary64, rotated in place, row r at position pos[r] */
int v4ao_rope(double* rows, long long n, long long d, const double* pos, long long rope_dims, double base)
{
    if (!rows || !pos || n < 0 || d < 1 || rope_dims < 0 || rope_dims > d || rope_dims % 2) return OR_ERR_ARG;
    for (long long r = 0; r < n; ++r) rope_rotate(rows + r * d, d, rope_dims, base, pos[r]);
    return OR_OK;
}

static void attend_item(void* vctx, long long item)
{
    attend_ctx* a = (attend_ctx*)vctx;
    long long ngroups = (a->heads + a->hgroup - 1) / a->hgroup;
    long long g = item % ngroups;
    long long bj = item / ngroups;
    long long b = bj / a->n_q, j = bj % a->n_q;
    long long cap = (a->idx ? a->k_sel : a->n_ent) + a->window + 1;
    size_t* rows = (size_t*)malloc(sizeof(size_t) * cap);
    int* src = (int*)malloc(sizeof(int) * cap);
    double* wts = (double*)malloc(sizeof(double) * cap);
    int bad = 0;
    long long n = gather_candidates(a, b, j, rows, src, &bad);
    if (bad) a->bad_index = 1;
    double* mat = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * (size_t)a->d);
    decode_rows(a, rows, src, n, mat);
    for (long long h = g * a->hgroup; h < (g + 1) * a->hgroup && h < a->heads; ++h) {
        double* o = a->out + ((b * a->n_q + j) * a->heads + h) * a->d;
        for (long long c = 0; c < a->d; ++c) o[c] = 0.0;
        if (n == 0) continue;                         /* empty candidate set: zeros */
        head_weights(a, b, j, h, mat, n, wts);
        for (long long i = 0; i < n; ++i)
            for (long long c = 0; c < a->d; ++c) o[c] += wts[i] * mat[i * a->d + c];
        if (a->rope_dims > 0) rope_rotate(o, a->d, a->rope_dims, a->rope_base, -(double)(a->ctx_len - a->n_q + j));
    }
    free(mat);
    free(wts);
    free(src);
    free(rows);
}

/* q: [batch][n_q][heads][d]; entries: [batch][ctx_len/m][d]; idx: [batch][n_q][k_sel]
 * int32 (-1 = empty slot) or NULL for dense attention over every visible
 * entry; token_kv: [batch][l_tok][d] whose row r holds position tok_pos0 + r;
 * all of q/entries/token_kv in dtype dt.  out: [batch][n_q][heads][d] binary64.
 * Returns OR_ERR_INDEX (after computing everything else) if an idx entry was
 * out of range or the window was not covered by token_kv. */
int v4ao_attend_ex(const void* q, const void* entries, const int32_t* idx, long long k_sel, const void* token_kv,
                   long long tok_pos0, long long l_tok, int dt, long long batch, long long n_q, long long heads,
                   long long d, long long m, long long window, long long ctx_len, const double* sink,
                   long long rope_dims, double rope_base, double* out)
{
    if (!q || !entries || !token_kv || !out || batch < 0 || n_q < 1 || heads < 1 || d < 1 || m < 1 || window < 0)
        return OR_ERR_ARG;
    if (n_q > ctx_len || (idx && k_sel < 1)) return OR_ERR_ARG;
    if (rope_dims < 0 || rope_dims > d || rope_dims % 2 || (rope_dims > 0 && !(rope_base > 0.0))) return OR_ERR_ARG;
    attend_ctx a = {q, entries, idx, k_sel, token_kv, tok_pos0, l_tok, dt, n_q, heads, d, m, window, ctx_len,
                    ctx_len / m, 8, out, 0, sink, rope_dims, rope_base};
    long long ngroups = (heads + a.hgroup - 1) / a.hgroup;
    parallel_for(batch * n_q * ngroups, attend_item, &a);
    return a.bad_index ? OR_ERR_INDEX : OR_OK;
}

int v4ao_attend(const void* q, const void* entries, const int32_t* idx, long long k_sel, const void* token_kv,
                long long tok_pos0, long long l_tok, int dt, long long batch, long long n_q, long long heads,
                long long d, long long m, long long window, long long ctx_len, double* out)
{
    return v4ao_attend_ex(q, entries, idx, k_sel, token_kv, tok_pos0, l_tok, dt, batch, n_q, heads, d, m, window,
                          ctx_len, NULL, 0, 10000.0, out);
}

/* Softmax weights of one (sequence b, query j, head h) over its candidate
 * list (selected or all visible entries first, then the window tokens in
 * increasing position).  wts must hold k_sel (or ctx_len/m) + window entries.
 * Returns the number of candidates, or -1 on a bad argument. */
long long v4ao_attend_weights(const void* q, const void* entries, const int32_t* idx, long long k_sel,
                              const void* token_kv, long long tok_pos0, long long l_tok, int dt, long long n_q,
                              long long heads, long long d, long long m, long long window, long long ctx_len,
                              long long b, long long j, long long h, double* wts)
{
    if (!q || !entries || !token_kv || !wts || j < 0 || j >= n_q || h < 0 || h >= heads) return -1;
    attend_ctx a = {q, entries, idx, k_sel, token_kv, tok_pos0, l_tok, dt, n_q, heads, d, m, window, ctx_len,
                    ctx_len / m, 8, NULL, 0, NULL, 0, 10000.0};
    long long cap = (idx ? k_sel : a.n_ent) + window + 1;
    size_t* rows = (size_t*)malloc(sizeof(size_t) * cap);
    int* src = (int*)malloc(sizeof(int) * cap);
    int bad = 0;
    long long n = gather_candidates(&a, b, j, rows, src, &bad);
    double* mat = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * (size_t)d);
    decode_rows(&a, rows, src, n, mat);
    if (n > 0) head_weights(&a, b, j, h, mat, n, wts);
    free(mat);
    free(src);
    free(rows);
    return n;
}
