/*
 * Paged-KV-cache attention oracle: a plain, slow, obviously correct CPU
 * reference in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load this library.  The product path
 * (libpagedkv and its Python binding) never calls it, and the two share no
 * code, headers, tables or helpers.
 *
 * Sources (four web pages on paged KV caches and FlashAttention; cited by
 * title and section):
 *   [KVFA]  "大模型推理优化：KV Cache与FlashAttention实战"
 *   [FAPKV] "Flash Attention与Paged KV Cache优化大模型计算效率"
 *   [KV3X]  "大模型推理优化实战：KV Cache + Flash Attention，让 Token 生成快 3 倍"
 *   [SYS]   "LLM推理系统优化：KV缓存管理与动态批处理技术"
 *
 * What is computed, and where it is defined:
 *   - attention of one query row over the cached keys,
 *     out = softmax(scale * q K^T) V, with the keys/values of all earlier
 *     tokens kept in a cache:  [KVFA] §2.1 "KV Cache的本质原理" and [KV3X]
 *     "KV Cache 的工作原理" (the TransformerWithKVCache forward: concatenate the
 *     cache, scores, softmax, weighted sum of values); the per-key loop of
 *     [KV3X] "先搞懂：大模型推理为什么慢？" (dot product per key, softmax,
 *     weighted sum).  The softmax here is the plain two-pass definition
 *     (max, exp, sum, divide), deliberately NOT the online recurrence.
 *   - the paged layout: K/V live in fixed-size pages of a physical pool and a
 *     per-sequence table maps logical page -> physical page:  [FAPKV] §3.2
 *     "分页式缓存设计" (fixed-size pages, central page table, PageTable with
 *     page = (page_size, d_model)) and [SYS] §3.1.  Pool layout
 *     [num_pages][page_size][num_kv_heads][head_dim]; logical token i of
 *     sequence b is row (i % page_size) of page block_tables[b][i / page_size].
 *   - grouped-query attention: query head h reads KV head h / (Hq / Hkv)
 *     (contiguous groups, the repeat_interleave of [SYS] §2.1).
 *   - chunked prefill: a chunk of n query rows of a sequence with context
 *     length ctx sits at absolute positions ctx-n .. ctx-1 (bottom-right
 *     alignment); with causal masking row r attends keys 0 .. ctx-n+r.
 *   - local (sliding-window) attention, the window_size argument of the
 *     attention call in [KVFA] §5.1 ("局部注意力"): with window w > 0 a query at
 *     position pos only sees keys pos-w+1 .. pos (keys below 0 do not exist);
 *     w <= 0 means no window.  Decode's query sits at pos = ctx-1.  The pages
 *     show the window only with causal masking; without it the window bounds
 *     the lower side alone (keys pos-w+1 .. ctx-1).
 *   - symmetric INT8 quantisation of a K/V row ([SYS] §3.2 "量化压缩的工程实践",
 *     bits = 8, one group = one (token, KV head) row):  a = max|x| (fp32),
 *     scale = fp16(a / 127) (round to nearest even), code =
 *     clamp(round_half_even(x / float(scale)), -127, 127); a zero scale gives
 *     zero codes.  Dequantised value = code * scale.  (Readings where the
 *     page is silent: NaN elements are ignored by the max and get code 0.)
 *   - the cache append (slot-mapping scatter): row t of the new K/V goes to
 *     slot slot_mapping[t] = page * page_size + offset; negative slots are
 *     skipped.  Byte copy.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_F16 = 2, OR_I8 = 3, OR_F64 = 4 };
enum { OR_OK = 0, OR_EBADARG = -1, OR_ERANGE = -2, OR_ENOMEM = -3 };

/* ---- element decoding (exact widening to double) ------------------------ */

static double or_from_bf16(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16 -> double, written out from the format's definition. */
static double or_from_f16(uint16_t h) {
    int sign = h >> 15;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);               /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25);   /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* float -> IEEE binary16 bits, round to nearest even. */
static uint16_t or_to_f16(float f) {
    uint32_t x;
    memcpy(&x, &f, sizeof x);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    double a = fabs((double)f);
    if (isnan(f)) return (uint16_t)(sign | 0x7e00u);
    if (a < ldexp(1.0, -14)) {                      /* subnormal range */
        double r = rint(a * ldexp(1.0, 24));        /* units of 2^-24 */
        return (uint16_t)(sign | (uint16_t)r);      /* r == 1024 is the smallest normal */
    }
    int ex;
    frexp(a, &ex);                                  /* a = mant * 2^ex, mant in [0.5,1) */
    int E = ex - 1;                                 /* a in [2^E, 2^(E+1)) */
    double r = rint(ldexp(a, 10 - E));              /* in [1024, 2048] */
    if (r >= 2048.0) { r = 1024.0; E += 1; }
    if (E > 15) return (uint16_t)(sign | 0x7c00u);  /* overflow -> inf */
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)(r - 1024.0));
}

static double or_elem(const void* base, int dtype, int64_t i) {
    switch (dtype) {
    case OR_F32: return (double)((const float*)base)[i];
    case OR_BF16: return or_from_bf16(((const uint16_t*)base)[i]);
    case OR_F16: return or_from_f16(((const uint16_t*)base)[i]);
    case OR_I8: return (double)((const int8_t*)base)[i];
    case OR_F64: return ((const double*)base)[i];
    default: return NAN;
    }
}

double oracle_bf16_to_double(uint16_t b) { return or_from_bf16(b); }
double oracle_f16_to_double(uint16_t h) { return or_from_f16(h); }
uint16_t oracle_float_to_f16(float f) { return or_to_f16(f); }

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- cache append ------------------------------------------------------- */

/* Copy row t of k (and v) to row slot_mapping[t] of the pools.  row_bytes is
 * num_kv_heads * head_dim * element size.  Negative slots are skipped; a slot
 * at or past num_slots is an error (nothing after it is written). */
int oracle_kv_cache_write(const void* k, const void* v, const int64_t* slot_mapping,
                          int64_t num_tokens, void* k_pool, void* v_pool,
                          int64_t row_bytes, int64_t num_slots) {
    if (num_tokens < 0 || row_bytes <= 0 || num_slots < 0) return OR_EBADARG;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t s = slot_mapping[t];
        if (s < 0) continue;
        if (s >= num_slots) return OR_ERANGE;
        memcpy((char*)k_pool + s * row_bytes, (const char*)k + t * row_bytes, (size_t)row_bytes);
        memcpy((char*)v_pool + s * row_bytes, (const char*)v + t * row_bytes, (size_t)row_bytes);
    }
    return OR_OK;
}

/* ---- symmetric INT8 quantisation of rows of d elements ------------------ */

int oracle_quantize_int8(const void* x, int x_dtype, int64_t rows, int d,
                         int8_t* codes, uint16_t* scales) {
    if (rows < 0 || d <= 0) return OR_EBADARG;
    if (x_dtype != OR_F32 && x_dtype != OR_BF16 && x_dtype != OR_F16) return OR_EBADARG;
    for (int64_t r = 0; r < rows; ++r) {
        float a = 0.0f;                         /* NaN elements are ignored */
        for (int j = 0; j < d; ++j) {
            float v = (float)or_elem(x, x_dtype, r * d + j);
            float av = fabsf(v);
            if (av > a) a = av;
        }
        float s32 = a / 127.0f;                /* fp32 division */
        uint16_t s16 = or_to_f16(s32);
        float s = (float)or_from_f16(s16);
        scales[r] = s16;
        for (int j = 0; j < d; ++j) {
            int8_t c = 0;
            if (s != 0.0f) {
                float v = (float)or_elem(x, x_dtype, r * d + j);
                float t = rintf(v / s);        /* fp32 division, ties to even */
                if (t != t) t = 0.0f;          /* NaN element -> code 0 */
                if (t > 127.0f) t = 127.0f;
                if (t < -127.0f) t = -127.0f;
                c = (int8_t)t;
            }
            codes[r * d + j] = c;
        }
    }
    return OR_OK;
}

/* ---- attention ---------------------------------------------------------- */

typedef struct {
    const void* k_pages; const void* v_pages; int kv_dtype;
    const uint16_t* k_scales; const uint16_t* v_scales;
    const int32_t* block_tables; int max_pages_per_seq;
    int num_kv_heads; int head_dim; int page_size; int64_t num_pages;
} or_cache;

/* Value of element d of key (is_v=0) or value (is_v=1) of logical token i of
 * sequence b, KV head kvh.  Sets *bad on an out-of-range page. */
static double or_kv(const or_cache* c, int is_v, int b, int i, int kvh, int d, int* bad) {
    int32_t page = c->block_tables[(int64_t)b * c->max_pages_per_seq + i / c->page_size];
    if (page < 0 || page >= c->num_pages) { *bad = 1; return 0.0; }
    int64_t slot = (int64_t)page * c->page_size + i % c->page_size;
    int64_t row = slot * c->num_kv_heads + kvh;
    double x = or_elem(is_v ? c->v_pages : c->k_pages, c->kv_dtype, row * c->head_dim + d);
    if (c->kv_dtype == OR_I8) x *= or_from_f16((is_v ? c->v_scales : c->k_scales)[row]);
    return x;
}

/* One query row (D values already in qd) against keys k_lo..k_hi-1 of
 * sequence b, KV head kvh.  Two-pass softmax in fp64. */
static int or_attend(const or_cache* c, const double* qd, int b, int kvh, int k_lo, int k_hi,
                     double scale, double* s, double* out, double* lse) {
    int D = c->head_dim, bad = 0;
    int nkeys = k_hi - k_lo;
    if (nkeys <= 0) {
        for (int d = 0; d < D; ++d) out[d] = 0.0;
        *lse = -INFINITY;
        return OR_OK;
    }
    for (int i = 0; i < nkeys; ++i) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += qd[d] * or_kv(c, 0, b, k_lo + i, kvh, d, &bad);
        s[i] = scale * dot;
    }
    double m = s[0];
    for (int i = 1; i < nkeys; ++i) if (s[i] > m) m = s[i];
    double L = 0.0;
    for (int i = 0; i < nkeys; ++i) { s[i] = exp(s[i] - m); L += s[i]; }
    for (int d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int i = 0; i < nkeys; ++i) acc += s[i] * or_kv(c, 1, b, k_lo + i, kvh, d, &bad);
        out[d] = acc / L;
    }
    *lse = m + log(L);
    return bad ? OR_ERANGE : OR_OK;
}

static int or_check_common(int num_seqs, int Hq, int Hkv, int D, int ps, int mp, int64_t P,
                           int kv_dtype, const uint16_t* ks, const uint16_t* vs) {
    if (num_seqs < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || ps <= 0 || mp < 0 || P < 0) return OR_EBADARG;
    if (Hq % Hkv) return OR_EBADARG;
    if (kv_dtype < OR_F32 || kv_dtype > OR_F64) return OR_EBADARG;
    if (kv_dtype == OR_I8 && (!ks || !vs)) return OR_EBADARG;
    return OR_OK;
}

/*
 * Decode: one query row per sequence, q [num_seqs][Hq][D], attending all
 * context_lens[b] keys.  context_lens[b] == 0 gives a zero row (reading of a
 * case the pages leave open).  If sel_items is NULL every (b, h) is computed
 * into out[(b*Hq + h)*D ...]; otherwise item i = sel_items[i] = b*Hq + h goes
 * to out[i*D ...].  lse (natural log of the softmax denominator plus the max)
 * may be NULL.
 */
int oracle_decode(const void* q, int q_dtype, const void* k_pages, const void* v_pages,
                  int kv_dtype, const uint16_t* k_scales, const uint16_t* v_scales,
                  const int32_t* block_tables, const int32_t* context_lens, double scale, int window,
                  int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int page_size,
                  int max_pages_per_seq, int64_t num_pages,
                  const int64_t* sel_items, int64_t n_sel, double* out, double* lse) {
    int rc = or_check_common(num_seqs, num_q_heads, num_kv_heads, head_dim, page_size,
                             max_pages_per_seq, num_pages, kv_dtype, k_scales, v_scales);
    if (rc) return rc;
    int maxctx = 0;
    for (int b = 0; b < num_seqs; ++b) {
        int ctx = context_lens[b];
        if (ctx < 0 || ctx > max_pages_per_seq * page_size) return OR_EBADARG;
        if (ctx > maxctx) maxctx = ctx;
    }
    or_cache c = {k_pages, v_pages, kv_dtype, k_scales, v_scales, block_tables,
                  max_pages_per_seq, num_kv_heads, head_dim, page_size, num_pages};
    int64_t n_items = sel_items ? n_sel : (int64_t)num_seqs * num_q_heads;
    int G = num_q_heads / num_kv_heads;
    int err = OR_OK;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(maxctx > 0 ? maxctx : 1));
        double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);
        if (!s || !qd) {
#pragma omp critical
            err = OR_ENOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t it = 0; it < n_items; ++it) {
            if (!s || !qd) continue;
            int64_t item = sel_items ? sel_items[it] : it;
            if (item < 0 || item >= (int64_t)num_seqs * num_q_heads) {
#pragma omp critical
                err = OR_EBADARG;
                continue;
            }
            int b = (int)(item / num_q_heads), h = (int)(item % num_q_heads);
            for (int d = 0; d < head_dim; ++d)
                qd[d] = or_elem(q, q_dtype, item * head_dim + d);
            double l;
            int ctx = context_lens[b];
            int k_lo = (window > 0 && ctx - window > 0) ? ctx - window : 0;
            int r = or_attend(&c, qd, b, h / G, k_lo, ctx, scale, s, out + it * head_dim, &l);
            if (lse) lse[it] = l;
            if (r) {
#pragma omp critical
                err = r;
            }
        }
        free(s);
        free(qd);
    }
    return err;
}

/*
 * Prefill: packed query rows q [total_q][Hq][D]; rows q_start[b] ..
 * q_start[b+1]-1 belong to sequence b and sit at absolute positions
 * ctx-n .. ctx-1 (n = chunk length, ctx = context_lens[b], n <= ctx
 * required).  causal != 0: row r attends keys 0 .. ctx-n+r; otherwise all
 * ctx keys.  Items are t*Hq + h over packed rows t; selection as in decode.
 */
int oracle_prefill(const void* q, int q_dtype, const void* k_pages, const void* v_pages,
                   int kv_dtype, const uint16_t* k_scales, const uint16_t* v_scales,
                   const int32_t* block_tables, const int32_t* q_start,
                   const int32_t* context_lens, int causal, double scale, int window,
                   int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int page_size,
                   int max_pages_per_seq, int64_t num_pages,
                   const int64_t* sel_items, int64_t n_sel, double* out, double* lse) {
    int rc = or_check_common(num_seqs, num_q_heads, num_kv_heads, head_dim, page_size,
                             max_pages_per_seq, num_pages, kv_dtype, k_scales, v_scales);
    if (rc) return rc;
    if (q_start[0] != 0) return OR_EBADARG;
    int maxctx = 0;
    for (int b = 0; b < num_seqs; ++b) {
        int n = q_start[b + 1] - q_start[b], ctx = context_lens[b];
        if (n < 0 || ctx < 0 || n > ctx || ctx > max_pages_per_seq * page_size) return OR_EBADARG;
        if (ctx > maxctx) maxctx = ctx;
    }
    int64_t total_q = q_start[num_seqs];
    or_cache c = {k_pages, v_pages, kv_dtype, k_scales, v_scales, block_tables,
                  max_pages_per_seq, num_kv_heads, head_dim, page_size, num_pages};
    int64_t n_items = sel_items ? n_sel : total_q * num_q_heads;
    int G = num_q_heads / num_kv_heads;
    int err = OR_OK;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(maxctx > 0 ? maxctx : 1));
        double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);
        if (!s || !qd) {
#pragma omp critical
            err = OR_ENOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t it = 0; it < n_items; ++it) {
            if (!s || !qd) continue;
            int64_t item = sel_items ? sel_items[it] : it;
            if (item < 0 || item >= total_q * num_q_heads) {
#pragma omp critical
                err = OR_EBADARG;
                continue;
            }
            int64_t t = item / num_q_heads;
            int h = (int)(item % num_q_heads);
            int lo = 0, hi = num_seqs - 1;              /* sequence owning row t */
            while (lo < hi) {
                int mid = (lo + hi + 1) / 2;
                if (q_start[mid] <= t) lo = mid; else hi = mid - 1;
            }
            int b = lo;
            int n = q_start[b + 1] - q_start[b], ctx = context_lens[b];
            int r = (int)(t - q_start[b]);
            int pos = ctx - n + r;
            int k_hi = causal ? pos + 1 : ctx;
            int k_lo = (window > 0 && pos - window + 1 > 0) ? pos - window + 1 : 0;
            for (int d = 0; d < head_dim; ++d)
                qd[d] = or_elem(q, q_dtype, item * head_dim + d);
            double l;
            int rr = or_attend(&c, qd, b, h / G, k_lo, k_hi, scale, s, out + it * head_dim, &l);
            if (lse) lse[it] = l;
            if (rr) {
#pragma omp critical
                err = rr;
            }
        }
        free(s);
        free(qd);
    }
    return err;
}
