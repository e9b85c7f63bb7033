/*
 * CPU oracle for paged KV-cache attention — TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load this library.  The product path (the CUDA library and its Python
 * binding) never calls it and shares no code, header or constant table with it.
 *
 * What it computes, and where the pages define it:
 *   - The cache write: every new token's K/V row is stored at the physical
 *     slot the scheduler chose for it (slot = physical block * block_size +
 *     offset).  "PagedAttention 与 Continuous Batching", §3.3 (数据结构: the
 *     token-18 -> block 42, offset 2 example and the three decode steps) and
 *     §2.5 (step 4 builds block_tables and slot_mapping).
 *   - Attention over the paged cache: for each query row, walk the request's
 *     block table, fetch every cached key/value, and take exact softmax
 *     attention.  §3.6 (PagedAttention Kernel) says paging only changes where
 *     K/V live; §10.8 (FAQ) says a prefix-cache hit equals recomputation up to
 *     rounding.  So this oracle is the plain definition: gather, then a
 *     two-pass softmax in fp64, with no online rescaling and no partitions.
 *   - Packed mixed prefill/decode rows delimited by cu_seqlens:
 *     "推理优化与服务：从 PagedAttention 到分离式部署", section 最新进展 (the V1
 *     unified step packs query tokens as [total_q, H, D] with cu_seqlens).
 *     Causality is aligned bottom-right: row i of a request with q_len rows and
 *     kv_len keys (cached + new) sees keys 0 .. kv_len - q_len + i.
 *   - FP8 KV ("kv_cache_dtype=fp8", §8.8 of the tutorial page): OCP FP8 E4M3
 *     (bias 7, largest finite 448, S.1111.111 is NaN, no infinities), written
 *     here from that format definition.  One fp32 scale per KV head for K and
 *     one for V; quantise = round-to-nearest-even with saturation of
 *     float(x) / scale, dequantise = e4m3 * scale.
 *
 * Readings taken where the pages are silent: KV pool layout
 * [num_blocks][num_kv_heads][block_size][head_dim] (one contiguous tile per
 * block and head, "per layer, per head" in §3.2); GQA maps query head hq to
 * KV head hq / (Hq / Hkv); a row with no visible key yields zeros.
 *
 * Pins: every function here is checked by the CPU tests against closed forms,
 * exhaustive codec tables, brute force on tiny inputs, an independent NumPy
 * fp64 twin and float64 scaled-dot-product attention in PyTorch.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Element formats understood by the oracle. */
enum { OR_F16 = 0, OR_BF16 = 1, OR_FP8_E4M3 = 2, OR_F32 = 3 };

/* Error codes returned by the oracle. */
enum { OR_OK = 0, OR_BAD_ARG = -1, OR_BAD_BLOCK = -2, OR_NO_MEMORY = -3 };

/* ------------------------------------------------------------------------ */
/* Element codecs, each written from its format definition.                  */
/* ------------------------------------------------------------------------ */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double or_f16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0x1F)
        v = f ? NAN : INFINITY;
    else if (e == 0)
        v = ldexp((double)f, -24);            /* subnormal: f * 2^-14 / 2^10 */
    else
        v = ldexp(1024.0 + f, e - 25);        /* (1 + f/2^10) * 2^(e-15)     */
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
double or_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float x;
    memcpy(&x, &u, sizeof x);
    return (double)x;
}

double or_f32_to_double(float x) { return (double)x; }

/* OCP FP8 E4M3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits.
 * Exponent field 0 encodes subnormals m * 2^-9; S.1111.111 is NaN;
 * there is no infinity, so 0x7E (448) is the largest finite value. */
double or_e4m3_to_double(uint8_t x)
{
    int sign = (x >> 7) & 1;
    int e = (x >> 3) & 0xF;
    int m = x & 7;
    double v;
    if (e == 0xF && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(8.0 + m, e - 10);           /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* Round a non-negative double that is an exact multiple of 1/2 or finer
 * to the nearest integer, ties to even. */
static double round_half_even(double q)
{
    double n = floor(q);
    double frac = q - n;
    if (frac > 0.5)
        return n + 1.0;
    if (frac < 0.5)
        return n;
    return fmod(n, 2.0) == 0.0 ? n : n + 1.0;
}

/* float -> E4M3, round to nearest even, saturating to +-448 (inf included);
 * NaN maps to the canonical 0x7F. */
uint8_t or_e4m3_from_float(float xf)
{
    double x = (double)xf;
    uint8_t sign = signbit(xf) ? 0x80 : 0x00;
    double a = fabs(x);
    if (isnan(xf))
        return 0x7F;
    if (a >= 448.0)
        return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: spacing 2^-9; code n = multiple of 2^-9
         * (n = 8 is the smallest normal, whose code is also 8). */
        double n = round_half_even(ldexp(a, 9));
        return sign | (uint8_t)n;
    }
    int E;
    (void)frexp(a, &E);                        /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1;                             /* a in [2^e, 2^(e+1))        */
    double n = round_half_even(ldexp(a, 3 - e)); /* in [8, 16]               */
    int code = ((e + 7) << 3) + ((int)n - 8);  /* n == 16 carries into e     */
    return sign | (uint8_t)code;
}

/* ------------------------------------------------------------------------ */
/* Element access.                                                          */
/* ------------------------------------------------------------------------ */

static size_t elem_bytes(int dtype)
{
    switch (dtype) {
    case OR_F16: case OR_BF16: return 2;
    case OR_FP8_E4M3: return 1;
    case OR_F32: return 4;
    default: return 0;
    }
}

static double load_as_double(const void *base, int64_t idx, int dtype)
{
    switch (dtype) {
    case OR_F16: return or_f16_to_double(((const uint16_t *)base)[idx]);
    case OR_BF16: return or_bf16_to_double(((const uint16_t *)base)[idx]);
    case OR_FP8_E4M3: return or_e4m3_to_double(((const uint8_t *)base)[idx]);
    case OR_F32: return or_f32_to_double(((const float *)base)[idx]);
    default: return NAN;
    }
}

/* ------------------------------------------------------------------------ */
/* Cache write (reshape_and_cache).                                          */
/* ------------------------------------------------------------------------ */

/*
 * key, value : [num_tokens] rows, token i starting at element i*token_stride,
 *              each row [num_kv_heads][head_dim] contiguous, in src_dtype.
 * slot_mapping: [num_tokens]; slot < 0 skips the token (padding).
 * k_cache, v_cache: [num_blocks][num_kv_heads][block_size][head_dim] in kv_dtype.
 * kv_dtype equals src_dtype (bit copy) or is OR_FP8_E4M3 (quantise with
 * k_scale[h] / v_scale[h]).
 */
int oracle_reshape_and_cache(const void *key, const void *value, int src_dtype,
                             int64_t num_tokens, int64_t token_stride,
                             const int64_t *slot_mapping, void *k_cache, void *v_cache,
                             int32_t num_blocks, int32_t block_size,
                             int32_t num_kv_heads, int32_t head_dim, int kv_dtype,
                             const float *k_scale, const float *v_scale)
{
    if (!key || !value || !slot_mapping || !k_cache || !v_cache)
        return OR_BAD_ARG;
    if (num_tokens < 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
        return OR_BAD_ARG;
    int fp8 = (kv_dtype == OR_FP8_E4M3);
    if (!fp8 && kv_dtype != src_dtype)
        return OR_BAD_ARG;
    if (fp8 && (!k_scale || !v_scale))
        return OR_BAD_ARG;
    size_t sb = elem_bytes(src_dtype), kb = elem_bytes(kv_dtype);
    if (!sb || !kb || src_dtype == OR_FP8_E4M3)
        return OR_BAD_ARG;

    for (int64_t i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        int64_t blk = slot / block_size;
        int64_t off = slot % block_size;
        if (blk >= num_blocks)
            return OR_BAD_BLOCK;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            for (int32_t d = 0; d < head_dim; ++d) {
                int64_t src = i * token_stride + (int64_t)h * head_dim + d;
                int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim + d;
                if (!fp8) {
                    memcpy((char *)k_cache + dst * kb, (const char *)key + src * sb, sb);
                    memcpy((char *)v_cache + dst * kb, (const char *)value + src * sb, sb);
                } else {
                    /* One IEEE division, rounded once to fp32: the fp64
                     * quotient of two floats rounds to the correctly rounded
                     * fp32 quotient (53 >= 2*24 + 2). */
                    float kq = (float)(load_as_double(key, src, src_dtype) / (double)k_scale[h]);
                    float vq = (float)(load_as_double(value, src, src_dtype) / (double)v_scale[h]);
                    ((uint8_t *)k_cache)[dst] = or_e4m3_from_float(kq);
                    ((uint8_t *)v_cache)[dst] = or_e4m3_from_float(vq);
                }
            }
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Attention over the paged cache.                                           */
/* ------------------------------------------------------------------------ */

typedef struct {
    const void *q; int q_dtype;
    int32_t total_q, num_seqs, num_q_heads;
    const int32_t *cu_seqlens_q, *seqlens_k;
    const void *k_cache, *v_cache;
    int32_t num_blocks, block_size, num_kv_heads, head_dim;
    int kv_dtype;
    const float *k_scale, *v_scale;
    const int32_t *block_tables; int32_t max_blocks_per_seq;
    double scale;
    const int64_t *pair_rows; const int32_t *pair_heads; int64_t num_pairs;
    int32_t window;                  /* > 0: keys pos-window+1 .. pos only */
    const float *alibi_slopes;       /* [num_q_heads] or NULL */
    double *out; double *lse;
    int error;               /* first error seen by any worker */
    pthread_mutex_t lock;
} attn_job;

/* The request that owns packed query row `row` (linear scan of cu_seqlens). */
static int32_t request_of_row(const attn_job *J, int64_t row)
{
    for (int32_t r = 0; r < J->num_seqs; ++r)
        if (row >= J->cu_seqlens_q[r] && row < J->cu_seqlens_q[r + 1])
            return r;
    return -1;
}

/* Dequantised cached element (token t of request r, KV head h, dim d). */
static int cached(const attn_job *J, const void *cache, const float *sc, int32_t r,
                  int32_t h, int64_t t, int32_t d, double *v)
{
    int32_t blk = J->block_tables[(int64_t)r * J->max_blocks_per_seq + t / J->block_size];
    int64_t off = t % J->block_size;
    if (blk < 0 || blk >= J->num_blocks)
        return OR_BAD_BLOCK;
    int64_t idx = (((int64_t)blk * J->num_kv_heads + h) * J->block_size + off) * J->head_dim + d;
    *v = load_as_double(cache, idx, J->kv_dtype);
    if (J->kv_dtype == OR_FP8_E4M3)
        *v *= (double)sc[h];
    return OR_OK;
}

/* One (query row, query head) pair: out[0..D) and optionally its log-sum-exp. */
static int attend_one(const attn_job *J, int64_t row, int32_t hq, double *out, double *lse)
{
    int32_t D = J->head_dim;
    int32_t r = request_of_row(J, row);
    if (r < 0 || hq < 0 || hq >= J->num_q_heads)
        return OR_BAD_ARG;
    int64_t q_len = J->cu_seqlens_q[r + 1] - J->cu_seqlens_q[r];
    int64_t kv_len = J->seqlens_k[r];
    int64_t i = row - J->cu_seqlens_q[r];
    int64_t last = kv_len - q_len + i;          /* last visible key, inclusive */
    int64_t n = last + 1 < kv_len ? last + 1 : kv_len;
    if (n < 0)
        n = 0;
    /* sliding window: only the `window` most recent keys up to the query's
     * own position are visible */
    int64_t first = 0;
    if (J->window > 0 && last - J->window + 1 > 0)
        first = last - J->window + 1;
    if (first > n)
        first = n;
    int32_t h = hq / (J->num_q_heads / J->num_kv_heads);
    double slope = J->alibi_slopes ? (double)J->alibi_slopes[hq] : 0.0;

    for (int32_t d = 0; d < D; ++d)
        out[d] = 0.0;
    if (lse)
        *lse = -INFINITY;
    if (n == 0 || first >= n)
        return OR_OK;

    double *qv = (double *)malloc(sizeof(double) * D);
    double *s = (double *)malloc(sizeof(double) * n);
    if (!qv || !s) {
        free(qv); free(s);
        return OR_NO_MEMORY;
    }
    for (int32_t d = 0; d < D; ++d)
        qv[d] = load_as_double(J->q, (row * J->num_q_heads + hq) * (int64_t)D + d, J->q_dtype);

    int rc = OR_OK;
    /* pass 1: scores s_t = scale * <q, k_t> (+ ALiBi bias slope * (t - pos)) */
    for (int64_t t = first; t < n && rc == OR_OK; ++t) {
        double dot = 0.0;
        for (int32_t d = 0; d < D; ++d) {
            double k;
            rc = cached(J, J->k_cache, J->k_scale, r, h, t, d, &k);
            if (rc != OR_OK)
                break;
            dot += qv[d] * k;
        }
        s[t] = J->scale * dot + slope * (double)(t - last);
    }
    if (rc == OR_OK) {
        double m = s[first];
        for (int64_t t = first + 1; t < n; ++t)
            if (s[t] > m)
                m = s[t];
        double denom = 0.0;
        for (int64_t t = first; t < n; ++t) {
            s[t] = exp(s[t] - m);              /* s now holds the weights */
            denom += s[t];
        }
        /* pass 2: out = sum_t w_t v_t / sum_t w_t */
        for (int64_t t = first; t < n && rc == OR_OK; ++t) {
            for (int32_t d = 0; d < D; ++d) {
                double v;
                rc = cached(J, J->v_cache, J->v_scale, r, h, t, d, &v);
                if (rc != OR_OK)
                    break;
                out[d] += s[t] * v;
            }
        }
        for (int32_t d = 0; d < D; ++d)
            out[d] /= denom;
        if (lse)
            *lse = m + log(denom);
    }
    free(qv);
    free(s);
    return rc;
}

typedef struct { attn_job *J; int64_t begin, end; } attn_slice;

static void *attn_worker(void *arg)
{
    attn_slice *S = (attn_slice *)arg;
    attn_job *J = S->J;
    int32_t D = J->head_dim;
    for (int64_t p = S->begin; p < S->end; ++p) {
        int64_t row; int32_t hq; int64_t o;
        if (J->pair_rows) {
            row = J->pair_rows[p];
            hq = J->pair_heads[p];
            o = p;
        } else {
            row = p / J->num_q_heads;
            hq = (int32_t)(p % J->num_q_heads);
            o = p;
        }
        int rc = attend_one(J, row, hq, J->out + o * D, J->lse ? J->lse + o : NULL);
        if (rc != OR_OK) {
            pthread_mutex_lock(&J->lock);
            if (J->error == OR_OK)
                J->error = rc;
            pthread_mutex_unlock(&J->lock);
            return NULL;
        }
    }
    return NULL;
}

/*
 * Attention over the paged cache for packed query rows.
 *
 * q         : [total_q][num_q_heads][head_dim] in q_dtype.
 * cu_seqlens_q: [num_seqs + 1], rows of request r are cu[r] .. cu[r+1]-1.
 * seqlens_k : [num_seqs], keys of request r (cached + this step's new ones).
 * block_tables: [num_seqs][max_blocks_per_seq]; entries past ceil(kv_len/bs)
 *             are never read.
 * scale     : the logit scale (the caller's fp32 value, widened).
 * pair_rows/pair_heads: NULL for every (row, head) pair, writing
 *             out[total_q][num_q_heads][head_dim]; otherwise num_pairs chosen
 *             pairs, writing out[num_pairs][head_dim].
 * lse       : optional log-sum-exp of the scaled logits per pair (-inf when
 *             a row sees no key).
 * num_threads: worker threads over independent pairs (<= 1: the caller's).
 * Decode is the special case cu_seqlens_q = 0,1,..,B and seqlens_k = context_lens.
 */
int oracle_paged_attention_ex(double *out, double *lse, const void *q, int q_dtype,
                              int32_t total_q, int32_t num_seqs, int32_t num_q_heads,
                              const int32_t *cu_seqlens_q, const int32_t *seqlens_k,
                              const void *k_cache, const void *v_cache, int32_t num_blocks,
                              int32_t block_size, int32_t num_kv_heads, int32_t head_dim,
                              int kv_dtype, const float *k_scale, const float *v_scale,
                              const int32_t *block_tables, int32_t max_blocks_per_seq,
                              double scale, const int64_t *pair_rows, const int32_t *pair_heads,
                              int64_t num_pairs, int num_threads, int32_t window,
                              const float *alibi_slopes)
{
    if (!out || !q || !cu_seqlens_q || !seqlens_k || !k_cache || !v_cache || !block_tables)
        return OR_BAD_ARG;
    if (num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads || head_dim <= 0 ||
        block_size <= 0 || num_seqs < 0 || total_q < 0)
        return OR_BAD_ARG;
    if (kv_dtype == OR_FP8_E4M3 && (!k_scale || !v_scale))
        return OR_BAD_ARG;
    if (!elem_bytes(q_dtype) || q_dtype == OR_FP8_E4M3 || !elem_bytes(kv_dtype))
        return OR_BAD_ARG;
    if (pair_rows && !pair_heads)
        return OR_BAD_ARG;

    attn_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.q_dtype = q_dtype; J.total_q = total_q; J.num_seqs = num_seqs;
    J.num_q_heads = num_q_heads; J.cu_seqlens_q = cu_seqlens_q; J.seqlens_k = seqlens_k;
    J.k_cache = k_cache; J.v_cache = v_cache; J.num_blocks = num_blocks;
    J.block_size = block_size; J.num_kv_heads = num_kv_heads; J.head_dim = head_dim;
    J.kv_dtype = kv_dtype; J.k_scale = k_scale; J.v_scale = v_scale;
    J.block_tables = block_tables; J.max_blocks_per_seq = max_blocks_per_seq; J.scale = scale;
    J.pair_rows = pair_rows; J.pair_heads = pair_heads; J.num_pairs = num_pairs;
    J.window = window; J.alibi_slopes = alibi_slopes;
    J.out = out; J.lse = lse; J.error = OR_OK;
    pthread_mutex_init(&J.lock, NULL);
    int64_t total = pair_rows ? num_pairs : (int64_t)total_q * num_q_heads;
    int nt = num_threads < 1 ? 1 : num_threads;
    if (nt > total)
        nt = total > 0 ? (int)total : 1;

    attn_slice *slices = (attn_slice *)calloc((size_t)nt, sizeof(attn_slice));
    pthread_t *tids = (pthread_t *)calloc((size_t)nt, sizeof(pthread_t));
    if (!slices || !tids) {
        free(slices); free(tids);
        pthread_mutex_destroy(&J.lock);
        return OR_NO_MEMORY;
    }
    for (int w = 0; w < nt; ++w) {
        slices[w].J = &J;
        slices[w].begin = total * w / nt;
        slices[w].end = total * (w + 1) / nt;
    }
    if (nt == 1) {
        attn_worker(&slices[0]);
    } else {
        /* a slice whose thread could not be started runs here instead;
           started[w] says which threads there are to join */
        unsigned char *started = (unsigned char *)calloc((size_t)nt, 1);
        for (int w = 0; w < nt; ++w) {
            if (started && pthread_create(&tids[w], NULL, attn_worker, &slices[w]) == 0)
                started[w] = 1;
            else
                attn_worker(&slices[w]);
        }
        for (int w = 0; w < nt; ++w)
            if (started && started[w])
                pthread_join(tids[w], NULL);
        free(started);
    }
    free(slices);
    free(tids);
    pthread_mutex_destroy(&J.lock);
    return J.error;
}

/* Plain attention (no window, no ALiBi): the definition the pages give. */
int oracle_paged_attention(double *out, double *lse, const void *q, int q_dtype,
                           int32_t total_q, int32_t num_seqs, int32_t num_q_heads,
                           const int32_t *cu_seqlens_q, const int32_t *seqlens_k,
                           const void *k_cache, const void *v_cache, int32_t num_blocks,
                           int32_t block_size, int32_t num_kv_heads, int32_t head_dim,
                           int kv_dtype, const float *k_scale, const float *v_scale,
                           const int32_t *block_tables, int32_t max_blocks_per_seq,
                           double scale, const int64_t *pair_rows, const int32_t *pair_heads,
                           int64_t num_pairs, int num_threads)
{
    return oracle_paged_attention_ex(out, lse, q, q_dtype, total_q, num_seqs, num_q_heads,
                                     cu_seqlens_q, seqlens_k, k_cache, v_cache, num_blocks,
                                     block_size, num_kv_heads, head_dim, kv_dtype, k_scale,
                                     v_scale, block_tables, max_blocks_per_seq, scale,
                                     pair_rows, pair_heads, num_pairs, num_threads, 0, NULL);
}

/* ------------------------------------------------------------------------ */
/* Whole-block copies (copy-on-write, swap).                                 */
/* ------------------------------------------------------------------------ */

/*
 * For each pair (src, dst): block dst of dst_k/dst_v takes the bytes of
 * block src of src_k/src_v.  A block is block_bytes contiguous bytes
 * ([num_kv_heads][block_size][head_dim] elements).  Copy-on-write passes the
 * same pool as source and destination ("PagedAttention 与 Continuous
 * Batching", §3.8); swapping passes a device-side and a host-side pool (§3.9).
 */
int oracle_copy_blocks(void *dst_k, void *dst_v, const void *src_k, const void *src_v,
                       int64_t src_num_blocks, int64_t dst_num_blocks, int64_t block_bytes,
                       const int64_t *pairs, int64_t num_pairs)
{
    if (!dst_k || !dst_v || !src_k || !src_v || (!pairs && num_pairs) || block_bytes <= 0)
        return OR_BAD_ARG;
    for (int64_t i = 0; i < num_pairs; ++i) {
        int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
        if (s < 0 || s >= src_num_blocks || d < 0 || d >= dst_num_blocks)
            return OR_BAD_BLOCK;
        memmove((char *)dst_k + d * block_bytes, (const char *)src_k + s * block_bytes,
                (size_t)block_bytes);
        memmove((char *)dst_v + d * block_bytes, (const char *)src_v + s * block_bytes,
                (size_t)block_bytes);
    }
    return OR_OK;
}
