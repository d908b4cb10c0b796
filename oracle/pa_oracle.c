/*
 * pa_oracle.c -- fp64 CPU oracle for paged-KV decode attention and the
 * slot-mapped cache append.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  The
 * product path (paged_kv_attention_36_b200/) never imports, links or calls
 * it, and it shares no code, header or constant with that path.
 *
 * What it computes (the plainest reading of the pages, which name the
 * method but never print its formula):
 *   - "paged attention for decode" over a "KV cache ... managed in
 *     fixed-size pages" (miniVLLM docs index, "What is miniVLLM?" and
 *     "Explore by topic"; tiny-vllm write-up, "Chi tiet"): for sequence b
 *     and query head h, with kv head g = h / (Hq/Hkv),
 *         K_t = k_cache[block_tables[b][t / bs]][g][t % bs][:]   (same for V)
 *         s_t = scale * sum_d q[b][h][d] * K_t[d]        t = 0 .. L_b-1
 *         out[b][h][:] = sum_t softmax(s)_t * V_t[:]
 *     computed in double precision on the bf16 inputs widened exactly,
 *     with the stable softmax (subtract the max, exponentiate, sum), in
 *     order of logical token index t.
 *   - the split-KV partial of one token range [t0, t1): the normalised
 *     partial output o, its max logit m (natural-log units) and
 *     l = sum_t exp(s_t - m), and the log-sum-exp merge of such partials
 *     (flash-decoding; the online-softmax rescaling named on the miniVLLM
 *     docs index, "Explore by topic").
 *   - the append: k_cache[slot / bs][g][slot % bs][:] = k_new[t][g][:]
 *     (same for V) for every token t whose slot is >= 0 (a KV-caching
 *     engine writing each decode step's new token, miniVLLM review,
 *     "What main.py actually does").
 *
 * Cache layout read here (written out independently of the GPU code from
 * the documented layout): k_cache and v_cache are [NB][Hkv][bs][D] bf16,
 * row-major; block_tables is [B][M] int32; q and out are [B][Hq][D].
 *
 * fp8 KV cache (the pages' quantization theme applied to the KV cache:
 * MiniVLLM write-up, "量化层" and "量化支持"): each cached value is one
 * OCP FP8 E4M3 code c (the "fn" variant: 4 exponent bits with bias 7, 3
 * mantissa bits, no infinities, 0x7F/0xFF NaN, largest finite 448) with a
 * per-kv-head scale, value = e4m3(c) * scale[g].  The append encodes
 * x / scale[g] (one IEEE binary32 division of the widened bf16 value) by
 * rounding to the nearest representable value, ties to even, and
 * saturating magnitudes beyond 448 to 448.  Layouts (uint8):
 *   k_cache8 [NB][Hkv][16][D]   token-major, like the bf16 cache;
 *   v_cache8 [NB][Hkv][D][16]   each (block, head) tile transposed: row d
 *                               holds the 16 tokens' values of column d at
 *                               position pos(t) = 4*((t % 8) / 2) + 2*(t / 8) + t % 2.
 * The fp8 decode is the formula above with K_t, V_t the dequantized values.
 *
 * Multi-query (chunked prefill) attention over the paged cache, the step
 * beside decode in the pages' engines (miniVLLM docs index, "What is
 * miniVLLM?": flash attention for prefill; Mini-SGLang write-up, "Key
 * optimizations": chunked prefill): sequence b brings q_len_b query tokens
 * (rows cu_q_lens[b] .. cu_q_lens[b+1]-1 of q[total][Hq][D]), which are the
 * last q_len_b of its L_b cached tokens; query token i (position
 * p = L_b - q_len_b + i) attends causally to tokens t = 0 .. p.
 *
 * Parity pins: tests/test_oracle_pins.py checks every function here
 * against torch's scaled_dot_product_attention on contiguous K/V, block
 * permutation and block-size invariance, the closed forms for
 * context_len == 1, equal keys, scale == 0 and a two-token worked example,
 * a dominant key, the split/merge identity, and an append round trip.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define PAO_OK 0
#define PAO_ERR_ARG (-1)
#define PAO_ERR_BLOCK (-2)   /* a block id inside [0, L) is outside [0, NB) */
#define PAO_ERR_LEN (-3)     /* context_len outside [0, M*bs] */
#define PAO_ERR_SLOT (-4)    /* an append slot beyond the pool */
#define PAO_ERR_NOMEM (-5)

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    const uint16_t *q, *k_cache, *v_cache;
    const int32_t *block_tables, *context_lens;
    int64_t B, Hq, Hkv, D, bs, NB, M;
    double scale;
} problem_t;

/* Address of row (token t of sequence b, kv head g) inside a cache, or
 * NULL when its block id is out of range. */
static const uint16_t *cache_row(const problem_t *p, const uint16_t *cache,
                                 int64_t b, int64_t g, int64_t t)
{
    int64_t logical_block = t / p->bs;
    int64_t offset = t % p->bs;
    int64_t block = p->block_tables[b * p->M + logical_block];
    if (block < 0 || block >= p->NB) return NULL;
    return cache + ((block * p->Hkv + g) * p->bs + offset) * p->D;
}

/* Attention of the query row q (D bf16 values) against kv head g of
 * sequence b over tokens [t0, t1).  Writes the normalised output o[D];
 * *m_out = max logit, *l_out = sum of exp(s - m).  An empty range gives
 * o = 0, m = -inf, l = 0. */
static int attend_tokens(const problem_t *p, int64_t b, int64_t g, const uint16_t *q,
                         int64_t t0, int64_t t1, double *s_buf,
                         double *o, double *m_out, double *l_out)
{
    for (int64_t d = 0; d < p->D; ++d) o[d] = 0.0;
    if (t1 <= t0) {
        *m_out = -INFINITY;
        *l_out = 0.0;
        return PAO_OK;
    }
    /* logits */
    double m = -INFINITY;
    for (int64_t t = t0; t < t1; ++t) {
        const uint16_t *k = cache_row(p, p->k_cache, b, g, t);
        if (!k) return PAO_ERR_BLOCK;
        double dot = 0.0;
        for (int64_t d = 0; d < p->D; ++d)
            dot += bf16_bits_to_double(q[d]) * bf16_bits_to_double(k[d]);
        double s = p->scale * dot;
        s_buf[t - t0] = s;
        if (s > m) m = s;
    }
    /* weights, their sum, and the weighted sum of values */
    double l = 0.0;
    for (int64_t t = t0; t < t1; ++t) {
        double w = exp(s_buf[t - t0] - m);
        l += w;
        const uint16_t *v = cache_row(p, p->v_cache, b, g, t);
        for (int64_t d = 0; d < p->D; ++d) o[d] += w * bf16_bits_to_double(v[d]);
    }
    for (int64_t d = 0; d < p->D; ++d) o[d] /= l;
    *m_out = m;
    *l_out = l;
    return PAO_OK;
}

/* Query head h of sequence b (its row of q[B][Hq][D]) over tokens [t0, t1). */
static int attend_range(const problem_t *p, int64_t b, int64_t h,
                        int64_t t0, int64_t t1, double *s_buf,
                        double *o, double *m_out, double *l_out)
{
    const int64_t G = p->Hq / p->Hkv;
    return attend_tokens(p, b, h / G, p->q + (b * p->Hq + h) * p->D, t0, t1, s_buf, o, m_out, l_out);
}

/* ---------------------------------------------------------------------
 * Full decode, threaded over (b, h) rows.
 * ------------------------------------------------------------------- */
typedef struct {
    const problem_t *p;
    double *out;
    int64_t first, stride;
    int status;
} decode_job_t;

static void *decode_worker(void *arg)
{
    decode_job_t *job = (decode_job_t *)arg;
    const problem_t *p = job->p;
    int64_t max_len = p->M * p->bs;
    double *s_buf = (double *)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
    if (!s_buf) { job->status = PAO_ERR_NOMEM; return NULL; }
    job->status = PAO_OK;
    for (int64_t row = job->first; row < p->B * p->Hq; row += job->stride) {
        int64_t b = row / p->Hq, h = row % p->Hq;
        double m, l;
        int rc = attend_range(p, b, h, 0, p->context_lens[b], s_buf,
                              job->out + row * p->D, &m, &l);
        if (rc != PAO_OK) { job->status = rc; break; }
    }
    free(s_buf);
    return NULL;
}

static int check_problem(const problem_t *p)
{
    if (!p->q || !p->k_cache || !p->v_cache || !p->block_tables || !p->context_lens)
        return PAO_ERR_ARG;
    if (p->B < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->D <= 0 || p->bs <= 0 ||
        p->NB < 0 || p->M < 0 || p->Hq % p->Hkv != 0)
        return PAO_ERR_ARG;
    for (int64_t b = 0; b < p->B; ++b)
        if (p->context_lens[b] < 0 || p->context_lens[b] > p->M * p->bs) return PAO_ERR_LEN;
    return PAO_OK;
}

int pa_oracle_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                     const int32_t *block_tables, const int32_t *context_lens,
                     int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t bs,
                     int64_t NB, int64_t M, double scale, double *out, int nthreads)
{
    problem_t p = {q, k_cache, v_cache, block_tables, context_lens,
                   B, Hq, Hkv, D, bs, NB, M, scale};
    int rc = check_problem(&p);
    if (rc != PAO_OK) return rc;
    if (!out) return PAO_ERR_ARG;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t tid[256];
    decode_job_t jobs[256];
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = (decode_job_t){&p, out, i, nthreads, PAO_OK};
        if (nthreads == 1) decode_worker(&jobs[i]);
        else pthread_create(&tid[i], NULL, decode_worker, &jobs[i]);
    }
    if (nthreads > 1)
        for (int i = 0; i < nthreads; ++i) pthread_join(tid[i], NULL);
    for (int i = 0; i < nthreads; ++i)
        if (jobs[i].status != PAO_OK) return jobs[i].status;
    return PAO_OK;
}

/* ---------------------------------------------------------------------
 * Partials of arbitrary (b, h, [t0, t1)) ranges: o[n][D], m[n], l[n].
 * ------------------------------------------------------------------- */
int pa_oracle_partials(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                       const int32_t *block_tables, const int32_t *context_lens,
                       int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t bs,
                       int64_t NB, int64_t M, double scale,
                       const int32_t *range_b, const int32_t *range_h,
                       const int32_t *range_t0, const int32_t *range_t1, int64_t n,
                       double *o, double *m, double *l)
{
    problem_t p = {q, k_cache, v_cache, block_tables, context_lens,
                   B, Hq, Hkv, D, bs, NB, M, scale};
    int rc = check_problem(&p);
    if (rc != PAO_OK) return rc;
    double *s_buf = (double *)malloc(sizeof(double) * (size_t)(M * bs > 0 ? M * bs : 1));
    if (!s_buf) return PAO_ERR_NOMEM;
    for (int64_t i = 0; i < n && rc == PAO_OK; ++i) {
        int64_t b = range_b[i], h = range_h[i], t0 = range_t0[i], t1 = range_t1[i];
        if (b < 0 || b >= B || h < 0 || h >= Hq || t0 < 0 || t1 < t0 ||
            t1 > context_lens[b]) { rc = PAO_ERR_ARG; break; }
        rc = attend_range(&p, b, h, t0, t1, s_buf, o + i * D, m + i, l + i);
    }
    free(s_buf);
    return rc;
}

/* ---------------------------------------------------------------------
 * Log-sum-exp merge of n partials of one output row.
 *   M_ = max_i m_i;  w_i = l_i * exp(m_i - M_);  out = sum_i w_i o_i / sum_i w_i
 * Partials with l_i == 0 (empty ranges) carry no weight.
 * ------------------------------------------------------------------- */
int pa_oracle_lse_merge(const double *o, const double *m, const double *l,
                        int64_t n, int64_t D, double *out)
{
    if (n < 0 || D <= 0 || !out) return PAO_ERR_ARG;
    double mx = -INFINITY;
    for (int64_t i = 0; i < n; ++i)
        if (l[i] > 0.0 && m[i] > mx) mx = m[i];
    for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
    if (mx == -INFINITY) return PAO_OK;
    double wsum = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        if (!(l[i] > 0.0)) continue;
        double w = l[i] * exp(m[i] - mx);
        wsum += w;
        for (int64_t d = 0; d < D; ++d) out[d] += w * o[i * D + d];
    }
    for (int64_t d = 0; d < D; ++d) out[d] /= wsum;
    return PAO_OK;
}

/* ---------------------------------------------------------------------
 * Slot-mapped append (bit copy).  Negative slots are padding and skipped.
 * Slots beyond the pool are skipped and reported.
 * ------------------------------------------------------------------- */
int pa_oracle_append(const uint16_t *k_new, const uint16_t *v_new, const int32_t *slot_mapping,
                     int64_t T, uint16_t *k_cache, uint16_t *v_cache,
                     int64_t Hkv, int64_t D, int64_t bs, int64_t NB)
{
    if (T < 0 || Hkv <= 0 || D <= 0 || bs <= 0 || NB < 0) return PAO_ERR_ARG;
    if (T > 0 && (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache)) return PAO_ERR_ARG;
    int rc = PAO_OK;
    for (int64_t t = 0; t < T; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t block = slot / bs, offset = slot % bs;
        if (block >= NB) { rc = PAO_ERR_SLOT; continue; }
        for (int64_t g = 0; g < Hkv; ++g) {
            int64_t dst = ((block * Hkv + g) * bs + offset) * D;
            int64_t src = (t * Hkv + g) * D;
            for (int64_t d = 0; d < D; ++d) {
                k_cache[dst + d] = k_new[src + d];
                v_cache[dst + d] = v_new[src + d];
            }
        }
    }
    return rc;
}

/* ---------------------------------------------------------------------
 * OCP FP8 E4M3 ("fn": no infinities, NaN = 0x7F / 0xFF, max finite 448).
 * Normal codes: (1 + m/8) * 2^(e-7), e = 1..15 (e = 15, m = 7 is NaN);
 * subnormal codes (e = 0): (m/8) * 2^-6.
 * ------------------------------------------------------------------- */
double pa_oracle_e4m3_decode(uint8_t c)
{
    const int e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    const double mag = e == 0 ? ldexp((double)m, -9) : ldexp(8.0 + m, e - 10);
    return (c & 0x80) ? -mag : mag;
}

/* Round half to even of a non-negative double to an integer (exact). */
static double round_half_even(double v)
{
    double f = floor(v);
    double r = v - f;
    if (r > 0.5) return f + 1.0;
    if (r < 0.5) return f;
    return fmod(f, 2.0) == 0.0 ? f : f + 1.0;
}

/* Nearest E4M3 code to x (ties to even), |x| beyond 448 saturating to 448,
 * NaN to 0x7F. */
uint8_t pa_oracle_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a == 0.0) return sign;
    if (a >= 448.0) return sign | 0x7E;
    int ex;
    frexp(a, &ex);                 /* a = f * 2^ex, f in [0.5, 1) */
    int E = ex - 1;                /* a in [2^E, 2^(E+1)) */
    if (E < -6) {                  /* subnormal range: multiples of 2^-9 */
        double n = round_half_even(ldexp(a, 9));
        if (n >= 8.0) return sign | 0x08;          /* rounded up to 2^-6 */
        return sign | (uint8_t)n;
    }
    double n = round_half_even(ldexp(a, 3 - E)); /* in [8, 16] */
    if (n == 16.0) { n = 8.0; E += 1; }
    if (E > 8 || (E == 8 && n > 14.0)) return sign | 0x7E;  /* beyond 448 */
    return sign | (uint8_t)(((E + 7) << 3) | ((int)n - 8));
}

void pa_oracle_e4m3_encode_array(const float *x, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = pa_oracle_e4m3_encode(x[i]);
}

void pa_oracle_e4m3_decode_array(const uint8_t *c, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = pa_oracle_e4m3_decode(c[i]);
}

static int64_t vt_pos(int64_t t) { return 4 * ((t % 8) / 2) + 2 * (t / 8) + t % 2; }

/* Slot-mapped append into the fp8 caches (block size 16): the row of token
 * t, kv head g is encoded as e4m3(x / scale[g]). */
int pa_oracle_append_fp8(const uint16_t *k_new, const uint16_t *v_new, const int32_t *slot_mapping,
                         int64_t T, uint8_t *k_cache, uint8_t *v_cache, const float *k_scale,
                         const float *v_scale, int64_t Hkv, int64_t D, int64_t NB)
{
    const int64_t bs = 16;
    if (T < 0 || Hkv <= 0 || D <= 0 || NB < 0) return PAO_ERR_ARG;
    if (T > 0 && (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache || !k_scale || !v_scale))
        return PAO_ERR_ARG;
    int rc = PAO_OK;
    for (int64_t t = 0; t < T; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t block = slot / bs, offset = slot % bs;
        if (block >= NB) { rc = PAO_ERR_SLOT; continue; }
        for (int64_t g = 0; g < Hkv; ++g) {
            int64_t src = (t * Hkv + g) * D;
            int64_t tile = block * Hkv + g;
            for (int64_t d = 0; d < D; ++d) {
                float kx = (float)bf16_bits_to_double(k_new[src + d]);
                float vx = (float)bf16_bits_to_double(v_new[src + d]);
                k_cache[(tile * bs + offset) * D + d] = pa_oracle_e4m3_encode(kx / k_scale[g]);
                v_cache[(tile * D + d) * bs + vt_pos(offset)] = pa_oracle_e4m3_encode(vx / v_scale[g]);
            }
        }
    }
    return rc;
}

/* fp8 decode, same formula as pa_oracle_decode on the dequantized values
 * (codes looked up in a table built from pa_oracle_e4m3_decode), threaded
 * over (b, h) rows. */
typedef struct {
    const uint16_t *q;
    const uint8_t *k_cache, *v_cache;
    const float *k_scale, *v_scale;
    const int32_t *block_tables, *context_lens;
    int64_t B, Hq, Hkv, D, NB, M;
    double scale;
    const double *table;
    double *out;
    int64_t first, stride;
    int status;
} fp8_job_t;

static void *decode_fp8_worker(void *arg)
{
    fp8_job_t *j = (fp8_job_t *)arg;
    const int64_t bs = 16, G = j->Hq / j->Hkv, D = j->D;
    double *s_buf = (double *)malloc(sizeof(double) * (size_t)(j->M * bs > 0 ? j->M * bs : 1));
    if (!s_buf) { j->status = PAO_ERR_NOMEM; return NULL; }
    j->status = PAO_OK;
    for (int64_t row = j->first; row < j->B * j->Hq; row += j->stride) {
        const int64_t b = row / j->Hq, h = row % j->Hq, g = h / G;
        const int64_t L = j->context_lens[b];
        const uint16_t *qr = j->q + row * D;
        double *o = j->out + row * D;
        for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
        if (L == 0) continue;
        const double ks = (double)j->k_scale[g], vs = (double)j->v_scale[g];
        double mx = -INFINITY;
        for (int64_t t = 0; t < L; ++t) {
            const int64_t block = j->block_tables[b * j->M + t / bs];
            if (block < 0 || block >= j->NB) { j->status = PAO_ERR_BLOCK; break; }
            const uint8_t *k = j->k_cache + ((block * j->Hkv + g) * bs + t % bs) * D;
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d) dot += bf16_bits_to_double(qr[d]) * (j->table[k[d]] * ks);
            s_buf[t] = j->scale * dot;
            if (s_buf[t] > mx) mx = s_buf[t];
        }
        if (j->status != PAO_OK) break;
        double l = 0.0;
        for (int64_t t = 0; t < L; ++t) {
            const int64_t block = j->block_tables[b * j->M + t / bs];
            const uint8_t *vt = j->v_cache + (block * j->Hkv + g) * D * bs;
            const double w = exp(s_buf[t] - mx);
            l += w;
            const int64_t pos = vt_pos(t % bs);
            for (int64_t d = 0; d < D; ++d) o[d] += w * (j->table[vt[d * bs + pos]] * vs);
        }
        for (int64_t d = 0; d < D; ++d) o[d] /= l;
    }
    free(s_buf);
    return NULL;
}

int pa_oracle_decode_fp8(const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                         const float *k_scale, const float *v_scale,
                         const int32_t *block_tables, const int32_t *context_lens,
                         int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t NB, int64_t M,
                         double scale, double *out, int nthreads)
{
    if (!q || !k_cache || !v_cache || !k_scale || !v_scale || !block_tables || !context_lens || !out)
        return PAO_ERR_ARG;
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || NB < 0 || M < 0 || Hq % Hkv != 0) return PAO_ERR_ARG;
    for (int64_t b = 0; b < B; ++b)
        if (context_lens[b] < 0 || context_lens[b] > M * 16) return PAO_ERR_LEN;
    double table[256];
    for (int c = 0; c < 256; ++c) table[c] = pa_oracle_e4m3_decode((uint8_t)c);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t tid[256];
    fp8_job_t jobs[256];
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = (fp8_job_t){q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                              B, Hq, Hkv, D, NB, M, scale, table, out, i, nthreads, PAO_OK};
        if (nthreads == 1) decode_fp8_worker(&jobs[i]);
        else pthread_create(&tid[i], NULL, decode_fp8_worker, &jobs[i]);
    }
    if (nthreads > 1)
        for (int i = 0; i < nthreads; ++i) pthread_join(tid[i], NULL);
    for (int i = 0; i < nthreads; ++i)
        if (jobs[i].status != PAO_OK) return jobs[i].status;
    return PAO_OK;
}

/* ---------------------------------------------------------------------
 * Multi-query (chunked prefill) attention, threaded over query rows.
 * ------------------------------------------------------------------- */
typedef struct {
    const problem_t *p;
    const int32_t *cu_q_lens;
    double *out;
    int64_t total_rows, first, stride;
    int status;
} prefill_job_t;

static void *prefill_worker(void *arg)
{
    prefill_job_t *job = (prefill_job_t *)arg;
    const problem_t *p = job->p;
    const int64_t G = p->Hq / p->Hkv;
    double *s_buf = (double *)malloc(sizeof(double) * (size_t)(p->M * p->bs > 0 ? p->M * p->bs : 1));
    if (!s_buf) { job->status = PAO_ERR_NOMEM; return NULL; }
    job->status = PAO_OK;
    int64_t b = 0;
    for (int64_t row = job->first; row < job->total_rows; row += job->stride) {
        const int64_t tok = row / p->Hq, h = row % p->Hq;
        while (job->cu_q_lens[b + 1] <= tok) ++b;          /* sequence of query token `tok` */
        const int64_t q_len = job->cu_q_lens[b + 1] - job->cu_q_lens[b];
        const int64_t pos = p->context_lens[b] - q_len + (tok - job->cu_q_lens[b]);
        double m, l;
        int rc = attend_tokens(p, b, h / G, p->q + row * p->D, 0, pos + 1, s_buf,
                               job->out + row * p->D, &m, &l);
        if (rc != PAO_OK) { job->status = rc; break; }
    }
    free(s_buf);
    return NULL;
}

int pa_oracle_prefill(const uint16_t *q, const int32_t *cu_q_lens, const uint16_t *k_cache,
                      const uint16_t *v_cache, const int32_t *block_tables, const int32_t *context_lens,
                      int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t bs, int64_t NB, int64_t M,
                      double scale, double *out, int nthreads)
{
    problem_t p = {q, k_cache, v_cache, block_tables, context_lens, B, Hq, Hkv, D, bs, NB, M, scale};
    int rc = check_problem(&p);
    if (rc != PAO_OK) return rc;
    if (!cu_q_lens || !out || cu_q_lens[0] != 0) return PAO_ERR_ARG;
    for (int64_t b = 0; b < B; ++b) {
        const int64_t q_len = cu_q_lens[b + 1] - cu_q_lens[b];
        if (q_len < 0 || q_len > context_lens[b]) return PAO_ERR_LEN;
    }
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t tid[256];
    prefill_job_t jobs[256];
    const int64_t total_rows = (int64_t)cu_q_lens[B] * Hq;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = (prefill_job_t){&p, cu_q_lens, out, total_rows, i, nthreads, PAO_OK};
        if (nthreads == 1) prefill_worker(&jobs[i]);
        else pthread_create(&tid[i], NULL, prefill_worker, &jobs[i]);
    }
    if (nthreads > 1)
        for (int i = 0; i < nthreads; ++i) pthread_join(tid[i], NULL);
    for (int i = 0; i < nthreads; ++i)
        if (jobs[i].status != PAO_OK) return jobs[i].status;
    return PAO_OK;
}
