/*
 * lazy_oracle.c -- plain, slow, fp64 CPU oracle for deferred-RoPE attention
 * over a shared paged KV cache (LazyAttention).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the
 * CUDA library is checked against.  Only the test suite, the smoke check and
 * the benchmark's CPU-baseline leg may load it.  It shares no code, header,
 * table or constant with the CUDA library, and the library never calls it.
 *
 * Sources (three web pages about arXiv 2606.04302):
 *   [ABS]  shd-paper.top, "LazyAttention: Efficient Retrieval-Augmented
 *          Generation with Deferred Positional Encoding" -- the English
 *          abstract (section "摘要（原文）").
 *   [CORE] gist.science, same title -- Technical Summary, Methodology,
 *          "Core Concept: Deferred Positional Encoding".
 *   [PRE]  same page -- Technical Implementation, "Prefilling".
 *   [DEC]  same page -- Technical Implementation, "Decoding".
 *   [EQV]  same page -- "Mathematical Equivalence".
 *   [CON]  same page -- "Key Contributions" (GQA/MQA compatibility).
 *
 * What it computes.  [EQV] states that deferring RoPE to the kernel gives the
 * same scores and outputs as attending over keys that were rotated eagerly at
 * their logical positions.  The oracle therefore computes the eager
 * (materialised) definition directly: for every request it rebuilds each key
 * as RoPE(k_raw, o + j) at its logical position (segment offset o plus local
 * index j), rotates each query at its own position, and runs causal GQA
 * softmax attention in double precision.  No paging, no deferred rotation, no
 * tiling, no online softmax: those are what the CUDA path does and what this
 * file checks.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - RoPE uses the rotate-half pairing (component i with component i + d/2)
 *     and frequencies theta_i = base^(-2i/d) unless a frequency table is set
 *     (RoPE variants such as Llama-3.1 frequency scaling, computed here by
 *     oracle_llama31_theta from the published rule).
 *   - Softmax scale 1/sqrt(d) unless given; no soft-cap.
 *   - Causal rule: key at position t is visible to a query at position p iff
 *     t <= p.  A query that sees no key produces a zero row.
 *   - GQA: query head h reads KV head h / G with G = Hq / Hkv ([CON]).
 *   - Table word: low 17 bits physical block id, high 15 bits the segment's
 *     logical offset in tokens ([DEC] states only that the block id and
 *     the offset are packed together into one register word).
 *   - Block metadata word: (j0 / 16) << 8 | n_valid, where j0 is the local
 *     index of the block's first token inside its segment and n_valid (1..16)
 *     the number of written slots.
 *   - bf16 values round to nearest, ties to even.
 *   - ALiBi ([CON] names it among the relative encodings the method extends
 *     to): when per-head slopes m_h are set, nothing is rotated and the score
 *     of query head h at position p for the key at position t gets the linear
 *     penalty -m_h * (p - t), with the distance p - t = p - o - j taken from
 *     the same logical positions the RoPE path uses (Press, Smith and Lewis,
 *     "Train Short, Test Long: Attention with Linear Biases", 2022, for the
 *     bias and for the default slopes, oracle_alibi_slopes).
 *
 * Every function is plain C99; OpenMP (if enabled) only splits independent
 * output rows across threads.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef M_PI
#define M_PI 3.14159265358979323846
#endif

#define OR_OK 0
#define OR_EINVAL (-1)
#define OR_ERANGE (-2)
#define OR_ENOMEM (-3)

#define OR_BLOCK_BITS 17
#define OR_OFFSET_BITS 15
#define OR_BLOCK_TOKENS 16

/* ------------------------------------------------------------------------- */
/* bf16 <-> double                                                           */
/* ------------------------------------------------------------------------- */

/* A bf16 value is the top half of an IEEE binary32; widening is exact. */
double oracle_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to bf16 (8 significant bits, binary32 exponent range) with
 * one rounding step, to nearest, ties to even.  Written from the format's
 * definition: find the quantum of x's binade, divide, round, multiply. */
uint16_t oracle_f64_to_bf16(double x)
{
    float f;
    uint32_t u;
    if (isnan(x)) return 0x7FC0;
    if (x == 0.0) {
        f = (float)x; /* keeps the sign of zero */
        memcpy(&u, &f, sizeof u);
        return (uint16_t)(u >> 16);
    }
    double ax = fabs(x);
    int e;
    frexp(ax, &e);               /* ax = m * 2^e, m in [0.5, 1) */
    int q_exp = e - 8;           /* quantum for 8 significant bits */
    if (q_exp < -133) q_exp = -133; /* subnormal range of binary32/bf16 */
    double scaled = ldexp(ax, -q_exp);   /* exact: power-of-two scaling */
    double r = nearbyint(scaled);        /* default mode: nearest, ties even */
    double y = ldexp(r, q_exp);
    if (y > 3.3895313892515355e38) y = INFINITY; /* beyond bf16 max finite */
    f = (float)y;                 /* exact: y has <= 8 significant bits */
    if (x < 0) f = -f;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------- */
/* Segment-table word codec ([DEC]: block id and offset share one 32-bit word). */
/* ------------------------------------------------------------------------- */

int oracle_pack_word(int64_t block, int64_t offset, uint32_t *word)
{
    if (block < 0 || block >= ((int64_t)1 << OR_BLOCK_BITS)) return OR_ERANGE;
    if (offset < 0 || offset >= ((int64_t)1 << OR_OFFSET_BITS)) return OR_ERANGE;
    *word = (uint32_t)offset * (uint32_t)(1u << OR_BLOCK_BITS) + (uint32_t)block;
    return OR_OK;
}

void oracle_unpack_word(uint32_t word, int32_t *block, int32_t *offset)
{
    *block = (int32_t)(word % (1u << OR_BLOCK_BITS));
    *offset = (int32_t)(word / (1u << OR_BLOCK_BITS));
}

uint32_t oracle_pack_meta(int32_t block_index_in_segment, int32_t n_valid)
{
    return (uint32_t)block_index_in_segment * 256u + (uint32_t)n_valid;
}

/* ------------------------------------------------------------------------- */
/* RoPE ([CORE]: positional encoding applied to keys and queries).           */
/* ------------------------------------------------------------------------- */

/* Optional frequency table: when set for d/2 components, theta_i = table[i].
 * Set before a call and cleared after it by the Python wrapper (one call at a
 * time; OpenMP threads only read it). */
static double g_theta[512];
static int g_theta_n = 0;

void oracle_set_rope_theta(const double *theta, int half)
{
    if (!theta || half <= 0 || half > 512) {
        g_theta_n = 0;
        return;
    }
    memcpy(g_theta, theta, sizeof(double) * (size_t)half);
    g_theta_n = half;
}

/* Optional ALiBi slopes, one per query head; set and cleared around a call
 * like the frequency table.  While set, oracle_attend rotates nothing. */
static double g_alibi[4096];
static int g_alibi_n = 0;

void oracle_set_alibi(const double *slopes, int n)
{
    if (!slopes || n <= 0 || n > 4096) {
        g_alibi_n = 0;
        return;
    }
    memcpy(g_alibi, slopes, sizeof(double) * (size_t)n);
    g_alibi_n = n;
}

/* The ALiBi paper's head slopes for n heads: for n a power of two, the
 * geometric sequence whose first term and ratio are both 2^(-8/n); otherwise
 * the slopes of the largest power of two m below n, followed by the first
 * n - m terms at even positions (0, 2, 4, ...) of the sequence for 2m. */
static double alibi_geometric(int n, int k)
{
    return pow(2.0, -8.0 * (double)(k + 1) / (double)n);
}

void oracle_alibi_slopes(int n, double *out)
{
    int m = 1;
    while (2 * m <= n) m *= 2;
    for (int k = 0; k < m && k < n; ++k) out[k] = alibi_geometric(m, k);
    for (int k = m; k < n; ++k) out[k] = alibi_geometric(2 * m, 2 * (k - m));
}

static double rope_theta(int i, int d, double base)
{
    if (g_theta_n == d / 2) return g_theta[i];
    return pow(base, -2.0 * (double)i / (double)d);
}

/* Llama-3.1 frequency scaling of the RoPE frequencies (the "llama3" rope type
 * of the Llama 3.1 model configuration): with f_i = base^(-2i/d) and its
 * wavelength 2*pi/f_i, components whose wavelength is below
 * original_max/high_factor keep f_i, those above original_max/low_factor get
 * f_i/factor, and in between f_i is interpolated linearly in the ratio
 * original_max/wavelength, from f_i/factor at low_factor to f_i at
 * high_factor. */
void oracle_llama31_theta(double base, int d, double factor, double low_factor, double high_factor,
                          double original_max, double *theta)
{
    const double lo_wl = original_max / low_factor, hi_wl = original_max / high_factor;
    for (int i = 0; i < d / 2; ++i) {
        const double f = pow(base, -(2.0 * i) / d);   /* the unscaled frequency */
        const double wl = 2.0 * M_PI / f;
        if (wl < hi_wl) {
            theta[i] = f;
        } else if (wl > lo_wl) {
            theta[i] = f / factor;
        } else {
            const double s = (original_max / wl - low_factor) / (high_factor - low_factor);
            theta[i] = (1.0 - s) * f / factor + s * f;
        }
    }
}

/* y = RoPE(x, pos): for each pair (i, i + d/2) rotate by angle pos*theta_i. */
void oracle_rope(const double *x, int d, double base, int64_t pos, double *y)
{
    int half = d / 2;
    for (int i = 0; i < half; ++i) {
        double ang = (double)pos * rope_theta(i, d, base);
        double c = cos(ang), s = sin(ang);
        double a = x[i], b = x[i + half];
        y[i] = a * c - b * s;
        y[i + half] = b * c + a * s;
    }
}

/* ------------------------------------------------------------------------- */
/* Expected pool contents after writes ([CORE], [ABS]: one physical copy per  */
/* document, keys rotated at their document-local index j).                  */
/* ------------------------------------------------------------------------- */

/* For each token t: block = slot[t] / 16, s = slot[t] % 16.
 *   k_pool[block][h][s][:] = bf16(RoPE(k_raw[t][h][:], local_j[t]))
 *   v_pool[block][h][s][:] = v_raw[t][h][:]
 *   blk_meta[block] = max(blk_meta[block], meta(local_j[t] / 16, s + 1))
 * A token whose local index is not congruent to its slot modulo 16 breaks the
 * block alignment of segments and is reported (OR_ERANGE); so is a slot
 * outside the pool.  Pools and metadata are read-modify-written in place. */
int oracle_kv_write(int n_tok, int num_kv_heads, int head_dim, double rope_base,
                    const uint16_t *k_raw, const uint16_t *v_raw,
                    const int32_t *slot, const int32_t *local_j,
                    int64_t num_blocks, uint16_t *k_pool, uint16_t *v_pool,
                    uint32_t *blk_meta)
{
    int d = head_dim;
    double *x = (double *)malloc(sizeof(double) * 2 * (size_t)d);
    if (!x) return OR_ENOMEM;
    double *y = x + d;
    int rc = OR_OK;
    for (int t = 0; t < n_tok; ++t) {
        int64_t sl = slot[t];
        if (sl < 0 || sl >= num_blocks * OR_BLOCK_TOKENS || local_j[t] < 0 ||
            (local_j[t] % OR_BLOCK_TOKENS) != (int)(sl % OR_BLOCK_TOKENS)) {
            rc = OR_ERANGE;
            continue;
        }
        int64_t blk = sl / OR_BLOCK_TOKENS;
        int s = (int)(sl % OR_BLOCK_TOKENS);
        for (int h = 0; h < num_kv_heads; ++h) {
            const uint16_t *kr = k_raw + ((size_t)t * num_kv_heads + h) * d;
            const uint16_t *vr = v_raw + ((size_t)t * num_kv_heads + h) * d;
            size_t dst = (((size_t)blk * num_kv_heads + h) * OR_BLOCK_TOKENS + s) * d;
            for (int i = 0; i < d; ++i) x[i] = oracle_bf16_to_f64(kr[i]);
            oracle_rope(x, d, rope_base, local_j[t], y);
            for (int i = 0; i < d; ++i) {
                k_pool[dst + i] = oracle_f64_to_bf16(y[i]);
                v_pool[dst + i] = vr[i];
            }
        }
        uint32_t m = oracle_pack_meta(local_j[t] / OR_BLOCK_TOKENS, s + 1);
        if (m > blk_meta[blk]) blk_meta[blk] = m;
    }
    free(x);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Table expansion: what every table word means, slot by slot ([DEC]).       */
/* ------------------------------------------------------------------------- */

/* For table word w (block b, offset o) and slot s in 0..15:
 *   out_block[16w+s] = b
 *   out_slot [16w+s] = 16*b + s
 *   out_pos  [16w+s] = o + 16*(meta index of b) + s   if s < n_valid(b), else -1
 * A block id outside the pool gives OR_ERANGE and -1 entries. */
int oracle_expand_table(int64_t n_words, const uint32_t *words, const uint32_t *blk_meta,
                        int64_t num_blocks, int32_t *out_block, int32_t *out_slot,
                        int32_t *out_pos)
{
    int rc = OR_OK;
    for (int64_t w = 0; w < n_words; ++w) {
        int32_t b, o;
        oracle_unpack_word(words[w], &b, &o);
        int valid = b < num_blocks;
        uint32_t meta = valid ? blk_meta[b] : 0;
        int32_t idx = (int32_t)(meta / 256u), nv = (int32_t)(meta % 256u);
        if (!valid) rc = OR_ERANGE;
        for (int s = 0; s < OR_BLOCK_TOKENS; ++s) {
            out_block[w * OR_BLOCK_TOKENS + s] = valid ? b : -1;
            out_slot[w * OR_BLOCK_TOKENS + s] = valid ? b * OR_BLOCK_TOKENS + s : -1;
            out_pos[w * OR_BLOCK_TOKENS + s] =
                (valid && s < nv) ? o + idx * OR_BLOCK_TOKENS + s : -1;
        }
    }
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Attention, materialised semantics ([EQV], [PRE], [DEC], [CON]).           */
/* ------------------------------------------------------------------------- */

/* Inputs describe each request as a list of segments over a token store of
 * raw (unrotated) keys and values:
 *   segment g of request r (seg_indptr[r] <= g < seg_indptr[r+1]) covers
 *   store rows seg_src[g] .. seg_src[g] + seg_len[g] - 1, whose local index j
 *   sits at logical position seg_off[g] + j.
 * Queries: q_raw[q][h][:] for q in cu_q[r] .. cu_q[r+1]-1, at q_pos[q].
 * Rows computed: (sel_q[i], sel_h[i]) for i < n_sel; n_sel < 0 means every
 * (query, head) pair in order q-major, h-minor.
 * out[i][:] receives the attention output of row i.  If scores != NULL it
 * receives, per row, the scaled scores of the request's keys in segment
 * order (masked keys: -INFINITY), scores_ld doubles apart. */
int oracle_attend(int num_req, int num_q_heads, int num_kv_heads, int head_dim,
                  double rope_base, double softmax_scale,
                  const uint16_t *q_raw, const int32_t *cu_q, const int32_t *q_pos,
                  const int32_t *seg_indptr, const int32_t *seg_src,
                  const int32_t *seg_off, const int32_t *seg_len,
                  const uint16_t *k_tok, const uint16_t *v_tok,
                  int64_t n_sel, const int32_t *sel_q, const int32_t *sel_h,
                  double *out, double *scores, int64_t scores_ld)
{
    const int d = head_dim, Hq = num_q_heads, Hkv = num_kv_heads;
    if (d <= 0 || (d % 2) != 0 || Hkv <= 0 || Hq <= 0 || (Hq % Hkv) != 0) return OR_EINVAL;
    const int G = Hq / Hkv;
    const double scale = softmax_scale > 0 ? softmax_scale : 1.0 / sqrt((double)d);
    const int64_t total_q = cu_q[num_req];
    const int64_t n_rows = n_sel >= 0 ? n_sel : total_q * Hq;
    const int alibi = g_alibi_n == Hq;   /* linear position penalty in place of RoPE */
    int rc = OR_OK;

    for (int r = 0; r < num_req; ++r) {
        /* rows of this request */
        int64_t cnt = 0;
        for (int64_t i = 0; i < n_rows; ++i) {
            int64_t q = n_sel >= 0 ? sel_q[i] : i / Hq;
            if (q >= cu_q[r] && q < cu_q[r + 1]) ++cnt;
        }
        if (cnt == 0) continue;

        /* 1. keys rotated eagerly at logical positions, values as given */
        int64_t kv_len = 0;
        for (int g = seg_indptr[r]; g < seg_indptr[r + 1]; ++g) kv_len += seg_len[g];
        double *K = (double *)malloc(sizeof(double) * (size_t)(kv_len > 0 ? kv_len : 1) * Hkv * d);
        double *V = (double *)malloc(sizeof(double) * (size_t)(kv_len > 0 ? kv_len : 1) * Hkv * d);
        int64_t *P = (int64_t *)malloc(sizeof(int64_t) * (size_t)(kv_len > 0 ? kv_len : 1));
        int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)cnt);
        if (!K || !V || !P || !rows) {
            free(K); free(V); free(P); free(rows);
            return OR_ENOMEM;
        }
        int64_t t = 0;
        for (int g = seg_indptr[r]; g < seg_indptr[r + 1]; ++g) {
            for (int j = 0; j < seg_len[g]; ++j, ++t) {
                P[t] = (int64_t)seg_off[g] + j;
                for (int h = 0; h < Hkv; ++h) {
                    const uint16_t *kr = k_tok + (((size_t)seg_src[g] + j) * Hkv + h) * d;
                    const uint16_t *vr = v_tok + (((size_t)seg_src[g] + j) * Hkv + h) * d;
                    double x[1024];
                    if (d > 1024) { rc = OR_EINVAL; continue; }
                    for (int i = 0; i < d; ++i) x[i] = oracle_bf16_to_f64(kr[i]);
                    if (alibi)
                        memcpy(K + ((size_t)t * Hkv + h) * d, x, sizeof(double) * (size_t)d);
                    else
                        oracle_rope(x, d, rope_base, P[t], K + ((size_t)t * Hkv + h) * d);
                    for (int i = 0; i < d; ++i) V[((size_t)t * Hkv + h) * d + i] = oracle_bf16_to_f64(vr[i]);
                }
            }
        }
        int64_t c = 0;
        for (int64_t i = 0; i < n_rows; ++i) {
            int64_t q = n_sel >= 0 ? sel_q[i] : i / Hq;
            if (q >= cu_q[r] && q < cu_q[r + 1]) rows[c++] = i;
        }

        /* 2-5. per (query, head) row: rotate q, score, mask, softmax, output */
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t ci = 0; ci < cnt; ++ci) {
            int64_t i = rows[ci];
            int64_t q = n_sel >= 0 ? sel_q[i] : i / Hq;
            int h = n_sel >= 0 ? sel_h[i] : (int)(i % Hq);
            int kvh = h / G;
            int64_t p = q_pos[q];
            double xq[1024], qr[1024];
            for (int k = 0; k < d; ++k) xq[k] = oracle_bf16_to_f64(q_raw[((size_t)q * Hq + h) * d + k]);
            if (alibi)
                memcpy(qr, xq, sizeof(double) * (size_t)d);
            else
                oracle_rope(xq, d, rope_base, p, qr);
            double *s = (double *)malloc(sizeof(double) * (size_t)(kv_len > 0 ? kv_len : 1));
            double m = -INFINITY;
            for (int64_t u = 0; u < kv_len; ++u) {
                if (P[u] <= p) {
                    const double *kk = K + ((size_t)u * Hkv + kvh) * d;
                    double acc = 0.0;
                    for (int k = 0; k < d; ++k) acc += qr[k] * kk[k];
                    s[u] = acc * scale;
                    if (alibi) s[u] -= g_alibi[h] * (double)(p - P[u]);
                    if (s[u] > m) m = s[u];
                } else {
                    s[u] = -INFINITY;
                }
                if (scores) scores[i * scores_ld + u] = s[u];
            }
            double *o = out + i * d;
            for (int k = 0; k < d; ++k) o[k] = 0.0;
            if (m != -INFINITY) {
                double l = 0.0;
                for (int64_t u = 0; u < kv_len; ++u) {
                    if (s[u] == -INFINITY) continue;
                    double w = exp(s[u] - m);
                    l += w;
                    const double *vv = V + ((size_t)u * Hkv + kvh) * d;
                    for (int k = 0; k < d; ++k) o[k] += w * vv[k];
                }
                for (int k = 0; k < d; ++k) o[k] /= l;
            }
            free(s);
        }
        free(K); free(V); free(P); free(rows);
    }
    return rc;
}

/* Number of OpenMP threads the oracle will use (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Keys rotated eagerly at given logical positions and rounded to bf16: the
 * content a position-aware cache would hold ([ABS]: a copy re-encoded for its
 * positions, the cost the method avoids).  Used to check a materialised-key
 * copy.
 *   out[n][h][:] = bf16(RoPE(k_raw[n][h][:], pos[n])) */
int oracle_rope_rows_bf16(int64_t n, int num_kv_heads, int head_dim, double rope_base,
                          const uint16_t *k_raw, const int32_t *pos, uint16_t *out)
{
    int d = head_dim;
    if (d <= 0 || d > 1024 || (d % 2) != 0) return OR_EINVAL;
    for (int64_t t = 0; t < n; ++t) {
        for (int h = 0; h < num_kv_heads; ++h) {
            double x[1024], y[1024];
            const uint16_t *kr = k_raw + ((size_t)t * num_kv_heads + h) * d;
            for (int i = 0; i < d; ++i) x[i] = oracle_bf16_to_f64(kr[i]);
            oracle_rope(x, d, rope_base, pos[t], y);
            for (int i = 0; i < d; ++i) out[((size_t)t * num_kv_heads + h) * d + i] = oracle_f64_to_bf16(y[i]);
        }
    }
    return OR_OK;
}
