/*
 * oracle.c -- plain float64 CPU oracle for attention with a KV cache and RoPE.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library under rotary_embedding_b200/csrc) never calls it, and
 * the two share no code: no headers, no helpers, no tables.
 *
 * Everything here is the plain definition, written so that a reader can
 * check it against the pages by eye: single-threaded, no blocking, no
 * fusion, exact (two-pass) softmax, all arithmetic in double precision.
 *
 * Sources (page title, then section):
 *  [P1] flash-attention issue #1402 "is flash_attn_with_kvcache() supposed
 *       to work for seqlen > 1 ?" -- the no-RoPE reproducer (cache passed
 *       as [batch, seq, heads, dim] views, cache_seqlens) and the RoPE
 *       reproducer (inv_freq table, rotate_half, apply_rotary_emb with the
 *       result cast back to the input type).
 *  [P2] ROCm/flash-attention PR #99 "Added Support for Rotary Positional
 *       Embeddings (both non-fused and fused kernel)" -- COS/SIN of shape
 *       (seqlen, rotary_dim/2), SEQLEN_OFFSET as int or per-batch tensor,
 *       INTERLEAVED flag, rotary_fraction, and the "Motivation" section
 *       (each 2-D chunk of q and k rotated by an angle set by the token's
 *       position m and the chunk index).
 *  [P3] s2.cpp PR #40 "feat: Flash Attention and modernized KV Cache layout
 *       for Slow-AR" -- write the new k/v rows into the cache at their
 *       offsets, then attend (the write must precede the read).
 *  [P4] flash-attention PR #1604 "Support hdimQK != hdimV backward" --
 *       d_qk may differ from d_v (DeepSeek 192/128).
 *  [P5] "optimizing-attention-flash" skill page -- Workflow 1 Step 2
 *       (softmax(q k^T / sqrt(d)) v), Workflow 2 Step 2 (layout
 *       [batch, seq, heads, dim], causal flag, softmax_scale=None means
 *       1/sqrt(d)) and Step 3 (fewer KV heads than query heads).
 *
 * Readings where the pages are silent:
 *  - the query row i of batch b sits at position cache_seqlens[b] + i, the
 *    same position as new key row i;
 *  - half-split pairs (j, j + r/2) inside the first r dims, interleaved
 *    pairs (2j, 2j+1); dims >= r pass through;
 *  - query head h reads kv head h / (h_q / h_kv);
 *  - causal masking is aligned bottom-right: query i of s_q sees key j of
 *    N keys iff j <= i + N - s_q;
 *  - lse is the natural-log log-sum-exp of the scaled scores; a row with no
 *    visible key gives out = 0 and lse = -inf;
 *  - rounding to fp16/bf16 is round-to-nearest-even.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ORACLE_PLANT selects a deliberately wrong variant, built only by the
 * tests that check the pins catch such mistakes (0 = the real oracle). */
#ifndef ORACLE_PLANT
#define ORACLE_PLANT 0
#endif

#define ORACLE_NO_ROUND 0
#define ORACLE_FP16 1
#define ORACLE_BF16 2

/* ------------------------------------------------------------------ */
/* Rounding a double to the nearest fp16 / bf16 value (ties to even),  */
/* from the IEEE 754 binary16 definition (11 significant bits, normal  */
/* exponents -14..15) and the bfloat16 definition (8 significant bits, */
/* the binary32 exponent range).  The result is returned as a double.  */
/* ------------------------------------------------------------------ */
static double round_to_format(double x, int sig_bits, int emin_frexp, double maxval)
{
    if (x == 0.0 || isnan(x) || isinf(x)) return x;
    int e;
    frexp(x, &e);                 /* x = m * 2^e with 0.5 <= |m| < 1 */
    if (e < emin_frexp) e = emin_frexp;   /* subnormal range: fixed quantum */
    double quantum = ldexp(1.0, e - sig_bits);
    double r = rint(x / quantum) * quantum;   /* rint: nearest, ties to even */
    if (fabs(r) > maxval) r = copysign(INFINITY, x);
    return r;
}

double oracle_round_one(double x, int fmt)
{
    if (fmt == ORACLE_FP16)
        /* binary16: min normal 2^-14 = 0.5 * 2^-13; max 65504 */
        return round_to_format(x, 11, -13, 65504.0);
    if (fmt == ORACLE_BF16)
        /* bfloat16: min normal 2^-126 = 0.5 * 2^-125; max (2 - 2^-7) * 2^127 */
        return round_to_format(x, 8, -125, ldexp(2.0 - ldexp(1.0, -7), 127));
    return x;
}

void oracle_round(double *x, int64_t n, int fmt)
{
    for (int64_t i = 0; i < n; ++i) x[i] = oracle_round_one(x[i], fmt);
}

/* ------------------------------------------------------------------ */
/* RoPE of one row of d values at table row `pos` ([P1] RoPE         */
/* reproducer, rotate_half; [P2] COS/SIN (seqlen, r/2), INTERLEAVED,  */
/* "Motivation").  For each angle index j < r/2 the pair (a, b) is     */
/* rotated by the table angle: a' = a c - b s, b' = a s + b c.         */
/* ------------------------------------------------------------------ */
void oracle_rope_row(const double *x, double *y, int d, int r, int interleaved,
                     const double *cos_row, const double *sin_row)
{
    for (int t = 0; t < d; ++t) y[t] = x[t];
    int half = r / 2;
    for (int j = 0; j < half; ++j) {
        int ia, ib;
        if (interleaved) { ia = 2 * j; ib = 2 * j + 1; }
        else             { ia = j;     ib = j + half;  }
#if ORACLE_PLANT == 3            /* planted: half-split partner from the full head dim */
        if (!interleaved) ib = j + d / 2;
#endif
        double c = cos_row[j], s = sin_row[j];
        double a = x[ia], b = x[ib];
#if ORACLE_PLANT == 1            /* planted: rotation sign flipped */
        y[ia] = a * c + b * s;
        y[ib] = -a * s + b * c;
#elif ORACLE_PLANT == 2          /* planted: sin and cos swapped */
        y[ia] = a * s - b * c;
        y[ib] = a * c + b * s;
#else
        y[ia] = a * c - b * s;
        y[ib] = a * s + b * c;
#endif
    }
}

/* Rotate `rows` rows of length d, row i at table row pos[i].  The
 * tables are [tab_rows, r/2] row-major.  Returns -1 if a position is
 * outside the table. */
int oracle_rope(const double *x, double *y, int64_t rows, int d, const int64_t *pos,
                const double *cos_tab, const double *sin_tab, int64_t tab_rows,
                int r, int interleaved)
{
    int half = r / 2;
    for (int64_t i = 0; i < rows; ++i) {
        if (r > 0 && (pos[i] < 0 || pos[i] >= tab_rows)) return -1;
        const double *cr = r > 0 ? cos_tab + pos[i] * half : NULL;
        const double *sr = r > 0 ? sin_tab + pos[i] * half : NULL;
        oracle_rope_row(x + i * d, y + i * d, d, r, interleaved, cr, sr);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Standalone rotary ([P2] "both non-fused and fused kernel": COS/SIN, */
/* SEQLEN_OFFSET, INTERLEAVED, CONJUGATE).  Row i of x (length d) is   */
/* rotated at table row pos[i]; with `conjugate` every pair is rotated */
/* by the negated angle (sin replaced by -sin: the inverse rotation),   */
/* then the result is rounded to `fmt`.  Returns -1 if a position is   */
/* outside the table.                                                  */
/* ------------------------------------------------------------------ */
int oracle_rotary(const double *x, double *y, int64_t rows, int d, const int64_t *pos,
                  const double *cos_tab, const double *sin_tab, int64_t tab_rows,
                  int r, int interleaved, int conjugate, int fmt)
{
    int half = r / 2;
    double *neg = half > 0 ? (double *)malloc(sizeof(double) * half) : NULL;
    for (int64_t i = 0; i < rows; ++i) {
        if (r > 0 && (pos[i] < 0 || pos[i] >= tab_rows)) { free(neg); return -1; }
        const double *cr = r > 0 ? cos_tab + pos[i] * half : NULL;
        const double *sr = r > 0 ? sin_tab + pos[i] * half : NULL;
#if ORACLE_PLANT == 11           /* planted: the conjugate flag ignored */
        conjugate = 0;
#endif
        if (r > 0 && conjugate) {
            for (int j = 0; j < half; ++j) neg[j] = -sr[j];
            sr = neg;
        }
        oracle_rope_row(x + i * d, y + i * d, d, r, interleaved, cr, sr);
        oracle_round(y + i * d, d, fmt);
    }
    free(neg);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Keys lo .. hi visible to query row i of s_q over N keys (hi < lo:   */
/* none).  The rows are aligned bottom-right at a = i + N - s_q: with  */
/* causal, hi = a; with a window ("optimizing-attention-flash",        */
/* window_size=(left, right), -1 = unbounded), lo = a - left and hi is */
/* at most a + right.                                                  */
/* ------------------------------------------------------------------ */
static void visible_range(int64_t i, int64_t N, int64_t s_q, int causal,
                          int64_t win_left, int64_t win_right, int64_t *lo_out, int64_t *hi_out)
{
    int64_t a = i + N - s_q;
    int64_t hi = N - 1, lo = 0;
    if (causal) {
        int64_t last = a;                    /* last visible key index */
#if ORACLE_PLANT == 4            /* planted: top-left instead of bottom-right alignment */
        last = i;
#elif ORACLE_PLANT == 5          /* planted: diagonal excluded */
        last = a - 1;
#endif
        hi = last;
    }
    if (win_right >= 0 && a + win_right < hi) hi = a + win_right;
    if (win_left >= 0) lo = a - win_left;
#if ORACLE_PLANT == 12           /* planted: left window one key short */
    if (win_left >= 0) lo = a - win_left + 1;
#endif
    if (lo < 0) lo = 0;
    if (hi > N - 1) hi = N - 1;
    *lo_out = lo;
    *hi_out = hi;
}

/* ------------------------------------------------------------------ */
/* Exact masked softmax attention for one (batch, query head) pair     */
/* ([P5] Workflow 1 Step 2; causal flag of Workflow 2 Step 2).         */
/*   q_rows  [s_q, d_qk] with row stride q_ld                          */
/*   k_rows  [N, d_qk]   with row stride k_ld                          */
/*   v_rows  [N, d_v]    with row stride v_ld                          */
/*   out     [s_q, d_v]  with row stride o_ld                          */
/*   lse     [s_q]                                                     */
/* ------------------------------------------------------------------ */
static void attend_one_head(const double *q_rows, int64_t q_ld,
                            const double *k_rows, int64_t k_ld,
                            const double *v_rows, int64_t v_ld,
                            int64_t s_q, int64_t N, int d_qk, int d_v,
                            int causal, int64_t win_left, int64_t win_right, double scale,
                            double *out, int64_t o_ld, double *lse, double *scores)
{
    for (int64_t i = 0; i < s_q; ++i) {
        int64_t lo, hi;
        visible_range(i, N, s_q, causal, win_left, win_right, &lo, &hi);
        double *o = out + i * o_ld;
        if (hi < lo) {
            for (int t = 0; t < d_v; ++t) o[t] = 0.0;
            lse[i] = -INFINITY;
            continue;
        }
        const double *qi = q_rows + i * q_ld;
        double m = -INFINITY;
        for (int64_t j = lo; j <= hi; ++j) {
            const double *kj = k_rows + j * k_ld;
            double dot = 0.0;
            for (int t = 0; t < d_qk; ++t) dot += qi[t] * kj[t];
#if ORACLE_PLANT == 6            /* planted: scale dropped */
            scores[j - lo] = dot;
#else
            scores[j - lo] = scale * dot;
#endif
            if (scores[j - lo] > m) m = scores[j - lo];
        }
        double l = 0.0;
        for (int64_t j = lo; j <= hi; ++j) {
            scores[j - lo] = exp(scores[j - lo] - m);
            l += scores[j - lo];
        }
        for (int t = 0; t < d_v; ++t) o[t] = 0.0;
        for (int64_t j = lo; j <= hi; ++j) {
            const double *vj = v_rows + j * v_ld;
            double p = scores[j - lo] / l;
            for (int t = 0; t < d_v; ++t) o[t] += p * vj[t];
        }
#if ORACLE_PLANT == 7            /* planted: max term dropped from lse */
        lse[i] = log(l);
#else
        lse[i] = m + log(l);
#endif
    }
}

/* ------------------------------------------------------------------ */
/* attn_with_kvcache, the whole path:                                  */
/*  1. rotate q rows and new k rows at positions L_b + i ([P1], [P2]), */
/*     rounding the result to the element type ([P1]: .type_as);      */
/*  2. write rotated k and raw v into cache rows L_b .. L_b+s_new-1   */
/*     ([P1] cache_seqlens, [P3] write then attend);                  */
/*  3. attend over cache rows 0 .. L_b+s_new-1 with GQA head mapping  */
/*     and the bottom-right causal mask ([P4], [P5]).                 */
/* Layouts (all contiguous):                                          */
/*   q [b, s_q, h_q, d_qk]; k_cache [b, cap, h_kv, d_qk];              */
/*   v_cache [b, cap, h_kv, d_v]; k_new [b, s_new, h_kv, d_qk];         */
/*   v_new [b, s_new, h_kv, d_v]; cos/sin [tab_rows, r/2];             */
/*   out [b, s_q, h_q, d_v]; lse [b, h_q, s_q].                        */
/* k_cache / v_cache are updated in place.  k_new may be NULL          */
/* (s_new must then be 0).  r == 0 disables RoPE.                      */
/* Returns 0, or a negative value for an argument the definition       */
/* cannot evaluate (a row past the cache or the table).                */
/* ------------------------------------------------------------------ */
int oracle_kvcache_fwd(int64_t b, int64_t s_q, int64_t s_new, int64_t h_q, int64_t h_kv,
                       int d_qk, int d_v, int64_t cap,
                       const double *q, double *k_cache, double *v_cache,
                       const double *k_new, const double *v_new,
                       const double *cos_tab, const double *sin_tab, int64_t tab_rows,
                       int r, int interleaved, const int32_t *cache_seqlens,
                       int causal, double scale, int fmt,
                       double *out, double *lse, int64_t win_left, int64_t win_right)
{
    if (h_kv <= 0 || h_q % h_kv != 0) return -1;
    if (r < 0 || r % 2 != 0 || r > d_qk) return -2;
    int64_t group = h_q / h_kv;
    double *qrot = (double *)malloc(sizeof(double) * (size_t)(s_q * h_q * d_qk > 0 ? s_q * h_q * d_qk : 1));
    double *scores = (double *)malloc(sizeof(double) * (size_t)(cap + 1));
    if (!qrot || !scores) { free(qrot); free(scores); return -4; }
    int rc = 0;
    for (int64_t bi = 0; bi < b && rc == 0; ++bi) {
        int64_t L = cache_seqlens[bi];
        int64_t N = L + s_new;
        if (L < 0 || N > cap) { rc = -3; break; }
        if (r > 0 && N > tab_rows) { rc = -3; break; }
        if (r > 0 && L + s_q > tab_rows) { rc = -3; break; }
        /* step 1+2: rotate the new key rows and append them with the raw v rows */
        for (int64_t i = 0; i < s_new; ++i) {
            for (int64_t h = 0; h < h_kv; ++h) {
                const double *kn = k_new + ((bi * s_new + i) * h_kv + h) * d_qk;
                const double *vn = v_new + ((bi * s_new + i) * h_kv + h) * d_v;
                double *kc = k_cache + ((bi * cap + L + i) * h_kv + h) * d_qk;
                double *vc = v_cache + ((bi * cap + L + i) * h_kv + h) * d_v;
                if (r > 0)
                    oracle_rope_row(kn, kc, d_qk, r, interleaved,
                                    cos_tab + (L + i) * (r / 2), sin_tab + (L + i) * (r / 2));
                else
                    for (int t = 0; t < d_qk; ++t) kc[t] = kn[t];
                for (int t = 0; t < d_qk; ++t) kc[t] = oracle_round_one(kc[t], fmt);
#if ORACLE_PLANT == 10           /* planted: v rows written one row late */
                if (L + i + 1 < cap)
                    vc += h_kv * d_v;
#endif
                for (int t = 0; t < d_v; ++t) vc[t] = vn[t];
            }
        }
        /* step 1: rotate the query rows at the same positions */
        for (int64_t i = 0; i < s_q; ++i) {
            for (int64_t h = 0; h < h_q; ++h) {
                const double *qs = q + ((bi * s_q + i) * h_q + h) * d_qk;
                double *qd = qrot + (i * h_q + h) * d_qk;
                int64_t pos = L + i;
#if ORACLE_PLANT == 9            /* planted: every query row at position L */
                pos = L;
#endif
                if (r > 0)
                    oracle_rope_row(qs, qd, d_qk, r, interleaved,
                                    cos_tab + pos * (r / 2), sin_tab + pos * (r / 2));
                else
                    for (int t = 0; t < d_qk; ++t) qd[t] = qs[t];
                for (int t = 0; t < d_qk; ++t) qd[t] = oracle_round_one(qd[t], fmt);
            }
        }
        /* step 3: attention over the N keys now in the cache */
        for (int64_t h = 0; h < h_q; ++h) {
#if ORACLE_PLANT == 8            /* planted: kv head chosen modulo instead of by group */
            int64_t hk = h % h_kv;
#else
            int64_t hk = h / group;
#endif
            attend_one_head(qrot + h * d_qk, h_q * d_qk,
                            k_cache + (bi * cap * h_kv + hk) * d_qk, h_kv * d_qk,
                            v_cache + (bi * cap * h_kv + hk) * d_v, h_kv * d_v,
                            s_q, N, d_qk, d_v, causal, win_left, win_right, scale,
                            out + (bi * s_q * h_q + h) * d_v, h_q * d_v,
                            lse + (bi * h_q + h) * s_q, scores);
        }
    }
    free(qrot);
    free(scores);
    return rc;
}

/* ------------------------------------------------------------------ */
/* Cache-less attention ([P5] Quick start, flash_attn_func):           */
/*   q [b, s_q, h_q, d_qk], k [b, s_k, h_kv, d_qk], v [b, s_k, h_kv, d_v] */
/*   out [b, s_q, h_q, d_v], lse [b, h_q, s_q].                        */
/* ------------------------------------------------------------------ */
int oracle_fwd(int64_t b, int64_t s_q, int64_t s_k, int64_t h_q, int64_t h_kv,
               int d_qk, int d_v, const double *q, const double *k, const double *v,
               int causal, double scale, double *out, double *lse, int64_t win_left, int64_t win_right)
{
    if (h_kv <= 0 || h_q % h_kv != 0) return -1;
    int64_t group = h_q / h_kv;
    double *scores = (double *)malloc(sizeof(double) * (size_t)(s_k + 1));
    if (!scores) return -4;
    for (int64_t bi = 0; bi < b; ++bi)
        for (int64_t h = 0; h < h_q; ++h) {
            int64_t hk = h / group;
            attend_one_head(q + (bi * s_q * h_q + h) * d_qk, h_q * d_qk,
                            k + (bi * s_k * h_kv + hk) * d_qk, h_kv * d_qk,
                            v + (bi * s_k * h_kv + hk) * d_v, h_kv * d_v,
                            s_q, s_k, d_qk, d_v, causal, win_left, win_right, scale,
                            out + (bi * s_q * h_q + h) * d_v, h_q * d_v,
                            lse + (bi * h_q + h) * s_q, scores);
        }
    free(scores);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Backward of cache-less attention ([P4] "Support hdimQK != hdimV     */
/* backward": the gradients of q, k and v when d_qk != d_v).  The     */
/* pages give no formula; this is the gradient of the forward's        */
/* definition, out_i = sum_j P_ij v_j with P_i = softmax_j(scale q_i.k_j) */
/* over the visible keys, for an upstream gradient dout:               */
/*   dv_j  += P_ij dout_i                                              */
/*   dP_ij  = dout_i . v_j                                             */
/*   dS_ij  = P_ij (dP_ij - sum_t P_it dP_it)   (softmax Jacobian)     */
/*   dq_i   = scale sum_j dS_ij k_j                                    */
/*   dk_j  += scale dS_ij q_i                                          */
/* with P recomputed exactly (two-pass softmax) from q and k.  A kv    */
/* head's dk and dv sum over the query heads that read it (GQA).       */
/* Layouts (contiguous): q, dq [b, s_q, h_q, d_qk]; k, dk              */
/* [b, s_k, h_kv, d_qk]; v, dv [b, s_k, h_kv, d_v]; dout               */
/* [b, s_q, h_q, d_v].  Returns 0, or a negative value for arguments   */
/* the definition cannot evaluate.                                     */
/* ------------------------------------------------------------------ */
int oracle_bwd(int64_t b, int64_t s_q, int64_t s_k, int64_t h_q, int64_t h_kv,
               int d_qk, int d_v, const double *q, const double *k, const double *v,
               const double *dout, int causal, double scale, int64_t win_left, int64_t win_right,
               double *dq, double *dk, double *dv)
{
    if (h_kv <= 0 || h_q % h_kv != 0) return -1;
    int64_t group = h_q / h_kv;
    double *P = (double *)malloc(sizeof(double) * (size_t)(s_k + 1));
    double *dP = (double *)malloc(sizeof(double) * (size_t)(s_k + 1));
    if (!P || !dP) {
        free(P);
        free(dP);
        return -4;
    }
    memset(dq, 0, sizeof(double) * (size_t)(b * s_q * h_q * d_qk));
    memset(dk, 0, sizeof(double) * (size_t)(b * s_k * h_kv * d_qk));
    memset(dv, 0, sizeof(double) * (size_t)(b * s_k * h_kv * d_v));
    for (int64_t bi = 0; bi < b; ++bi)
        for (int64_t h = 0; h < h_q; ++h) {
            int64_t hk = h / group;
#if ORACLE_PLANT == 15           /* planted: only the group's last query head reaches dk, dv */
            if (h % group != group - 1) continue;
#endif
            for (int64_t i = 0; i < s_q; ++i) {
                int64_t lo, hi;
                visible_range(i, s_k, s_q, causal, win_left, win_right, &lo, &hi);
                if (hi < lo) continue;            /* no visible key: out is 0, no gradient */
                const double *qi = q + ((bi * s_q + i) * h_q + h) * d_qk;
                const double *doi = dout + ((bi * s_q + i) * h_q + h) * d_v;
                double *dqi = dq + ((bi * s_q + i) * h_q + h) * d_qk;
                /* P_i: exact softmax over the visible keys */
                double m = -INFINITY;
                for (int64_t j = lo; j <= hi; ++j) {
                    const double *kj = k + ((bi * s_k + j) * h_kv + hk) * d_qk;
                    double dot = 0.0;
                    for (int t = 0; t < d_qk; ++t) dot += qi[t] * kj[t];
                    P[j - lo] = scale * dot;
                    if (P[j - lo] > m) m = P[j - lo];
                }
                double l = 0.0;
                for (int64_t j = lo; j <= hi; ++j) {
                    P[j - lo] = exp(P[j - lo] - m);
                    l += P[j - lo];
                }
                for (int64_t j = lo; j <= hi; ++j) P[j - lo] /= l;
                /* dP_ij = dout_i . v_j and the Jacobian's row term */
                double rowterm = 0.0;
                for (int64_t j = lo; j <= hi; ++j) {
                    const double *vj = v + ((bi * s_k + j) * h_kv + hk) * d_v;
                    double dot = 0.0;
                    for (int t = 0; t < d_v; ++t) dot += doi[t] * vj[t];
                    dP[j - lo] = dot;
                    rowterm += P[j - lo] * dot;
                }
#if ORACLE_PLANT == 13           /* planted: the Jacobian's row term dropped */
                rowterm = 0.0;
#endif
                for (int64_t j = lo; j <= hi; ++j) {
                    const double *kj = k + ((bi * s_k + j) * h_kv + hk) * d_qk;
                    double *dkj = dk + ((bi * s_k + j) * h_kv + hk) * d_qk;
                    double *dvj = dv + ((bi * s_k + j) * h_kv + hk) * d_v;
                    double pij = P[j - lo];
                    double ds = pij * (dP[j - lo] - rowterm);
                    for (int t = 0; t < d_v; ++t) dvj[t] += pij * doi[t];
                    for (int t = 0; t < d_qk; ++t) dqi[t] += scale * ds * kj[t];
#if ORACLE_PLANT == 14           /* planted: scale missing from dk */
                    for (int t = 0; t < d_qk; ++t) dkj[t] += ds * qi[t];
#else
                    for (int t = 0; t < d_qk; ++t) dkj[t] += scale * ds * qi[t];
#endif
                }
            }
        }
    free(P);
    free(dP);
    return 0;
}
