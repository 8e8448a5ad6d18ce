/*
 * oracle.c -- plain, slow fp64 CPU reference for the DiT attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or
 * call this file; only the tests, the entry point's smoke check and the
 * bench's CPU-baseline leg do. It shares no code with the CUDA library.
 *
 * What it computes, and where it comes from (ReGenVC, arXiv 2607.28144, as
 * summarised on the blog.captcha.la page, "Methodology -- deep read" and
 * "Technical innovations"): the decoder's diffusion transformer runs *exact*
 * attention, and its sequence parallelism (Ulysses x Ring) preserves that
 * exactness by streaming KV blocks and combining partial results. There is no
 * equation on the pages, so each function below writes out the textbook
 * definition it implements, in fp64, in the order the definition states:
 *
 *   oracle_attention_f64   softmax(scale * Q K^T) V per (batch, head, query),
 *                          with the natural-log LSE of the scaled logits.
 *   oracle_attention_bwd_f64  the gradients dQ, dK, dV of that attention for an
 *                          upstream dO (chain rule through the softmax).
 *   oracle_attention_bwd_block_f64  the same chain rule for one block of the
 *                          keys, with the whole attention's out and LSE given
 *                          (the step Ring attention's backward repeats per
 *                          key shard).
 *   oracle_lse_merge_f64   the two-block combination of (O, LSE) that Ring
 *                          attention applies between KV blocks.
 *   oracle_rope3d_f64      3D rotary position embedding of the Wan2.1 DiT
 *                          that the decoder's architecture matches (page 2,
 *                          "Methodology -- deep read": the student matches
 *                          the Wan2.1-Fun-Control teacher). The pages do not
 *                          print its formula; the reading used is stated at
 *                          the function. Parity of the pairing convention is
 *                          unpinned by the pages.
 *
 * bf16 inputs are widened exactly to double; bf16 outputs are rounded to
 * nearest-even directly from the double (no intermediate fp32 rounding).
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC oracle.c -o liboracle.so -lm
 * (no -ffast-math: the sums run in the plain order written here).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- bf16 --- */

double oracle_bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to bf16, nearest with ties to even, on its bit pattern. */
uint16_t oracle_f64_to_bf16(double x)
{
    uint64_t b;
    memcpy(&b, &x, sizeof b);
    uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
    uint64_t mag = b & 0x7FFFFFFFFFFFFFFFull;
    if (mag > 0x7FF0000000000000ull) return (uint16_t)(sign | 0x7FC0u);  /* NaN */
    if (mag == 0x7FF0000000000000ull) return (uint16_t)(sign | 0x7F80u); /* inf */
    if (mag >= 0x3810000000000000ull) {           /* |x| >= 2^-126: normal bf16 */
        uint64_t keep = mag >> 45;                /* exponent (11) + 7 mantissa bits */
        uint64_t rem = mag & ((1ull << 45) - 1);
        uint64_t half = 1ull << 44;
        if (rem > half || (rem == half && (keep & 1))) keep++;
        uint64_t r = keep - ((uint64_t)(1023 - 127) << 7);
        if (r >= 0x7F80u) return (uint16_t)(sign | 0x7F80u);              /* overflow */
        return (uint16_t)(sign | r);
    }
    /* bf16 subnormal range: integer multiples of 2^-133, round the multiple. */
    double s = ldexp(fabs(x), 133);
    double fl = floor(s);
    double fr = s - fl;
    uint64_t n = (uint64_t)fl;
    if (fr > 0.5 || (fr == 0.5 && (n & 1))) n++;
    return (uint16_t)(sign | n);
}

void oracle_bf16_to_f64_array(const uint16_t *h, double *x, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) x[i] = oracle_bf16_to_f64(h[i]);
}

void oracle_f64_to_bf16_array(const double *x, uint16_t *h, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) h[i] = oracle_f64_to_bf16(x[i]);
}

/* ----------------------------------------------------------- attention --- */

/* An input array that is either fp64 or bf16 bit patterns (widened on access). */
typedef struct {
    const void *p;
    int bf16;
} src_t;

static inline double at(src_t s, int64_t i)
{
    return s.bf16 ? oracle_bf16_to_f64(((const uint16_t *)s.p)[i]) : ((const double *)s.p)[i];
}

/*
 * One query row of exact softmax attention, by definition:
 *   s_j   = scale * sum_d q_d k_jd            for j < Skv
 *   m     = max_j s_j
 *   p_j   = exp(s_j - m)
 *   l     = sum_j p_j
 *   out_d = (sum_j p_j v_jd) / l
 *   lse   = m + ln l                          (natural log, scaled-logit units)
 * Skv == 0 gives out = 0 and lse = -inf (the empty softmax).
 * The query row starts at element qo of q, the head's keys/values at ko.
 * `p` is caller scratch of Skv doubles.
 */
static void attention_row(src_t q, int64_t qo, src_t k, src_t v, int64_t ko,
                          int64_t Skv, int64_t D, double scale,
                          double *p, double *out, double *lse)
{
    for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
    if (Skv == 0) {
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int64_t j = 0; j < Skv; ++j) {
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += at(q, qo + d) * at(k, ko + j * D + d);
        p[j] = scale * dot;
        if (p[j] > m) m = p[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < Skv; ++j) {
        p[j] = exp(p[j] - m);
        l += p[j];
    }
    for (int64_t j = 0; j < Skv; ++j)
        for (int64_t d = 0; d < D; ++d) out[d] += p[j] * at(v, ko + j * D + d);
    for (int64_t d = 0; d < D; ++d) out[d] /= l;
    *lse = m + log(l);
}

/*
 * Attention over BH independent (batch, head) problems laid out [BH][S][D].
 * rows == NULL: every query row, out [BH*Sq][D], lse [BH*Sq].
 * rows != NULL: only the nrows global rows rows[r] = bh*Sq + i, out [nrows][D].
 */
static int attention_rows(src_t q, src_t k, src_t v, int64_t BH, int64_t Sq, int64_t Skv,
                          int64_t D, double scale, const int64_t *rows, int64_t nrows,
                          double *out, double *lse)
{
    int64_t n = rows ? nrows : BH * Sq;
    int failed = 0;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
        if (!p) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n; ++r) {
            if (!p) continue;
            int64_t g = rows ? rows[r] : r;
            int64_t bh = g / Sq;
            attention_row(q, g * D, k, v, bh * Skv * D, Skv, D, scale, p, out + r * D, lse + r);
        }
        free(p);
    }
    return failed ? -1 : 0;
}

void oracle_attention_f64(const double *q, const double *k, const double *v,
                          int64_t BH, int64_t Sq, int64_t Skv, int64_t D, double scale,
                          const int64_t *rows, int64_t nrows,
                          double *out, double *lse)
{
    src_t sq = {q, 0}, sk = {k, 0}, sv = {v, 0};
    attention_rows(sq, sk, sv, BH, Sq, Skv, D, scale, rows, nrows, out, lse);
}

/* Same, on bf16 inputs (each element widened exactly to double when read). */
int oracle_attention_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          int64_t BH, int64_t Sq, int64_t Skv, int64_t D, double scale,
                          const int64_t *rows, int64_t nrows,
                          double *out, double *lse)
{
    src_t sq = {q, 1}, sk = {k, 1}, sv = {v, 1};
    return attention_rows(sq, sk, sv, BH, Sq, Skv, D, scale, rows, nrows, out, lse);
}

/* ------------------------------------------------------------ backward --- */

/*
 * Gradients of exact attention for one (batch, head), by the chain rule
 * applied to the definition above (no page prints them; the distillation
 * step that trains the decoder needs them). With s_ij = scale <q_i, k_j>,
 * P = softmax_j(s), O = P V and an upstream gradient dO:
 *   dV_j   = sum_i P_ij dO_i
 *   dP_ij  = <dO_i, v_j>
 *   delta_i = sum_j P_ij dP_ij            (= <dO_i, O_i>)
 *   dS_ij  = P_ij (dP_ij - delta_i)        (softmax Jacobian)
 *   dQ_i   = scale sum_j dS_ij k_j
 *   dK_j   = scale sum_i dS_ij q_i
 * Everything in fp64 from q, k, v, dO; P is recomputed exactly per row.
 * Inputs [Sq][D] / [Skv][D] of one head; outputs dq [Sq][D], dk, dv [Skv][D].
 */
static void attention_bwd_head(src_t q, int64_t qo, src_t k, src_t v, int64_t ko, src_t dout, int64_t doo,
                               int64_t Sq, int64_t Skv, int64_t D, double scale,
                               double *P, double *dS, double *dq, double *dk, double *dv)
{
    for (int64_t i = 0; i < Sq; ++i) {
        double m = -INFINITY;
        for (int64_t j = 0; j < Skv; ++j) {
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d) dot += at(q, qo + i * D + d) * at(k, ko + j * D + d);
            P[i * Skv + j] = scale * dot;
            if (P[i * Skv + j] > m) m = P[i * Skv + j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < Skv; ++j) {
            P[i * Skv + j] = exp(P[i * Skv + j] - m);
            l += P[i * Skv + j];
        }
        for (int64_t j = 0; j < Skv; ++j) P[i * Skv + j] /= l;
        double delta = 0.0;
        for (int64_t j = 0; j < Skv; ++j) {
            double dp = 0.0;
            for (int64_t d = 0; d < D; ++d) dp += at(dout, doo + i * D + d) * at(v, ko + j * D + d);
            dS[i * Skv + j] = dp;
            delta += P[i * Skv + j] * dp;
        }
        for (int64_t j = 0; j < Skv; ++j) dS[i * Skv + j] = P[i * Skv + j] * (dS[i * Skv + j] - delta);
    }
    for (int64_t x = 0; x < Sq * D; ++x) dq[x] = 0.0;
    for (int64_t x = 0; x < Skv * D; ++x) { dk[x] = 0.0; dv[x] = 0.0; }
    for (int64_t i = 0; i < Sq; ++i)
        for (int64_t j = 0; j < Skv; ++j)
            for (int64_t d = 0; d < D; ++d) {
                dv[j * D + d] += P[i * Skv + j] * at(dout, doo + i * D + d);
                dq[i * D + d] += scale * dS[i * Skv + j] * at(k, ko + j * D + d);
                dk[j * D + d] += scale * dS[i * Skv + j] * at(q, qo + i * D + d);
            }
}

static int attention_bwd(src_t q, src_t k, src_t v, src_t dout, int64_t BH, int64_t Sq, int64_t Skv, int64_t D,
                         double scale, double *dq, double *dk, double *dv)
{
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh) {
        double *P = (double *)malloc(sizeof(double) * (size_t)(Sq * Skv > 0 ? Sq * Skv : 1));
        double *dS = (double *)malloc(sizeof(double) * (size_t)(Sq * Skv > 0 ? Sq * Skv : 1));
        if (!P || !dS) {
#pragma omp atomic write
            failed = 1;
        } else {
            attention_bwd_head(q, bh * Sq * D, k, v, bh * Skv * D, dout, bh * Sq * D, Sq, Skv, D, scale, P, dS,
                               dq + bh * Sq * D, dk + bh * Skv * D, dv + bh * Skv * D);
        }
        free(P);
        free(dS);
    }
    return failed ? -1 : 0;
}

int oracle_attention_bwd_f64(const double *q, const double *k, const double *v, const double *dout,
                             int64_t BH, int64_t Sq, int64_t Skv, int64_t D, double scale,
                             double *dq, double *dk, double *dv)
{
    src_t sq = {q, 0}, sk = {k, 0}, sv = {v, 0}, sd = {dout, 0};
    return attention_bwd(sq, sk, sv, sd, BH, Sq, Skv, D, scale, dq, dk, dv);
}

int oracle_attention_bwd_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                              int64_t BH, int64_t Sq, int64_t Skv, int64_t D, double scale,
                              double *dq, double *dk, double *dv)
{
    src_t sq = {q, 1}, sk = {k, 1}, sv = {v, 1}, sd = {dout, 1};
    return attention_bwd(sq, sk, sv, sd, BH, Sq, Skv, D, scale, dq, dk, dv);
}

/*
 * The gradients contributed by one block of keys when the softmax runs over
 * more keys than the block holds, and its statistics are given: out_i and
 * lse_i of the whole attention (as Ring attention's backward receives them,
 * the merged result of every key block). By the chain rule of the full
 * attention, restricted to the block's keys j:
 *   P_ij   = exp(scale <q_i, k_j> - lse_i)      (the block's slice of the softmax)
 *   dP_ij  = <dO_i, v_j>
 *   delta_i = <dO_i, out_i>                      (= sum over ALL keys of P dP)
 *   dS_ij  = P_ij (dP_ij - delta_i)
 *   dq_i  += scale sum_j dS_ij k_j               (this block's share of dq)
 *   dk_j   = scale sum_i dS_ij q_i,  dv_j = sum_i P_ij dO_i   (complete)
 * Inputs per head [Sq][D] / [Skv][D], lse [Sq]; outputs dq [Sq][D] (the
 * share), dk, dv [Skv][D].
 */
static void attention_bwd_block_head(src_t q, int64_t qo, src_t k, src_t v, int64_t ko, src_t out, src_t dout,
                                     const double *lse, int64_t Sq, int64_t Skv, int64_t D, double scale,
                                     double *dq, double *dk, double *dv)
{
    for (int64_t x = 0; x < Sq * D; ++x) dq[x] = 0.0;
    for (int64_t x = 0; x < Skv * D; ++x) { dk[x] = 0.0; dv[x] = 0.0; }
    for (int64_t i = 0; i < Sq; ++i) {
        double delta = 0.0;
        for (int64_t d = 0; d < D; ++d) delta += at(dout, qo + i * D + d) * at(out, qo + i * D + d);
        for (int64_t j = 0; j < Skv; ++j) {
            double s = 0.0, dp = 0.0;
            for (int64_t d = 0; d < D; ++d) {
                s += at(q, qo + i * D + d) * at(k, ko + j * D + d);
                dp += at(dout, qo + i * D + d) * at(v, ko + j * D + d);
            }
            const double p = exp(scale * s - lse[i]);
            const double ds = p * (dp - delta);
            for (int64_t d = 0; d < D; ++d) {
                dq[i * D + d] += scale * ds * at(k, ko + j * D + d);
                dk[j * D + d] += scale * ds * at(q, qo + i * D + d);
                dv[j * D + d] += p * at(dout, qo + i * D + d);
            }
        }
    }
}

static void attention_bwd_block(src_t q, src_t k, src_t v, src_t out, src_t dout, const double *lse, int64_t BH,
                                int64_t Sq, int64_t Skv, int64_t D, double scale, double *dq, double *dk,
                                double *dv)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh)
        attention_bwd_block_head(q, bh * Sq * D, k, v, bh * Skv * D, out, dout, lse + bh * Sq, Sq, Skv, D, scale,
                                 dq + bh * Sq * D, dk + bh * Skv * D, dv + bh * Skv * D);
}

void oracle_attention_bwd_block_f64(const double *q, const double *k, const double *v, const double *out,
                                    const double *lse, const double *dout, int64_t BH, int64_t Sq, int64_t Skv,
                                    int64_t D, double scale, double *dq, double *dk, double *dv)
{
    src_t sq = {q, 0}, sk = {k, 0}, sv = {v, 0}, so = {out, 0}, sd = {dout, 0};
    attention_bwd_block(sq, sk, sv, so, sd, lse, BH, Sq, Skv, D, scale, dq, dk, dv);
}

void oracle_attention_bwd_block_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *out,
                                     const double *lse, const uint16_t *dout, int64_t BH, int64_t Sq, int64_t Skv,
                                     int64_t D, double scale, double *dq, double *dk, double *dv)
{
    src_t sq = {q, 1}, sk = {k, 1}, sv = {v, 1}, so = {out, 1}, sd = {dout, 1};
    attention_bwd_block(sq, sk, sv, so, sd, lse, BH, Sq, Skv, D, scale, dq, dk, dv);
}

/*
 * The same gradients for chosen rows only, at sizes where the full Sq x Skv
 * matrices do not fit: dq for the query rows qrows[0..nqr), dk and dv for the
 * key rows krows[0..nkr), of every (b, h). dk_j and dv_j sum over every query
 * row, so each query row's max m_i, sum l_i and delta_i are computed first
 * (one pass over its logits), then P_ij = exp(s_ij - m_i) / l_i is recomputed
 * where it is needed. Outputs dq [BH][nqr][D], dk, dv [BH][nkr][D].
 */
static double dot_f64(const double *a, const double *b, int64_t D)
{
    double acc = 0.0;
    for (int64_t d = 0; d < D; ++d) acc += a[d] * b[d];
    return acc;
}

int oracle_attention_bwd_rows_bf16(const uint16_t *q16, const uint16_t *k16, const uint16_t *v16,
                                   const uint16_t *do16, int64_t BH, int64_t Sq, int64_t Skv, int64_t D,
                                   double scale, const int64_t *qrows, int64_t nqr, const int64_t *krows,
                                   int64_t nkr, double *dq, double *dk, double *dv)
{
    /* one head at a time, widened to fp64 (exact) */
    size_t nq = (size_t)(Sq * D > 0 ? Sq * D : 1), nk = (size_t)(Skv * D > 0 ? Skv * D : 1);
    size_t ns = (size_t)(Sq > 0 ? Sq : 1);
    double *q = (double *)malloc(sizeof(double) * nq), *g = (double *)malloc(sizeof(double) * nq);
    double *k = (double *)malloc(sizeof(double) * nk), *v = (double *)malloc(sizeof(double) * nk);
    double *m = (double *)malloc(sizeof(double) * ns), *l = (double *)malloc(sizeof(double) * ns);
    double *delta = (double *)malloc(sizeof(double) * ns);
    int rc = (q && g && k && v && m && l && delta) ? 0 : -1;
    for (int64_t bh = 0; rc == 0 && bh < BH; ++bh) {
        oracle_bf16_to_f64_array(q16 + bh * Sq * D, q, Sq * D);
        oracle_bf16_to_f64_array(do16 + bh * Sq * D, g, Sq * D);
        oracle_bf16_to_f64_array(k16 + bh * Skv * D, k, Skv * D);
        oracle_bf16_to_f64_array(v16 + bh * Skv * D, v, Skv * D);
        /* per query row: m_i, l_i, then delta_i = sum_j P_ij dP_ij */
#pragma omp parallel
        {
            double *srow = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
#pragma omp for schedule(dynamic, 16)
            for (int64_t i = 0; i < Sq; ++i) {
                if (!srow) continue;
                double mi = -INFINITY;
                for (int64_t j = 0; j < Skv; ++j) {
                    srow[j] = scale * dot_f64(q + i * D, k + j * D, D);
                    if (srow[j] > mi) mi = srow[j];
                }
                double li = 0.0, di = 0.0;
                for (int64_t j = 0; j < Skv; ++j) {
                    double e = exp(srow[j] - mi);
                    li += e;
                    di += e * dot_f64(g + i * D, v + j * D, D);
                }
                m[i] = mi;
                l[i] = li;
                delta[i] = di / li;
            }
            if (!srow) {
#pragma omp atomic write
                rc = -1;
            }
            free(srow);
        }
        /* dq_i = scale sum_j dS_ij k_j */
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t r = 0; r < nqr; ++r) {
            int64_t i = qrows[r];
            double *o = dq + (bh * nqr + r) * D;
            for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
            for (int64_t j = 0; j < Skv; ++j) {
                double p = exp(scale * dot_f64(q + i * D, k + j * D, D) - m[i]) / l[i];
                double ds = p * (dot_f64(g + i * D, v + j * D, D) - delta[i]);
                for (int64_t d = 0; d < D; ++d) o[d] += scale * ds * k[j * D + d];
            }
        }
        /* dv_j = sum_i P_ij dO_i,  dk_j = scale sum_i dS_ij q_i */
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t r = 0; r < nkr; ++r) {
            int64_t j = krows[r];
            double *ov = dv + (bh * nkr + r) * D, *ok = dk + (bh * nkr + r) * D;
            for (int64_t d = 0; d < D; ++d) { ov[d] = 0.0; ok[d] = 0.0; }
            for (int64_t i = 0; i < Sq; ++i) {
                double p = exp(scale * dot_f64(q + i * D, k + j * D, D) - m[i]) / l[i];
                double ds = p * (dot_f64(g + i * D, v + j * D, D) - delta[i]);
                for (int64_t d = 0; d < D; ++d) {
                    ov[d] += p * g[i * D + d];
                    ok[d] += scale * ds * q[i * D + d];
                }
            }
        }
    }
    free(q); free(g); free(k); free(v); free(m); free(l); free(delta);
    return rc;
}

/* ------------------------------------------------------------ LSE merge --- */

/*
 * Combine two partial attentions of the same queries over disjoint key
 * blocks a and b (each normalised by its own softmax, with its own LSE):
 *   m   = max(lse_a, lse_b)
 *   w_a = exp(lse_a - m),  w_b = exp(lse_b - m)
 *   out = (w_a o_a + w_b o_b) / (w_a + w_b)
 *   lse = m + ln(w_a + w_b)
 * Both LSEs -inf (two empty blocks): out = 0, lse = -inf.
 */
void oracle_lse_merge_f64(const double *oa, const double *lsea,
                          const double *ob, const double *lseb,
                          int64_t rows, int64_t D, double *out, double *lse)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double m = lsea[r] > lseb[r] ? lsea[r] : lseb[r];
        if (m == -INFINITY) {
            for (int64_t d = 0; d < D; ++d) out[r * D + d] = 0.0;
            lse[r] = -INFINITY;
            continue;
        }
        double wa = exp(lsea[r] - m);
        double wb = exp(lseb[r] - m);
        for (int64_t d = 0; d < D; ++d)
            out[r * D + d] = (wa * oa[r * D + d] + wb * ob[r * D + d]) / (wa + wb);
        lse[r] = m + log(wa + wb);
    }
}

/* --------------------------------------------------------- projections --- */

static void rope_row(double *row, int64_t n, int64_t Hh, int64_t Ww, int64_t D, double theta, int transpose);

/*
 * The projections around the attention in a DiT block (the decoder's DiT
 * matches the Wan2.1 architecture: blog page, "Methodology -- deep read"):
 *   y = x W^T + b,  x one token's row of C model features, W [N][C] (the
 *   usual linear-layer layout), b [N] or none.
 * QKV (N = 3 H D): y = [q | k | v], head h of q at columns h D .. h D + D - 1.
 * q and k then get, per head, RMSNorm over its D values with a weight g
 * (x / sqrt(mean x^2 + eps) * g; g = 1 when none) and the 3D RoPE of the
 * token's latent grid position (rope_row above); v is left as is. Reading:
 * the norm is per head, as in the input preparation of every workload.
 * Tokens: x [B][S][C] bf16, S = T Hh Ww; rows[] are global token ids b S + s.
 * Outputs q, k, v [nrows][H][D] in fp64.
 */
int oracle_qkv_proj_rows(const uint16_t *x, const uint16_t *w, const double *bias, const double *gq,
                         const double *gk, int64_t B, int64_t S, int64_t C, int64_t H, int64_t D, int64_t T,
                         int64_t Hh, int64_t Ww, double theta, double eps, const int64_t *rows, int64_t nrows,
                         double *q, double *k, double *v)
{
    if (T * Hh * Ww != S || D < 6 || (D % 2) != 0) return -1;
    int64_t N = 3 * H * D;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t tok = rows[r];
        if (tok < 0 || tok >= B * S) {
#pragma omp atomic write
            failed = 1;
            continue;
        }
        double *y = (double *)malloc(sizeof(double) * (size_t)N);
        if (!y) {
#pragma omp atomic write
            failed = 1;
            continue;
        }
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t c = 0; c < C; ++c)
                acc += oracle_bf16_to_f64(x[tok * C + c]) * oracle_bf16_to_f64(w[n * C + c]);
            y[n] = acc + (bias ? bias[n] : 0.0);
        }
        for (int64_t which = 0; which < 3; ++which) {
            double *dst = which == 0 ? q : which == 1 ? k : v;
            const double *g = which == 0 ? gq : gk;
            for (int64_t h = 0; h < H; ++h) {
                double *src = y + which * H * D + h * D;
                double *o = dst + (r * H + h) * D;
                if (which < 2) {
                    double ms = 0.0;
                    for (int64_t d = 0; d < D; ++d) ms += src[d] * src[d];
                    ms /= (double)D;
                    double inv = 1.0 / sqrt(ms + eps);
                    for (int64_t d = 0; d < D; ++d) o[d] = src[d] * inv * (g ? g[h * D + d] : 1.0);
                    rope_row(o, tok % S, Hh, Ww, D, theta, 0);
                } else {
                    for (int64_t d = 0; d < D; ++d) o[d] = src[d];
                }
            }
        }
        free(y);
    }
    return failed ? -1 : 0;
}

/*
 * Output projection: y = o W^T + b for token rows o of H D values, the
 * attention output of that token with its heads concatenated:
 * o[h D + d] = O[b][h][s][d] for O [B][H][S][D]. W [N][H D], b [N] or none.
 * Output y [nrows][N] in fp64.
 */
int oracle_out_proj_rows(const uint16_t *O, const uint16_t *w, const double *bias, int64_t B, int64_t S,
                         int64_t H, int64_t D, int64_t N, const int64_t *rows, int64_t nrows, double *y)
{
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t tok = rows[r];
        if (tok < 0 || tok >= B * S) {
#pragma omp atomic write
            failed = 1;
            continue;
        }
        int64_t b = tok / S, s = tok % S;
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t h = 0; h < H; ++h)
                for (int64_t d = 0; d < D; ++d)
                    acc += oracle_bf16_to_f64(O[((b * H + h) * S + s) * D + d]) *
                           oracle_bf16_to_f64(w[n * H * D + h * D + d]);
            y[r * N + n] = acc + (bias ? bias[n] : 0.0);
        }
    }
    return failed ? -1 : 0;
}

/* ------------------------------------------------------ FP8 (e4m3) --- */

/*
 * OCP FP8 E4M3 ("fn": no infinities): 1 sign bit, 4 exponent bits with bias
 * 7, 3 mantissa bits. Exponent field 1..15 encodes 2^(e-7) (1 + m/8), except
 * field 15 with m = 7 which is NaN, so the largest finite value is 448;
 * field 0 encodes subnormals 2^-6 (m/8). Rounding here: to nearest, ties to
 * even, then saturation of finite values to +-448 (the "satfinite" rounding
 * of the FP8 variant). The FP8 attention variant is not on the pages; its
 * quantisation is defined here (see oracle_quantize_e4m3).
 */
double oracle_e4m3_to_f64(uint8_t c)
{
    int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);               /* 2^-6 * m/8 */
    else
        v = ldexp(8.0 + m, e - 7 - 3);          /* 2^(e-7) * (8+m)/8 */
    return sgn ? -v : v;
}

uint8_t oracle_f64_to_e4m3(double x)
{
    if (x != x) return 0x7F;
    uint8_t sgn = (x < 0) ? 0x80 : 0;
    double a = fabs(x);
    if (a >= 448.0) return sgn | 0x7E;           /* saturate */
    int e2;
    frexp(a, &e2);                               /* a = f 2^e2, f in [0.5, 1) */
    int e = e2 - 1;                              /* a in [2^e, 2^(e+1)) */
    if (e < -6) e = -6;                          /* subnormal spacing 2^-9 */
    double ulp = ldexp(1.0, e - 3);
    double n = nearbyint(a / ulp);               /* exact quotient, ties to even */
    double r = n * ulp;
    if (r >= 448.0) return sgn | 0x7E;
    if (r == 0.0) return sgn;
    int re2;
    frexp(r, &re2);
    int re = re2 - 1;
    if (re < -6) return sgn | (uint8_t)(r / ldexp(1.0, -9));     /* subnormal: m = r / 2^-9 */
    int mant = (int)(r / ldexp(1.0, re - 3)) - 8;                 /* 0..7 */
    return sgn | (uint8_t)(((re + 7) << 3) | mant);
}

void oracle_f64_to_e4m3_array(const double *x, uint8_t *c, int64_t n)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) c[i] = oracle_f64_to_e4m3(x[i]);
}

/*
 * Blockwise quantisation of x [BH][S][D] (bf16) for the FP8 attention: each
 * block of `block_rows` consecutive rows of one (b, h) -- the last one
 * ragged -- gets amax = max |x| over the block, scale = amax / 448 and
 * inv = 448 / amax, both rounded to fp32; every element is multiplied by inv
 * in fp32 and rounded to e4m3 as above; x is represented by code * scale. An
 * all-zero block gets scale = inv = 1. Outputs codes [BH][S][D] and scales
 * [BH][ceil(S / block_rows)].
 */
int oracle_quantize_e4m3(const uint16_t *x, int64_t BH, int64_t S, int64_t D, int64_t block_rows,
                         uint8_t *codes, float *scales)
{
    if (block_rows <= 0) return -1;
    int64_t nb = (S + block_rows - 1) / block_rows;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < BH * nb; ++t) {
        int64_t bh = t / nb, b = t % nb;
        int64_t r0 = b * block_rows, r1 = r0 + block_rows < S ? r0 + block_rows : S;
        const uint16_t *xb = x + (bh * S + r0) * D;
        uint8_t *cb = codes + (bh * S + r0) * D;
        int64_t n = (r1 - r0) * D;
        float amax = 0.0f;
        for (int64_t i = 0; i < n; ++i) {
            float a = fabsf((float)oracle_bf16_to_f64(xb[i]));
            if (a > amax) amax = a;
        }
        volatile float scale = 1.0f, inv = 1.0f;   /* volatile: each op rounded to fp32 */
        if (amax > 0.0f) {
            scale = amax / 448.0f;
            inv = 448.0f / amax;
        }
        scales[t] = scale;
        for (int64_t i = 0; i < n; ++i) {
            volatile float y = (float)oracle_bf16_to_f64(xb[i]) * inv;
            cb[i] = oracle_f64_to_e4m3((double)y);
        }
    }
    return 0;
}

/* ---------------------------------------------------------------- RoPE --- */

/*
 * 3D rotary position embedding, in place on x [BH][S][D], S = T*Hh*Ww.
 *
 * Reading (the pages give no formula; this is the Wan2.1 DiT's 3D RoPE that
 * the decoder's architecture matches):
 *  - token n sits at latent grid position (t, y, x) with n = (t*Hh + y)*Ww + x;
 *  - the head dimension splits into three axis blocks, in the order t, h, w:
 *    d_h = d_w = 2*floor(D/6) and d_t = D - 2*d_h (44/42/42 at D = 128);
 *  - inside an axis block of width d_a, the pair (2j, 2j+1) is rotated by
 *    angle pos_a * theta^(-2j/d_a), j = 0 .. d_a/2 - 1:
 *        x'_{2j}   = x_{2j} cos(angle) - x_{2j+1} sin(angle)
 *        x'_{2j+1} = x_{2j} sin(angle) + x_{2j+1} cos(angle)
 *    (the product of the pair, read as a complex number, with e^{i angle}).
 */
/* Rotate one row of D values of token n in place (R, or R^T with transpose). */
static void rope_row(double *row, int64_t n, int64_t Hh, int64_t Ww, int64_t D, double theta, int transpose)
{
    int64_t dh = 2 * (D / 6);
    int64_t dt = D - 2 * dh;
    int64_t base[3] = {0, dt, dt + dh};
    int64_t width[3] = {dt, dh, dh};
    int64_t pos[3];
    pos[0] = n / (Hh * Ww);
    pos[1] = (n / Ww) % Hh;
    pos[2] = n % Ww;
    for (int a = 0; a < 3; ++a) {
        for (int64_t j = 0; j < width[a] / 2; ++j) {
            double angle = (double)pos[a] * pow(theta, -2.0 * (double)j / (double)width[a]);
            double c = cos(angle), s = sin(angle);
            double x0 = row[base[a] + 2 * j];
            double x1 = row[base[a] + 2 * j + 1];
            if (!transpose) {
                row[base[a] + 2 * j] = x0 * c - x1 * s;
                row[base[a] + 2 * j + 1] = x0 * s + x1 * c;
            } else {
                /* R^T: the same rotation matrix, transposed */
                row[base[a] + 2 * j] = c * x0 + s * x1;
                row[base[a] + 2 * j + 1] = c * x1 - s * x0;
            }
        }
    }
}

static int rope3d_apply(double *x, int64_t BH, int64_t T, int64_t Hh, int64_t Ww,
                        int64_t D, double theta, int transpose)
{
    if (D < 6 || (D % 2) != 0) return -1;
    int64_t S = T * Hh * Ww;
#pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < BH * S; ++g) rope_row(x + g * D, g % S, Hh, Ww, D, theta, transpose);
    return 0;
}

int oracle_rope3d_f64(double *x, int64_t BH, int64_t T, int64_t Hh, int64_t Ww,
                      int64_t D, double theta)
{
    return rope3d_apply(x, BH, T, Hh, Ww, D, theta, 0);
}

/*
 * Gradient of the 3D RoPE: x' = R x with R orthogonal and block-diagonal
 * (one 2x2 rotation per pair), so dL/dx = R^T dL/dx' -- every pair turned
 * back by its angle. In place on g [BH][S][D].
 */
int oracle_rope3d_bwd_f64(double *g, int64_t BH, int64_t T, int64_t Hh, int64_t Ww,
                          int64_t D, double theta)
{
    return rope3d_apply(g, BH, T, Hh, Ww, D, theta, 1);
}

static int rope3d_bf16(uint16_t *x, int64_t BH, int64_t T, int64_t Hh, int64_t Ww,
                       int64_t D, double theta, int transpose)
{
    int64_t n = BH * T * Hh * Ww * D;
    double *xd = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (!xd) return -2;
    oracle_bf16_to_f64_array(x, xd, n);
    int rc = rope3d_apply(xd, BH, T, Hh, Ww, D, theta, transpose);
    if (rc == 0) oracle_f64_to_bf16_array(xd, x, n);
    free(xd);
    return rc;
}

/* In place on bf16: widen, rotate in fp64, round to nearest-even bf16. */
int oracle_rope3d_bf16(uint16_t *x, int64_t BH, int64_t T, int64_t Hh, int64_t Ww,
                       int64_t D, double theta)
{
    return rope3d_bf16(x, BH, T, Hh, Ww, D, theta, 0);
}

int oracle_rope3d_bwd_bf16(uint16_t *g, int64_t BH, int64_t T, int64_t Hh, int64_t Ww,
                           int64_t D, double theta)
{
    return rope3d_bf16(g, BH, T, Hh, Ww, D, theta, 1);
}

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
