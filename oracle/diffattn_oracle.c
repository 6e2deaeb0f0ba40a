/*
 * diffattn_oracle.c -- plain float64 CPU oracle for the differential-attention
 * forward pass (prefill, grouped prefill, single-query decode).
 *
 * TEST INFRASTRUCTURE ONLY.  This file exists so that tests, the package's
 * smoke check and the benchmark's CPU-baseline leg have an obviously correct
 * result to compare against.  It shares no code, header, table or helper with
 * the CUDA path, and the CUDA path never calls it.
 *
 * What it computes (one output row = one batch b, one signal head h, one query
 * position i), step by step, with no tiling, no online softmax and no fusion:
 *
 *   1. Key range J.  Causal prefill: keys 0..i (the diagonal is included, so
 *      no row is empty).  Non-causal prefill: keys 0..N-1.  Decode: the query
 *      sits at position kv_len-1 and sees keys 0..kv_len-1.  A sliding window
 *      of W > 0 keys (causal only; Motif 3 summary, sections 2.1 and
 *      "Practical Implications": sliding-window layers with 128-token
 *      windows) keeps the W most recent of those keys: i-W < j <= i.
 *      (Motif 2.6B is a decoder-only Transformer: edgentiq Motif-2.6B blog;
 *      Motif 3 summary, section 2.1 "full causal-attention layer".)
 *   2. For each map t in {1,2}: z_j = s * <q_t, k_t[j]>, m = max_j z_j,
 *      w_j = exp(z_j - m), l = sum_j w_j, A_t[c] = sum_j w_j v[j][c] / l.
 *      This is softmax(Q_t K_t^T) V written out row by row
 *      (Motif 2.6B explainer, section "Differential attention", the formula
 *      attn = [softmax(Q1 K1^T) - lambda softmax(Q2 K2^T)] V; both maps use
 *      the same V).  The scale s is a parameter (the pages print none).
 *   3. D[c] = A_1[c] - lambda_h * A_2[c]   (same formula, the subtraction).
 *      Grouped form: the noise map of signal head h is that of noise head
 *      n(h) = h / g, i.e. Repeat_g interleaves the noise heads (Motif 3
 *      summary, section 2.2, eq. "grouped differential output"
 *      D_t = H_S,t - lambda_t (.) Repeat_g(H_N,t)).  The V head of signal head
 *      h is v(h) = h / (H / H_V).
 *   4. Norm after the subtraction (Motif 2.6B explainer, figure 1 caption and
 *      the paragraph on the GroupNorm that "keeps the ... scores stable"),
 *      read as one RMS group per head and token over its dv channels:
 *      Y[c] = D[c] / sqrt(mean_c D[c]^2 + eps) * gain[h][c].
 *      With apply_norm == 0 the pre-norm D is returned.
 *   0. Rotary position embedding (optional; Motif 2.6B explainer, "The
 *      block": RoPE with theta = 500,000).  With rope_theta > 0 every 64-wide
 *      row of Q1, K1, Q2, K2 at token position n is rotated before step 2,
 *      pair by pair: for c < d/2, with angle a = n * theta^(-2c/d),
 *        x'[2c]   = x[2c] cos a - x[2c+1] sin a
 *        x'[2c+1] = x[2c] sin a + x[2c+1] cos a.
 *      (The pages give the base only; interleaved pairs within each map's
 *      own 64 dimensions are this oracle's reading.)
 *   5. Token-dependent lambda and output gate (Motif 3 summary, section 2.2):
 *      lambda_t = sigma(x_t W^lambda) per signal head and token, and
 *      GDLA(x_t) = vec(sigma(G_t) (.) D_t) W^O.  The projections are outside
 *      this path, so their outputs -- the logits x_t W^lambda [B][N][H] and
 *      G_t [B][N][H][dv] -- are the inputs; sigma is the logistic function.
 *      With lambda logits given they replace lambda[h] in step 3.  With gate
 *      logits given, step 4's result (normalised or not) is multiplied
 *      element-wise by sigma(G_t), i.e. the gate is the last operation before
 *      W^O.
 *
 * Every input is float64 (the exact bf16 / fp32 values widened by the caller)
 * and every intermediate is float64.  Built with -ffp-contract=off so that the
 * compiler does not fuse multiplies and adds behind the reader's back.
 *
 * Layouts (all contiguous, row-major, element counts not bytes):
 *   prefill: q1,k1 [B][N][H][d]; q2,k2 [B][N][H_N][d]; v [B][N][H_V][dv];
 *            out [B][N][H][dv]; lambda [H]; gain [H][dv] or NULL (= 1);
 *            lambda_logit [B][N][H] or NULL; gate_logit [B][N][H][dv] or NULL.
 *   decode:  q1,q2 [B][H][d]; k1,k2 [B][H][L][d]; v [B][H][L][dv];
 *            kv_len [B] or NULL (= L); out [B][H][dv];
 *            lambda_logit [B][H] or NULL; gate_logit [B][H][dv] or NULL.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Softmax weights of one query row against nkeys keys (step 2 above, before
 * the product with V).  w receives exp(z_j - m); the return value is l.       */
static double softmax_weights(const double *q, const double *k, int64_t k_row_stride,
                              int64_t nkeys, int64_t d, double scale, double *w)
{
    double m = -INFINITY;
    for (int64_t j = 0; j < nkeys; ++j) {
        const double *kj = k + j * k_row_stride;
        double dot = 0.0;
        for (int64_t c = 0; c < d; ++c) dot += q[c] * kj[c];
        w[j] = scale * dot;
        if (w[j] > m) m = w[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < nkeys; ++j) {
        w[j] = exp(w[j] - m);
        l += w[j];
    }
    return l;
}

/* Step 0: rotate every d-wide row of x [B][N][heads][d] by its token
 * position; returns a new array (caller frees) or NULL on allocation failure. */
static double *rope_copy(const double *x, int64_t B, int64_t N, int64_t heads, int64_t d,
                         double theta)
{
    double *y = (double *)malloc(sizeof(double) * (size_t)(B * N * heads * d > 0 ? B * N * heads * d : 1));
    if (!y) return NULL;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t h = 0; h < heads; ++h) {
                const double *xr = x + ((b * N + n) * heads + h) * d;
                double *yr = y + ((b * N + n) * heads + h) * d;
                for (int64_t c = 0; c < d / 2; ++c) {
                    const double a = (double)n * pow(theta, -2.0 * (double)c / (double)d);
                    const double cs = cos(a), sn = sin(a);
                    yr[2 * c] = xr[2 * c] * cs - xr[2 * c + 1] * sn;
                    yr[2 * c + 1] = xr[2 * c] * sn + xr[2 * c + 1] * cs;
                }
            }
    return y;
}

/* The logistic function sigma(x) = 1 / (1 + e^-x) of step 5.                 */
static double logistic(double x)
{
    return 1.0 / (1.0 + exp(-x));
}

/* One output row: steps 2-5 above.  a1, a2 are scratch of length dv; w1, w2 of
 * length nkeys.                                                               */
static void diff_row(const double *q1, const double *k1, int64_t k1_rs,
                     const double *q2, const double *k2, int64_t k2_rs,
                     const double *v, int64_t v_rs,
                     int64_t nkeys, int64_t d, int64_t dv, double scale,
                     double lambda, const double *gain, double eps, int apply_norm,
                     const double *gate_logit,
                     double *w1, double *w2, double *a1, double *a2, double *out)
{
    double l1 = softmax_weights(q1, k1, k1_rs, nkeys, d, scale, w1);
    double l2 = softmax_weights(q2, k2, k2_rs, nkeys, d, scale, w2);
    for (int64_t c = 0; c < dv; ++c) { a1[c] = 0.0; a2[c] = 0.0; }
    for (int64_t j = 0; j < nkeys; ++j) {
        const double *vj = v + j * v_rs;
        for (int64_t c = 0; c < dv; ++c) {
            a1[c] += w1[j] * vj[c];
            a2[c] += w2[j] * vj[c];
        }
    }
    for (int64_t c = 0; c < dv; ++c) out[c] = a1[c] / l1 - lambda * (a2[c] / l2);
    if (apply_norm) {
        double ss = 0.0;
        for (int64_t c = 0; c < dv; ++c) ss += out[c] * out[c];
        double r = 1.0 / sqrt(ss / (double)dv + eps);
        for (int64_t c = 0; c < dv; ++c) out[c] = out[c] * r * (gain ? gain[c] : 1.0);
    }
    if (gate_logit)
        for (int64_t c = 0; c < dv; ++c) out[c] = logistic(gate_logit[c]) * out[c];
}

/* Number of OpenMP threads the oracle will use (reported beside its timings). */
int diffattn_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Softmax weights w_j / l of one query row (one map), for the "each row sums
 * to 1" check.  q [d]; k [nkeys][d]; out [nkeys].                             */
void diffattn_oracle_softmax_row(const double *q, const double *k, int64_t nkeys, int64_t d,
                                 double scale, double *out)
{
    double l = softmax_weights(q, k, d, nkeys, d, scale, out);
    for (int64_t j = 0; j < nkeys; ++j) out[j] /= l;
}

/* Prefill (and grouped prefill).  rows: NULL for every (b, i, h), otherwise
 * nrows triples (b, i, h) whose outputs are written; other rows of out are not
 * touched.  Returns 0, or -1 on an invalid argument.                          */
int diffattn_oracle_prefill(const double *q1, const double *q2, const double *k1,
                            const double *k2, const double *v,
                            int64_t B, int64_t N, int64_t H, int64_t H_N, int64_t H_V,
                            int64_t d, int64_t dv,
                            const double *lambda, const double *gain,
                            const double *lambda_logit, const double *gate_logit,
                            double scale, double eps, int causal, int apply_norm, int64_t window,
                            double rope_theta, const int64_t *rows, int64_t nrows, double *out)
{
    if (B < 0 || N < 0 || H <= 0 || H_N <= 0 || H_V <= 0 || d <= 0 || dv <= 0) return -1;
    if (window < 0 || (window > 0 && !causal) || rope_theta < 0 || (rope_theta > 0 && d % 2)) return -1;
    if (H % H_N != 0 || H % H_V != 0) return -1;  /* before anything is allocated */
    double *rq1 = NULL, *rq2 = NULL, *rk1 = NULL, *rk2 = NULL;
    if (rope_theta > 0) {  /* step 0 */
        rq1 = rope_copy(q1, B, N, H, d, rope_theta);
        rk1 = rope_copy(k1, B, N, H, d, rope_theta);
        rq2 = rope_copy(q2, B, N, H_N, d, rope_theta);
        rk2 = rope_copy(k2, B, N, H_N, d, rope_theta);
        if (!rq1 || !rk1 || !rq2 || !rk2) {
            free(rq1); free(rk1); free(rq2); free(rk2);
            return -1;
        }
        q1 = rq1; k1 = rk1; q2 = rq2; k2 = rk2;
    }
    const int64_t g = H / H_N;       /* signal heads per noise head */
    const int64_t gv = H / H_V;      /* signal heads per V head */
    const int64_t total = rows ? nrows : B * N * H;
    int bad = 0;
#pragma omp parallel
    {
        double *w1 = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        double *w2 = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        double *a1 = (double *)malloc(sizeof(double) * (size_t)dv);
        double *a2 = (double *)malloc(sizeof(double) * (size_t)dv);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < total; ++r) {
            int64_t b, i, h;
            if (rows) { b = rows[3 * r]; i = rows[3 * r + 1]; h = rows[3 * r + 2]; }
            else { b = r / (N * H); i = (r / H) % N; h = r % H; }
            if (b < 0 || b >= B || i < 0 || i >= N || h < 0 || h >= H) { bad = 1; continue; }
            const int64_t n = h / g, hv = h / gv;
            const int64_t nkeys = causal ? i + 1 : N;
            /* first visible key: i - W + 1 under a window of W keys */
            const int64_t j0 = (window > 0 && i + 1 > window) ? i + 1 - window : 0;
            const double *q1r = q1 + ((b * N + i) * H + h) * d;
            const double *q2r = q2 + ((b * N + i) * H_N + n) * d;
            const double *k1b = k1 + ((b * N + j0) * H + h) * d;
            const double *k2b = k2 + ((b * N + j0) * H_N + n) * d;
            const double *vb = v + ((b * N + j0) * H_V + hv) * dv;
            const int64_t row = (b * N + i) * H + h;   /* index of (b, i, h) */
            const double lam = lambda_logit ? logistic(lambda_logit[row]) : lambda[h];
            const double *gate = gate_logit ? gate_logit + row * dv : NULL;
            diff_row(q1r, k1b, H * d, q2r, k2b, H_N * d, vb, H_V * dv, nkeys - j0, d, dv, scale,
                     lam, gain ? gain + h * dv : NULL, eps, apply_norm, gate, w1, w2, a1, a2,
                     out + row * dv);
        }
        free(w1); free(w2); free(a1); free(a2);
    }
    free(rq1); free(rk1); free(rq2); free(rk2);
    return bad ? -1 : 0;
}

/* Single-query decode.  kv_len: NULL (every sequence has L keys) or [B] with
 * 1 <= kv_len[b] <= L.  Returns 0, or -1 on an invalid argument.              */
int diffattn_oracle_decode(const double *q1, const double *q2, const double *k1,
                           const double *k2, const double *v,
                           int64_t B, int64_t H, int64_t L, int64_t d, int64_t dv,
                           const int64_t *kv_len, const double *lambda, const double *gain,
                           const double *lambda_logit, const double *gate_logit,
                           double scale, double eps, int apply_norm, int64_t window, double *out)
{
    if (B < 0 || H <= 0 || L <= 0 || d <= 0 || dv <= 0 || window < 0) return -1;
    for (int64_t b = 0; b < B; ++b)
        if (kv_len && (kv_len[b] < 1 || kv_len[b] > L)) return -1;
#pragma omp parallel
    {
        double *w1 = (double *)malloc(sizeof(double) * (size_t)L);
        double *w2 = (double *)malloc(sizeof(double) * (size_t)L);
        double *a1 = (double *)malloc(sizeof(double) * (size_t)dv);
        double *a2 = (double *)malloc(sizeof(double) * (size_t)dv);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < B * H; ++r) {
            const int64_t b = r / H, h = r % H;
            const int64_t nkeys = kv_len ? kv_len[b] : L;
            /* under a window of W keys: the W most recent cached keys */
            const int64_t j0 = (window > 0 && nkeys > window) ? nkeys - window : 0;
            const double lam = lambda_logit ? logistic(lambda_logit[r]) : lambda[h];
            diff_row(q1 + r * d, k1 + (r * L + j0) * d, d, q2 + r * d, k2 + (r * L + j0) * d, d,
                     v + (r * L + j0) * dv, dv, nkeys - j0, d, dv, scale, lam,
                     gain ? gain + h * dv : NULL, eps, apply_norm,
                     gate_logit ? gate_logit + r * dv : NULL, w1, w2, a1, a2, out + r * dv);
        }
        free(w1); free(w2); free(a1); free(a2);
    }
    return 0;
}
