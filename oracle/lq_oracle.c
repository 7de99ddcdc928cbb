/*
 * lq_oracle.c -- CPU oracle for int8 per-window recurrent-state decode of
 * delta-rule linear attention (LeapQuant).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference legs load this library.  It shares no
 * code, header, table or constant with the CUDA library, and the CUDA library
 * never calls it.
 *
 * Everything is computed in FP64, one head at a time, in plain loops.  A value
 * that the method stores in a narrower format (int8 codes, FP32 row scales,
 * FP32 smoothing factors, FP32 compensators, FP32 buffered records) is rounded
 * to that format when it is stored and read back from the stored value.  The
 * `exact` switch of lqo_window keeps records in FP64 (used by the exact-
 * arithmetic pins only).
 *
 * Sources (page title, then the part of the page):
 *  [LQ] "LeapQuant: Efficient Linear Attention with Accurate Recurrent State
 *       Quantization" -- Abstract; Figure 2 (per-token versus per-window
 *       quantization); Figure 4 (per-window state reconstruction with
 *       Compensator Tokens); Appendix, Table 4 (instances of equation 1 and the
 *       size of one buffered update (d_i, k~_i, u_i)).
 *  [KP] "LeapQuant: Near-Lossless 8-Bit Recurrent State Quantization for Linear
 *       Attention LLMs" -- Key points (Per-Window Quantization, Compensator
 *       Tokens, Residual Smoothing).
 *  [CN] "LeapQuant trims the memory burden of linear-attention models" --
 *       "Quantize less often, protect the outliers".
 *
 * Equation 1 is not printed on the pages; only its instances are (Table 4).
 * The form used here is the one every Table 4 row is an instance of:
 *      S_t = S_{t-1} D_t + (v_t - S_{t-1} b_t) k~_t^T ,   o_t = S_t q_t ,
 * with S in R^{d_v x d_k} (row i = value channel, column j = key channel) and
 * D_t = Diag(d_t) diagonal.  With u_t = v_t - S_{t-1} b_t the update is
 * S_t = S_{t-1} D_t + u_t k~_t^T, so the buffered record (d_t, k~_t, u_t) of
 * Table 4 is all a window needs.
 *
 * Pinning (what ties each function to something other than itself):
 *  lqo_eq1_steps  -- Table 4 rows against each model's published update
 *                    (DeltaNet, Gated DeltaNet, Mamba2, GLA, RetNet, linear
 *                    attention), brute-force exact rational products.
 *  lqo_window     -- exact rational unrolled products on tiny heads; explicit
 *                    stepping of the dequantized boundary state; the
 *                    quantization-off chain equals the exact recurrence.
 *  lqo_rebuild    -- same pins as lqo_window (the rebuilt S_n is compared).
 *  lqo_quantize   -- closed-form error bound, exact compensator rows, the
 *                    top-r norm property, column-max identity of the
 *                    smoothing, hand cases (zero, constant, spike rows).
 *                    The compensator-selection and smoothing RULES themselves
 *                    are not fixed by the pages (parity unpinned by the pages:
 *                    our definition, written below); the implementation is
 *                    pinned to that definition by the properties above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Round an FP64 value to the nearest FP32 value (ties to even). */
static double f32(double x) { return (double)(float)x; }

/* Round a finite value to the nearest value with 8 significant bits (the
 * BF16 significand), ties to even: x = m 2^e with 0.5 <= |m| < 1, so
 * rint(m 2^8) 2^(e-8) keeps 8 bits (rint rounds half to even).  Values in
 * the FP32 normal range only (BF16 shares FP32's exponent range). */
static double bf16(double x)
{
    int e;
    double m = frexp(x, &e);
    return ldexp(rint(ldexp(m, 8)), e - 8);
}

/* ------------------------------------------------------------------------ */
/* Equation 1, explicit stepping ([LQ] Table 4).                             */
/* ------------------------------------------------------------------------ */

/* Runs n steps of equation 1 on each of nh heads, in FP64.
 *   S  [nh][dv][dk]  in/out state
 *   d  [nh][n][dk]   diagonal of D_t (a scalar gate is passed repeated)
 *   kt [nh][n][dk]   k~_t
 *   b  [nh][n][dk]   b_t
 *   v  [nh][n][dv]
 *   q  [nh][n][dk]   may be NULL (no outputs)
 *   o  [nh][n][dv]   o_t = S_t q_t, may be NULL                          */
void lqo_eq1_steps(int nh, int dv, int dk, int n, double *S, const double *d,
                   const double *kt, const double *b, const double *v,
                   const double *q, double *o)
{
#pragma omp parallel for schedule(dynamic)
    for (int h = 0; h < nh; ++h) {
        double *Sh = S + (size_t)h * dv * dk;
        double *u = malloc(sizeof(double) * dv);
        for (int t = 0; t < n; ++t) {
            const double *dt = d + ((size_t)h * n + t) * dk;
            const double *kk = kt + ((size_t)h * n + t) * dk;
            const double *bt = b + ((size_t)h * n + t) * dk;
            const double *vt = v + ((size_t)h * n + t) * dv;
            /* u_t = v_t - S_{t-1} b_t */
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += Sh[(size_t)i * dk + j] * bt[j];
                u[i] = vt[i] - acc;
            }
            /* S_t = S_{t-1} D_t + u_t k~_t^T */
            for (int i = 0; i < dv; ++i)
                for (int j = 0; j < dk; ++j)
                    Sh[(size_t)i * dk + j] = Sh[(size_t)i * dk + j] * dt[j] + u[i] * kk[j];
            if (q && o) {
                const double *qt = q + ((size_t)h * n + t) * dk;
                double *ot = o + ((size_t)h * n + t) * dv;
                for (int i = 0; i < dv; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dk; ++j) acc += Sh[(size_t)i * dk + j] * qt[j];
                    ot[i] = acc;
                }
            }
        }
        free(u);
    }
}

/* ------------------------------------------------------------------------ */
/* Quantizer: compensator selection, residual smoothing, int8 codes.        */
/* ------------------------------------------------------------------------ */

/* Quantizes nh FP32 states S [nh][dv][dk] into the int8 snapshot format.
 *
 * [LQ] Abstract and Figure 4, [KP] Key points, [CN]: the largest outliers are
 * kept in a few high-precision Compensator Tokens, which flattens the row
 * l2 norms of the residual; the residual is smoothed across channels and
 * quantized once to 8 bits.  The pages fix neither rule; ours is:
 *
 *  C2  n_i = ||S[i,:]||_2.  The r rows with the largest n_i become
 *      compensators, largest first; an exact tie goes to the smaller row
 *      index.  comp_row[c] = that row, comp_val[c] = the row itself (FP32).
 *      R = S with those rows set to zero.
 *  C3  m_j = max_i |R_ij|;  c_j = fp32(sqrt(m_j)), or 1 when m_j = 0 or when
 *      smoothing is off (SmoothQuant-style migration with strength 1/2 along
 *      the key channels).  R'_ij = fp32(R_ij / c_j).
 *  C4  with q = 2^(bits-1) - 1 (127 for 8 bits; the 6- and 4-bit states of
 *      [LQ] Table 1's lower-precision groups give 31 and 7):
 *      sigma_i = fp32(max_j |R'_ij| / q) (the stored scale);
 *      Q_ij = clamp(rne(fp32(R'_ij / sigma_i)), -q, q), Q_i. = 0 when
 *      sigma_i = 0.  Round half to even; no zero point; -q-1 unused.  The
 *      codes come back one per int8 whatever the width (the packing of a
 *      narrower code is a storage format, not arithmetic).
 *  bits = 16 is the BF16 state of [LQ] Table 2 ("BF16 per-step" and its
 *      per-window row): C2 as above, then no smoothing (c = 1) and no integer
 *      codes (sigma = 1): the residual itself is stored rounded to BF16,
 *      dense_ij = bf16(R_ij), in `dense` [nh][dv][dk] (FP32 array).
 *
 * Every division and square root above is one IEEE FP32 operation on FP32
 * operands: the FP64 result rounded once to FP32 is the correctly rounded
 * FP32 result, because FP64 carries more than 2 x 24 + 2 significant bits
 * (double rounding is then innocuous for a quotient or a square root).  So
 * the quantization decision is taken in FP32, the precision of the stored
 * format.  The row norms (an argmax decision) are computed in
 * FP64; when two norms are within rounding of each other either selection is
 * correct.
 *
 * row_norm [nh][dv] (optional) receives n_i.                               */
void lqo_quantize(int nh, int dv, int dk, int r, int smoothing, int bits, const float *S,
                  int8_t *codes, float *row_scale, float *col_smooth,
                  int32_t *comp_row, float *comp_val, double *row_norm, float *dense)
{
    const double qmax = (double)((1 << (bits - 1)) - 1);
#pragma omp parallel for schedule(dynamic)
    for (int h = 0; h < nh; ++h) {
        const float *Sh = S + (size_t)h * dv * dk;
        double *R = malloc(sizeof(double) * dv * dk);
        double *norm = malloc(sizeof(double) * dv);
        char *taken = calloc((size_t)dv, 1);
        for (int i = 0; i < dv; ++i) {
            double ss = 0.0;
            for (int j = 0; j < dk; ++j) {
                double x = Sh[(size_t)i * dk + j];
                R[(size_t)i * dk + j] = x;
                ss += x * x;
            }
            norm[i] = sqrt(ss);
            if (row_norm) row_norm[(size_t)h * dv + i] = norm[i];
        }
        /* C2: top-r rows by l2 norm, ties to the smaller index. */
        for (int c = 0; c < r; ++c) {
            int best = -1;
            for (int i = 0; i < dv; ++i)
                if (!taken[i] && (best < 0 || norm[i] > norm[best])) best = i;
            taken[best] = 1;
            comp_row[(size_t)h * r + c] = best;
            for (int j = 0; j < dk; ++j) {
                comp_val[((size_t)h * r + c) * dk + j] = Sh[(size_t)best * dk + j];
                R[(size_t)best * dk + j] = 0.0;
            }
        }
        if (bits == 16) {
            /* BF16 residual: no smoothing, unit scales, rounded values. */
            for (int j = 0; j < dk; ++j) col_smooth[(size_t)h * dk + j] = 1.0f;
            for (int i = 0; i < dv; ++i) {
                row_scale[(size_t)h * dv + i] = 1.0f;
                for (int j = 0; j < dk; ++j) {
                    codes[((size_t)h * dv + i) * dk + j] = 0;
                    dense[((size_t)h * dv + i) * dk + j] = (float)bf16(R[(size_t)i * dk + j]);
                }
            }
            free(R);
            free(norm);
            free(taken);
            continue;
        }
        /* C3: smoothing factor per key channel. */
        float *c = col_smooth + (size_t)h * dk;
        for (int j = 0; j < dk; ++j) {
            double m = 0.0;
            for (int i = 0; i < dv; ++i) {
                double a = fabs(R[(size_t)i * dk + j]);
                if (a > m) m = a;
            }
            c[j] = (smoothing && m > 0.0) ? (float)sqrt(m) : 1.0f;
        }
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j)
                R[(size_t)i * dk + j] = f32(R[(size_t)i * dk + j] / (double)c[j]);
        /* C4: per-row symmetric codes in [-qmax, qmax]. */
        for (int i = 0; i < dv; ++i) {
            double mx = 0.0;
            for (int j = 0; j < dk; ++j) {
                double a = fabs(R[(size_t)i * dk + j]);
                if (a > mx) mx = a;
            }
            double sigma = f32(mx / qmax);
            row_scale[(size_t)h * dv + i] = (float)sigma;
            for (int j = 0; j < dk; ++j) {
                double qv = 0.0;
                if (sigma > 0.0) {
                    qv = rint(f32(R[(size_t)i * dk + j] / sigma)); /* ties to even */
                    if (qv > qmax) qv = qmax;
                    if (qv < -qmax) qv = -qmax;
                }
                codes[((size_t)h * dv + i) * dk + j] = (int8_t)qv;
            }
        }
        free(R);
        free(norm);
        free(taken);
    }
}

/* Dequantized boundary state S^_0 [nh][dv][dk] in FP64:
 *   S^_0 = Diag(sigma) Q Diag(c) + sum_c e_{comp_row[c]} comp_val[c]^T .
 * A compensator is a pseudo-token with u = e_row and k~ = comp_val placed at
 * window position 0 ([LQ] Abstract: the Compensator Tokens share the update
 * path of real tokens; Figure 4: the state is the quantized residual plus the
 * Compensator Tokens plus the buffered real-token updates).                */
/* Compensators are rank-one pseudo-tokens u_c k~_c^T at window position 0.
 * The row rule stores k~_c = comp_val[c] and u_c = e_{comp_row[c]}; the
 * rank-r SVD rule stores u_c = comp_u[c] [dv] (comp_u != NULL) as well.    */
static void dequantize_head(int dv, int dk, int r, const int8_t *codes,
                            const float *row_scale, const float *col_smooth,
                            const int32_t *comp_row, const float *comp_val,
                            const float *dense, const float *comp_u, double *Sh)
{
    for (int i = 0; i < dv; ++i)
        for (int j = 0; j < dk; ++j)
            Sh[(size_t)i * dk + j] = dense ? (double)dense[(size_t)i * dk + j]
                                           : (double)row_scale[i] *
                                                 (double)codes[(size_t)i * dk + j] *
                                                 (double)col_smooth[j];
    for (int c = 0; c < r; ++c) {
        if (comp_u) {
            for (int i = 0; i < dv; ++i)
                for (int j = 0; j < dk; ++j)
                    Sh[(size_t)i * dk + j] += (double)comp_u[(size_t)c * dv + i] *
                                              (double)comp_val[(size_t)c * dk + j];
            continue;
        }
        int row = comp_row[c];
        for (int j = 0; j < dk; ++j)
            Sh[(size_t)row * dk + j] += (double)comp_val[(size_t)c * dk + j];
    }
}

void lqo_dequantize(int nh, int dv, int dk, int r, const int8_t *codes,
                    const float *row_scale, const float *col_smooth,
                    const int32_t *comp_row, const float *comp_val,
                    const float *dense, const float *comp_u, double *S_hat)
{
#pragma omp parallel for schedule(dynamic)
    for (int h = 0; h < nh; ++h)
        dequantize_head(dv, dk, r, codes + (size_t)h * dv * dk,
                        row_scale + (size_t)h * dv, col_smooth + (size_t)h * dk,
                        comp_row + (size_t)h * r, comp_val + (size_t)h * r * dk,
                        dense ? dense + (size_t)h * dv * dk : NULL,
                        comp_u ? comp_u + (size_t)h * r * dv : NULL,
                        S_hat + (size_t)h * dv * dk);
}

/* ------------------------------------------------------------------------ */
/* Per-window decode in buffered form ([LQ] Figure 2).                      */
/* ------------------------------------------------------------------------ */

/* Decay of the gate from just after window position m to position t:
 * D_{m+1..t} = Diag(exp(L_t - L_m)), with L the cumulative log gate stored in
 * the records (L_0 = 0).  Channel j of a scalar gate (gdim = 1) is channel 0. */
static double decay(const double *L, int gdim, int t, int m, int j)
{
    int jj = gdim == 1 ? 0 : j;
    double Lt = t > 0 ? L[(size_t)(t - 1) * gdim + jj] : 0.0;
    double Lm = m > 0 ? L[(size_t)(m - 1) * gdim + jj] : 0.0;
    return exp(Lt - Lm);
}

/* Runs n decode steps of one window on each of nh heads.
 *
 * The boundary state S^_0 (the int8 snapshot plus compensators) stays fixed;
 * step t (window position pos+1 .. pos+n) uses only S^_0 and the records
 * 1..t-1 already buffered ([LQ] Figure 2: outputs come from the fixed
 * low-bit state together with the high-precision buffered updates):
 *
 *   L_t        = L_{t-1} + log d_t                       (stored FP32)
 *   S_{t-1}b_t = S^_0 (D_{1..t-1} b_t) + sum_{m<t} u_m (k~_m . D_{m+1..t-1} b_t)
 *   u_t        = v_t - S_{t-1} b_t                      (stored FP32)
 *   k~_t                                                 (stored FP32)
 *   o_t = S_t q_t = S^_0 (D_{1..t} q_t) + sum_{m<=t} u_m (k~_m . D_{m+1..t} q_t)
 *
 * The record of position m is (L_m, k~_m, u_m); it encodes Table 4's
 * (d_m, k~_m, u_m) with the gate kept as a running log so that ratios of gate
 * products are exponentials of differences.
 *
 * Layouts (head-major):
 *   snapshot: codes [nh][dv][dk], row_scale [nh][dv], col_smooth [nh][dk],
 *             comp_row [nh][r], comp_val [nh][r][dk]
 *   records : rec_L [nh][W][gdim], rec_k [nh][W][dk], rec_u [nh][W][dv];
 *             positions 1..pos are read, pos+1..pos+n are written
 *   tokens  : d, kt, b, q [nh][n][dk]  (d holds gdim values per token:
 *             [nh][n][gdim]), v [nh][n][dv]
 *   o       : [nh][n][dv]
 * exact != 0 keeps records in FP64 instead of rounding them to FP32.        */
void lqo_window(int nh, int dv, int dk, int r, int gdim, int W, int pos, int n,
                int exact, const int8_t *codes, const float *row_scale,
                const float *col_smooth, const int32_t *comp_row,
                const float *comp_val, const float *dense, const float *comp_u,
                double *rec_L, double *rec_k, double *rec_u, const double *d, const double *kt,
                const double *b, const double *v, const double *q, double *o)
{
#pragma omp parallel for schedule(dynamic)
    for (int h = 0; h < nh; ++h) {
        double *S0 = malloc(sizeof(double) * dv * dk);
        double *x = malloc(sizeof(double) * dk);
        double *hb = malloc(sizeof(double) * dv);
        dequantize_head(dv, dk, r, codes + (size_t)h * dv * dk,
                        row_scale + (size_t)h * dv, col_smooth + (size_t)h * dk,
                        comp_row + (size_t)h * r, comp_val + (size_t)h * r * dk,
                        dense ? dense + (size_t)h * dv * dk : NULL,
                        comp_u ? comp_u + (size_t)h * r * dv : NULL, S0);
        double *L = rec_L + (size_t)h * W * gdim;
        double *K = rec_k + (size_t)h * W * dk;
        double *U = rec_u + (size_t)h * W * dv;
        for (int s = 0; s < n; ++s) {
            int t = pos + s + 1; /* window position, 1-based */
            const double *dt = d + ((size_t)h * n + s) * gdim;
            const double *kk = kt + ((size_t)h * n + s) * dk;
            const double *bt = b + ((size_t)h * n + s) * dk;
            const double *vt = v + ((size_t)h * n + s) * dv;
            const double *qt = q + ((size_t)h * n + s) * dk;
            /* L_t */
            for (int g = 0; g < gdim; ++g) {
                double prev = t > 1 ? L[(size_t)(t - 2) * gdim + g] : 0.0;
                double Lt = prev + log(dt[g]);
                L[(size_t)(t - 1) * gdim + g] = exact ? Lt : f32(Lt);
            }
            /* S_{t-1} b_t from the boundary state ... */
            for (int j = 0; j < dk; ++j) x[j] = decay(L, gdim, t - 1, 0, j) * bt[j];
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S0[(size_t)i * dk + j] * x[j];
                hb[i] = acc;
            }
            /* ... plus the buffered updates 1..t-1 */
            for (int m = 1; m < t; ++m) {
                double a = 0.0;
                for (int j = 0; j < dk; ++j)
                    a += K[(size_t)(m - 1) * dk + j] * decay(L, gdim, t - 1, m, j) * bt[j];
                for (int i = 0; i < dv; ++i) hb[i] += U[(size_t)(m - 1) * dv + i] * a;
            }
            /* record t = (L_t, k~_t, u_t) */
            for (int j = 0; j < dk; ++j)
                K[(size_t)(t - 1) * dk + j] = exact ? kk[j] : f32(kk[j]);
            for (int i = 0; i < dv; ++i) {
                double ui = vt[i] - hb[i];
                U[(size_t)(t - 1) * dv + i] = exact ? ui : f32(ui);
            }
            /* o_t = S_t q_t */
            double *ot = o + ((size_t)h * n + s) * dv;
            for (int j = 0; j < dk; ++j) x[j] = decay(L, gdim, t, 0, j) * qt[j];
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S0[(size_t)i * dk + j] * x[j];
                ot[i] = acc;
            }
            for (int m = 1; m <= t; ++m) {
                double a = 0.0;
                for (int j = 0; j < dk; ++j)
                    a += K[(size_t)(m - 1) * dk + j] * decay(L, gdim, t, m, j) * qt[j];
                for (int i = 0; i < dv; ++i) ot[i] += U[(size_t)(m - 1) * dv + i] * a;
            }
        }
        free(S0);
        free(x);
        free(hb);
    }
}

/* Rebuilds the full state at window position n from the boundary snapshot
 * and the n buffered records ([LQ] Figure 2: the state is reconstructed from
 * the buffered updates; Figure 4: quantized residual + Compensator Tokens +
 * buffered real-token updates):
 *   S_n = S^_0 D_{1..n} + sum_{m<=n} u_m (D_{m+1..n} k~_m)^T      (FP64) */
void lqo_rebuild(int nh, int dv, int dk, int r, int gdim, int W, int n,
                 const int8_t *codes, const float *row_scale,
                 const float *col_smooth, const int32_t *comp_row,
                 const float *comp_val, const float *dense, const float *comp_u,
                 const double *rec_L, const double *rec_k, const double *rec_u, double *S_out)
{
#pragma omp parallel for schedule(dynamic)
    for (int h = 0; h < nh; ++h) {
        double *Sh = S_out + (size_t)h * dv * dk;
        dequantize_head(dv, dk, r, codes + (size_t)h * dv * dk,
                        row_scale + (size_t)h * dv, col_smooth + (size_t)h * dk,
                        comp_row + (size_t)h * r, comp_val + (size_t)h * r * dk,
                        dense ? dense + (size_t)h * dv * dk : NULL,
                        comp_u ? comp_u + (size_t)h * r * dv : NULL, Sh);
        const double *L = rec_L + (size_t)h * W * gdim;
        const double *K = rec_k + (size_t)h * W * dk;
        const double *U = rec_u + (size_t)h * W * dv;
        for (int j = 0; j < dk; ++j) {
            double g = decay(L, gdim, n, 0, j);
            for (int i = 0; i < dv; ++i) Sh[(size_t)i * dk + j] *= g;
        }
        for (int m = 1; m <= n; ++m)
            for (int j = 0; j < dk; ++j) {
                double kh = K[(size_t)(m - 1) * dk + j] * decay(L, gdim, n, m, j);
                for (int i = 0; i < dv; ++i)
                    Sh[(size_t)i * dk + j] += U[(size_t)(m - 1) * dv + i] * kh;
            }
    }
}
