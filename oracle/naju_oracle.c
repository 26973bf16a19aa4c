/*
 * Naju fp64 oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, sequential double-precision CPU implementation of the Naju
 * block's scan path, written from the equations of the Naju reproduction
 * README ("Naju: A native discrete SSM with independent retention and
 * writing", section "Core equations" and the block flowchart) and the
 * arXiv 2607.21000 abstract.  Only the test suite, the package's smoke()
 * check and bench.py's CPU-baseline leg may load this library; the CUDA
 * product path never does, and the two share no code.
 *
 * Conventions (row-major, contiguous):
 *   u, h, a, b, z, out, dout, dh, da, db, dz : [Bt, L, d]
 *   B, C, dB, dC                             : [Bt, L, N]
 *   x0, xL, dxL, dx0, state                  : [Bt, d, N]
 *   D, dD, conv_b, dconv_b                   : [d]
 *   conv_w, dconv_w                          : [d, W]
 *
 * Readings of the pages (each is a choice where the pages are silent):
 *   - state x_n is d x N; the write is the outer product h_n B_n^T
 *     (README, Core equations, first display);
 *   - the gates f_n = sigma(a_n), i_n = sigma(b_n) are per (token, channel)
 *     and broadcast over the N state columns;
 *   - B_n, C_n are one N-vector per (batch, token), shared by all channels;
 *   - readout y_n = x_n C_n / sqrt(N) + D (.) h_n (README, Core equations,
 *     second display); the 1/sqrt(N) scale touches only x_n C_n;
 *   - output modulation out_n = y_n * SiLU(z_n) (README flowchart node
 *     "SiLU output modulation"); no z means no modulation;
 *   - causal depthwise conv (README flowchart node "causal depthwise conv +
 *     SiLU"): p[t] = bias + sum_k w[k] u[t-(W-1)+k], zero left padding,
 *     then h = SiLU(p);
 *   - zero initial state unless x0 is given.
 *
 * The loops below follow the recurrence literally, token by token.  OpenMP
 * only splits independent (batch, channel) rows across host threads; the
 * per-row arithmetic and its order are those of the equations.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double sigm(double v) { return 1.0 / (1.0 + exp(-v)); }
static double silu(double v) { return v * sigm(v); }
/* d/dv [v * sigma(v)] = sigma(v) * (1 + v * (1 - sigma(v))) */
static double dsilu(double v) {
    double s = sigm(v);
    return s * (1.0 + v * (1.0 - s));
}

int naju_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Causal depthwise conv + SiLU (README flowchart, "causal depthwise conv +
 * SiLU").  p_out may be NULL. */
void naju_oracle_conv_silu_fwd(int64_t Bt, int64_t L, int64_t d, int64_t W,
                               const double* u, const double* w, const double* bias,
                               double* p_out, double* h) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bb = 0; bb < Bt; ++bb)
        for (int64_t c = 0; c < d; ++c)
            for (int64_t t = 0; t < L; ++t) {
                double p = bias ? bias[c] : 0.0;
                for (int64_t k = 0; k < W; ++k) {
                    int64_t s = t - (W - 1) + k;
                    if (s >= 0) p += w[c * W + k] * u[(bb * L + s) * d + c];
                }
                if (p_out) p_out[(bb * L + t) * d + c] = p;
                h[(bb * L + t) * d + c] = silu(p);
            }
}

/* One decode token of the conv + SiLU above (README flowchart, "causal
 * depthwise conv + SiLU"): cs [Bt][d][W-1] holds the previous W-1 inputs of
 * each channel, oldest first; h = SiLU(bias + sum_{k<W-1} w[k] cs[k] +
 * w[W-1] u), then cs shifts by one and ends with u. */
void naju_oracle_conv_silu_step(int64_t Bt, int64_t d, int64_t W, const double* u,
                                const double* w, const double* bias, double* cs, double* h) {
    for (int64_t bb = 0; bb < Bt; ++bb)
        for (int64_t c = 0; c < d; ++c) {
            const int64_t e = bb * d + c;
            double* s = cs + e * (W - 1);
            double p = bias ? bias[c] : 0.0;
            for (int64_t k = 0; k < W - 1; ++k) p += w[c * W + k] * s[k];
            p += w[c * W + W - 1] * u[e];
            h[e] = silu(p);
            for (int64_t k = 0; k + 1 < W - 1; ++k) s[k] = s[k + 1];
            s[W - 2] = u[e];
        }
}

/* Gradient of the conv + SiLU above, given dL/dh.  dw, dbias are
 * accumulated over batch and time (overwritten, not added to). */
void naju_oracle_conv_silu_bwd(int64_t Bt, int64_t L, int64_t d, int64_t W,
                               const double* u, const double* w, const double* bias,
                               const double* dh, double* du, double* dw, double* dbias) {
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < d; ++c) {
        double* dp = (double*)malloc(sizeof(double) * (size_t)L);
        double dbc = 0.0;
        for (int64_t k = 0; k < W; ++k) dw[c * W + k] = 0.0;
        for (int64_t bb = 0; bb < Bt; ++bb) {
            for (int64_t t = 0; t < L; ++t) {
                double p = bias ? bias[c] : 0.0;
                for (int64_t k = 0; k < W; ++k) {
                    int64_t s = t - (W - 1) + k;
                    if (s >= 0) p += w[c * W + k] * u[(bb * L + s) * d + c];
                }
                dp[t] = dh[(bb * L + t) * d + c] * dsilu(p);
                dbc += dp[t];
            }
            /* p[t] depends on u[t-(W-1)+k] through w[k]; transpose that map. */
            for (int64_t s = 0; s < L; ++s) {
                double acc = 0.0;
                for (int64_t k = 0; k < W; ++k) {
                    int64_t t = s + (W - 1) - k;
                    if (t < L) acc += w[c * W + k] * dp[t];
                }
                du[(bb * L + s) * d + c] = acc;
            }
            for (int64_t k = 0; k < W; ++k) {
                double acc = 0.0;
                for (int64_t t = 0; t < L; ++t) {
                    int64_t s = t - (W - 1) + k;
                    if (s >= 0) acc += dp[t] * u[(bb * L + s) * d + c];
                }
                dw[c * W + k] += acc;
            }
        }
        if (dbias) dbias[c] = dbc;
        free(dp);
    }
}

/* Write gate.  b == NULL selects the coupled single gate i = 1 - f
 * (= sigma(-a)), the complementary gating analysed in the paper's abstract
 * (|r| + w <= 1); otherwise i = sigma(b). */
static double wgate(const double* a, const double* b, int64_t e) {
    return b ? sigm(b[e]) : sigm(-a[e]);
}

/* Forward scan (README, Core equations):
 *   x_n = f_n (.) x_{n-1} + i_n (.) (h_n B_n^T),  f = sigma(a), i = sigma(b)
 *   y_n = x_n C_n / sqrt(N) + D (.) h_n
 *   out_n = y_n * SiLU(z_n)
 * y_pre (the readout before modulation) and xL (state after the last token)
 * are optional outputs.  b == NULL: coupled gate i = 1 - f. */
void naju_oracle_scan_fwd(int64_t Bt, int64_t L, int64_t d, int64_t N,
                          const double* h, const double* a, const double* b,
                          const double* B, const double* C, const double* z,
                          const double* D, const double* x0,
                          double* y_pre, double* out, double* xL) {
    const double scale = 1.0 / sqrt((double)N);
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bb = 0; bb < Bt; ++bb)
        for (int64_t c = 0; c < d; ++c) {
            double* x = (double*)malloc(sizeof(double) * (size_t)N);
            for (int64_t j = 0; j < N; ++j) x[j] = x0 ? x0[(bb * d + c) * N + j] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t e = (bb * L + t) * d + c;
                const double f = sigm(a[e]);
                const double i = wgate(a, b, e);
                const double* Bn = B + (bb * L + t) * N;
                const double* Cn = C + (bb * L + t) * N;
                double r = 0.0;
                for (int64_t j = 0; j < N; ++j) {
                    x[j] = f * x[j] + i * (h[e] * Bn[j]);
                    r += x[j] * Cn[j];
                }
                const double y = r * scale + (D ? D[c] * h[e] : 0.0);
                if (y_pre) y_pre[e] = y;
                out[e] = z ? y * silu(z[e]) : y;
            }
            if (xL)
                for (int64_t j = 0; j < N; ++j) xL[(bb * d + c) * N + j] = x[j];
            free(x);
        }
}

/* Reverse-mode gradient of naju_oracle_scan_fwd, written out by hand from the
 * forward recurrence.  For one (batch, channel) row, with G_n = dL/dx_n:
 *   dy_n   = dout_n * SiLU(z_n)
 *   dz_n   = dout_n * y_n * SiLU'(z_n)
 *   G_n    = dy_n C_n / sqrt(N) + f_{n+1} G_{n+1}      (G_{L-1} also gets dxL)
 *   dh_n   = D dy_n + i_n (G_n . B_n)
 *   di_n   = h_n (G_n . B_n),  db_n = di_n i_n (1 - i_n)
 *   df_n   = G_n . x_{n-1},    da_n = df_n f_n (1 - f_n)
 *   dB_n  += G_n i_n h_n,      dC_n += dy_n x_n / sqrt(N)   (summed over d)
 *   dD    += dy_n h_n,         dx0 = f_0 G_0
 * Coupled gate (b == NULL, i = 1 - f): a reaches the loss through f and i,
 *   da_n = (df_n - di_n) f_n (1 - f_n), and there is no db (db may be NULL).
 * All states x_n of a row are kept, so the reverse sweep reads them exactly.
 * dD is overwritten.  dz may be NULL only when z is NULL. */
void naju_oracle_scan_bwd(int64_t Bt, int64_t L, int64_t d, int64_t N,
                          const double* h, const double* a, const double* b,
                          const double* B, const double* C, const double* z,
                          const double* D, const double* x0,
                          const double* dout, const double* dxL,
                          double* dh, double* da, double* db, double* dB, double* dC,
                          double* dz, double* dD, double* dx0) {
    const double scale = 1.0 / sqrt((double)N);
    int nthr = naju_oracle_num_threads();
    const size_t LN = (size_t)L * (size_t)N;
    double* accB = (double*)calloc((size_t)nthr * LN, sizeof(double));
    double* accC = (double*)calloc((size_t)nthr * LN, sizeof(double));
    if (dD)
        for (int64_t c = 0; c < d; ++c) dD[c] = 0.0;

    for (int64_t bb = 0; bb < Bt; ++bb) {
        memset(accB, 0, sizeof(double) * (size_t)nthr * LN);
        memset(accC, 0, sizeof(double) * (size_t)nthr * LN);
#pragma omp parallel
        {
            int tid = 0;
#ifdef _OPENMP
            tid = omp_get_thread_num();
#endif
            double* myB = accB + (size_t)tid * LN;
            double* myC = accC + (size_t)tid * LN;
            /* xs[(t+1)*N + j] = x_t[j]; row 0 is the initial state. */
            double* xs = (double*)malloc(sizeof(double) * (size_t)(L + 1) * (size_t)N);
            double* G = (double*)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(static)
            for (int64_t c = 0; c < d; ++c) {
                for (int64_t j = 0; j < N; ++j) xs[j] = x0 ? x0[(bb * d + c) * N + j] : 0.0;
                for (int64_t t = 0; t < L; ++t) {
                    const int64_t e = (bb * L + t) * d + c;
                    const double f = sigm(a[e]), i = wgate(a, b, e);
                    const double* Bn = B + (bb * L + t) * N;
                    for (int64_t j = 0; j < N; ++j)
                        xs[(t + 1) * N + j] = f * xs[t * N + j] + i * (h[e] * Bn[j]);
                }
                for (int64_t j = 0; j < N; ++j) G[j] = dxL ? dxL[(bb * d + c) * N + j] : 0.0;
                double dDc = 0.0;
                for (int64_t t = L - 1; t >= 0; --t) {
                    const int64_t e = (bb * L + t) * d + c;
                    const double f = sigm(a[e]), i = wgate(a, b, e);
                    const double* Bn = B + (bb * L + t) * N;
                    const double* Cn = C + (bb * L + t) * N;
                    const double* xt = xs + (t + 1) * N;
                    const double* xp = xs + t * N;
                    double r = 0.0;
                    for (int64_t j = 0; j < N; ++j) r += xt[j] * Cn[j];
                    const double y = r * scale + (D ? D[c] * h[e] : 0.0);
                    const double g = z ? silu(z[e]) : 1.0;
                    const double dy = dout[e] * g;
                    if (dz) dz[e] = z ? dout[e] * y * dsilu(z[e]) : 0.0;
                    /* G currently holds f_{t+1} G_{t+1} (+ dxL at the end). */
                    double GB = 0.0, Gx = 0.0;
                    for (int64_t j = 0; j < N; ++j) {
                        G[j] += dy * scale * Cn[j];
                        GB += G[j] * Bn[j];
                        Gx += G[j] * xp[j];
                        myB[t * N + j] += G[j] * i * h[e];
                        myC[t * N + j] += dy * scale * xt[j];
                    }
                    dh[e] = (D ? D[c] * dy : 0.0) + i * GB;
                    const double di = h[e] * GB;
                    if (b) {
                        db[e] = di * i * (1.0 - i);
                        da[e] = Gx * f * (1.0 - f);
                    } else {
                        if (db) db[e] = 0.0;
                        da[e] = (Gx - di) * f * (1.0 - f);
                    }
                    dDc += dy * h[e];
                    for (int64_t j = 0; j < N; ++j) G[j] *= f;
                }
                if (dD) dD[c] += dDc;
                if (dx0)
                    for (int64_t j = 0; j < N; ++j) dx0[(bb * d + c) * N + j] = G[j];
            }
            free(xs);
            free(G);
        }
        /* Sum the per-thread partials in thread order. */
        for (size_t k = 0; k < LN; ++k) {
            double sb = 0.0, sc = 0.0;
            for (int t = 0; t < nthr; ++t) {
                sb += accB[(size_t)t * LN + k];
                sc += accC[(size_t)t * LN + k];
            }
            dB[(size_t)bb * LN + k] = sb;
            dC[(size_t)bb * LN + k] = sc;
        }
    }
    free(accB);
    free(accC);
}

/* One decode step on a carried state (the recurrence for a single token).
 * state [Bt, d, N] is updated in place; h, a, b, z, out are [Bt, d];
 * B, C are [Bt, N]. */
void naju_oracle_scan_step(int64_t Bt, int64_t d, int64_t N,
                           const double* h, const double* a, const double* b,
                           const double* B, const double* C, const double* z,
                           const double* D, double* state, double* out) {
    const double scale = 1.0 / sqrt((double)N);
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bb = 0; bb < Bt; ++bb)
        for (int64_t c = 0; c < d; ++c) {
            const int64_t e = bb * d + c;
            const double f = sigm(a[e]), i = wgate(a, b, e);
            double* x = state + e * N;
            double r = 0.0;
            for (int64_t j = 0; j < N; ++j) {
                x[j] = f * x[j] + i * (h[e] * B[bb * N + j]);
                r += x[j] * C[bb * N + j];
            }
            const double y = r * scale + (D ? D[c] * h[e] : 0.0);
            out[e] = z ? y * silu(z[e]) : y;
        }
}
