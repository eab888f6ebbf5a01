/*
 * bdscan oracle: a plain, sequential, fp64 CPU restatement of the partially
 * bidirectional (block-confined reverse) selective-scan mixer of BDLM Mamba-H.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline / reference legs load this library. It shares no
 * code, header, table or helper with the CUDA path, and the CUDA path never
 * calls it.
 *
 * What the method computes, and where it is stated:
 *   "Training Hybrid Block Diffusion Language Models with Partial
 *   Bidirectionality" (arXiv 2607.02805):
 *   - Abstract: the reverse Mamba scan is restricted to the active denoising
 *     block, which makes the forward states prefix-only and exactly cacheable
 *     across blocks.
 *   - gist.science technical summary, "Methodik", cache-aligned objective:
 *     the Mamba layers cache only forward boundary (recurrent) states; the
 *     reverse scan is confined to the active block b_t, so the prefix cache
 *     C_l(c) depends on the clean prefix alone.
 *   - same summary, "Wesentliche Beitraege": the cached objects of the
 *     all-block training objective equal the inference-time block caches.
 *
 * The pages never write the recurrence. This file adopts the standard Mamba
 * selective-scan discretisation, used identically by both directions:
 *     delta_t = softplus(dt_raw_t)             (or dt_t itself)
 *     a_t[n]  = exp(delta_t * A[d,n])
 *     b_t[n]  = delta_t * x_t * B_t[n]
 *     forward : h_t = a_t * h_{t-1} + b_t,   h_{-1} = h0 (cache) or 0
 *               y_fwd_t = sum_n C_t[n] h_t[n] + Dskip[d] x_t
 *     reverse : inside block j = [jK, (j+1)K):
 *               g_t = a_t * g_{t+1} + b_t,   g_{(j+1)K} = 0
 *               y_rev_t = sum_n C_t[n] g_t[n] + Dskip[d] x_t
 *     output  : y_t = (y_fwd_t + y_rev_t) * (z ? silu(z_t) : 1)
 * Readings where the pages are silent: both directions share delta, A, B, C
 * and Dskip; the reverse step uses the decay of its own token t (the time
 * mirror image of the forward step); the sum y_fwd + y_rev therefore holds
 * Dskip*x twice; the gate multiplies the sum once.
 *
 * Layouts (row-major, contiguous): x, dt, z, y [Bt, L, D]; B, C [Bt, L, N];
 * A [D, N]; Dskip [D]; states [Bt, D, N]; boundary states [Bt, L/K, D, N]
 * (the state after the last token of each block).
 *
 * All inputs arrive as doubles already widened exactly from their storage
 * type; all arithmetic is double with libm exp/log1p. Channels (b, d) are
 * independent and are processed one after another.
 *
 * Build with -DORACLE_MUTANT=k to plant one deliberate mistake (tests use
 * this to show that the pins catch each plausible error):
 *   1 reverse decay taken from token t+1 instead of t
 *   2 Dskip*x left out of the reverse term
 *   3 reverse state not reset at block boundaries
 *   4 reverse scan exclusive (token t does not feed its own state)
 *   5 B and C swapped in the readout
 *   6 softplus replaced by exp
 *   7 forward state not carried from h0
 * and, in the backward pass (oracle_train_blocks_backward):
 *   8 reverse-state adjoint carried with the decay of token t, not t-1
 *   9 forward-state adjoint restarted at every block boundary
 *  10 decay gradient without the reverse-state term
 *  11 dt gradient without the softplus derivative
 *  12 initial-state gradient without the first token's decay
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

#define IDX3(a, b, c, nb, nc) ((((int64_t)(a)) * (nb) + (b)) * (nc) + (c))

/* softplus(v) = log(1 + e^v), written in the overflow-free form
 * max(v, 0) + log1p(exp(-|v|)). */
double oracle_softplus(double v) {
#if ORACLE_MUTANT == 6
    return exp(v);
#else
    double m = v > 0.0 ? v : 0.0;
    return m + log1p(exp(-fabs(v)));
#endif
}

/* silu(z) = z * sigmoid(z) */
double oracle_silu(double z) { return z / (1.0 + exp(-z)); }

static double delta_of(double dt_raw, int dt_softplus) {
    return dt_softplus ? oracle_softplus(dt_raw) : dt_raw;
}

/* Forward (causal) scan over tokens [0, L) of every channel.
 *   y_fwd    [Bt, L, D]       nullable
 *   h_out    [Bt, D, N]       nullable; may alias h0 (read before written)
 *   boundary [Bt, L/K, D, N]  nullable; state after tokens K-1, 2K-1, ...
 * Returns 0, or -1 on bad sizes / allocation failure. */
int oracle_forward(int64_t Bt, int64_t L, int64_t D, int64_t N, int64_t K,
                   const double *x, const double *dt, int dt_softplus,
                   const double *A, const double *B, const double *C,
                   const double *Dskip, const double *h0,
                   double *y_fwd, double *h_out, double *boundary) {
    if (Bt < 0 || L < 0 || D < 0 || N <= 0 || K <= 0 || (L % K) != 0) return -1;
    double *h = (double *)malloc(sizeof(double) * (size_t)N);
    if (!h) return -1;
    const int64_t nblk = L / K;
    for (int64_t b = 0; b < Bt; ++b) {
        for (int64_t d = 0; d < D; ++d) {
            for (int64_t n = 0; n < N; ++n) {
#if ORACLE_MUTANT == 7
                h[n] = 0.0;
#else
                h[n] = h0 ? h0[IDX3(b, d, n, D, N)] : 0.0;
#endif
            }
            for (int64_t t = 0; t < L; ++t) {
                const double xv = x[IDX3(b, t, d, L, D)];
                const double dl = delta_of(dt[IDX3(b, t, d, L, D)], dt_softplus);
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double a = exp(dl * A[d * N + n]);
                    h[n] = a * h[n] + dl * xv * B[IDX3(b, t, n, L, N)];
#if ORACLE_MUTANT == 5
                    acc += B[IDX3(b, t, n, L, N)] * h[n];
#else
                    acc += C[IDX3(b, t, n, L, N)] * h[n];
#endif
                }
                if (y_fwd) y_fwd[IDX3(b, t, d, L, D)] = acc + Dskip[d] * xv;
                if (boundary && ((t + 1) % K) == 0) {
                    const int64_t j = (t + 1) / K - 1;
                    for (int64_t n = 0; n < N; ++n)
                        boundary[((b * nblk + j) * D + d) * N + n] = h[n];
                }
            }
            if (h_out)
                for (int64_t n = 0; n < N; ++n) h_out[IDX3(b, d, n, D, N)] = h[n];
        }
    }
    free(h);
    return 0;
}

/* Block-confined reverse scan: for every block [jK, (j+1)K) the state starts
 * at zero after the block's last token and runs backwards to its first.
 *   y_rev [Bt, L, D] (required). */
int oracle_reverse_blocks(int64_t Bt, int64_t L, int64_t D, int64_t N, int64_t K,
                          const double *x, const double *dt, int dt_softplus,
                          const double *A, const double *B, const double *C,
                          const double *Dskip, double *y_rev) {
    if (Bt < 0 || L < 0 || D < 0 || N <= 0 || K <= 0 || (L % K) != 0 || !y_rev) return -1;
    double *g = (double *)malloc(sizeof(double) * (size_t)N);
    if (!g) return -1;
    for (int64_t b = 0; b < Bt; ++b) {
        for (int64_t d = 0; d < D; ++d) {
#if ORACLE_MUTANT == 3
            for (int64_t n = 0; n < N; ++n) g[n] = 0.0;
#endif
            for (int64_t j = L / K - 1; j >= 0; --j) {
#if ORACLE_MUTANT != 3
                for (int64_t n = 0; n < N; ++n) g[n] = 0.0;
#endif
                for (int64_t t = (j + 1) * K - 1; t >= j * K; --t) {
                    const double xv = x[IDX3(b, t, d, L, D)];
                    const double dl = delta_of(dt[IDX3(b, t, d, L, D)], dt_softplus);
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) {
#if ORACLE_MUTANT == 1
                        /* decay of the later token */
                        const double dnext = (t + 1 < (j + 1) * K)
                            ? delta_of(dt[IDX3(b, t + 1, d, L, D)], dt_softplus) : 0.0;
                        const double a = exp(dnext * A[d * N + n]);
#else
                        const double a = exp(dl * A[d * N + n]);
#endif
                        const double bt = dl * xv * B[IDX3(b, t, n, L, N)];
#if ORACLE_MUTANT == 4
                        acc += C[IDX3(b, t, n, L, N)] * g[n];
                        g[n] = a * g[n] + bt;
#else
                        g[n] = a * g[n] + bt;
                        acc += C[IDX3(b, t, n, L, N)] * g[n];
#endif
                    }
#if ORACLE_MUTANT == 2
                    y_rev[IDX3(b, t, d, L, D)] = acc;
#else
                    y_rev[IDX3(b, t, d, L, D)] = acc + Dskip[d] * xv;
#endif
                }
            }
        }
    }
    free(g);
    return 0;
}

/* y = (y_fwd + y_rev) * gate, gate = silu(z) when z is given, else 1.
 * y_rev may be NULL (forward-only output). n = element count. */
void oracle_combine(int64_t n, const double *y_fwd, const double *y_rev,
                    const double *z, double *y) {
    for (int64_t i = 0; i < n; ++i) {
        double v = y_fwd[i] + (y_rev ? y_rev[i] : 0.0);
        y[i] = z ? v * oracle_silu(z[i]) : v;
    }
}

/* Closed-form (matrix) evaluation for tiny sequences, in long double.
 * For each channel the output is written without any recurrence:
 *   y_t = sum_{s<=t} Mf[t,s] x_s + sum_{s>=t, same block} Mr[t,s] x_s
 *         + sum_n C_t[n] (prod_{r<=t} a_r[n]) h0[n] + 2 Dskip x_t,
 *   Mf[t,s] = sum_n C_t[n] (prod_{r=s+1..t} a_r[n]) delta_s B_s[n]
 *   Mr[t,s] = sum_n C_t[n] (prod_{r=t..s-1} a_r[n]) delta_s B_s[n]
 * then gated. Boundary states are the same explicit sums taken at block ends:
 *   h_e[n] = sum_{s<=e} (prod_{r=s+1..e} a_r[n]) delta_s x_s B_s[n]
 *            + (prod_{r<=e} a_r[n]) h0[n].
 * Every product is formed by explicit multiplication of exp() factors.
 * Requires L <= 64. y [Bt, L, D]; boundary [Bt, L/K, D, N] nullable. */
int oracle_bruteforce(int64_t Bt, int64_t L, int64_t D, int64_t N, int64_t K,
                      const double *x, const double *dt, int dt_softplus,
                      const double *A, const double *B, const double *C,
                      const double *Dskip, const double *z, const double *h0,
                      double *y, double *boundary) {
    if (Bt < 0 || L < 0 || L > 64 || D < 0 || N <= 0 || K <= 0 || (L % K) != 0 || !y) return -1;
    long double dl[64];
    for (int64_t b = 0; b < Bt; ++b) {
        for (int64_t d = 0; d < D; ++d) {
            for (int64_t t = 0; t < L; ++t) {
                double raw = dt[IDX3(b, t, d, L, D)];
                dl[t] = dt_softplus ? (long double)(raw > 0 ? raw : 0) + log1pl(expl(-fabsl((long double)raw)))
                                    : (long double)raw;
            }
            for (int64_t t = 0; t < L; ++t) {
                const int64_t blk0 = (t / K) * K, blk1 = blk0 + K; /* block of t */
                long double yt = 0.0L;
                for (int64_t s = 0; s < L; ++s) {
                    long double m = 0.0L;
                    for (int64_t n = 0; n < N; ++n) {
                        const long double An = (long double)A[d * N + n];
                        long double coef = 0.0L;
                        if (s <= t) { /* causal term */
                            long double p = 1.0L;
                            for (int64_t r = s + 1; r <= t; ++r) p *= expl(dl[r] * An);
                            coef += p;
                        }
                        if (s >= t && s >= blk0 && s < blk1) { /* in-block anti-causal term */
                            long double p = 1.0L;
                            for (int64_t r = t; r <= s - 1; ++r) p *= expl(dl[r] * An);
                            coef += p;
                        }
                        m += (long double)C[IDX3(b, t, n, L, N)] * coef * dl[s] *
                             (long double)B[IDX3(b, s, n, L, N)];
                    }
                    yt += m * (long double)x[IDX3(b, s, d, L, D)];
                }
                if (h0) {
                    for (int64_t n = 0; n < N; ++n) {
                        long double p = 1.0L;
                        for (int64_t r = 0; r <= t; ++r) p *= expl(dl[r] * (long double)A[d * N + n]);
                        yt += (long double)C[IDX3(b, t, n, L, N)] * p * (long double)h0[IDX3(b, d, n, D, N)];
                    }
                }
                yt += 2.0L * (long double)Dskip[d] * (long double)x[IDX3(b, t, d, L, D)];
                if (z) {
                    long double zv = (long double)z[IDX3(b, t, d, L, D)];
                    yt *= zv / (1.0L + expl(-zv));
                }
                y[IDX3(b, t, d, L, D)] = (double)yt;
            }
            if (boundary) {
                const int64_t nblk = L / K;
                for (int64_t j = 0; j < nblk; ++j) {
                    const int64_t e = (j + 1) * K - 1;
                    for (int64_t n = 0; n < N; ++n) {
                        const long double An = (long double)A[d * N + n];
                        long double hs = 0.0L;
                        for (int64_t s = 0; s <= e; ++s) {
                            long double p = 1.0L;
                            for (int64_t r = s + 1; r <= e; ++r) p *= expl(dl[r] * An);
                            hs += p * dl[s] * (long double)x[IDX3(b, s, d, L, D)] *
                                  (long double)B[IDX3(b, s, n, L, N)];
                        }
                        if (h0) {
                            long double p = 1.0L;
                            for (int64_t r = 0; r <= e; ++r) p *= expl(dl[r] * An);
                            hs += p * (long double)h0[IDX3(b, d, n, D, N)];
                        }
                        boundary[((b * nblk + j) * D + d) * N + n] = (double)hs;
                    }
                }
            }
        }
    }
    return 0;
}

/* Gradients of the all-block training output (forward over the whole
 * sequence plus the block-confined reverse scan, combined and gated) with
 * respect to every input, given dy = dLoss/dy [Bt, L, D]. The pages define
 * only the forward computation; the backward pass is its adjoint, derived
 * here by reverse-mode differentiation of the definition above:
 *   s_t  = sum_n C_t[n] (h_t[n] + g_t[n]) + 2 Dskip x_t,  y_t = s_t * gate_t
 *   ds_t = dy_t * gate_t,   dz_t = dy_t * s_t * silu'(z_t)
 *   lambda_t = dL/dh_t  = ds_t C_t + a_{t+1} lambda_{t+1}   (whole sequence,
 *              backwards from lambda_{L-1} = ds_{L-1} C_{L-1})
 *   mu_t     = dL/dg_t  = ds_t C_t + a_{t-1} mu_{t-1}       (inside the block,
 *              forwards from mu = ds C at the block's first token)
 *   db_t = lambda_t + mu_t,
 *   da_t = lambda_t h_{t-1} + mu_t g_{t+1}   (g after the block's last token = 0)
 *   dx_t     = 2 Dskip ds_t + sum_n db_t delta_t B_t
 *   ddelta_t = sum_n (da_t a_t A + db_t x_t B_t),  ddt_t = ddelta_t * sigmoid(dt_t)
 *              when delta = softplus(dt), else ddelta_t
 *   dB_t[n] = sum_d db_t delta_t x_t,  dC_t[n] = sum_d ds_t (h_t + g_t)
 *   dA[d,n] = sum_{b,t} da_t a_t delta_t,  dDskip[d] = sum_{b,t} 2 x_t ds_t
 *   dh0 = a_0 lambda_0.
 * Every h_t and g_t is stored for the whole sequence (no recomputation).
 * Outputs: dx, ddt [Bt, L, D]; dz [Bt, L, D] (only with z, else ignored);
 * dB, dC [Bt, L, N]; dA [D, N]; dDskip [D]; dh0 [Bt, D, N] (nullable).
 * All are overwritten. Returns 0, or -1 on bad sizes / allocation failure. */
int oracle_train_blocks_backward(int64_t Bt, int64_t L, int64_t D, int64_t N, int64_t K,
                                 const double *x, const double *dt, int dt_softplus,
                                 const double *A, const double *B, const double *C,
                                 const double *Dskip, const double *z, const double *h0,
                                 const double *dy,
                                 double *dx, double *ddt, double *dz, double *dB, double *dC,
                                 double *dA, double *dDskip, double *dh0) {
    if (Bt < 0 || L < 0 || D < 0 || N <= 0 || K <= 0 || (L % K) != 0) return -1;
    if (!dx || !ddt || !dB || !dC || !dA || !dDskip || (z && !dz)) return -1;
    const size_t LN = (size_t)(L > 0 ? L : 1) * (size_t)N;
    double *dl = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double *a = (double *)malloc(sizeof(double) * LN);    /* a_t[n] */
    double *h = (double *)malloc(sizeof(double) * (LN + (size_t)N)); /* h_{t-1}: row t holds h_{t-1}, row L holds h_{L-1} */
    double *g = (double *)malloc(sizeof(double) * LN);    /* g_t[n] */
    double *ds = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double *lam = (double *)malloc(sizeof(double) * LN);
    double *mu = (double *)malloc(sizeof(double) * LN);
    if (!dl || !a || !h || !g || !ds || !lam || !mu) {
        free(dl); free(a); free(h); free(g); free(ds); free(lam); free(mu);
        return -1;
    }
    memset(dB, 0, sizeof(double) * (size_t)(Bt * L * N));
    memset(dC, 0, sizeof(double) * (size_t)(Bt * L * N));
    memset(dA, 0, sizeof(double) * (size_t)(D * N));
    memset(dDskip, 0, sizeof(double) * (size_t)D);
    for (int64_t b = 0; b < Bt; ++b) {
        for (int64_t d = 0; d < D; ++d) {
            /* recompute the forward quantities of this channel */
            for (int64_t t = 0; t < L; ++t) {
                dl[t] = delta_of(dt[IDX3(b, t, d, L, D)], dt_softplus);
                for (int64_t n = 0; n < N; ++n) a[t * N + n] = exp(dl[t] * A[d * N + n]);
            }
            for (int64_t n = 0; n < N; ++n) h[n] = h0 ? h0[IDX3(b, d, n, D, N)] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const double xv = x[IDX3(b, t, d, L, D)];
                for (int64_t n = 0; n < N; ++n)
                    h[(t + 1) * N + n] = a[t * N + n] * h[t * N + n] + dl[t] * xv * B[IDX3(b, t, n, L, N)];
            }
            for (int64_t t = L - 1; t >= 0; --t) {
                const int block_end = ((t + 1) % K) == 0;
                const double xv = x[IDX3(b, t, d, L, D)];
                for (int64_t n = 0; n < N; ++n) {
                    const double gnext = block_end ? 0.0 : g[(t + 1) * N + n];
                    g[t * N + n] = a[t * N + n] * gnext + dl[t] * xv * B[IDX3(b, t, n, L, N)];
                }
            }
            /* output stage: s, the gate and its derivative */
            for (int64_t t = 0; t < L; ++t) {
                const int64_t i = IDX3(b, t, d, L, D);
                double s = 2.0 * Dskip[d] * x[i];
                for (int64_t n = 0; n < N; ++n)
                    s += C[IDX3(b, t, n, L, N)] * (h[(t + 1) * N + n] + g[t * N + n]);
                if (z) {
                    const double sg = 1.0 / (1.0 + exp(-z[i]));
                    ds[t] = dy[i] * z[i] * sg;
                    dz[i] = dy[i] * s * sg * (1.0 + z[i] * (1.0 - sg));
                } else {
                    ds[t] = dy[i];
                }
            }
            /* adjoint of the forward state, over the whole sequence */
            for (int64_t t = L - 1; t >= 0; --t) {
                for (int64_t n = 0; n < N; ++n) {
                    double v = ds[t] * C[IDX3(b, t, n, L, N)];
#if ORACLE_MUTANT == 9
                    if (t + 1 < L && ((t + 1) % K) != 0) v += a[(t + 1) * N + n] * lam[(t + 1) * N + n];
#else
                    if (t + 1 < L) v += a[(t + 1) * N + n] * lam[(t + 1) * N + n];
#endif
                    lam[t * N + n] = v;
                }
            }
            /* adjoint of the reverse state, inside each block */
            for (int64_t t = 0; t < L; ++t) {
                const int block_start = (t % K) == 0;
                for (int64_t n = 0; n < N; ++n) {
                    double v = ds[t] * C[IDX3(b, t, n, L, N)];
#if ORACLE_MUTANT == 8
                    if (!block_start) v += a[t * N + n] * mu[(t - 1) * N + n];
#else
                    if (!block_start) v += a[(t - 1) * N + n] * mu[(t - 1) * N + n];
#endif
                    mu[t * N + n] = v;
                }
            }
            /* gradients of the inputs */
            double dskip_acc = 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t i = IDX3(b, t, d, L, D);
                const double xv = x[i];
                const int block_end = ((t + 1) % K) == 0;
                double dxv = 2.0 * Dskip[d] * ds[t];
                double ddl = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double Bv = B[IDX3(b, t, n, L, N)];
                    const double dbv = lam[t * N + n] + mu[t * N + n];
                    const double gnext = block_end ? 0.0 : g[(t + 1) * N + n];
#if ORACLE_MUTANT == 10
                    const double dav = lam[t * N + n] * h[t * N + n];
                    (void)gnext;
#else
                    const double dav = lam[t * N + n] * h[t * N + n] + mu[t * N + n] * gnext;
#endif
                    dxv += dbv * dl[t] * Bv;
                    ddl += dav * a[t * N + n] * A[d * N + n] + dbv * xv * Bv;
                    dB[IDX3(b, t, n, L, N)] += dbv * dl[t] * xv;
                    dC[IDX3(b, t, n, L, N)] += ds[t] * (h[(t + 1) * N + n] + g[t * N + n]);
                    dA[d * N + n] += dav * a[t * N + n] * dl[t];
                }
                dx[i] = dxv;
#if ORACLE_MUTANT == 11
                ddt[i] = ddl;
#else
                ddt[i] = dt_softplus ? ddl / (1.0 + exp(-dt[i])) : ddl;
#endif
                dskip_acc += 2.0 * xv * ds[t];
            }
            dDskip[d] += dskip_acc;
            if (dh0)
                for (int64_t n = 0; n < N; ++n)
#if ORACLE_MUTANT == 12
                    dh0[IDX3(b, d, n, D, N)] = L > 0 ? lam[n] : 0.0;
#else
                    dh0[IDX3(b, d, n, D, N)] = L > 0 ? a[n] * lam[n] : 0.0;
#endif
        }
    }
    free(dl); free(a); free(h); free(g); free(ds); free(lam); free(mu);
    return 0;
}

int oracle_mutant_id(void) { return ORACLE_MUTANT; }
