/*
 * oracle_ssm.c -- plain, slow, sequential fp64 oracle of the Mamba-1 selective
 * scan (S6) and of its one-token decode state update.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; it is used by the tests, by the smoke check and by the CPU
 * baseline leg of the benchmark.  It shares no code, header, table or constant
 * with the CUDA library.
 *
 * What it computes (sources):
 *   - "Jamba: A Hybrid Transformer-Mamba Language Model" (obsidian-dorae222
 *     notes), section "Mamba 레이어" (Mamba layer): the selective SSM
 *         h_t = Abar_t h_{t-1} + Bbar_t x_t ,   y_t = C_t h_t ,
 *     with Bbar_t, C_t, Delta_t produced from the input (selectivity), state
 *     size d_state = 16, expansion factor 2.
 *   - "Jamba -- Hybrid SSM-Transformer" (factory.pai-world.com lesson), section
 *     "한 페이지로 보는 SSM" (SSM on one page): y_t needs only h_{t-1} and x_t,
 *     constant memory, O(1) work per token -- the decode update below.
 *   - same lesson, "Mamba-3" item 2: Mamba's state matrix is real diagonal, so
 *     every (channel d, state n) pair is an independent scalar recurrence.
 * The pages print only the symbols Abar, Bbar.  Readings taken where they are
 * silent:
 *   - discretisation: Abar = exp(Delta * A[d,n]),  Bbar x = Delta * B[t,n] * x;
 *   - Delta = softplus(delta + delta_bias[d]) when delta_softplus != 0, else
 *     Delta = delta + delta_bias[d];
 *   - output: out = (sum_n C[t,n] h[n] + D[d] x) * silu(z), silu(z) = z/(1+e^-z).
 *
 * Everything is evaluated in the order the definition states: channel by
 * channel, step by step, state by state, in double precision.
 *
 * Parity: this file is pinned by tests/test_oracle_pins.py (brute-force
 * unrolled sums, the geometric-series closed form, the Delta->0 and large-Delta
 * limits, libm softplus/silu, split-scan and decode==scan identities) and, for
 * the projection that produces Delta, B and C, by tests/oracle_proj_pins.py
 * (basis-vector selections, associativity, rank, RMSNorm closed forms), and the
 * reverse-mode gradient of the scan by tests/oracle_bwd_pins.py (central finite
 * differences of the forward scan, closed forms of the state gradient).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

/* softplus(v) = log(1 + e^v), written in the form that does not overflow. */
double oracle_softplus(double v) {
    if (v > 0.0) return v + log1p(exp(-v));
    return log1p(exp(v));
}

/* silu(z) = z * sigmoid(z) = z / (1 + e^-z). */
double oracle_silu(double z) {
    return z / (1.0 + exp(-z));
}

/* Delta for one (t, d): the raw input plus the per-channel bias, through
 * softplus when requested. */
static double oracle_delta(double raw, const double *delta_bias, int64_t d,
                           int delta_softplus) {
    double v = raw + (delta_bias ? delta_bias[d] : 0.0);
    return delta_softplus ? oracle_softplus(v) : v;
}

/*
 * Prefill scan over channels [d_lo, d_hi) of every sequence.
 *   x, delta, z : [batch, seqlen, d_inner]
 *   B, C        : [batch, seqlen, d_state]
 *   A           : [d_inner, d_state]
 *   D, delta_bias : [d_inner] or NULL (zero)
 *   h0          : [batch, d_inner, d_state] or NULL (zero initial state)
 *   out         : [batch, seqlen, d_inner]             (written for d in range)
 *   h_final     : [batch, d_inner, d_state] or NULL    (written for d in range)
 * The channel range only selects which independent recurrences to run, so a
 * caller may split [0, d_inner) across threads.  Returns 0, or -1 on a bad
 * argument.
 */
int oracle_scan_f64(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                    int64_t d_lo, int64_t d_hi,
                    const double *x, const double *delta, const double *z,
                    const double *B, const double *C, const double *A,
                    const double *D, const double *delta_bias, int delta_softplus,
                    const double *h0, double *out, double *h_final) {
    if (batch < 0 || seqlen < 0 || d_inner < 0 || d_state < 1 || d_state > 64)
        return -1;
    if (d_lo < 0 || d_hi > d_inner || d_lo > d_hi) return -1;
    double h[64];
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = d_lo; d < d_hi; ++d) {
            for (int64_t n = 0; n < d_state; ++n)
                h[n] = h0 ? h0[(b * d_inner + d) * d_state + n] : 0.0;
            for (int64_t t = 0; t < seqlen; ++t) {
                int64_t i = (b * seqlen + t) * d_inner + d;
                const double *Bt = B + (b * seqlen + t) * d_state;
                const double *Ct = C + (b * seqlen + t) * d_state;
                double xv = x[i];
                double dv = oracle_delta(delta[i], delta_bias, d, delta_softplus);
                double y = 0.0;
                for (int64_t n = 0; n < d_state; ++n) {
                    double abar = exp(dv * A[d * d_state + n]);
                    double bbar_x = dv * Bt[n] * xv;
                    h[n] = abar * h[n] + bbar_x;
                    y += Ct[n] * h[n];
                }
                double skip = D ? D[d] * xv : 0.0;
                out[i] = (y + skip) * oracle_silu(z[i]);
            }
            if (h_final)
                for (int64_t n = 0; n < d_state; ++n)
                    h_final[(b * d_inner + d) * d_state + n] = h[n];
        }
    }
    return 0;
}

/*
 * One decode step for every request: the same recurrence for a single token,
 * reading the cached state and writing the new state in place.
 *   state : [batch, d_inner, d_state]  (in/out)
 *   x, delta, z, out : [batch, d_inner]
 *   B, C  : [batch, d_state]
 */
int oracle_state_update_f64(int64_t batch, int64_t d_inner, int64_t d_state,
                            double *state,
                            const double *x, const double *delta, const double *z,
                            const double *B, const double *C, const double *A,
                            const double *D, const double *delta_bias,
                            int delta_softplus, double *out) {
    if (batch < 0 || d_inner < 0 || d_state < 1) return -1;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < d_inner; ++d) {
            int64_t i = b * d_inner + d;
            double *h = state + i * d_state;
            double xv = x[i];
            double dv = oracle_delta(delta[i], delta_bias, d, delta_softplus);
            double y = 0.0;
            for (int64_t n = 0; n < d_state; ++n) {
                double abar = exp(dv * A[d * d_state + n]);
                double bbar_x = dv * B[b * d_state + n] * xv;
                h[n] = abar * h[n] + bbar_x;
                y += C[b * d_state + n] * h[n];
            }
            double skip = D ? D[d] * xv : 0.0;
            out[i] = (y + skip) * oracle_silu(z[i]);
        }
    }
    return 0;
}

/*
 * The step before the scan: "Bbar_t, C_t, Delta_t = f(x_t)" (obsidian-dorae222
 * notes, section "Mamba 레이어"), with the RMSNorm the same section says Jamba
 * adds to the Mamba layer against training instability.  The pages do not
 * spell f out; the reading taken is the Mamba-1 one:
 *   xdbl_t  = W_x u_t                        (one linear map of the token)
 *   dt_low  = xdbl_t[0 .. R-1],  B_t = xdbl_t[R .. R+N-1],  C_t = xdbl_t[R+N .. R+2N-1]
 *   each of dt_low, B_t, C_t optionally RMS-normalised over its own entries:
 *       v_i <- w_i * v_i / sqrt(mean_j v_j^2 + eps)
 *   delta_t = W_dt dt_low                    (low-rank, rank R = dt_rank)
 * delta is the raw input of the scan: the per-channel bias and the softplus are
 * the scan's own first step, so they are not applied here.
 *   u      : [ntok, d_inner]
 *   W_x    : [dt_rank + 2 * d_state, d_inner]
 *   W_dt   : [d_inner, dt_rank]
 *   w_dt, w_B, w_C : RMSNorm weights [dt_rank], [d_state], [d_state], or NULL
 *            (no normalisation of that part)
 *   delta  : [ntok, d_inner]      B, C : [ntok, d_state]
 *   dt_low_out : [ntok, dt_rank] (after its RMSNorm), or NULL
 * Tokens [t_lo, t_hi) are computed, so a caller may split them across threads.
 * Returns 0, or -1 on a bad argument.
 */
static void oracle_rmsnorm(double *v, int64_t len, const double *w, double eps) {
    double ss = 0.0;
    for (int64_t i = 0; i < len; ++i) ss += v[i] * v[i];
    double inv = 1.0 / sqrt(ss / (double)len + eps);
    for (int64_t i = 0; i < len; ++i) v[i] = w[i] * (v[i] * inv);
}

/* delta_row[d] = sum_r W_dt[d, r] * dt_low[r]: the rank-R map of one token. */
static void oracle_low_rank_row(int64_t d_inner, int64_t dt_rank, const double *W_dt,
                                const double *dt_low, double *delta_row) {
    for (int64_t d = 0; d < d_inner; ++d) {
        double acc = 0.0;
        for (int64_t r = 0; r < dt_rank; ++r) acc += W_dt[d * dt_rank + r] * dt_low[r];
        delta_row[d] = acc;
    }
}

int oracle_project_f64(int64_t ntok, int64_t d_inner, int64_t dt_rank, int64_t d_state,
                       int64_t t_lo, int64_t t_hi,
                       const double *u, const double *W_x, const double *W_dt,
                       const double *w_dt, const double *w_B, const double *w_C, double eps,
                       double *delta, double *B, double *C, double *dt_low_out) {
    if (ntok < 0 || d_inner < 1 || dt_rank < 1 || d_state < 1) return -1;
    if (t_lo < 0 || t_hi > ntok || t_lo > t_hi || !(eps >= 0.0)) return -1;
    int64_t rows = dt_rank + 2 * d_state;
    double *xdbl = (double *)malloc((size_t)rows * sizeof(double));
    if (!xdbl) return -1;
    for (int64_t t = t_lo; t < t_hi; ++t) {
        const double *ut = u + t * d_inner;
        for (int64_t j = 0; j < rows; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < d_inner; ++k) acc += W_x[j * d_inner + k] * ut[k];
            xdbl[j] = acc;
        }
        double *dt_low = xdbl, *Bv = xdbl + dt_rank, *Cv = xdbl + dt_rank + d_state;
        if (w_dt) oracle_rmsnorm(dt_low, dt_rank, w_dt, eps);
        if (w_B) oracle_rmsnorm(Bv, d_state, w_B, eps);
        if (w_C) oracle_rmsnorm(Cv, d_state, w_C, eps);
        for (int64_t n = 0; n < d_state; ++n) {
            B[t * d_state + n] = Bv[n];
            C[t * d_state + n] = Cv[n];
        }
        if (dt_low_out)
            for (int64_t r = 0; r < dt_rank; ++r) dt_low_out[t * dt_rank + r] = dt_low[r];
        oracle_low_rank_row(d_inner, dt_rank, W_dt, dt_low, delta + t * d_inner);
    }
    free(xdbl);
    return 0;
}

/*
 * The last product of the step alone, for tokens [t_lo, t_hi):
 *   delta[t, d] = sum_r W_dt[d, r] * dt_low[t, r]
 *   dt_low : [ntok, dt_rank]   W_dt : [d_inner, dt_rank]   delta : [ntok, d_inner]
 */
int oracle_dt_proj_f64(int64_t ntok, int64_t d_inner, int64_t dt_rank, int64_t t_lo,
                       int64_t t_hi, const double *dt_low, const double *W_dt, double *delta) {
    if (ntok < 0 || d_inner < 1 || dt_rank < 1) return -1;
    if (t_lo < 0 || t_hi > ntok || t_lo > t_hi) return -1;
    for (int64_t t = t_lo; t < t_hi; ++t)
        oracle_low_rank_row(d_inner, dt_rank, W_dt, dt_low + t * dt_rank, delta + t * d_inner);
    return 0;
}

/*
 * Reverse-mode gradient of the prefill scan (training: the backward pass of
 * the layer).  The caller's scalar loss has gradient dout with respect to out
 * [batch, seqlen, d_inner] and dh_final with respect to h_final [batch,
 * d_inner, d_state] (NULL: zero).  For the channels in [d_lo, d_hi):
 *   written:      dx, ddelta, dz   [batch, seqlen, d_inner]   (ddelta is the
 *                 gradient of the raw step input)
 *                 dh0              [batch, d_inner, d_state] or NULL
 *   accumulated:  dA [d_inner, d_state], dD [d_inner], ddelta_bias [d_inner]
 *                 (each may be NULL), dB, dC [batch, seqlen, d_state]
 *                 (summed over the channels in range; the caller zeroes them).
 * The forward recurrence is re-run per channel, keeping every state, and the
 * chain rule is applied in reverse time:
 *   g      = dL/dh_t  = dy_t C_t + Abar_{t+1} * g_{t+1}   (g_L = dh_final)
 *   dAbar  = g * h_{t-1},  dDelta += dAbar * Abar * A + g * B_t x_t,
 *   dA    += dAbar * Abar * Delta,  dB_t += g Delta x_t,  dx_t += g Delta B_t,
 * with dy_t = dout_t silu(z_t), dz_t = dout_t y_t silu'(z_t),
 * silu'(z) = s (1 + z (1 - s)) for s = 1/(1+e^-z), and softplus'(v) = 1/(1+e^-v).
 */
int oracle_scan_bwd_f64(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                        int64_t d_lo, int64_t d_hi,
                        const double *x, const double *delta, const double *z,
                        const double *B, const double *C, const double *A,
                        const double *D, const double *delta_bias, int delta_softplus,
                        const double *h0, const double *dout, const double *dh_final,
                        double *dx, double *ddelta, double *dz, double *dB, double *dC,
                        double *dA, double *dD, double *ddelta_bias, double *dh0) {
    if (batch < 0 || seqlen < 0 || d_inner < 0 || d_state < 1 || d_state > 64) return -1;
    if (d_lo < 0 || d_hi > d_inner || d_lo > d_hi) return -1;
    double *hs = (double *)malloc((size_t)(seqlen + 1) * (size_t)d_state * sizeof(double));
    if (!hs) return -1;
    double g[64];
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = d_lo; d < d_hi; ++d) {
            /* forward, keeping h_{-1} = h0 in hs[0..N) and h_t in hs[(t+1)N ..) */
            for (int64_t n = 0; n < d_state; ++n)
                hs[n] = h0 ? h0[(b * d_inner + d) * d_state + n] : 0.0;
            for (int64_t t = 0; t < seqlen; ++t) {
                int64_t i = (b * seqlen + t) * d_inner + d;
                const double *Bt = B + (b * seqlen + t) * d_state;
                double dv = oracle_delta(delta[i], delta_bias, d, delta_softplus);
                for (int64_t n = 0; n < d_state; ++n)
                    hs[(t + 1) * d_state + n] = exp(dv * A[d * d_state + n]) * hs[t * d_state + n] +
                                                dv * Bt[n] * x[i];
            }
            /* backward */
            for (int64_t n = 0; n < d_state; ++n)
                g[n] = dh_final ? dh_final[(b * d_inner + d) * d_state + n] : 0.0;
            for (int64_t t = seqlen - 1; t >= 0; --t) {
                int64_t i = (b * seqlen + t) * d_inner + d;
                const double *Bt = B + (b * seqlen + t) * d_state;
                const double *Ct = C + (b * seqlen + t) * d_state;
                double *dBt = dB + (b * seqlen + t) * d_state;
                double *dCt = dC + (b * seqlen + t) * d_state;
                const double *h_now = hs + (t + 1) * d_state, *h_prev = hs + t * d_state;
                double v = delta[i] + (delta_bias ? delta_bias[d] : 0.0);
                double dv = delta_softplus ? oracle_softplus(v) : v;
                double xv = x[i], Dd = D ? D[d] : 0.0;
                double y = Dd * xv;
                for (int64_t n = 0; n < d_state; ++n) y += Ct[n] * h_now[n];
                double sz = 1.0 / (1.0 + exp(-z[i]));
                double dy = dout[i] * (z[i] * sz);
                dz[i] = dout[i] * y * sz * (1.0 + z[i] * (1.0 - sz));
                if (dD) dD[d] += dy * xv;
                double dxi = dy * Dd, dDelta = 0.0;
                for (int64_t n = 0; n < d_state; ++n) {
                    g[n] += dy * Ct[n];
                    dCt[n] += dy * h_now[n];
                }
                for (int64_t n = 0; n < d_state; ++n) {
                    double an = A[d * d_state + n];
                    double abar = exp(dv * an);
                    double dabar = g[n] * h_prev[n];
                    dDelta += dabar * abar * an + g[n] * Bt[n] * xv;
                    if (dA) dA[d * d_state + n] += dabar * abar * dv;
                    dBt[n] += g[n] * dv * xv;
                    dxi += g[n] * dv * Bt[n];
                    g[n] = abar * g[n];
                }
                double draw = delta_softplus ? dDelta / (1.0 + exp(-v)) : dDelta;
                ddelta[i] = draw;
                if (ddelta_bias) ddelta_bias[d] += draw;
                dx[i] = dxi;
            }
            if (dh0)
                for (int64_t n = 0; n < d_state; ++n) dh0[(b * d_inner + d) * d_state + n] = g[n];
        }
    }
    free(hs);
    return 0;
}

/*
 * The scalar-identity variant of the selective SSM (Mamba-2's state matrix):
 * "Jamba -- Hybrid SSM-Transformer" (factory.pai-world.com lesson), section
 * "Mamba-3: 2026년의 순수 SSM 기준선", item 2: the state matrix went from
 * complex (S4) to real diagonal (Mamba) to a scaled identity (Mamba-2); item 1
 * of the same list: Mamba-2 discretises with the Euler method.  Reading (the
 * pages print no equations of this variant): d_inner = nheads * headdim
 * channels, channel d = head * headdim + p; each head has one scalar A[head]
 * and one step size per token, Delta[t, head] = softplus(delta[t, head] +
 * delta_bias[head]) (or without softplus); every channel of the head keeps
 * d_state states
 *     h[n] = exp(Delta A[head]) h[n] + Delta B[t, n] x[t, d],
 *     out  = (sum_n C[t, n] h[n] + D[d] x[t, d]) silu(z[t, d]).
 *
 * Heads [h_lo, h_hi) of every sequence; layouts:
 *   x, z, out : [batch, seqlen, nheads * headdim]
 *   delta     : [batch, seqlen, nheads]
 *   B, C      : [batch, seqlen, d_state]
 *   A, delta_bias : [nheads] (delta_bias may be NULL)
 *   D         : [nheads * headdim] or NULL
 *   h0, h_final : [batch, nheads * headdim, d_state] (h0, h_final may be NULL)
 */
int oracle_ssd_scan_f64(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                        int64_t d_state, int64_t h_lo, int64_t h_hi, const double *x,
                        const double *delta, const double *z, const double *B, const double *C,
                        const double *A, const double *D, const double *delta_bias,
                        int delta_softplus, const double *h0, double *out, double *h_final) {
    if (batch < 0 || seqlen < 0 || nheads < 0 || headdim < 1 || d_state < 1 || d_state > 64)
        return -1;
    if (h_lo < 0 || h_hi > nheads || h_lo > h_hi) return -1;
    const int64_t d_inner = nheads * headdim;
    double h[64];
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t hd = h_lo; hd < h_hi; ++hd) {
            for (int64_t p = 0; p < headdim; ++p) {
                const int64_t d = hd * headdim + p;
                for (int64_t n = 0; n < d_state; ++n)
                    h[n] = h0 ? h0[(b * d_inner + d) * d_state + n] : 0.0;
                for (int64_t t = 0; t < seqlen; ++t) {
                    const double v = delta[(b * seqlen + t) * nheads + hd] +
                                     (delta_bias ? delta_bias[hd] : 0.0);
                    const double dv = delta_softplus ? oracle_softplus(v) : v;
                    const double decay = exp(dv * A[hd]);  /* one scalar for every state */
                    const int64_t i = (b * seqlen + t) * d_inner + d;
                    const double *Bt = B + (b * seqlen + t) * d_state;
                    const double *Ct = C + (b * seqlen + t) * d_state;
                    double y = 0.0;
                    for (int64_t n = 0; n < d_state; ++n) {
                        h[n] = decay * h[n] + dv * Bt[n] * x[i];
                        y += Ct[n] * h[n];
                    }
                    y += (D ? D[d] : 0.0) * x[i];
                    out[i] = y * oracle_silu(z[i]);
                }
                if (h_final)
                    for (int64_t n = 0; n < d_state; ++n) h_final[(b * d_inner + d) * d_state + n] = h[n];
            }
        }
    }
    return 0;
}
