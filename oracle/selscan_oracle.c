/*
 * selscan_oracle.c -- plain float64 CPU reference of the Mamba-1 selective
 * scan and of its single-token recurrent state update.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the ground truth the CUDA library is
 * checked against. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg load it. It shares no code, header, table or constant with
 * the CUDA sources, and the product path never calls it.
 *
 * Every loop below is the plain definition, one (batch, channel) chain at a
 * time, each chain strictly sequential in t. OpenMP only spreads independent
 * chains over cores; it does not reorder any chain's arithmetic.
 *
 * Pages followed (title, section):
 *  [Guide] "Mamba & State Space Models — Guide Complet" (skillsmp.com skill
 *          "mamba-ssm"):
 *          §1 "Discrétisation": ZOH, A_bar = exp(Δ·A),
 *             B_bar = (exp(Δ·A) − I)·A⁻¹·B; h_k = A_bar·h_{k−1} + B_bar·u_k,
 *             y_k = C·h_k + D·u_k.
 *          §4 "Implémentation du SSM sélectif (S6)": Δ = softplus(dt_proj(x))
 *             with the bias inside the softplus; per token A_bar = exp(Δ_t·A)
 *             with A diagonal per channel; h starts at zero; y_t = h·C_t + D·x_t
 *             with D a per-channel vector.
 *          §4 "Parallel Associative Scan": (a,b)⊕(a',b') = (a·a', a·b' + b).
 *  [Johe]  "Mamba и State Space Models: альтернатива Transformer"
 *          (johe.ru/blog/mamba-ssm):
 *          "SSM as RNN": input term scaled by delta, y read after the update.
 *          "Discretization": delta_bias added to the projected Δ.
 *          "Hardware-Aware Scan": the state is carried across fixed-size
 *             blocks of the sequence.
 *          "Mamba Block": output gated by silu(gate).
 *
 * Readings where the pages are garbled or silent:
 *  - The input term on the hot path is B_bar·x = Δ·B·x (the delta-scaled B of
 *    [Johe] "SSM as RNN"), with the x that page's ssm_step drops restored.
 *    The ZOH coefficient (exp(Δ·A) − 1)/A of [Guide] §1 is kept as a second
 *    mode (bbar_mode = 1) for the discretization pins.
 *  - A is used as given (negative for a stable scan); no epsilon or clamp is
 *    added to Δ; D·x is added before the gate; silu is applied once.
 *
 * Layouts (row-major, last index fastest): x, delta, z, y [batch, L, D];
 * B, C [batch, L, N]; A [D, N]; Dv, delta_bias [D]; states [batch, D, N].
 * Null Dv / delta_bias / h0 mean zero; null z means no gate; null
 * final_state means the final state is not returned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BBAR_DELTA 0 /* B_bar = Δ·B   ([Johe] "SSM as RNN")        */
#define ORACLE_BBAR_ZOH 1   /* B_bar = (exp(Δ·A) − 1)/A·B ([Guide] §1)    */

/* softplus(v) = log(1 + e^v), written so that neither branch overflows. */
static double softplus(double v)
{
    return v > 0.0 ? v + log1p(exp(-v)) : log1p(exp(v));
}

/* silu(z) = z·sigmoid(z) ([Johe] "Mamba Block", y * silu(gate)). */
static double silu(double z)
{
    return z / (1.0 + exp(-z));
}

/* Δ for one (token, channel): bias inside the softplus ([Guide] §4,
 * [Johe] "Discretization"). */
static double step_size(double delta, const double *delta_bias, int64_t d,
                        int softplus_flag)
{
    double v = delta + (delta_bias ? delta_bias[d] : 0.0);
    return softplus_flag ? softplus(v) : v;
}

/* Input coefficient multiplying B[n]·x: Δ, or the diagonal ZOH factor
 * (exp(Δ·a) − 1)/a, whose a → 0 limit is Δ. */
static double bbar_coeff(double dt, double a, int bbar_mode)
{
    if (bbar_mode == ORACLE_BBAR_ZOH)
        return a == 0.0 ? dt : expm1(dt * a) / a;
    return dt;
}

/* The ZOH coefficient c = (exp(Δ·a) − 1)/a of [Guide] §1 and its partial
 * derivatives: ∂c/∂Δ = exp(Δ·a) (for every a, including the limit a → 0),
 * ∂c/∂a = (z·exp(z) − (exp(z) − 1))/a² = Δ²·(z·exp(z) − expm1(z))/z² with
 * z = Δ·a, whose z → 0 limit is Δ²/2 (the series 1/2 + z/3 + z²/8 below
 * |z| = 1e-4). */
static void zoh_coeff_grads(double dt, double a, double *c, double *c_dt, double *c_a)
{
    double z = dt * a;
    *c = a == 0.0 ? dt : expm1(z) / a;
    *c_dt = exp(z);
    if (fabs(z) < 1e-4)
        *c_a = dt * dt * (0.5 + z / 3.0 + z * z / 8.0);
    else
        *c_a = dt * dt * (z * exp(z) - expm1(z)) / (z * z);
}

/*
 * One token of one channel: the discrete recurrence of [Guide] §1/§4 with the
 * selective (per-token) Δ, B, C. Updates h[0..N) in place and returns the
 * gated output.
 */
static double token_update(double *h, double xv, double dt, const double *Arow,
                           const double *Bt, const double *Ct, double dskip,
                           const double *zv, int64_t N, int bbar_mode)
{
    double acc = 0.0;
    for (int64_t n = 0; n < N; ++n) {
        double a_bar = exp(dt * Arow[n]);
        double b_bar = bbar_coeff(dt, Arow[n], bbar_mode) * Bt[n];
        h[n] = a_bar * h[n] + b_bar * xv;
        acc += Ct[n] * h[n]; /* y reads the state after the update */
    }
    double out = acc + dskip * xv;
    if (zv)
        out *= silu(*zv);
    return out;
}

/*
 * Selective scan over a whole sequence.
 * h0 (nullable, [batch, D, N]) is the state before token 0 (zero if null).
 */
void oracle_selscan_fwd(const double *x, const double *delta, const double *A,
                        const double *B, const double *C, const double *Dv,
                        const double *z, const double *delta_bias,
                        int softplus_flag, int bbar_mode, const double *h0,
                        double *y, double *final_state, int64_t batch,
                        int64_t L, int64_t D, int64_t N, int nthreads)
{
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for collapse(2) schedule(dynamic, 1) num_threads(nthreads)
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < D; ++d) {
            double *h = (double *)malloc((size_t)N * sizeof(double));
            for (int64_t n = 0; n < N; ++n)
                h[n] = h0 ? h0[(b * D + d) * N + n] : 0.0;
            const double *Arow = A + d * N;
            double dskip = Dv ? Dv[d] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                int64_t i = (b * L + t) * D + d;
                int64_t j = (b * L + t) * N;
                double dt = step_size(delta[i], delta_bias, d, softplus_flag);
                y[i] = token_update(h, x[i], dt, Arow, B + j, C + j, dskip,
                                    z ? z + i : NULL, N, bbar_mode);
            }
            if (final_state)
                for (int64_t n = 0; n < N; ++n)
                    final_state[(b * D + d) * N + n] = h[n];
            free(h);
        }
    }
}

/*
 * Single-token recurrent update used at inference: the same token step,
 * applied in place to a carried state ([Johe] "SSM as Convolution":
 * recurrent mode for inference; [Guide] §6: O(1) state instead of a cache).
 * x, delta, z [batch, D]; B, C [batch, N]; state [batch, D, N]; y [batch, D].
 */
void oracle_state_update(double *state, const double *x, const double *delta,
                         const double *A, const double *B, const double *C,
                         const double *Dv, const double *z,
                         const double *delta_bias, int softplus_flag,
                         double *y, int64_t batch, int64_t D, int64_t N)
{
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < D; ++d) {
            int64_t i = b * D + d;
            double dt = step_size(delta[i], delta_bias, d, softplus_flag);
            y[i] = token_update(state + i * N, x[i], dt, A + d * N, B + b * N,
                                C + b * N, Dv ? Dv[d] : 0.0, z ? z + i : NULL, N,
                                ORACLE_BBAR_DELTA);
        }
    }
}

/*
 * The associative operator of [Guide] §4 "Parallel Associative Scan" for the
 * affine maps h -> a·h + b. The page writes (a,b)⊕(a',b') = (a·a', a·b' + b),
 * which composes correctly when the left operand is the LATER element; here
 * the later element is named explicitly: the result applies `earlier` first,
 * then `later`.
 */
void oracle_compose(double a_later, double b_later, double a_earlier,
                    double b_earlier, double *a_out, double *b_out)
{
    *a_out = a_later * a_earlier;
    *b_out = a_later * b_earlier + b_later;
}

/*
 * Chunked form of the same scan ([Johe] "Hardware-Aware Scan": fixed-size
 * blocks with the state carried between them; [Guide] §4 operator):
 *   1. per chunk c, from a zero state: P_c[n] = product of A_bar over the
 *      chunk, H_c[n] = the chunk's own final state;
 *   2. carry: hin_0 = h0, hin_{c+1} = (P_c, H_c) ∘ hin_c;
 *   3. rescan every chunk from hin_c to produce y.
 * The final state is hin after the last chunk. Must equal oracle_selscan_fwd
 * up to rounding order.
 */
void oracle_selscan_fwd_chunked(const double *x, const double *delta,
                                const double *A, const double *B,
                                const double *C, const double *Dv,
                                const double *z, const double *delta_bias,
                                int softplus_flag, int bbar_mode,
                                const double *h0, double *y,
                                double *final_state, int64_t batch, int64_t L,
                                int64_t D, int64_t N, int64_t chunk,
                                int nthreads)
{
    if (chunk < 1)
        chunk = 1;
    if (nthreads < 1)
        nthreads = 1;
    int64_t nchunks = (L + chunk - 1) / chunk;
#pragma omp parallel for collapse(2) schedule(dynamic, 1) num_threads(nthreads)
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < D; ++d) {
            const double *Arow = A + d * N;
            double dskip = Dv ? Dv[d] : 0.0;
            double *P = (double *)malloc((size_t)(nchunks * N) * sizeof(double));
            double *H = (double *)malloc((size_t)(nchunks * N) * sizeof(double));
            double *hin = (double *)malloc((size_t)((nchunks + 1) * N) * sizeof(double));
            /* 1. chunk aggregates from a zero state */
            for (int64_t c = 0; c < nchunks; ++c) {
                double *Pc = P + c * N, *Hc = H + c * N;
                for (int64_t n = 0; n < N; ++n) {
                    Pc[n] = 1.0;
                    Hc[n] = 0.0;
                }
                int64_t t1 = (c + 1) * chunk < L ? (c + 1) * chunk : L;
                for (int64_t t = c * chunk; t < t1; ++t) {
                    int64_t i = (b * L + t) * D + d;
                    int64_t j = (b * L + t) * N;
                    double dt = step_size(delta[i], delta_bias, d, softplus_flag);
                    for (int64_t n = 0; n < N; ++n) {
                        double a_bar = exp(dt * Arow[n]);
                        double b_bar = bbar_coeff(dt, Arow[n], bbar_mode) * B[j + n];
                        /* (a_bar, b_bar·x) ∘ (P, H): this token comes later */
                        oracle_compose(a_bar, b_bar * x[i], Pc[n], Hc[n],
                                       &Pc[n], &Hc[n]);
                    }
                }
            }
            /* 2. carry across chunks */
            for (int64_t n = 0; n < N; ++n)
                hin[n] = h0 ? h0[(b * D + d) * N + n] : 0.0;
            for (int64_t c = 0; c < nchunks; ++c) {
                for (int64_t n = 0; n < N; ++n) {
                    double a_unused;
                    oracle_compose(P[c * N + n], H[c * N + n], 1.0,
                                   hin[c * N + n], &a_unused,
                                   &hin[(c + 1) * N + n]);
                }
            }
            /* 3. rescan each chunk from its carried-in state (hin[c] is
             *    consumed in place; hin[c + 1] was already read above) */
            for (int64_t c = 0; c < nchunks; ++c) {
                double *h = hin + c * N;
                int64_t t1 = (c + 1) * chunk < L ? (c + 1) * chunk : L;
                for (int64_t t = c * chunk; t < t1; ++t) {
                    int64_t i = (b * L + t) * D + d;
                    int64_t j = (b * L + t) * N;
                    double dt = step_size(delta[i], delta_bias, d, softplus_flag);
                    y[i] = token_update(h, x[i], dt, Arow, B + j, C + j, dskip,
                                        z ? z + i : NULL, N, bbar_mode);
                }
            }
            if (final_state)
                for (int64_t n = 0; n < N; ++n)
                    final_state[(b * D + d) * N + n] = hin[nchunks * N + n];
            free(P);
            free(H);
            free(hin);
        }
    }
}

/*
 * Diagonal ZOH input matrix for one step ([Guide] §1 "Discrétisation"):
 * B_bar[n] = (exp(Δ·A[n]) − 1)/A[n] · B[n], the a → 0 limit being Δ·B[n].
 * Also returns A_bar[n] = exp(Δ·A[n]).
 */
void oracle_zoh_discretize(double dt, const double *A, const double *B,
                           double *A_bar, double *B_bar, int64_t N)
{
    for (int64_t n = 0; n < N; ++n) {
        A_bar[n] = exp(dt * A[n]);
        B_bar[n] = bbar_coeff(dt, A[n], ORACLE_BBAR_ZOH) * B[n];
    }
}

/* d silu(z)/dz = σ(z)·(1 + z·(1 − σ(z))). */
static double silu_grad(double z)
{
    double sg = 1.0 / (1.0 + exp(-z));
    return sg * (1.0 + z * (1.0 - sg));
}

/* d softplus(v)/dv = σ(v). */
static double sigmoid(double v)
{
    return 1.0 / (1.0 + exp(-v));
}

/*
 * Gradient of oracle_selscan_fwd (input term Δ·B·x) by reverse-mode
 * differentiation of the recurrence: the loss is Σ dy·y + Σ dfinal·final_state
 * for given dy [batch, L, D] and dfinal [batch, D, N] (null: 0).
 *
 * The backward pass with recomputation that [Infer] "Cena selekcji" names is
 * the reverse sweep of the recurrence [Guide] §4 / [Johe] "SSM as RNN":
 * with λ_t = ∂loss/∂h_t,
 *   λ_{L−1} = ds_{L−1}·C_{L−1} + dfinal,   λ_t = ds_t·C_t + Abar_{t+1}·λ_{t+1},
 * where ds_t = dy_t·silu(z_t) is the gradient of the pre-gate output
 * s_t = Σ_n C_t[n]·h_t[n] + D·x_t. Each token then contributes
 *   dB_t[n] += λ_t[n]·Δ_t·x_t          (summed over channels)
 *   dC_t[n] += ds_t·h_t[n]             (summed over channels)
 *   du_t     = Σ_n λ_t[n]·B_t[n]       (u_t = Δ_t·x_t)
 *   dΔ_t     = Σ_n λ_t[n]·h_{t−1}[n]·Abar_t[n]·A[n] + du_t·x_t
 *   dA[n]   += λ_t[n]·h_{t−1}[n]·Abar_t[n]·Δ_t
 *   dx_t     = du_t·Δ_t + ds_t·D,   dD += ds_t·x_t,   dz_t = dy_t·s_t·silu'(z_t)
 *   ddelta_t = dΔ_t·σ(delta_t + bias) (softplus on; dΔ_t otherwise),
 *   dbias   += ddelta_t
 * and dh0 = Abar_0·λ_0. With the ZOH input term (bbar_mode = 1) the input
 * of token t is c_t[n]·B_t[n]·x_t with c = (exp(Δ·A[n]) − 1)/A[n] instead of
 * Δ·B_t[n]·x_t; then dB_t[n] += λ_t[n]·c_t[n]·x_t, dx_t = Σ_n λ_t[n]·c_t[n]·
 * B_t[n] + ds_t·D, the input part of dΔ_t is Σ_n λ_t[n]·(∂c/∂Δ)·B_t[n]·x_t
 * and dA[n] gains λ_t[n]·(∂c/∂A)·B_t[n]·x_t (zoh_coeff_grads). The forward
 * states h_t are kept per chain (this is the plain definition, not a
 * memory-saving schedule).
 *
 * Outputs: dx, ddelta, dz [batch, L, D] (dz only when z is given); dB, dC
 * [batch, L, N]; dA [D, N]; dDv, ddelta_bias [D]; dh0 [batch, D, N]
 * (nullable). Every output is overwritten.
 */
void oracle_selscan_bwd(const double *x, const double *delta, const double *A,
                        const double *B, const double *C, const double *Dv,
                        const double *z, const double *delta_bias,
                        int softplus_flag, int bbar_mode, const double *h0, const double *dy,
                        const double *dfinal, double *dx, double *ddelta,
                        double *dA, double *dB, double *dC, double *dDv,
                        double *dz, double *ddelta_bias, double *dh0,
                        int64_t batch, int64_t L, int64_t D, int64_t N,
                        int nthreads)
{
    if (nthreads < 1)
        nthreads = 1;
    for (int64_t i = 0; i < D * N; ++i)
        dA[i] = 0.0;
    for (int64_t d = 0; d < D; ++d) {
        dDv[d] = 0.0;
        ddelta_bias[d] = 0.0;
    }
    for (int64_t i = 0; i < batch * L * N; ++i) {
        dB[i] = 0.0;
        dC[i] = 0.0;
    }
    /* dB and dC sum over channels: every thread accumulates its channels into
     * a private [L, N] pair, added to the outputs in thread order. */
    double *priv = (double *)calloc((size_t)(nthreads * 2 * L * N), sizeof(double));
    for (int64_t b = 0; b < batch; ++b) {
#pragma omp parallel num_threads(nthreads)
        {
            int tid = 0;
#ifdef _OPENMP
            tid = omp_get_thread_num();
#endif
            double *pB = priv + (size_t)tid * 2 * L * N, *pC = pB + L * N;
            double *hs = (double *)malloc((size_t)((L + 1) * N) * sizeof(double));
            double *dts = (double *)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
            double *ss = (double *)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
            double *lam = (double *)malloc((size_t)N * sizeof(double));
#pragma omp for schedule(static)
            for (int64_t d = 0; d < D; ++d) {
                const double *Arow = A + d * N;
                double dskip = Dv ? Dv[d] : 0.0;
                /* forward, keeping h_{t} for every t (hs[t + 1]) */
                for (int64_t n = 0; n < N; ++n)
                    hs[n] = h0 ? h0[(b * D + d) * N + n] : 0.0;
                for (int64_t t = 0; t < L; ++t) {
                    int64_t i = (b * L + t) * D + d;
                    int64_t j = (b * L + t) * N;
                    double dt = step_size(delta[i], delta_bias, d, softplus_flag);
                    double acc = 0.0;
                    dts[t] = dt;
                    for (int64_t n = 0; n < N; ++n) {
                        double h = exp(dt * Arow[n]) * hs[t * N + n] +
                                   bbar_coeff(dt, Arow[n], bbar_mode) * B[j + n] * x[i];
                        hs[(t + 1) * N + n] = h;
                        acc += C[j + n] * h;
                    }
                    ss[t] = acc + dskip * x[i];
                }
                /* reverse sweep */
                for (int64_t n = 0; n < N; ++n)
                    lam[n] = dfinal ? dfinal[(b * D + d) * N + n] : 0.0;
                for (int64_t t = L - 1; t >= 0; --t) {
                    int64_t i = (b * L + t) * D + d;
                    int64_t j = (b * L + t) * N;
                    double dt = dts[t];
                    double ds = z ? dy[i] * silu(z[i]) : dy[i];
                    if (z)
                        dz[i] = dy[i] * ss[t] * silu_grad(z[i]);
                    dDv[d] += ds * x[i];
                    double du = 0.0, ddt = 0.0;
                    if (bbar_mode == ORACLE_BBAR_ZOH) {
                        for (int64_t n = 0; n < N; ++n) {
                            double h = hs[(t + 1) * N + n], hprev = hs[t * N + n];
                            double a_bar = exp(dt * Arow[n]);
                            double c, c_dt, c_a;
                            zoh_coeff_grads(dt, Arow[n], &c, &c_dt, &c_a);
                            lam[n] += ds * C[j + n]; /* λ_t */
                            pC[t * N + n] += ds * h;
                            pB[t * N + n] += lam[n] * c * x[i];
                            du += lam[n] * c * B[j + n]; /* here: dx without the D term */
                            ddt += lam[n] * hprev * a_bar * Arow[n] +
                                   lam[n] * c_dt * B[j + n] * x[i];
                            dA[d * N + n] += lam[n] * hprev * a_bar * dt +
                                             lam[n] * c_a * B[j + n] * x[i];
                            lam[n] *= a_bar;
                        }
                        dx[i] = du + ds * dskip;
                    } else {
                        for (int64_t n = 0; n < N; ++n) {
                            double h = hs[(t + 1) * N + n], hprev = hs[t * N + n];
                            double a_bar = exp(dt * Arow[n]);
                            lam[n] += ds * C[j + n]; /* λ_t */
                            pC[t * N + n] += ds * h;
                            pB[t * N + n] += lam[n] * dt * x[i];
                            du += lam[n] * B[j + n];
                            ddt += lam[n] * hprev * a_bar * Arow[n];
                            dA[d * N + n] += lam[n] * hprev * a_bar * dt;
                            lam[n] *= a_bar; /* Abar_t·λ_t, the part of λ_{t−1} from h_t */
                        }
                        ddt += du * x[i];
                        dx[i] = du * dt + ds * dskip;
                    }
                    double v = delta[i] + (delta_bias ? delta_bias[d] : 0.0);
                    double dv = softplus_flag ? ddt * sigmoid(v) : ddt;
                    ddelta[i] = dv;
                    ddelta_bias[d] += dv;
                }
                if (dh0)
                    for (int64_t n = 0; n < N; ++n)
                        dh0[(b * D + d) * N + n] = lam[n];
            }
            free(hs);
            free(dts);
            free(ss);
            free(lam);
        }
        for (int k = 0; k < nthreads; ++k) {
            double *pB = priv + (size_t)k * 2 * L * N, *pC = pB + L * N;
            for (int64_t i = 0; i < L * N; ++i) {
                dB[b * L * N + i] += pB[i];
                dC[b * L * N + i] += pC[i];
                pB[i] = 0.0;
                pC[i] = 0.0;
            }
        }
    }
    free(priv);
}

/*
 * Causal depthwise convolution in front of the scan: the Conv1d with one
 * filter per channel, kernel width K and K − 1 leading zeros of "Mamba и State
 * Space Models: альтернатива Transformer" ("Mamba Block": groups = channels,
 * padding d_conv − 1) and of "Mamba & State Space Models — Guide Complet" §7
 * (kernel_size 4, keeping the first L outputs), followed by the SiLU of that
 * page's block diagram (Conv1D → SiLU → SSM):
 *   x[b, t, d] = silu( cb[d] + Σ_{k<K} w[d, k] · x_in[b, t − (K−1) + k, d] ),
 * with x_in = 0 before the first token. Like torch's Conv1d this is a
 * cross-correlation (w[d, K−1] multiplies the current token).
 * x_in, x_out [batch, L, D]; w [D, K]; cb [D] (nullable: zero).
 */
void oracle_causal_conv1d(const double *x_in, const double *w, const double *cb,
                          double *x_out, int64_t batch, int64_t L, int64_t D,
                          int64_t K, int silu_flag)
{
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t t = 0; t < L; ++t)
            for (int64_t d = 0; d < D; ++d) {
                double acc = cb ? cb[d] : 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    int64_t s = t - (K - 1) + k;
                    if (s >= 0)
                        acc += w[d * K + k] * x_in[(b * L + s) * D + d];
                }
                x_out[(b * L + t) * D + d] = silu_flag ? silu(acc) : acc;
            }
}

/*
 * Gradient of oracle_causal_conv1d for the loss Σ dxc·x (x the conv output):
 * with pre = cb + Σ_k w[k]·x_in[t − (K−1) + k] and dpre = dxc·silu'(pre)
 * (dxc itself when silu_flag is 0),
 *   dx_in[s]  = Σ_k w[d, k] · dpre[s + (K−1) − k]   (tokens past the end: 0)
 *   dw[d, k]  = Σ_{b,t} dpre[b, t, d] · x_in[b, t − (K−1) + k, d]
 *   dcb[d]    = Σ_{b,t} dpre[b, t, d].
 * dx_in [batch, L, D]; dw [D, K]; dcb [D] (nullable). Outputs overwritten.
 */
void oracle_causal_conv1d_bwd(const double *x_in, const double *w, const double *cb,
                              const double *dxc, double *dx_in, double *dw, double *dcb,
                              int64_t batch, int64_t L, int64_t D, int64_t K,
                              int silu_flag)
{
    double *dpre = (double *)malloc((size_t)(batch * L * D > 0 ? batch * L * D : 1) *
                                    sizeof(double));
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t t = 0; t < L; ++t)
            for (int64_t d = 0; d < D; ++d) {
                double pre = cb ? cb[d] : 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    int64_t s = t - (K - 1) + k;
                    if (s >= 0)
                        pre += w[d * K + k] * x_in[(b * L + s) * D + d];
                }
                int64_t i = (b * L + t) * D + d;
                dpre[i] = silu_flag ? dxc[i] * silu_grad(pre) : dxc[i];
            }
    for (int64_t i = 0; i < D * K; ++i)
        dw[i] = 0.0;
    if (dcb)
        for (int64_t d = 0; d < D; ++d)
            dcb[d] = 0.0;
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t s = 0; s < L; ++s)
            for (int64_t d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    int64_t t = s + (K - 1) - k; /* the output token x_in[s] feeds via w[k] */
                    if (t < L)
                        acc += w[d * K + k] * dpre[(b * L + t) * D + d];
                }
                dx_in[(b * L + s) * D + d] = acc;
            }
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t t = 0; t < L; ++t)
            for (int64_t d = 0; d < D; ++d) {
                double g = dpre[(b * L + t) * D + d];
                if (dcb)
                    dcb[d] += g;
                for (int64_t k = 0; k < K; ++k) {
                    int64_t s = t - (K - 1) + k;
                    if (s >= 0)
                        dw[d * K + k] += g * x_in[(b * L + s) * D + d];
                }
            }
    free(dpre);
}
