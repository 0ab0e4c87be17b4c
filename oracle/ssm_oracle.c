/*
 * fp64 CPU oracle for the selective scan (S6).  TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, sequential code that states what the scan computes.  It shares
 * no code, header, table or helper with the CUDA library; nothing in the
 * product path may call it.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg load it.
 *
 * Sources (the pages this follows):
 *  [SEL]  booiljung.github.io, "3.2 선택적 스캔(Selective Scan) 알고리즘과
 *         정보의 압축 및 선별" -- §1.1 the recurrence h_t = Ā h_{t-1} + B̄ x_t,
 *         y_t = C h_t; §1.2 the selection equations (Δ_t = Softplus(Parameter
 *         + Linear_1(x_t)), B_t, C_t per token); §2.1 ZOH, Ā_t = exp(Δ_t A)
 *         with A diagonal so the exponential is elementwise; §3.3 the backward
 *         pass recomputes the states instead of storing them.
 *  [SSM]  정보관리기술사 학습 노트, "상태공간 모델(SSM)과 Mamba 아키텍처" --
 *         §2 the discrete recurrence x_k = Ā x_{k-1} + B̄ u_k, y_k = C x_k;
 *         §3 flowchart: the SSM output is multiplied by a SiLU gate branch.
 *  [MAM]  honbul.tistory.com/130, summary of "Mamba: Linear-Time Sequence
 *         Modeling with Selective State Spaces" -- §2 S6: B_t, C_t, Δ_t =
 *         softplus(Δ + s_Δ(x_t)) are functions of the input.
 *
 * Readings where the pages leave a step open:
 *  - B̄_t = Δ_t B_t (the simplified discretisation of B; the ZOH form of [SEL]
 *    §2.1 is provided separately as the `zoh` flag of ssm_oracle_fwd, and the
 *    two agree as A -> 0).
 *  - h_0 = 0 unless an initial state is given.
 *  - the skip term D[d] x_t is added to y before the gate; the gate is
 *    out = y * z * sigmoid(z).
 *  - softplus(r) = log(1 + e^r), with the bias added before the softplus.
 *
 * Layouts (row-major): u, delta, z, out, dout: [batch][dim][seqlen];
 * B, C: [batch][dstate][seqlen]; A: [dim][dstate]; D, delta_bias: [dim];
 * h0, last_state: [batch][dim][dstate].
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double softplus(double r) {
    /* log(1 + e^r), written so that neither branch overflows */
    return r > 0.0 ? r + log1p(exp(-r)) : log1p(exp(r));
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

#define IDX3(a, b, c, nb, nc) (((size_t)(a) * (nb) + (b)) * (nc) + (c))

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int ssm_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Forward pass.  For each batch row b and channel d, walk t = 0..L-1:
 *   Δ_t   = softplus(delta[b,d,t] + bias[d])      (or the raw sum if !softplus)
 *   Ā_t[n] = exp(Δ_t A[d,n])                       ([SEL] §2.1)
 *   B̄_t[n] = Δ_t B[b,n,t]   or, with zoh, (Ā_t[n] - 1) / A[d,n] * B[b,n,t]
 *   h_t[n] = Ā_t[n] h_{t-1}[n] + B̄_t[n] u[b,d,t]  ([SEL] §1.1, [SSM] §2)
 *   y_t    = sum_n C[b,n,t] h_t[n] + D[d] u[b,d,t]
 *   out_t  = y_t * z_t * sigmoid(z_t)  if z given, else y_t   ([SSM] §3)
 * D, z, delta_bias, h0, last_state may be NULL.  Returns 0.
 */
int ssm_oracle_fwd(int batch, int dim, int seqlen, int dstate,
                   const double *u, const double *delta, const double *A,
                   const double *B, const double *C, const double *D,
                   const double *z, const double *delta_bias, int delta_softplus,
                   int zoh, const double *h0, double *out, double *last_state,
                   int nthreads) {
    set_threads(nthreads);
    long npair = (long)batch * dim;
#pragma omp parallel
    {
        double *h = (double *)malloc(sizeof(double) * (size_t)dstate);
#pragma omp for schedule(dynamic, 4)
        for (long p = 0; p < npair; ++p) {
            int b = (int)(p / dim), d = (int)(p % dim);
            const double *ub = u + IDX3(b, d, 0, dim, seqlen);
            const double *db = delta + IDX3(b, d, 0, dim, seqlen);
            const double *zb = z ? z + IDX3(b, d, 0, dim, seqlen) : NULL;
            double *ob = out + IDX3(b, d, 0, dim, seqlen);
            const double *Bb = B + IDX3(b, 0, 0, dstate, seqlen);
            const double *Cb = C + IDX3(b, 0, 0, dstate, seqlen);
            for (int n = 0; n < dstate; ++n)
                h[n] = h0 ? h0[IDX3(b, d, n, dim, dstate)] : 0.0;
            for (int t = 0; t < seqlen; ++t) {
                double r = db[t] + (delta_bias ? delta_bias[d] : 0.0);
                double dt = delta_softplus ? softplus(r) : r;
                double x = ub[t];
                double y = 0.0;
                for (int n = 0; n < dstate; ++n) {
                    double a = A[(size_t)d * dstate + n];
                    double abar = exp(dt * a);
                    double bbar;
                    if (zoh && a != 0.0) /* (Ā - 1)/A, via expm1 to avoid cancellation */
                        bbar = expm1(dt * a) / a * Bb[(size_t)n * seqlen + t];
                    else
                        bbar = dt * Bb[(size_t)n * seqlen + t];
                    h[n] = abar * h[n] + bbar * x;
                    y += Cb[(size_t)n * seqlen + t] * h[n];
                }
                if (D) y += D[d] * x;
                if (zb) y *= zb[t] * sigmoid(zb[t]);
                ob[t] = y;
            }
            if (last_state)
                for (int n = 0; n < dstate; ++n)
                    last_state[IDX3(b, d, n, dim, dstate)] = h[n];
        }
        free(h);
    }
    return 0;
}

/* d/dA of (exp(Δ a) - 1)/a, the zero-order-hold input factor: Δ² ψ(Δ a)
 * with ψ(x) = (x e^x - (e^x - 1)) / x² = Σ_{j>=0} (j+1) x^j / (j+2)!,
 * summed as a series near 0 where the closed form cancels. */
static double zoh_dk_da(double dt, double a) {
    double x = dt * a, psi;
    if (fabs(x) < 1e-3)
        psi = 0.5 + x * (1.0 / 3.0 + x * (1.0 / 8.0 + x * (1.0 / 30.0 + x / 144.0)));
    else
        psi = (x * exp(x) - expm1(x)) / (x * x);
    return dt * dt * psi;
}

/*
 * Backward pass (the adjoint of ssm_oracle_fwd with h0 = 0),
 * obtained by reverse-mode differentiation of the loop above.  The pages
 * give no backward formulas; only that the backward recomputes the states
 * ([SEL] §3.3), which this code does by re-running the forward recurrence
 * per (b, d) and keeping its states in a local buffer.
 *
 * With g_t = dout[b,d,t], s = sigmoid(z_t), and y_t the pre-gate output:
 *   gy_t = g_t z_t s            (g_t if no gate)
 *   dz_t = g_t y_t s (1 + z_t (1 - s))
 *   lam_t[n] = C_t[n] gy_t + Ā_{t+1}[n] lam_{t+1}[n],   lam_L = 0
 *   du_t = gy_t D + sum_n lam_t[n] Δ_t B_t[n]
 *   dΔ_t = sum_n lam_t[n] (A[n] Ā_t[n] h_{t-1}[n] + B_t[n] u_t)
 *   ddelta_t = dΔ_t sigmoid(r_t) with softplus (dΔ_t otherwise)
 *   dA[d,n] += lam_t[n] Δ_t Ā_t[n] h_{t-1}[n]     dD[d] += gy_t u_t
 *   dB[b,n,t] += lam_t[n] Δ_t u_t                 dC[b,n,t] += gy_t h_t[n]
 *   dbias[d] += ddelta_t
 * With zoh the input factor Δ_t above becomes k_t[n] = (Ā_t[n] - 1)/A[n]
 * (Δ_t where A[n] = 0): du and dB use k, the B term of dΔ gains the factor
 * dk/dΔ = Ā_t[n], and dA gains lam_t[n] B_t[n] u_t dk/dA (zoh_dk_da).
 * Gradients are written (not accumulated into).  dD / dz / dbias may be NULL
 * (and must be when the matching input is NULL).  Returns 0, or -1 if a
 * scratch allocation fails.
 */
int ssm_oracle_bwd(int batch, int dim, int seqlen, int dstate,
                   const double *u, const double *delta, const double *A,
                   const double *B, const double *C, const double *D,
                   const double *z, const double *delta_bias, int delta_softplus,
                   const double *dout, double *du, double *ddelta, double *dA,
                   double *dB, double *dC, double *dD, double *dz, double *dbias,
                   int zoh, int nthreads) {
    set_threads(nthreads);
    long npair = (long)batch * dim;
    size_t bcsz = (size_t)batch * dstate * seqlen;
    int nt = ssm_oracle_max_threads();
    /* per-thread partial sums for dB and dC (reduced over d afterwards) */
    double *pdB = (double *)calloc((size_t)nt * bcsz, sizeof(double));
    double *pdC = (double *)calloc((size_t)nt * bcsz, sizeof(double));
    if (!pdB || !pdC) { free(pdB); free(pdC); return -1; }
    memset(dA, 0, sizeof(double) * (size_t)dim * dstate);
    if (dD) memset(dD, 0, sizeof(double) * (size_t)dim);
    if (dbias) memset(dbias, 0, sizeof(double) * (size_t)dim);
    /* dA, dD, dbias are sums over (b, t): accumulate per (b, d) then add per d */
    double *pdA = (double *)calloc((size_t)npair * dstate, sizeof(double));
    double *pdD = (double *)calloc((size_t)npair, sizeof(double));
    double *pdb = (double *)calloc((size_t)npair, sizeof(double));
    if (!pdA || !pdD || !pdb) {
        free(pdB); free(pdC); free(pdA); free(pdD); free(pdb); return -1;
    }
    int fail = 0;
#pragma omp parallel
    {
        int tid = 0;
#ifdef _OPENMP
        tid = omp_get_thread_num();
#endif
        double *myB = pdB + (size_t)tid * bcsz, *myC = pdC + (size_t)tid * bcsz;
        /* hs[t][n] = h_t[n] for t = -1..L-1 (row 0 is h_{-1} = 0) */
        double *hs = (double *)malloc(sizeof(double) * (size_t)(seqlen + 1) * dstate);
        double *dts = (double *)malloc(sizeof(double) * (size_t)seqlen);
        double *lam = (double *)malloc(sizeof(double) * (size_t)dstate);
        if (!hs || !dts || !lam) {
#pragma omp atomic write
            fail = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (long p = 0; p < npair; ++p) {
            if (!hs || !dts || !lam) continue;
            int b = (int)(p / dim), d = (int)(p % dim);
            const double *ub = u + IDX3(b, d, 0, dim, seqlen);
            const double *db = delta + IDX3(b, d, 0, dim, seqlen);
            const double *zb = z ? z + IDX3(b, d, 0, dim, seqlen) : NULL;
            const double *gb = dout + IDX3(b, d, 0, dim, seqlen);
            const double *Bb = B + IDX3(b, 0, 0, dstate, seqlen);
            const double *Cb = C + IDX3(b, 0, 0, dstate, seqlen);
            const double *Ad = A + (size_t)d * dstate;
            double *dub = du + IDX3(b, d, 0, dim, seqlen);
            double *ddb = ddelta + IDX3(b, d, 0, dim, seqlen);
            double *dzb = dz ? dz + IDX3(b, d, 0, dim, seqlen) : NULL;
            double *bB = myB + IDX3(b, 0, 0, dstate, seqlen);
            double *bC = myC + IDX3(b, 0, 0, dstate, seqlen);
            double bias = delta_bias ? delta_bias[d] : 0.0;
            /* forward recompute of the states */
            for (int n = 0; n < dstate; ++n) hs[n] = 0.0;
            for (int t = 0; t < seqlen; ++t) {
                double r = db[t] + bias;
                double dt = delta_softplus ? softplus(r) : r;
                dts[t] = dt;
                for (int n = 0; n < dstate; ++n) {
                    double abar = exp(dt * Ad[n]);
                    double k = (zoh && Ad[n] != 0.0) ? expm1(dt * Ad[n]) / Ad[n] : dt;
                    hs[(size_t)(t + 1) * dstate + n] =
                        abar * hs[(size_t)t * dstate + n] + k * Bb[(size_t)n * seqlen + t] * ub[t];
                }
            }
            /* reverse sweep */
            for (int n = 0; n < dstate; ++n) lam[n] = 0.0;
            double accD = 0.0, accb = 0.0;
            double *accA = pdA + (size_t)p * dstate;
            for (int t = seqlen - 1; t >= 0; --t) {
                double dt = dts[t], x = ub[t];
                const double *hprev = hs + (size_t)t * dstate;
                const double *hcur = hs + (size_t)(t + 1) * dstate;
                double y = 0.0;
                for (int n = 0; n < dstate; ++n) y += Cb[(size_t)n * seqlen + t] * hcur[n];
                if (D) y += D[d] * x;
                double gy = gb[t];
                if (zb) {
                    double s = sigmoid(zb[t]);
                    dzb[t] = gb[t] * y * s * (1.0 + zb[t] * (1.0 - s));
                    gy = gb[t] * zb[t] * s;
                }
                double dx = D ? gy * D[d] : 0.0;
                double ddt = 0.0;
                if (D) accD += gy * x;
                for (int n = 0; n < dstate; ++n) {
                    double Bt = Bb[(size_t)n * seqlen + t];
                    double Ct = Cb[(size_t)n * seqlen + t];
                    double abar = exp(dt * Ad[n]);
                    int zn = zoh && Ad[n] != 0.0;
                    double k = zn ? expm1(dt * Ad[n]) / Ad[n] : dt;   /* B̄ = k B */
                    double dk_ddt = zoh ? abar : 1.0;
                    /* lam_t = C_t gy_t + Ā_{t+1} lam_{t+1}; lam[] holds
                       Ā_{t+1} lam_{t+1} on entry (see the update below) */
                    double l = Ct * gy + lam[n];
                    dx += l * k * Bt;
                    ddt += l * (Ad[n] * abar * hprev[n] + Bt * x * dk_ddt);
                    accA[n] += l * dt * abar * hprev[n];
                    if (zoh) accA[n] += l * Bt * x * zoh_dk_da(dt, Ad[n]);
                    bB[(size_t)n * seqlen + t] += l * k * x;
                    bC[(size_t)n * seqlen + t] += gy * hcur[n];
                    lam[n] = abar * l; /* becomes Ā_t lam_t for step t-1 */
                }
                dub[t] = dx;
                double r = db[t] + bias;
                double dr = delta_softplus ? ddt * sigmoid(r) : ddt;
                ddb[t] = dr;
                accb += dr;
            }
            pdD[p] = accD;
            pdb[p] = accb;
        }
        free(hs); free(dts); free(lam);
    }
    if (fail) {
        free(pdB); free(pdC); free(pdA); free(pdD); free(pdb); return -1;
    }
    /* deterministic reductions */
    for (size_t i = 0; i < bcsz; ++i) {
        double sb = 0.0, sc = 0.0;
        for (int k = 0; k < nt; ++k) { sb += pdB[(size_t)k * bcsz + i]; sc += pdC[(size_t)k * bcsz + i]; }
        dB[i] = sb; dC[i] = sc;
    }
    for (long p = 0; p < npair; ++p) {
        int d = (int)(p % dim);
        for (int n = 0; n < dstate; ++n) dA[(size_t)d * dstate + n] += pdA[(size_t)p * dstate + n];
        if (dD) dD[d] += pdD[p];
        if (dbias) dbias[d] += pdb[p];
    }
    free(pdB); free(pdC); free(pdA); free(pdD); free(pdb);
    return 0;
}
