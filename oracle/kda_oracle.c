/*
 * kda_oracle.c -- fp64 CPU reference for the Kimi Delta Attention (KDA)
 * recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file; only the test-suite, the package's smoke check and the
 * CPU-baseline leg of the benchmark do.  It shares no code, header or
 * constant with the CUDA library.
 *
 * What it computes (per batch b and head h, state S in R^{dk x dv}):
 *
 *   S_t = (I - e_t k_t k_t^T) Diag(alpha_t) S_{t-1} + w_t k_t v_t^T
 *   o_t = scale * S_t^T q_t,          alpha_t = exp(g_t)  (per channel)
 *
 * KDA itself uses e_t = w_t = beta_t.  The update is the "combined form" of
 * "Kimi Linear's Hybrid Linear Attention Architecture: A Technical
 * Breakdown", section 3.3 (decay first, then directional erasure, then the
 * write), written with the state oriented dk x dv as in the update printed
 * in "Kimi Linear: How Moonshot AI Built a Hybrid Attention Architecture
 * That Beats Full Attention" (beta_t k_t v_t^T).  The readout is the
 * "Step 4: Query" block of the "Kimi Linear" explainer (math.kryvik.com):
 * the query reads the state after the token's own write.
 *
 * Two independent evaluations are provided, plus the gradients:
 *   kda_oracle_fwd        -- the recurrence as column operations:
 *                            decay rows, p = S^T k, u = w v - e p,
 *                            S += k u^T, o = scale S^T q.
 *   kda_oracle_bruteforce -- builds every transition matrix
 *                            M_t = (I - e_t k_t k_t^T) Diag(alpha_t)
 *                            explicitly (dk x dk) and forms M_t S + w k v^T
 *                            with a dense triple loop.  O(T dk^2 dv): small
 *                            cases only.
 *   kda_oracle_bwd        -- reverse-mode gradients of kda_oracle_fwd.
 *
 * Layouts (row-major, contiguous, all double):
 *   q, k, g : [B, T, H, dk]      v, out : [B, T, H, dv]
 *   e, w    : [B, T, H]          h0, hT : [B, H, dk, dv]
 * h0 == NULL means a zero initial state; hT == NULL means "not written";
 * out == NULL means "not written".  Returns 0, or -1 on bad sizes.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int sizes_ok(long B, long T, long H, long dk, long dv)
{
    return B >= 0 && T >= 0 && H >= 0 && dk > 0 && dv > 0;
}

int kda_oracle_fwd(const double *q, const double *k, const double *v,
                   const double *g, const double *e, const double *w,
                   double scale, const double *h0, double *out, double *hT,
                   long B, long T, long H, long dk, long dv, int nthreads)
{
    if (!sizes_ok(B, T, H, dk, dv)) return -1;
    long BH = B * H;
    if (nthreads < 1) nthreads = 1;
    int failed = 0;

#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        long b = bh / H, h = bh % H;
        double *S = (double *)malloc(sizeof(double) * dk * dv);
        double *p = (double *)malloc(sizeof(double) * dv);
        double *u = (double *)malloc(sizeof(double) * dv);
        if (!S || !p || !u) {
            failed = 1;
            free(S); free(p); free(u);
            continue;
        }
        if (h0) memcpy(S, h0 + bh * dk * dv, sizeof(double) * dk * dv);
        else    memset(S, 0, sizeof(double) * dk * dv);

        for (long t = 0; t < T; ++t) {
            long row = (b * T + t) * H + h;
            const double *qt = q + row * dk, *kt = k + row * dk;
            const double *vt = v + row * dv, *gt = g + row * dk;
            double et = e[row], wt = w[row];

            /* 1. per-channel decay of the old memory: row r scaled by alpha_r */
            for (long r = 0; r < dk; ++r) {
                double a = exp(gt[r]);
                for (long c = 0; c < dv; ++c) S[r * dv + c] *= a;
            }
            /* 2. what the decayed memory returns for the key: p = S^T k */
            for (long c = 0; c < dv; ++c) p[c] = 0.0;
            for (long r = 0; r < dk; ++r)
                for (long c = 0; c < dv; ++c) p[c] += kt[r] * S[r * dv + c];
            /* 3. erase along k and write v: u = w v - e p */
            for (long c = 0; c < dv; ++c) u[c] = wt * vt[c] - et * p[c];
            /* 4. rank-1 update S += k u^T */
            for (long r = 0; r < dk; ++r)
                for (long c = 0; c < dv; ++c) S[r * dv + c] += kt[r] * u[c];
            /* 5. readout after the write: o = scale * S^T q */
            if (out) {
                double *ot = out + row * dv;
                for (long c = 0; c < dv; ++c) ot[c] = 0.0;
                for (long r = 0; r < dk; ++r)
                    for (long c = 0; c < dv; ++c) ot[c] += qt[r] * S[r * dv + c];
                for (long c = 0; c < dv; ++c) ot[c] *= scale;
            }
        }
        if (hT) memcpy(hT + bh * dk * dv, S, sizeof(double) * dk * dv);
        free(S); free(p); free(u);
    }
    return failed ? -1 : 0;
}

int kda_oracle_bruteforce(const double *q, const double *k, const double *v,
                          const double *g, const double *e, const double *w,
                          double scale, const double *h0, double *out,
                          double *hT, long B, long T, long H, long dk, long dv)
{
    if (!sizes_ok(B, T, H, dk, dv)) return -1;
    double *M = (double *)malloc(sizeof(double) * dk * dk);
    double *S = (double *)malloc(sizeof(double) * dk * dv);
    double *N = (double *)malloc(sizeof(double) * dk * dv);
    if (!M || !S || !N) { free(M); free(S); free(N); return -1; }

    for (long b = 0; b < B; ++b)
    for (long h = 0; h < H; ++h) {
        long bh = b * H + h;
        if (h0) memcpy(S, h0 + bh * dk * dv, sizeof(double) * dk * dv);
        else    memset(S, 0, sizeof(double) * dk * dv);
        for (long t = 0; t < T; ++t) {
            long row = (b * T + t) * H + h;
            const double *qt = q + row * dk, *kt = k + row * dk;
            const double *vt = v + row * dv, *gt = g + row * dk;
            /* M = (I - e k k^T) Diag(alpha): entry (r, c) = (delta_rc - e k_r k_c) alpha_c */
            for (long r = 0; r < dk; ++r)
                for (long c = 0; c < dk; ++c)
                    M[r * dk + c] = ((r == c ? 1.0 : 0.0) - e[row] * kt[r] * kt[c]) * exp(gt[c]);
            /* N = M S + w k v^T */
            for (long r = 0; r < dk; ++r)
                for (long c = 0; c < dv; ++c) {
                    double acc = 0.0;
                    for (long m = 0; m < dk; ++m) acc += M[r * dk + m] * S[m * dv + c];
                    N[r * dv + c] = acc + w[row] * kt[r] * vt[c];
                }
            memcpy(S, N, sizeof(double) * dk * dv);
            if (out) {
                double *ot = out + row * dv;
                for (long c = 0; c < dv; ++c) {
                    double acc = 0.0;
                    for (long r = 0; r < dk; ++r) acc += S[r * dv + c] * qt[r];
                    ot[c] = scale * acc;
                }
            }
        }
        if (hT) memcpy(hT + bh * dk * dv, S, sizeof(double) * dk * dv);
    }
    free(M); free(S); free(N);
    return 0;
}

/*
 * kda_oracle_bwd -- gradients of the forward above, by reverse-mode
 * differentiation of the same token loop (the plain definition of the
 * backward pass; the pages state no formula for it).  For a loss
 *   L = sum(dout * out) + sum(dhT * hT)
 * it returns dL/dq, dL/dk, dL/dv, dL/dg, dL/de, dL/dw and dL/dh0 in the
 * inputs' layouts (KDA's dL/dbeta is de + dw).  dout or dhT may be NULL
 * (zero).  Per (b, h) it first runs the loop forward keeping every state,
 * then walks the tokens backwards with the adjoint dS of the state:
 *   readout   o = scale S_t^T q:   dq = scale S_t do,   dS += scale q do^T
 *   write     S_t = S' + k u^T:    du = dS^T k,         dk += dS u
 *   u = w v - e p:                 dw = du.v, dv = w du, de = -du.p, dp = -e du
 *   p = S'^T k:                    dS' = dS + k dp^T,   dk += S' dp
 *   S' = Diag(alpha) S_{t-1}:      dg_r = alpha_r sum_c dS'_rc S_{t-1,rc},
 *                                  dS_{t-1} = Diag(alpha) dS'
 * and dh0 is the adjoint left after the first token.  Memory: (T + 1) dk dv
 * doubles per (b, h) at a time (small problems only).
 */
int kda_oracle_bwd(const double *q, const double *k, const double *v,
                   const double *g, const double *e, const double *w,
                   double scale, const double *h0,
                   const double *dout, const double *dhT,
                   double *dq, double *dkk, double *dvv, double *dg,
                   double *de, double *dw, double *dh0,
                   long B, long T, long H, long dk, long dv, int nthreads)
{
    if (!sizes_ok(B, T, H, dk, dv)) return -1;
    long BH = B * H;
    if (nthreads < 1) nthreads = 1;
    int failed = 0;

#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        long b = bh / H, h = bh % H;
        long SZ = dk * dv;
        double *St = (double *)malloc(sizeof(double) * SZ * (T + 1));
        double *dS = (double *)malloc(sizeof(double) * SZ);
        double *Sd = (double *)malloc(sizeof(double) * SZ);
        double *p = (double *)malloc(sizeof(double) * dv);
        double *u = (double *)malloc(sizeof(double) * dv);
        double *du = (double *)malloc(sizeof(double) * dv);
        if (!St || !dS || !Sd || !p || !u || !du) {
            failed = 1;
            free(St); free(dS); free(Sd); free(p); free(u); free(du);
            continue;
        }
        /* forward, keeping S_0 .. S_T */
        if (h0) memcpy(St, h0 + bh * SZ, sizeof(double) * SZ);
        else    memset(St, 0, sizeof(double) * SZ);
        for (long t = 0; t < T; ++t) {
            long row = (b * T + t) * H + h;
            const double *kt = k + row * dk, *vt = v + row * dv, *gt = g + row * dk;
            const double *S0 = St + t * SZ;
            double *S1 = St + (t + 1) * SZ;
            for (long r = 0; r < dk; ++r) {
                double a = exp(gt[r]);
                for (long c = 0; c < dv; ++c) S1[r * dv + c] = a * S0[r * dv + c];
            }
            for (long c = 0; c < dv; ++c) p[c] = 0.0;
            for (long r = 0; r < dk; ++r)
                for (long c = 0; c < dv; ++c) p[c] += kt[r] * S1[r * dv + c];
            for (long c = 0; c < dv; ++c) u[c] = w[row] * vt[c] - e[row] * p[c];
            for (long r = 0; r < dk; ++r)
                for (long c = 0; c < dv; ++c) S1[r * dv + c] += kt[r] * u[c];
        }
        /* backward */
        if (dhT) memcpy(dS, dhT + bh * SZ, sizeof(double) * SZ);
        else     memset(dS, 0, sizeof(double) * SZ);
        for (long t = T - 1; t >= 0; --t) {
            long row = (b * T + t) * H + h;
            const double *qt = q + row * dk, *kt = k + row * dk;
            const double *vt = v + row * dv, *gt = g + row * dk;
            const double *S0 = St + t * SZ, *S1 = St + (t + 1) * SZ;
            double et = e[row], wt = w[row];
            double *dqt = dq + row * dk, *dkt = dkk + row * dk, *dgt = dg + row * dk;
            double *dvt = dvv + row * dv;
            /* recompute S' = Diag(alpha) S_{t-1}, p and u of this token */
            for (long r = 0; r < dk; ++r) {
                double a = exp(gt[r]);
                for (long c = 0; c < dv; ++c) Sd[r * dv + c] = a * S0[r * dv + c];
            }
            for (long c = 0; c < dv; ++c) p[c] = 0.0;
            for (long r = 0; r < dk; ++r)
                for (long c = 0; c < dv; ++c) p[c] += kt[r] * Sd[r * dv + c];
            for (long c = 0; c < dv; ++c) u[c] = wt * vt[c] - et * p[c];
            /* readout */
            for (long r = 0; r < dk; ++r) {
                double acc = 0.0;
                if (dout)
                    for (long c = 0; c < dv; ++c) acc += S1[r * dv + c] * dout[row * dv + c];
                dqt[r] = scale * acc;
            }
            if (dout)
                for (long r = 0; r < dk; ++r)
                    for (long c = 0; c < dv; ++c) dS[r * dv + c] += scale * qt[r] * dout[row * dv + c];
            /* write S_t = S' + k u^T */
            for (long c = 0; c < dv; ++c) du[c] = 0.0;
            for (long r = 0; r < dk; ++r)
                for (long c = 0; c < dv; ++c) du[c] += dS[r * dv + c] * kt[r];
            for (long r = 0; r < dk; ++r) {
                double acc = 0.0;
                for (long c = 0; c < dv; ++c) acc += dS[r * dv + c] * u[c];
                dkt[r] = acc;
            }
            /* u = w v - e p */
            double dwt = 0.0, det = 0.0;
            for (long c = 0; c < dv; ++c) {
                dwt += du[c] * vt[c];
                det -= du[c] * p[c];
                dvt[c] = wt * du[c];
            }
            dw[row] = dwt;
            de[row] = det;
            /* p = S'^T k with dp = -e du: dS' = dS + k dp^T, dk += S' dp */
            for (long r = 0; r < dk; ++r) {
                double acc = 0.0;
                for (long c = 0; c < dv; ++c) {
                    double dp = -et * du[c];
                    acc += Sd[r * dv + c] * dp;
                    dS[r * dv + c] += kt[r] * dp;
                }
                dkt[r] += acc;
            }
            /* S' = Diag(alpha) S_{t-1} */
            for (long r = 0; r < dk; ++r) {
                double a = exp(gt[r]), acc = 0.0;
                for (long c = 0; c < dv; ++c) {
                    acc += dS[r * dv + c] * S0[r * dv + c];
                    dS[r * dv + c] *= a;
                }
                dgt[r] = a * acc;
            }
        }
        if (dh0) memcpy(dh0 + bh * SZ, dS, sizeof(double) * SZ);
        free(St); free(dS); free(Sd); free(p); free(u); free(du);
    }
    return failed ? -1 : 0;
}

int kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
