/*
 * fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, token-by-token evaluation of the recurrences whose chunked
 * form the CUDA library computes.  No chunking, no blocking, no reordering:
 * each token is one rank-1 state update followed by one read-out.  Only the
 * tests, the package's smoke check and the benchmark's CPU-baseline leg may
 * load this file's library.  It shares no code with the CUDA path.
 *
 * State convention: the state S_t is d_v x d_k (it maps keys to values, so
 * o_t = S_t q_t).  Initial and final states are exchanged in the transposed
 * layout h = S^T, shape [B, H, d_k, d_v], row-major with d_v innermost.
 *
 * Sources (page title, then section):
 *   - Gated delta rule.  The pages name Gated DeltaNet and its chunkwise
 *     form ("Quando o 'Bom o Suficiente' e Otimo: Aproximacao de Inversao de
 *     Matriz Baseada Apenas em Multiplicacao para Gated DeltaNet Quantizado",
 *     section "Declaracao do Problema") and read the delta rule as an online
 *     SGD step on the least-squares loss 1/2 ||S k_t - v_t||^2 ("Resumo
 *     Tecnico: Preconditioned DeltaNet", section 1; the Arabic summary of
 *     the same paper, section 1), with alpha the decay axis and beta the gain
 *     axis of the DGPS taxonomy (Arabic summary, section 2c).  The update
 *     itself is not printed on the pages; the form used here is the standard
 *     one: S_t = S_{t-1} alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t q_t.
 *   - Preconditioned two-gate variant.  Diagonal curvature accumulator of the
 *     squared keys with the preconditioned write key ("Preconditioned
 *     DeltaNet: Curvature-aware Sequence Modeling for Linear Recurrences",
 *     Arabic summary, section 2b "the diagonal approximation"); separate read
 *     and write keys ("Resumo Tecnico: Preconditioned DeltaNet", section 2,
 *     "Estabilidade e Parametrizacao"); channel-wise erase gate b_t on the
 *     key axis and write gate w_t on the value axis ("NVIDIA Apresenta Gated
 *     DeltaNet-2", section "Como DeltaNet-2 Redesenhou a Arquitetura").  The
 *     accumulator used is the moving average rho_t = c rho_{t-1} + k_t (.) k_t
 *     with write key k_t / sqrt(rho_t + eps); c = 1 gives the pages' plain
 *     running sum.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC gdn_oracle.c -o libgdn_oracle.so -lm
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static size_t tok(int b, int t, int h, int T, int H) {
    return ((size_t)b * T + t) * H + h;
}

/*
 * Gated delta rule, one (batch, head) sequence per outer iteration.
 *   q, k  [B,T,H,dk]; v [B,T,H,dv]; alpha, beta [B,T,H] (alpha NULL => 1,
 *   beta NULL => 1); h0 [B,H,dk,dv] or NULL (=> 0);
 *   o [B,T,H,dv]; hT [B,H,dk,dv] or NULL.
 * Per token:  p = S k_t  (prediction of the undecayed state)
 *             S = alpha_t S - alpha_t beta_t p k_t^T + beta_t v_t k_t^T
 *             o_t = S q_t
 * which is S_{t-1} alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T.
 */
void oracle_gated_delta_fwd(int B, int T, int H, int dk, int dv,
                            const double *q, const double *k, const double *v,
                            const double *alpha, const double *beta,
                            const double *h0, double *o, double *hT,
                            int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int bh = 0; bh < B * H; ++bh) {
        const int b = bh / H, h = bh % H;
        double *S = (double *)calloc((size_t)dv * dk, sizeof(double));
        double *p = (double *)malloc((size_t)dv * sizeof(double));
        if (h0) {
            const double *src = h0 + (size_t)bh * dk * dv;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[(size_t)j * dk + i] = src[(size_t)i * dv + j];
        }
        for (int t = 0; t < T; ++t) {
            const size_t r = tok(b, t, h, T, H);
            const double *kt = k + r * dk, *qt = q + r * dk, *vt = v + r * dv;
            const double a = alpha ? alpha[r] : 1.0;
            const double be = beta ? beta[r] : 1.0;
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[(size_t)j * dk + i] * kt[i];
                p[j] = acc;
            }
            for (int j = 0; j < dv; ++j) {
                const double cp = a * be * p[j], cv = be * vt[j];
                double *row = S + (size_t)j * dk;
                for (int i = 0; i < dk; ++i)
                    row[i] = a * row[i] - cp * kt[i] + cv * kt[i];
            }
            double *ot = o + r * dv;
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[(size_t)j * dk + i] * qt[i];
                ot[j] = acc;
            }
        }
        if (hT) {
            double *dst = hT + (size_t)bh * dk * dv;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    dst[(size_t)i * dv + j] = S[(size_t)j * dk + i];
        }
        free(S);
        free(p);
    }
}

/*
 * Preconditioned two-gate delta rule.
 *   q (read key), k (raw key) [B,T,H,dk]; v [B,T,H,dv];
 *   alpha [B,T,H,dk] per key channel, or NULL (=> 1);
 *   erase b_t [B,T,H,dk] or NULL (=> 1); write w_t [B,T,H,dv] or NULL (=> 1);
 *   precond selects the per-channel preconditioner f of the curvature
 *   accumulator rho (0: none, f = 1):
 *     1  f = 1 / sqrt(rho + eps)                      (moving-average form)
 *     2  f = 1 / (rho + eps)                          (P_t = Diag(A_t)^-1, the
 *        pages' diagonal approximation, "Preconditioned DeltaNet ..." Arabic
 *        summary, section 2b)
 *     3  f = x^tanh(ln(1 / (rho + eps)) / ln x)      (2 squashed into [1/x, x]
 *        on a log scale, "Resumo Tecnico: Preconditioned DeltaNet", section 2,
 *        "Estabilidade e Parametrizacao"; the squash function is not printed)
 *   precond_query = 0 applies f to the write key (ATK), 1 to the query (ATQ)
 *   (Arabic summary, section 2a).
 * Per token:  rho   = rho_decay * rho + k_t (.) k_t          (rho_0 = 0)
 *   ATK:      kw    = f (.) k_t                               (write key)
 *             e     = b_t (.) kw  for precond 1,  b_t (.) k_t  for 2, 3
 *                     (the pages' forms read the state with the raw key and
 *                      write with the preconditioned one)
 *             qe    = q_t
 *   ATQ:      kw    = k_t,  e = b_t (.) k_t,  qe = f (.) q_t
 *             p     = S e
 *             S     = S diag(alpha_t) - p kw^T + (w_t (.) v_t) kw^T
 *             o_t   = S qe
 */
void oracle_precond_two_gate_fwd(int B, int T, int H, int dk, int dv,
                                 const double *q, const double *k, const double *v,
                                 const double *alpha, const double *erase,
                                 const double *write, int precond,
                                 double rho_decay, double rho_eps, double precond_x,
                                 int precond_query,
                                 const double *h0, double *o, double *hT,
                                 int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int bh = 0; bh < B * H; ++bh) {
        const int b = bh / H, h = bh % H;
        double *S = (double *)calloc((size_t)dv * dk, sizeof(double));
        double *rho = (double *)calloc((size_t)dk, sizeof(double));
        double *kw = (double *)malloc((size_t)dk * sizeof(double));
        double *e = (double *)malloc((size_t)dk * sizeof(double));
        double *qe = (double *)malloc((size_t)dk * sizeof(double));
        double *p = (double *)malloc((size_t)dv * sizeof(double));
        if (h0) {
            const double *src = h0 + (size_t)bh * dk * dv;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[(size_t)j * dk + i] = src[(size_t)i * dv + j];
        }
        for (int t = 0; t < T; ++t) {
            const size_t r = tok(b, t, h, T, H);
            const double *kt = k + r * dk, *qt = q + r * dk, *vt = v + r * dv;
            for (int i = 0; i < dk; ++i) {
                double f = 1.0;
                if (precond) {
                    rho[i] = rho_decay * rho[i] + kt[i] * kt[i];
                    const double a = rho[i] + rho_eps;
                    if (precond == 1) f = 1.0 / sqrt(a);
                    else if (precond == 2) f = 1.0 / a;
                    else f = pow(precond_x, tanh(log(1.0 / a) / log(precond_x)));
                }
                const double b = erase ? erase[r * dk + i] : 1.0;
                if (precond_query) {
                    kw[i] = kt[i];
                    e[i] = b * kt[i];
                    qe[i] = f * qt[i];
                } else {
                    kw[i] = f * kt[i];
                    e[i] = b * (precond == 1 ? kw[i] : kt[i]);
                    qe[i] = qt[i];
                }
            }
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[(size_t)j * dk + i] * e[i];
                p[j] = acc;
            }
            for (int j = 0; j < dv; ++j) {
                const double u = (write ? write[r * dv + j] : 1.0) * vt[j];
                double *row = S + (size_t)j * dk;
                for (int i = 0; i < dk; ++i) {
                    const double a = alpha ? alpha[r * dk + i] : 1.0;
                    row[i] = row[i] * a - p[j] * kw[i] + u * kw[i];
                }
            }
            double *ot = o + r * dv;
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[(size_t)j * dk + i] * qe[i];
                ot[j] = acc;
            }
        }
        if (hT) {
            double *dst = hT + (size_t)bh * dk * dv;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    dst[(size_t)i * dv + j] = S[(size_t)j * dk + i];
        }
        free(S);
        free(rho);
        free(kw);
        free(e);
        free(qe);
        free(p);
    }
}

/*
 * Reverse-mode gradient of oracle_gated_delta_fwd (the training use the pages
 * give chunkwise forms for: "Quando o 'Bom o Suficiente' e Otimo ...",
 * sections "Resumo" and "Declaracao do Problema").  The pages print no
 * backward pass; this is the adjoint of the token recurrence, one token at a
 * time in reverse order, derived by the chain rule from the forward update.
 *
 * Inputs as in the forward, plus
 *   dout [B,T,H,dv]           gradient of the loss with respect to o
 *   dhT  [B,H,dk,dv] or NULL  gradient with respect to the final state h_T
 * Outputs (all written in full; NULL skips one)
 *   dq, dkk [B,T,H,dk]; dvv [B,T,H,dv]; dalpha, dbeta [B,T,H]; dh0 [B,H,dk,dv]
 *
 * With S_t = alpha_t S_{t-1} + u_t k_t^T, u_t = beta_t (v_t - alpha_t p_t),
 * p_t = S_{t-1} k_t, o_t = S_t q_t, and D = dL/dS_t (d_v x d_k) the gradient
 * reaching S_t from later tokens:
 *   D      += do_t q_t^T                    (read-out of token t)
 *   dq_t    = S_t^T do_t
 *   du      = D k_t
 *   dv_t    = beta_t du
 *   dbeta_t = du . (v_t - alpha_t p_t)
 *   dalpha_t= <D, S_{t-1}> - beta_t du . p_t
 *   dk_t    = D^T u_t - alpha_t beta_t S_{t-1}^T du
 *   D      <- alpha_t D - alpha_t beta_t du k_t^T      (dL/dS_{t-1})
 * and dh0 = D^T after the first token.
 *
 * The states S_{t-1} are needed in reverse order.  They are recomputed from
 * checkpoints kept every SEG tokens: the recomputation repeats the forward's
 * operations in the forward's order, so every state is bit-identical to the
 * one the forward produced; only the memory footprint changes.
 */
#define ORACLE_SEG 64

static void fwd_token(double *S, double *p, int dk, int dv, const double *kt,
                      const double *vt, double a, double be)
{
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[(size_t)j * dk + i] * kt[i];
        p[j] = acc;
    }
    for (int j = 0; j < dv; ++j) {
        const double cp = a * be * p[j], cv = be * vt[j];
        double *row = S + (size_t)j * dk;
        for (int i = 0; i < dk; ++i)
            row[i] = a * row[i] - cp * kt[i] + cv * kt[i];
    }
}

void oracle_gated_delta_bwd(int B, int T, int H, int dk, int dv,
                            const double *q, const double *k, const double *v,
                            const double *alpha, const double *beta,
                            const double *h0, const double *dout, const double *dhT,
                            double *dq, double *dkk, double *dvv,
                            double *dalpha, double *dbeta, double *dh0,
                            int nthreads)
{
    const int nseg = (T + ORACLE_SEG - 1) / ORACLE_SEG;
    const size_t SZ = (size_t)dv * dk;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int bh = 0; bh < B * H; ++bh) {
        const int b = bh / H, h = bh % H;
        /* ckpt[s] = state before token s*SEG; seg[i] = state after token s*SEG+i-1 */
        double *ckpt = (double *)calloc((size_t)nseg * SZ, sizeof(double));
        double *seg = (double *)malloc((size_t)(ORACLE_SEG + 1) * SZ * sizeof(double));
        double *S = (double *)calloc(SZ, sizeof(double));
        double *D = (double *)calloc(SZ, sizeof(double));
        double *p = (double *)malloc((size_t)dv * sizeof(double));
        double *u = (double *)malloc((size_t)dv * sizeof(double));
        double *du = (double *)malloc((size_t)dv * sizeof(double));
        if (h0) {
            const double *src = h0 + (size_t)bh * dk * dv;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[(size_t)j * dk + i] = src[(size_t)i * dv + j];
        }
        /* forward sweep, keeping the checkpoints */
        for (int t = 0; t < T; ++t) {
            if (t % ORACLE_SEG == 0) memcpy(ckpt + (size_t)(t / ORACLE_SEG) * SZ, S, SZ * sizeof(double));
            const size_t r = tok(b, t, h, T, H);
            fwd_token(S, p, dk, dv, k + r * dk, v + r * dv,
                      alpha ? alpha[r] : 1.0, beta ? beta[r] : 1.0);
        }
        if (dhT) {
            const double *src = dhT + (size_t)bh * dk * dv;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    D[(size_t)j * dk + i] = src[(size_t)i * dv + j];
        }
        /* reverse sweep, one segment at a time */
        for (int s = nseg - 1; s >= 0; --s) {
            const int t0 = s * ORACLE_SEG;
            const int t1 = (t0 + ORACLE_SEG < T) ? t0 + ORACLE_SEG : T;
            memcpy(seg, ckpt + (size_t)s * SZ, SZ * sizeof(double));
            for (int t = t0; t < t1; ++t) {
                const size_t r = tok(b, t, h, T, H);
                double *Sn = seg + (size_t)(t - t0 + 1) * SZ;
                memcpy(Sn, Sn - SZ, SZ * sizeof(double));
                fwd_token(Sn, p, dk, dv, k + r * dk, v + r * dv,
                          alpha ? alpha[r] : 1.0, beta ? beta[r] : 1.0);
            }
            for (int t = t1 - 1; t >= t0; --t) {
                const size_t r = tok(b, t, h, T, H);
                const double *St = seg + (size_t)(t - t0 + 1) * SZ;  /* S_t */
                const double *Sp = St - SZ;                          /* S_{t-1} */
                const double *kt = k + r * dk, *qt = q + r * dk, *vt = v + r * dv;
                const double *dot = dout + r * dv;
                const double a = alpha ? alpha[r] : 1.0;
                const double be = beta ? beta[r] : 1.0;
                for (int j = 0; j < dv; ++j)
                    for (int i = 0; i < dk; ++i) D[(size_t)j * dk + i] += dot[j] * qt[i];
                if (dq)
                    for (int i = 0; i < dk; ++i) {
                        double acc = 0.0;
                        for (int j = 0; j < dv; ++j) acc += St[(size_t)j * dk + i] * dot[j];
                        dq[r * dk + i] = acc;
                    }
                for (int j = 0; j < dv; ++j) {
                    double pj = 0.0, dj = 0.0;
                    for (int i = 0; i < dk; ++i) {
                        pj += Sp[(size_t)j * dk + i] * kt[i];
                        dj += D[(size_t)j * dk + i] * kt[i];
                    }
                    p[j] = pj;
                    du[j] = dj;
                    u[j] = be * (vt[j] - a * pj);
                }
                if (dvv)
                    for (int j = 0; j < dv; ++j) dvv[r * dv + j] = be * du[j];
                if (dbeta) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += du[j] * (vt[j] - a * p[j]);
                    dbeta[r] = acc;
                }
                if (dalpha) {
                    double acc = 0.0;
                    for (size_t x = 0; x < SZ; ++x) acc += D[x] * Sp[x];
                    for (int j = 0; j < dv; ++j) acc -= be * du[j] * p[j];
                    dalpha[r] = acc;
                }
                if (dkk)
                    for (int i = 0; i < dk; ++i) {
                        double acc = 0.0;
                        for (int j = 0; j < dv; ++j)
                            acc += D[(size_t)j * dk + i] * u[j] - a * be * Sp[(size_t)j * dk + i] * du[j];
                        dkk[r * dk + i] = acc;
                    }
                for (int j = 0; j < dv; ++j) {
                    double *row = D + (size_t)j * dk;
                    const double c = a * be * du[j];
                    for (int i = 0; i < dk; ++i) row[i] = a * row[i] - c * kt[i];
                }
            }
        }
        if (dh0) {
            double *dst = dh0 + (size_t)bh * dk * dv;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    dst[(size_t)i * dv + j] = D[(size_t)j * dk + i];
        }
        free(ckpt);
        free(seg);
        free(S);
        free(D);
        free(p);
        free(u);
        free(du);
    }
}
