/*
 * gdn_oracle.c -- float64 CPU oracle for the Gated Delta Network (GDN) layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the CPU-baseline
 * leg of bench.py load this file's library.  It shares no code, header, table
 * or helper with the CUDA path and must never be reached from the product path.
 *
 * What it computes (the layer the FlashQLA pages accelerate: news.hamidun.com
 * "Qwen FlashQLA ... Hopper", section "What is FlashQLA": forward and backward
 * of GDN in chunked-prefill mode).  The pages do not print the rule; it is the
 * standard gated delta rule, per (sequence, value head):
 *
 *     S_t = exp(g_t) * S_{t-1} * (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t q_t
 *
 * S_t is dv x dk.  The oracle stores its transpose H = S^T (dk x dv, row-major,
 * the layout the library's S0/ST arrays use), so the rule reads, token by token:
 *
 *     H  <- exp(g_t) H                 (gate the previous state)
 *     p   = H^T k_t                    (what the gated state recalls for k_t)
 *     H  <- H + beta_t k_t (v_t - p)^T (delta-rule write)
 *     o_t = H^T q_t                    (read with the updated state)
 *
 * There is no chunking, no blocking and no reordering: one token at a time, in
 * float64.  Chunked prefill is the same computation split into calls whose
 * S_T feeds the next call's S0 (news.hamidun.com page, "Chunked Prefill"
 * scenario).
 *
 * Backward: the reverse-mode adjoint of the four token steps above, taken in
 * reverse token order.  Forward states are checkpointed every CKPT tokens and
 * re-run inside each checkpoint window, so memory stays O(T/CKPT * dk * dv).
 *
 * Layouts (all row-major, float64, tokens packed):
 *   q, k   [T_total, Hk, dk]      v, o   [T_total, Hv, dv]
 *   beta, g [T_total, Hv]         S0, ST [N, Hv, dk, dv]
 *   cu_seqlens int64 [N+1]: sequence n owns tokens [cu[n], cu[n+1]).
 *   Value head h reads q/k head h / (Hv / Hk)  (contiguous groups).
 * NULL S0 means a zero initial state; NULL ST skips writing the final state.
 * Return value: 0 on success, 1 on bad arguments, 2 on allocation failure.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define CKPT 64

static int check_args(int64_t N, const int64_t* cu, int Hk, int Hv, int dk, int dv) {
    if (N < 0 || !cu || Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0) return 1;
    if (Hv % Hk != 0) return 1;
    if (cu[0] != 0) return 1;
    for (int64_t n = 0; n < N; ++n)
        if (cu[n + 1] < cu[n]) return 1;
    return 0;
}

/* ---------------------------------------------------------------- forward */

int gdn_oracle_fwd(int64_t N, const int64_t* cu, int Hk, int Hv, int dk, int dv,
                   const double* q, const double* k, const double* v,
                   const double* beta, const double* g, const double* S0,
                   double* o, double* ST) {
    if (check_args(N, cu, Hk, Hv, dk, dv)) return 1;
    const int group = Hv / Hk;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t unit = 0; unit < N * Hv; ++unit) {
        const int64_t n = unit / Hv;
        const int h = (int)(unit % Hv);
        const int hk = h / group;
        double* H = (double*)malloc(sizeof(double) * dk * dv);
        double* p = (double*)malloc(sizeof(double) * dv);
        if (!H || !p) {
            free(H);
            free(p);
#pragma omp atomic write
            err = 2;
            continue;
        }
        if (S0)
            memcpy(H, S0 + (n * Hv + h) * (int64_t)dk * dv, sizeof(double) * dk * dv);
        else
            memset(H, 0, sizeof(double) * dk * dv);

        for (int64_t t = cu[n]; t < cu[n + 1]; ++t) {
            const double* kt = k + (t * Hk + hk) * (int64_t)dk;
            const double* qt = q + (t * Hk + hk) * (int64_t)dk;
            const double* vt = v + (t * Hv + h) * (int64_t)dv;
            const double a = exp(g[t * Hv + h]);
            const double b = beta[t * Hv + h];
            /* H <- a H */
            for (int i = 0; i < dk * dv; ++i) H[i] *= a;
            /* p = H^T k */
            for (int j = 0; j < dv; ++j) p[j] = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) p[j] += H[i * dv + j] * kt[i];
            /* H <- H + b k (v - p)^T */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) H[i * dv + j] += b * kt[i] * (vt[j] - p[j]);
            /* o = H^T q */
            double* ot = o + (t * Hv + h) * (int64_t)dv;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) ot[j] += H[i * dv + j] * qt[i];
        }
        if (ST) memcpy(ST + (n * Hv + h) * (int64_t)dk * dv, H, sizeof(double) * dk * dv);
        free(H);
        free(p);
    }
    return err;
}

/* --------------------------------------------------------------- backward */

/* One token step forward, keeping the gated state H1 = exp(g) H0 (needed by the
 * adjoint).  H is updated in place from H0 to H2. */
static void token_step(double* H, double* H1, double* p, int dk, int dv, const double* kt,
                       const double* vt, double a, double b) {
    for (int i = 0; i < dk * dv; ++i) H[i] *= a;
    if (H1) memcpy(H1, H, sizeof(double) * dk * dv);
    for (int j = 0; j < dv; ++j) p[j] = 0.0;
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) p[j] += H[i * dv + j] * kt[i];
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) H[i * dv + j] += b * kt[i] * (vt[j] - p[j]);
}

/*
 * Adjoint of one token, in reverse.  Forward sub-steps and their adjoints:
 *   H1 = a H0            ->  dg += <dH1, H1>,  dH0 = a dH1
 *   p  = H1^T k          ->  dH1 += k dp^T,    dk += H1 dp
 *   e  = v - p           ->  dv = de,          dp = -de
 *   H2 = H1 + b k e^T    ->  dH1 = dH2, db = k^T dH2 e, dk += b dH2 e, de = b dH2^T k
 *   o  = H2^T q          ->  dH2 += q do^T,    dq = H2 do
 * dH holds dH2 on entry and dH0 on exit.
 */
int gdn_oracle_bwd(int64_t N, const int64_t* cu, int Hk, int Hv, int dk, int dv,
                   const double* q, const double* k, const double* v,
                   const double* beta, const double* g, const double* S0,
                   const double* dout, const double* dST,
                   double* dq, double* dkey, double* dval, double* dbeta, double* dg,
                   double* dS0) {
    if (check_args(N, cu, Hk, Hv, dk, dv)) return 1;
    const int group = Hv / Hk;
    const int64_t T_total = cu[N];
    /* q/k gradients are sums over the value heads of a group; each (seq, k-head)
     * unit owns its rows, so units never write the same element. */
    memset(dq, 0, sizeof(double) * T_total * Hk * dk);
    memset(dkey, 0, sizeof(double) * T_total * Hk * dk);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t unit = 0; unit < N * Hk; ++unit) {
        const int64_t n = unit / Hk;
        const int hk = (int)(unit % Hk);
        const int64_t bos = cu[n], len = cu[n + 1] - cu[n];
        const int64_t nck = (len + CKPT - 1) / CKPT;
        const size_t S = (size_t)dk * dv;
        double* ck = (double*)malloc(sizeof(double) * S * (nck > 0 ? nck : 1));
        double* H1w = (double*)malloc(sizeof(double) * S * CKPT); /* gated states */
        double* H = (double*)malloc(sizeof(double) * S);
        double* H2 = (double*)malloc(sizeof(double) * S);
        double* dH = (double*)malloc(sizeof(double) * S);
        double* p = (double*)malloc(sizeof(double) * dv);
        double* e = (double*)malloc(sizeof(double) * dv);
        double* de = (double*)malloc(sizeof(double) * dv);
        if (!ck || !H1w || !H || !H2 || !dH || !p || !e || !de) {
            free(ck); free(H1w); free(H); free(H2); free(dH); free(p); free(e); free(de);
#pragma omp atomic write
            err = 2;
            continue;
        }
        for (int hh = 0; hh < group; ++hh) {
            const int h = hk * group + hh;
            /* forward with checkpoints: ck[c] = state before token bos + c*CKPT */
            if (S0) memcpy(H, S0 + (n * Hv + h) * S, sizeof(double) * S);
            else memset(H, 0, sizeof(double) * S);
            for (int64_t c = 0; c < nck; ++c) {
                memcpy(ck + c * S, H, sizeof(double) * S);
                int64_t t1 = bos + (c + 1) * CKPT;
                if (t1 > bos + len) t1 = bos + len;
                for (int64_t t = bos + c * CKPT; t < t1; ++t)
                    token_step(H, NULL, p, dk, dv, k + (t * Hk + hk) * (int64_t)dk,
                               v + (t * Hv + h) * (int64_t)dv, exp(g[t * Hv + h]),
                               beta[t * Hv + h]);
            }
            /* adjoint, starting from dS_T */
            if (dST) memcpy(dH, dST + (n * Hv + h) * S, sizeof(double) * S);
            else memset(dH, 0, sizeof(double) * S);
            for (int64_t c = nck - 1; c >= 0; --c) {
                const int64_t t0 = bos + c * CKPT;
                int64_t t1 = t0 + CKPT;
                if (t1 > bos + len) t1 = bos + len;
                /* re-run the window, keeping each token's gated state H1 */
                memcpy(H, ck + c * S, sizeof(double) * S);
                for (int64_t t = t0; t < t1; ++t)
                    token_step(H, H1w + (t - t0) * S, p, dk, dv,
                               k + (t * Hk + hk) * (int64_t)dk, v + (t * Hv + h) * (int64_t)dv,
                               exp(g[t * Hv + h]), beta[t * Hv + h]);
                for (int64_t t = t1 - 1; t >= t0; --t) {
                    const double* kt = k + (t * Hk + hk) * (int64_t)dk;
                    const double* qt = q + (t * Hk + hk) * (int64_t)dk;
                    const double* vt = v + (t * Hv + h) * (int64_t)dv;
                    const double* dot = dout + (t * Hv + h) * (int64_t)dv;
                    const double a = exp(g[t * Hv + h]);
                    const double b = beta[t * Hv + h];
                    const double* H1 = H1w + (t - t0) * S;
                    double* dqt = dq + (t * Hk + hk) * (int64_t)dk;
                    double* dkt = dkey + (t * Hk + hk) * (int64_t)dk;
                    /* recompute p, e and H2 from H1 */
                    for (int j = 0; j < dv; ++j) p[j] = 0.0;
                    for (int i = 0; i < dk; ++i)
                        for (int j = 0; j < dv; ++j) p[j] += H1[i * dv + j] * kt[i];
                    for (int j = 0; j < dv; ++j) e[j] = vt[j] - p[j];
                    for (int i = 0; i < dk; ++i)
                        for (int j = 0; j < dv; ++j) H2[i * dv + j] = H1[i * dv + j] + b * kt[i] * e[j];
                    /* o = H2^T q */
                    for (int i = 0; i < dk; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < dv; ++j) {
                            dH[i * dv + j] += qt[i] * dot[j];
                            s += H2[i * dv + j] * dot[j];
                        }
                        dqt[i] += s;
                    }
                    /* H2 = H1 + b k e^T */
                    double db = 0.0;
                    for (int j = 0; j < dv; ++j) de[j] = 0.0;
                    for (int i = 0; i < dk; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < dv; ++j) {
                            s += dH[i * dv + j] * e[j];
                            de[j] += b * dH[i * dv + j] * kt[i];
                        }
                        db += kt[i] * s;
                        dkt[i] += b * s;
                    }
                    dbeta[t * Hv + h] = db;
                    /* e = v - p, p = H1^T k */
                    double* dvt = dval + (t * Hv + h) * (int64_t)dv;
                    for (int j = 0; j < dv; ++j) dvt[j] = de[j];
                    for (int i = 0; i < dk; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < dv; ++j) {
                            dH[i * dv + j] -= kt[i] * de[j];
                            s += H1[i * dv + j] * de[j];
                        }
                        dkt[i] -= s;
                    }
                    /* H1 = a H0 */
                    double dgt = 0.0;
                    for (size_t i = 0; i < S; ++i) dgt += dH[i] * H1[i];
                    dg[t * Hv + h] = dgt;
                    for (size_t i = 0; i < S; ++i) dH[i] *= a;
                }
            }
            if (dS0) memcpy(dS0 + (n * Hv + h) * S, dH, sizeof(double) * S);
        }
        free(ck); free(H1w); free(H); free(H2); free(dH); free(p); free(e); free(de);
    }
    return err;
}

int gdn_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
