/*
 * Float64 CPU oracle for the Comba recurrence -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg may load this library.  The CUDA library never links, includes or calls
 * it, and it shares no code with the CUDA sources.
 *
 * What it computes is the plain token-by-token definition of Comba's
 * scalar-plus-low-rank (SPLR) bilinear RNN with output correction, as the
 * PaperWeekly write-up "Comba: Improving Bilinear RNNs with Closed-loop
 * Control" describes it (section "Comba架构：基于闭环控制理论": a scalar decay on
 * the identity plus a rank-1 key correction, then the same key used as the
 * output feedback) and the arXiv abstract of the same paper states
 * (scalar-plus-low-rank transition with state- and output-feedback
 * corrections).  The page's formulas were lost in extraction; the form used
 * here is
 *
 *     S_t = alpha_t * S_{t-1} - b_e,t * S_{t-1} k_t k_t^T + b_w,t * v_t k_t^T
 *     o_t = S_t (q_t - d_h k_t)
 *
 * with alpha_t = exp(log_alpha_t), S in R^{dv x dk}, and the output read from
 * the post-update state.  The product path ties b_e = b_w = beta; the two are
 * separate here only so that a self-test can switch the erase term off and
 * recover causal (gated) linear attention exactly.
 *
 * Layouts (row-major): q,k [B,T,H,dk]; v [B,T,H,dv]; log_alpha, beta_* [B,T,H];
 * d [H]; S0, S_final [B,H,dv,dk] (S0 may be NULL: zero state; S_final may be
 * NULL; S_final may alias S0); out [B,T,H,dv].
 *
 * Parity pins (closed forms, a hand-worked example, brute-force products,
 * invariants) live in the tests; every function here is pinned by them.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static void one_chain(const double* q, const double* k, const double* v,
                      const double* log_alpha, const double* beta_e,
                      const double* beta_w, double d_h, const double* S0,
                      double* out, double* S_final, long b, long h,
                      long T, long H, long dk, long dv,
                      double* S, double* Sk, double* qt) {
    if (S0) memcpy(S, S0 + (b * H + h) * dv * dk, sizeof(double) * dv * dk);
    else memset(S, 0, sizeof(double) * dv * dk);
    for (long t = 0; t < T; ++t) {
        const long bth = (b * T + t) * H + h;
        const double* kt = k + bth * dk;
        const double* qv = q + bth * dk;
        const double* vt = v + bth * dv;
        const double a = exp(log_alpha[bth]);
        const double be = beta_e[bth];
        const double bw = beta_w[bth];
        /* Sk = S_{t-1} k_t : the state's current read-out at the key. */
        for (long i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (long j = 0; j < dk; ++j) acc += S[i * dk + j] * kt[j];
            Sk[i] = acc;
        }
        /* The three terms of the SPLR transition, each written out. */
        for (long i = 0; i < dv; ++i)
            for (long j = 0; j < dk; ++j)
                S[i * dk + j] = a * S[i * dk + j] - be * Sk[i] * kt[j] + bw * vt[i] * kt[j];
        /* Output correction: query minus d_h times the key, read from S_t. */
        for (long j = 0; j < dk; ++j) qt[j] = qv[j] - d_h * kt[j];
        double* ot = out + bth * dv;
        for (long i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (long j = 0; j < dk; ++j) acc += S[i * dk + j] * qt[j];
            ot[i] = acc;
        }
    }
    if (S_final) memcpy(S_final + (b * H + h) * dv * dk, S, sizeof(double) * dv * dk);
}

/* Returns 0 on success, -1 on bad sizes, -2 on allocation failure. */
int comba_oracle_recurrence_f64(const double* q, const double* k, const double* v,
                                const double* log_alpha, const double* beta_e,
                                const double* beta_w, const double* d,
                                const double* S0, double* out, double* S_final,
                                long B, long T, long H, long dk, long dv,
                                int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    const long chains = B * H;
    int status = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double* S = (double*)malloc(sizeof(double) * dv * dk);
        double* Sk = (double*)malloc(sizeof(double) * dv);
        double* qt = (double*)malloc(sizeof(double) * dk);
        const int ok = S && Sk && qt;
        if (!ok) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = -2;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (long c = 0; c < chains; ++c)
            if (ok)
                one_chain(q, k, v, log_alpha, beta_e, beta_w, d[c % H], S0, out,
                          S_final, c / H, c % H, T, H, dk, dv, S, Sk, qt);
        free(S);
        free(Sk);
        free(qt);
    }
    return status;
}

int comba_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
