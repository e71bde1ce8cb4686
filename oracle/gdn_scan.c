/*
 * Oracle: fp64 sequential scan of the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or
 * call this file; only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference leg use it. It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes. The pages ("A Modern Multimodal Assistant on a 6 GB 2011
 * GPU", abstract, result (i)) name the recurrent layers of a hybrid
 * gated-delta-net backbone and a "sequential scan" of them, the token-by-token
 * form that the chunked delta-rule rewrite replaces (page 2, "Resumen
 * Tecnico", Metodologia, "Capas Recurrentes"). The recurrence itself is the
 * gated delta rule of the paper the pages cite by title ("Gated Delta
 * Networks: Improving Mamba2 with Delta Rule", page 3 reference list). Per
 * sequence n and head h, with S a dv x dk matrix (row = value index):
 *
 *     alpha_t = exp(g_t)
 *     S_t     = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t     = S_t q_t
 *
 * written out term by term below:
 *     S_t[i][j] = alpha S[i][j] - alpha beta (S k)[i] k[j] + beta v[i] k[j].
 * No blocking, no chunking, no reordering beyond this definition.
 *
 * Layouts (token-major, all contiguous, fp64):
 *   q, k : [T_tot][H][dk]     v, o : [T_tot][H][dv]
 *   g, beta : [T_tot][H]      S0, S_T : [N][H][dv][dk]
 *   cu_seqlens : [N+1] int64, sequence n covers tokens [cu[n], cu[n+1]).
 * S0 may be NULL (zero initial state). Parallel over (n, h) with OpenMP.
 * Returns 0 on success, -1 on a malformed cu_seqlens, -2 on allocation failure.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int gdn_oracle_scan_f64(const double *q, const double *k, const double *v,
                        const double *g, const double *beta, const double *S0,
                        const int64_t *cu_seqlens, int N, int H, int dk, int dv,
                        double *o, double *S_T)
{
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n] || cu_seqlens[0] != 0) return -1;

    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int nh = 0; nh < N * H; ++nh) {
        const int n = nh / H, h = nh % H;
        double *S = (double *)malloc(sizeof(double) * (size_t)dv * dk);
        double *Sk = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!S || !Sk) {
            free(S);
            free(Sk);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        const size_t sbase = ((size_t)n * H + h) * (size_t)dv * dk;
        if (S0)
            memcpy(S, S0 + sbase, sizeof(double) * (size_t)dv * dk);
        else
            memset(S, 0, sizeof(double) * (size_t)dv * dk);

        for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
            const double *qt = q + ((size_t)t * H + h) * dk;
            const double *kt = k + ((size_t)t * H + h) * dk;
            const double *vt = v + ((size_t)t * H + h) * dv;
            const double alpha = exp(g[(size_t)t * H + h]);
            const double b = beta[(size_t)t * H + h];

            /* (S_{t-1} k_t) */
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * kt[j];
                Sk[i] = acc;
            }
            /* S_t = alpha S_{t-1} - alpha beta (S_{t-1} k_t) k_t^T + beta v_t k_t^T */
            for (int i = 0; i < dv; ++i)
                for (int j = 0; j < dk; ++j)
                    S[(size_t)i * dk + j] = alpha * S[(size_t)i * dk + j]
                                            - alpha * b * Sk[i] * kt[j]
                                            + b * vt[i] * kt[j];
            /* o_t = S_t q_t */
            double *ot = o + ((size_t)t * H + h) * dv;
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * qt[j];
                ot[i] = acc;
            }
        }
        memcpy(S_T + sbase, S, sizeof(double) * (size_t)dv * dk);
        free(S);
        free(Sk);
    }
    return failed ? -2 : 0;
}

/* Number of OpenMP threads a parallel region of the scan uses (1 without OpenMP). */
int gdn_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Cap the OpenMP thread count used by later scans (ignored without OpenMP). */
void gdn_oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
