/*
 * CPU oracle for the gated delta-rule recurrence with channel-wise decay.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference leg load this file's library.  It
 * shares no code, header or constant with the GPU library and must never be
 * reached from the product path.
 *
 * What it computes (plain float64, token by token, no blocking or
 * reordering).  For every sequence n and head h:
 *
 *   S <- initial_state[n,h] or 0                       (document reset,
 *                                                       openarchlab "GDN, KDA
 *                                                       va Mamba-2" sec. 3)
 *   for each token t of the sequence, in order:
 *     (a~, m) from the variant:                        (Raon-1-mini-preview
 *        KDA   : a~ = beta_t k_t,   m = beta_t v_t      discussion, equations
 *        RDA   : a~ = e_t k_t,      m = w_t v_t         "KDA:", "RDA:",
 *        GDN-2 : a~ = b_t (.) k_t,  m = w_t (.) v_t     "GDN-2:")
 *     S' = Diag(alpha_t) S          decay first: every update on that page
 *                                   applies Diag(alpha_t) to S_{t-1} before
 *                                   the rank-one erase
 *     u  = m - S'^T a~              the delta rule's "value minus what the
 *                                   state predicts for this key" (openarchlab
 *                                   page, sec. 1 and the v - Sk remark, sec. 3)
 *     S  = S' + k_t u^T
 *     o_t = S^T q_t                 readout on the post-update state
 *
 * Expanding (I - k a~^T) S' + k m^T = S' + k (m - S'^T a~)^T shows this is the
 * pages' product form term for term; the Python side also carries the literal
 * product form and a brute-force dense form, and the tests pin all three
 * against each other and against closed forms.
 *
 * Layouts (row-major, C order):
 *   q, k, alpha : [B,T,H,dk]    v : [B,T,H,dv]    o : [B,T,H,dv]
 *   g1 : KDA beta / RDA e [B,T,H];  GDN-2 b [B,T,H,dk]
 *   g2 : KDA unused (NULL) / RDA w [B,T,H];  GDN-2 w [B,T,H,dv]
 *   state : [N,H,dk,dv]  (rows = key channel, columns = value channel)
 * With cu_seqlens (N+1 offsets into T) B must be 1 and sequence n spans
 * tokens [cu[n], cu[n+1]); otherwise sequence n is batch row n (N = B).
 */
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_KDA = 0, ORACLE_RDA = 1, ORACLE_GDN2 = 2 };

static void run_one(int variant, int T0, int len, int b, int T, int H, int h, int dk, int dv,
                    const double *q, const double *k, const double *v, const double *alpha,
                    const double *g1, const double *g2, const double *s0, double *sf,
                    double *o, double *S, double *at, double *mt, double *u)
{
    if (s0) memcpy(S, s0, sizeof(double) * (size_t)dk * dv);
    else memset(S, 0, sizeof(double) * (size_t)dk * dv);
    for (int t = T0; t < T0 + len; ++t) {
        size_t tok = ((size_t)b * T + t) * H + h;
        const double *qt = q + tok * dk, *kt = k + tok * dk, *vt = v + tok * dv;
        const double *al = alpha + tok * dk;
        /* erase direction a~ and written value m */
        for (int i = 0; i < dk; ++i) {
            double g = (variant == ORACLE_GDN2) ? g1[tok * dk + i] : g1[tok];
            at[i] = g * kt[i];
        }
        for (int j = 0; j < dv; ++j) {
            double g;
            if (variant == ORACLE_KDA) g = g1[tok];
            else if (variant == ORACLE_RDA) g = g2[tok];
            else g = g2[tok * dv + j];
            mt[j] = g * vt[j];
        }
        /* S' = Diag(alpha) S */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= al[i];
        /* u = m - S'^T a~ */
        for (int j = 0; j < dv; ++j) u[j] = mt[j];
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) u[j] -= S[(size_t)i * dv + j] * at[i];
        /* S = S' + k u^T */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += kt[i] * u[j];
        /* o_t = S^T q_t */
        double *ot = o + tok * dv;
        for (int j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) ot[j] += S[(size_t)i * dv + j] * qt[i];
    }
    if (sf) memcpy(sf, S, sizeof(double) * (size_t)dk * dv);
}

/* Returns 0 on success, -1 on a bad argument. */
int oracle_recurrence(int variant, int B, int T, int H, int dk, int dv,
                      const double *q, const double *k, const double *v, const double *alpha,
                      const double *g1, const double *g2,
                      const int *cu_seqlens, int num_seqs,
                      const double *s0, double *s_final, double *o, int n_threads)
{
    if (variant < 0 || variant > 2 || B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return -1;
    if (!q || !k || !v || !alpha || !g1 || !o) return -1;
    if (variant != ORACLE_KDA && !g2) return -1;
    int N = B;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 1 || cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T) return -1;
        for (int n = 0; n < num_seqs; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
        N = num_seqs;
    }
    long work = (long)N * H;
    /* the thread count applies to this call only (a num_threads clause, not
       omp_set_num_threads, which would persist into later calls) */
#ifdef _OPENMP
    const int nt = n_threads > 0 ? n_threads : omp_get_max_threads();
#else
    (void)n_threads;
#endif
    int err = 0;
#pragma omp parallel num_threads(nt)
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *at = (double *)malloc(sizeof(double) * (size_t)dk);
        double *mt = (double *)malloc(sizeof(double) * (size_t)dv);
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!S || !at || !mt || !u) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long w = 0; w < work; ++w) {
                int n = (int)(w / H), h = (int)(w % H);
                int b = cu_seqlens ? 0 : n;
                int T0 = cu_seqlens ? cu_seqlens[n] : 0;
                int len = cu_seqlens ? cu_seqlens[n + 1] - cu_seqlens[n] : T;
                size_t soff = ((size_t)n * H + h) * (size_t)dk * dv;
                run_one(variant, T0, len, b, T, H, h, dk, dv, q, k, v, alpha, g1, g2,
                        s0 ? s0 + soff : NULL, s_final ? s_final + soff : NULL, o, S, at, mt, u);
            }
        }
        free(S); free(at); free(mt); free(u);
    }
    return err ? -1 : 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
