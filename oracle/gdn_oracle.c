/*
 * Plain CPU oracle for the gated delta-rule (GDN) token mixer of a looped
 * linear-time transformer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may link,
 * load or call this file: only the test suite, the smoke check of the build
 * entry point and the benchmark's CPU-baseline leg use it.  It shares no code
 * with the CUDA kernels.
 *
 * What it computes ("LT2: Linear-Time Looped Transformers", §2, the "LT2."
 * paragraph: q_t, k_t in R^{dk}, v_t in R^{dv}, recurrent state
 * S_t in R^{dk x dv}; the mixer is Gated DeltaNet, named in Appendix C).
 * The page's display equations were lost, so the update is the gated delta
 * rule in its usual form, written in the page's dk x dv orientation
 * (Sigma = S^T of the dv x dk form):
 *
 *     Sigma_t = a_t (I - b_t k_t k_t^T) Sigma_{t-1} + b_t k_t v_t^T
 *     o_t     = scale * Sigma_t^T q_t
 *
 * evaluated token by token in double precision, exactly as written: the
 * product (I - b k k^T) Sigma is evaluated as Sigma - b k (k^T Sigma), which is
 * the same expression with the matrix-vector product done first.  No chunking,
 * no blocking, no reordering across tokens.  Independent (sequence, head)
 * chains run in parallel with OpenMP; each chain is sequential.
 *
 * Layouts (all dense, row-major, doubles):
 *   q, k  [n_tok][H][dk]      v, o  [n_tok][H][dv]      a, b  [n_tok][H]
 *   S0, ST [n_seq][H][dk][dv] (S0 may be NULL = zeros; ST may be NULL)
 *   cu_seqlens int32 [n_seq+1], token offsets of each packed sequence.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One step of the recurrence on one head's state.  sig is dk x dv, row-major.
 * y is caller scratch of length dv. */
static void gdn_token_step(double *sig, int dk, int dv,
                           const double *q, const double *k, const double *v,
                           double a, double b, double scale,
                           double *o, double *y)
{
    /* y = k^T Sigma_{t-1}  (a row vector over dv) */
    for (int j = 0; j < dv; ++j) y[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double ki = k[i];
        const double *row = sig + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) y[j] += ki * row[j];
    }
    /* Sigma_t = a (Sigma - b k y) + b k v^T */
    for (int i = 0; i < dk; ++i) {
        const double ki = k[i];
        double *row = sig + (size_t)i * dv;
        for (int j = 0; j < dv; ++j)
            row[j] = a * (row[j] - b * ki * y[j]) + b * ki * v[j];
    }
    /* o_t = scale * Sigma_t^T q */
    if (o) {
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double qi = q[i];
            const double *row = sig + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) o[j] += qi * row[j];
        }
        for (int j = 0; j < dv; ++j) o[j] *= scale;
    }
}

/* Prefill over packed sequences: every (sequence, head) chain starts from its
 * S0 (or zero) and walks its tokens in order. Returns 0, or -1 on bad args. */
int oracle_gdn_fwd(const double *q, const double *k, const double *v,
                   const double *a, const double *b, const double *S0,
                   double *o, double *ST, const int32_t *cu_seqlens,
                   int n_seq, int H, int dk, int dv, double scale)
{
    if (!q || !k || !v || !a || !b || !o || !cu_seqlens) return -1;
    if (n_seq < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    for (int s = 0; s < n_seq; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
    const long n_chain = (long)n_seq * H;
    int bad = 0;
#pragma omp parallel
    {
        double *sig = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *y = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!sig || !y) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long c = 0; c < n_chain; ++c) {
                const int s = (int)(c / H), h = (int)(c % H);
                const size_t sidx = ((size_t)s * H + h) * (size_t)dk * dv;
                if (S0) memcpy(sig, S0 + sidx, sizeof(double) * (size_t)dk * dv);
                else memset(sig, 0, sizeof(double) * (size_t)dk * dv);
                for (int t = cu_seqlens[s]; t < cu_seqlens[s + 1]; ++t) {
                    const size_t th = (size_t)t * H + h;
                    gdn_token_step(sig, dk, dv, q + th * dk, k + th * dk, v + th * dv,
                                   a[th], b[th], scale, o + th * dv, y);
                }
                if (ST) memcpy(ST + sidx, sig, sizeof(double) * (size_t)dk * dv);
            }
        }
        free(sig);
        free(y);
    }
    return bad ? -1 : 0;
}

/* Decode: one token for each of N independent slots (a slot is one
 * sequence x layer x loop state), H heads each; S [N][H][dk][dv] updated in
 * place, o [N][H][dv]. */
int oracle_gdn_decode(const double *q, const double *k, const double *v,
                      const double *a, const double *b, double *S, double *o,
                      int N, int H, int dk, int dv, double scale)
{
    if (!q || !k || !v || !a || !b || !S || !o) return -1;
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    const long n_chain = (long)N * H;
    int bad = 0;
#pragma omp parallel
    {
        double *y = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!y) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(static)
            for (long c = 0; c < n_chain; ++c) {
                gdn_token_step(S + (size_t)c * dk * dv, dk, dv, q + (size_t)c * dk,
                               k + (size_t)c * dk, v + (size_t)c * dv, a[c], b[c],
                               scale, o + (size_t)c * dv, y);
            }
        }
        free(y);
    }
    return bad ? -1 : 0;
}

/* Per-loop learned residual ("LT2: Linear-Time Looped Transformers", §2,
 * "LT2." paragraph): h = h_tilde + rho (.) h_prev, rho per channel.
 * h_tilde, h_prev, h_out [rows][d]; rho [d]. */
int oracle_loop_residual(const double *h_tilde, const double *h_prev,
                         const double *rho, double *h_out, long rows, int d)
{
    if (!h_tilde || !h_prev || !rho || !h_out || rows < 0 || d <= 0) return -1;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r)
        for (int c = 0; c < d; ++c)
            h_out[(size_t)r * d + c] =
                h_tilde[(size_t)r * d + c] + rho[c] * h_prev[(size_t)r * d + c];
    return 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
