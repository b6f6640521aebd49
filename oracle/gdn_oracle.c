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
#include <math.h>
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

/* Reverse mode of the prefill: gradients of a scalar loss that depends on the
 * outputs o (through dO = dloss/do) and on the final states (through
 * dST = dloss/dS_T, or NULL for none).  Per chain, token by token backwards,
 * with G_t the gradient with respect to Sigma_t (the part flowing back from
 * the later tokens and the final state, plus the readout of token t itself):
 *
 *     G_t          = dSigma_t + scale q_t dO_t^T
 *     x_t          = Sigma_{t-1}^T k_t,      y_t = G_t^T k_t          (dv)
 *     dq_t         = scale Sigma_t dO_t
 *     dv_t         = b_t y_t
 *     dk_t         = -a_t b_t (G_t x_t + Sigma_{t-1} y_t) + b_t G_t v_t
 *     da_t         = <G_t, Sigma_{t-1}> - b_t y_t . x_t
 *     db_t         = y_t . (v_t - a_t x_t)
 *     dSigma_{t-1} = a_t (G_t - b_t k_t y_t^T)
 *
 * and dS0 = dSigma_0.  Each term is the derivative of one factor of the
 * update Sigma_t = a_t (Sigma_{t-1} - b_t k_t x_t^T) + b_t k_t v_t^T or of the
 * readout.  The forward states Sigma_0 .. Sigma_L of a chain are recomputed
 * with the same token step and kept in memory ((L + 1) dk dv doubles per
 * chain in flight).  Output layouts as the inputs; dS0 may be NULL.
 * Returns 0, or -1 on bad arguments or memory exhaustion. */
int oracle_gdn_bwd(const double *q, const double *k, const double *v,
                   const double *a, const double *b, const double *S0,
                   const double *dO, const double *dST, const int32_t *cu_seqlens,
                   int n_seq, int H, int dk, int dv, double scale,
                   double *dq, double *dk_out, double *dv_out, double *da, double *db,
                   double *dS0)
{
    if (!q || !k || !v || !a || !b || !dO || !cu_seqlens) return -1;
    if (!dq || !dk_out || !dv_out || !da || !db) return -1;
    if (n_seq < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    for (int s = 0; s < n_seq; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
    const long n_chain = (long)n_seq * H;
    const size_t sz = (size_t)dk * dv;
    int bad = 0;
#pragma omp parallel
    {
        double *G = (double *)malloc(sizeof(double) * sz);
        double *x = (double *)malloc(sizeof(double) * (size_t)dv);
        double *y = (double *)malloc(sizeof(double) * (size_t)dv);
        double *scratch = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!G || !x || !y || !scratch) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long c = 0; c < n_chain; ++c) {
                const int s = (int)(c / H), h = (int)(c % H);
                const int t0 = cu_seqlens[s], t1 = cu_seqlens[s + 1];
                const int L = t1 - t0;
                const size_t sidx = ((size_t)s * H + h) * sz;
                /* forward states Sigma_0 .. Sigma_L of this chain */
                double *states = (double *)malloc(sizeof(double) * sz * (size_t)(L + 1));
                if (!states) {
#pragma omp atomic write
                    bad = 1;
                    continue;
                }
                if (S0) memcpy(states, S0 + sidx, sizeof(double) * sz);
                else memset(states, 0, sizeof(double) * sz);
                for (int i = 0; i < L; ++i) {
                    const size_t th = (size_t)(t0 + i) * H + h;
                    memcpy(states + sz * (size_t)(i + 1), states + sz * (size_t)i, sizeof(double) * sz);
                    gdn_token_step(states + sz * (size_t)(i + 1), dk, dv, q + th * dk, k + th * dk,
                                   v + th * dv, a[th], b[th], scale, NULL, scratch);
                }
                /* backwards: G starts as the final-state gradient */
                if (dST) memcpy(G, dST + sidx, sizeof(double) * sz);
                else memset(G, 0, sizeof(double) * sz);
                for (int i = L - 1; i >= 0; --i) {
                    const size_t th = (size_t)(t0 + i) * H + h;
                    const double *qt = q + th * dk, *kt = k + th * dk, *vt = v + th * dv;
                    const double *dOt = dO + th * dv;
                    const double at = a[th], bt = b[th];
                    const double *Sig = states + sz * (size_t)(i + 1);    /* Sigma_t     */
                    const double *Sp = states + sz * (size_t)i;           /* Sigma_{t-1} */
                    /* G_t += scale q_t dO_t^T */
                    for (int r = 0; r < dk; ++r)
                        for (int j = 0; j < dv; ++j) G[(size_t)r * dv + j] += scale * qt[r] * dOt[j];
                    /* dq_t = scale Sigma_t dO_t */
                    for (int r = 0; r < dk; ++r) {
                        double acc = 0.0;
                        for (int j = 0; j < dv; ++j) acc += Sig[(size_t)r * dv + j] * dOt[j];
                        dq[th * dk + r] = scale * acc;
                    }
                    /* x = Sigma_{t-1}^T k,  y = G^T k */
                    for (int j = 0; j < dv; ++j) x[j] = y[j] = 0.0;
                    for (int r = 0; r < dk; ++r)
                        for (int j = 0; j < dv; ++j) {
                            x[j] += kt[r] * Sp[(size_t)r * dv + j];
                            y[j] += kt[r] * G[(size_t)r * dv + j];
                        }
                    /* dv_t = b y */
                    for (int j = 0; j < dv; ++j) dv_out[th * dv + j] = bt * y[j];
                    /* dk_t = -a b (G x + Sigma_{t-1} y) + b G v */
                    for (int r = 0; r < dk; ++r) {
                        double gx = 0.0, sy = 0.0, gv = 0.0;
                        for (int j = 0; j < dv; ++j) {
                            gx += G[(size_t)r * dv + j] * x[j];
                            sy += Sp[(size_t)r * dv + j] * y[j];
                            gv += G[(size_t)r * dv + j] * vt[j];
                        }
                        dk_out[th * dk + r] = -at * bt * (gx + sy) + bt * gv;
                    }
                    /* da_t = <G, Sigma_{t-1}> - b y.x ;  db_t = y.(v - a x) */
                    double gs = 0.0, yx = 0.0, yv = 0.0;
                    for (size_t e = 0; e < sz; ++e) gs += G[e] * Sp[e];
                    for (int j = 0; j < dv; ++j) {
                        yx += y[j] * x[j];
                        yv += y[j] * vt[j];
                    }
                    da[th] = gs - bt * yx;
                    db[th] = yv - at * yx;
                    /* dSigma_{t-1} = a (G - b k y^T) */
                    for (int r = 0; r < dk; ++r)
                        for (int j = 0; j < dv; ++j)
                            G[(size_t)r * dv + j] = at * (G[(size_t)r * dv + j] - bt * kt[r] * y[j]);
                }
                if (dS0) memcpy(dS0 + sidx, G, sizeof(double) * sz);
                free(states);
            }
        }
        free(G);
        free(x);
        free(y);
        free(scratch);
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

/* ------------------------------------------------------------------------
 * Sliding-window softmax attention, the window mixer of the hybrid LT2 loops
 * ("LT2: Linear-Time Looped Transformers", §2: a sliding-window block of
 * window w; Appendix C: windowed variants attend to the w - 1 previous
 * tokens and the token itself, no future tokens).  For query t of a sequence
 * starting at t0, over the keys j in [max(t0, t - w + 1), t]:
 *
 *     s_j = scale q_t . k_j,   p_j = exp(s_j - max_j s_j),
 *     o_t = sum_j p_j v_j / sum_j p_j
 *
 * evaluated as written, one query at a time, in double precision.
 * Layouts: q, k [n_tok][H][d], v, o [n_tok][H][dv].
 * ------------------------------------------------------------------------ */
int oracle_swa_fwd(const double *q, const double *k, const double *v, double *o,
                   const int32_t *cu_seqlens, int n_seq, int H, int d, int dv,
                   int window, double scale)
{
    if (!q || !k || !v || !o || !cu_seqlens) return -1;
    if (n_seq < 0 || H <= 0 || d <= 0 || dv <= 0 || window < 1) return -1;
    for (int s = 0; s < n_seq; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
    const long n_tok = cu_seqlens[n_seq] - cu_seqlens[0];
    int bad = 0;
#pragma omp parallel
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)window);
        if (!sc) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long u = 0; u < n_tok * H; ++u) {
                const long t = cu_seqlens[0] + u / H;
                const int h = (int)(u % H);
                int s = 0;
                while (cu_seqlens[s + 1] <= t) ++s;
                const long lo = (t - window + 1 > cu_seqlens[s]) ? t - window + 1 : cu_seqlens[s];
                const double *qt = q + ((size_t)t * H + h) * d;
                double m = -1.0 / 0.0;
                for (long j = lo; j <= t; ++j) {
                    const double *kj = k + ((size_t)j * H + h) * d;
                    double acc = 0.0;
                    for (int c = 0; c < d; ++c) acc += qt[c] * kj[c];
                    sc[j - lo] = scale * acc;
                    if (sc[j - lo] > m) m = sc[j - lo];
                }
                double l = 0.0;
                double *ot = o + ((size_t)t * H + h) * dv;
                for (int c = 0; c < dv; ++c) ot[c] = 0.0;
                for (long j = lo; j <= t; ++j) {
                    const double p = exp(sc[j - lo] - m);
                    l += p;
                    const double *vj = v + ((size_t)j * H + h) * dv;
                    for (int c = 0; c < dv; ++c) ot[c] += p * vj[c];
                }
                for (int c = 0; c < dv; ++c) ot[c] /= l;
            }
        }
        free(sc);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------
 * Per-channel (diagonal) gate variant, the KDA mixer named among the LT2
 * mixers ("LT2: Linear-Time Looped Transformers", Appendix C; the DPLR block
 * of §2 and Appendix B.1 in its general diagonal form).  The pages print no
 * update rule for it; the reading taken here replaces the scalar decay a_t of
 * the gated delta rule by a diagonal Diag(a_t), a_t in (0, 1]^{dk}, acting on
 * the key side of the state before the delta step:
 *
 *     Sigma_t = (I - b_t k_t k_t^T) Diag(a_t) Sigma_{t-1} + b_t k_t v_t^T
 *     o_t     = scale * Sigma_t^T q_t
 *
 * which is the gated delta rule when every entry of a_t is the same.  It is
 * evaluated as written: Z = Diag(a) Sigma (row i scaled by a_i), y = k^T Z,
 * Sigma_t = Z - b k y + b k v^T.  Layout of a: [n_tok][H][dk].
 * ------------------------------------------------------------------------ */
static void kda_token_step(double *sig, int dk, int dv,
                           const double *q, const double *k, const double *v,
                           const double *a, double b, double scale,
                           double *o, double *y)
{
    /* Z = Diag(a) Sigma_{t-1}, in place */
    for (int i = 0; i < dk; ++i) {
        double *row = sig + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) row[j] *= a[i];
    }
    /* y = k^T Z */
    for (int j = 0; j < dv; ++j) y[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double kc = k[i];
        const double *row = sig + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) y[j] += kc * row[j];
    }
    /* Sigma_t = Z - b k y + b k v^T */
    for (int i = 0; i < dk; ++i) {
        const double kc = k[i];
        double *row = sig + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) row[j] = row[j] - b * kc * y[j] + b * kc * v[j];
    }
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

/* Prefill of the per-channel gate variant over packed sequences (as
 * oracle_gdn_fwd, with a [n_tok][H][dk]). */
int oracle_kda_fwd(const double *q, const double *k, const double *v,
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
                    kda_token_step(sig, dk, dv, q + th * dk, k + th * dk, v + th * dv,
                                   a + th * dk, b[th], scale, o + th * dv, y);
                }
                if (ST) memcpy(ST + sidx, sig, sizeof(double) * (size_t)dk * dv);
            }
        }
        free(sig);
        free(y);
    }
    return bad ? -1 : 0;
}

/* One decode step of the per-channel gate variant for N slots x H heads
 * (a [N][H][dk]); S is updated in place. */
int oracle_kda_decode(const double *q, const double *k, const double *v,
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
                kda_token_step(S + (size_t)c * dk * dv, dk, dv, q + (size_t)c * dk,
                               k + (size_t)c * dk, v + (size_t)c * dv, a + (size_t)c * dk, b[c],
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
