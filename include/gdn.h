/*
 * gdn.h -- C ABI of the looped gated delta-rule (GDN) mixer library for
 * NVIDIA B200 (sm_100a).
 *
 * The operation ("LT2: Linear-Time Looped Transformers", §2, "LT2."
 * paragraph): a looped transformer applies its shared block stack T times; in
 * LT2 the block's token mixer is a linear-attention recurrence with queries and
 * keys q_t, k_t in R^{dk}, values v_t in R^{dv} and a recurrent state
 * S_t in R^{dk x dv}.  The mixer used here is Gated DeltaNet (named among the
 * LT2 mixers, Appendix C).  In the page's dk x dv orientation the state update
 * and readout are
 *
 *     S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T,   o_t = scale * S_t^T q_t
 *
 * (a rank-1, diagonal-plus-low-rank update, §2 and Appendix B.1), and the
 * per-loop residual across iterations is h^(tau) = h~^(tau) + rho_tau (.) h^(tau-1)
 * with a per-channel gate rho_tau in R^d (§2, "LT2." paragraph).
 *
 * Conventions for every entry point
 *   - All pointers passed to the compute calls are DEVICE pointers unless a
 *     parameter says otherwise; the caller owns every buffer.  The compute calls
 *     never allocate, free or synchronise; they enqueue work on `stream` and
 *     return.
 *   - Tensors are dense and row-major in the layouts given below; every
 *     pointer must be 16-byte aligned.
 *   - Argument errors are detected on the host and returned before anything is
 *     launched (GDN_ERR_INVALID, GDN_ERR_UNSUPPORTED).  A failed launch returns
 *     GDN_ERR_CUDA.  A device-side wait that exceeds its iteration limit records
 *     GDN_ERR_TIMEOUT in a device status word, read (and cleared) by
 *     gdn_get_device_status().
 *   - Thread safety: calls on different streams may run concurrently; they share
 *     only read-only launch constants and the device status word.
 *   - Devices: the kernels' shared-memory launch attributes are set on the
 *     first call of the process, on the device current then; run one process
 *     per GPU (as the benchmark and the tests do).  Driving several GPUs from
 *     one process is not tested; a launch that the attributes do not cover
 *     fails with GDN_ERR_CUDA (no fault).
 */
#ifndef LOOPED_GDN_H
#define LOOPED_GDN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID = 1,     /* null pointer, bad size, misaligned pointer      */
    GDN_ERR_UNSUPPORTED = 2, /* shape/dtype combination this build does not run */
    GDN_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed     */
    GDN_ERR_TIMEOUT = 4,     /* a device-side wait hit its iteration limit      */
    GDN_ERR_WORKSPACE = 5    /* workspace pointer/size below the queried need   */
} gdn_status;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* Flags for gdn_fwd_params.flags and gdn_decode_step(). */
#define GDN_QK_L2NORM 0x1u /* normalise q and k per head in fp32 before use:
                              x / sqrt(sum x^2 + 1e-6).  The precise prefill
                              rounds the normalised vectors to io dtype; the
                              tensor-core prefill and decode apply the inverse
                              norms as fp32 factors to the products of the
                              inputs as given (the same map, one rounding
                              fewer)                                           */
#define GDN_PRECISE   0x2u /* prefill: use the fp32 CUDA-core chunk kernel even
                              for bf16 inputs (slower, fp32 operands)          */
#define GDN_SINGLE_PASS 0x4u /* prefill: run every (sequence, head) chain in one
                              pass even when a segmented schedule would be
                              chosen (see gdn_chunk_fwd)                       */
#define GDN_CHANNEL_GATE 0x8u /* per-channel (diagonal) decay, the KDA mixer of
                              the LT2 mixer list ("LT2: Linear-Time Looped
                              Transformers", Appendix C; the DPLR block of §2
                              with a diagonal decay).  a is [tokens][H][dk]
                              fp32, a_t in (0, 1]^{dk}, and the update reads
                                Sigma_t = (I - b_t k_t k_t^T) Diag(a_t)
                                          Sigma_{t-1} + b_t k_t v_t^T
                              (the gated delta rule when a_t's entries are
                              equal).  Prefill runs the fp32 CUDA-core KDA
                              chunk kernel; decode both decode kernels       */
#define GDN_TEST_WAIT_TIMEOUT 0x40000000u
                           /* test hook of the tensor-core prefill: one thread
                              waits on a barrier that nothing arrives, so the
                              bounded wait runs out (about 2 s); the call then
                              ends with GDN_ERR_TIMEOUT in the device status
                              word and no outputs, and the context stays
                              usable.  Other paths ignore it.                  */

/*
 * Prefill over packed or variable-length sequences.
 *
 *   q, k       [total_tokens][H][dk]   io_dtype
 *   v          [total_tokens][H][dv]   io_dtype
 *   a, b       [total_tokens][H]       fp32.  a_t in (0, 1] is the decay gate
 *                                      ([total_tokens][H][dk] with GDN_CHANNEL_GATE),
 *                                      b_t the write strength (any finite value;
 *                                      b in [0, 2] keeps ||I - b k k^T|| <= 1 for
 *                                      unit keys, Appendix B.1).
 *   S0         [n_seq][H][dk][dv]      fp32, or NULL for a zero initial state
 *   o          [total_tokens][H][dv]   io_dtype, written
 *   S_T        [n_seq][H][dk][dv]      fp32 final state, or NULL to skip; may
 *                                      alias S0 exactly (in-place update)
 *   cu_seqlens device int32 [n_seq+1] token offsets (0 = cu[0] <= ... <= cu[n_seq]
 *              = total_tokens), or NULL: n_seq sequences of seq_len tokens each
 *              (total_tokens = n_seq * seq_len).
 *   scale      multiplies every output (1.0 reproduces the recurrence as written).
 * Optional epilogue of the looped block, applied to each output in this order
 * (every pointer NULL = that step off):
 *   gate       [total_tokens][H] fp32 logits of the head-wise sigmoid output
 *              gate: o_t,h <- sigmoid(gate_t,h) o_t,h (one factor per token and
 *              head; "LT2: Linear-Time Looped Transformers", §3, the
 *              gated-attention paragraph: a head-specific sigmoid gate after the
 *              mixer).  The state is not gated.
 *   h_prev, rho  the loop residual of §2 ("LT2." paragraph) fused into the
 *              output: o <- round(o) + rho (.) h_prev, computed in fp32 and
 *              rounded to io_dtype (round(o) is the output as it would be
 *              stored, so the result equals gdn_chunk_fwd followed by
 *              loop_residual).  h_prev [total_tokens][H*dv] io_dtype (o's
 *              layout), rho [H*dv] fp32; both or neither.  o may be h_prev
 *              itself (exact aliasing, for an in-place loop state).
 * Each (sequence, head) chain starts from its S0 and runs the recurrence over its
 * own tokens; a sequence of length 0 writes no output and S_T = S0.
 * o must not overlap q, k, v, a, b, S0, S_T or gate, nor h_prev other than exactly.
 *
 * Supported: dk in {64, 128}; dv a multiple of 64, at most 512; H >= 1.
 * bf16 with dk = 128 and dv a multiple of 128 runs on the tensor-core (tcgen05)
 * kernel; fp32, or any other supported shape, or GDN_PRECISE, runs on the fp32
 * CUDA-core chunk kernel.
 */
typedef struct {
    const void *q, *k, *v;
    const float *a, *b;
    const float *S0;
    void *o;
    float *S_T;
    const int32_t *cu_seqlens;
    int n_seq, seq_len, total_tokens, H, dk, dv;
    gdn_dtype io_dtype;
    float scale;
    unsigned flags;
    const float *gate;       /* optional epilogue, see above */
    const void *h_prev;
    const float *rho;
} gdn_fwd_params;

/* Bytes of device workspace gdn_chunk_fwd needs for these parameters (may be 0).
 * Returns (size_t)-1 if the parameters are invalid.  The need is non-zero only
 * when the segmented schedule or, with GDN_CHANNEL_GATE, the two-launch
 * schedule is chosen (see below); it is a function of the shapes, flags and
 * the current device's SM count.  For GDN_CHANNEL_GATE it is, with
 * S = (floor(total_tokens / 64) + n_seq + 1) * H chunk slots and each array
 * rounded up to 256 bytes, 3 arrays of S * 64 * dk fp32, 2 of S * 64 * dv and
 * 1 of S * dk. */
size_t gdn_chunk_fwd_workspace(const gdn_fwd_params *p);

/* The schedule gdn_chunk_fwd takes for these parameters when it is given a
 * workspace of gdn_chunk_fwd_workspace(p) bytes (host only, no device memory
 * touched).  Any output pointer may be NULL.
 *   n_segs:   1 = one pass per chain; >= 2 = segment 0 of seg0_tok tokens,
 *             then segments of seg_tok tokens (the last one may be shorter).
 *   seg0_tok, seg_tok: 0 for one pass.
 *   launches: stream operations the call enqueues: 0 (nothing to do), 1 (one
 *             pass, or the copy or clear of S_T when every sequence is empty),
 *             2 or 3 (see the schedules below; a varlen call with its length
 *             sort takes 2, a GDN_CHANNEL_GATE call with a workspace 2).
 *   corrected: 1 for the corrected segmented schedule, else 0.
 * Parameters gdn_chunk_fwd would reject return the same error status. */
gdn_status gdn_chunk_fwd_schedule(const gdn_fwd_params *p, int *n_segs, int *seg0_tok,
                                  int *seg_tok, int *launches, int *corrected);

/* Chunkwise prefill (chunks of 64 tokens).
 *
 * Schedule.  Each (sequence, head, 128-wide dv slice) chain normally runs in
 * one pass.  When fixed-length sequences (cu_seqlens == NULL) give too few
 * chains to fill the GPU, every sequence is instead cut into segments whose
 * state update is affine in the start state, S_end = M S_start + B, with one
 * of two schedules (all launches on `stream`):
 *   corrected (the default): a first launch runs segment 0 in full from S0
 *     and, beside it, every later segment from a zero state, writing its
 *     zero-start outputs into o, its B, its dk x dk transition M, and the
 *     per-token rows qhat_i = M_i^T q_i (scaled like o_i) that carry the
 *     start state's share of each output; a second kernel chains the start
 *     states (and S_T) in fp32 (skipped when there is nothing to chain); a
 *     third adds qhat_i^T S_p to the outputs (tensor cores) and applies the
 *     output gate and the loop residual, to every segment: there the output
 *     is rounded to io_dtype before the gate factor multiplies it.
 *   output pass (when o is h_prev itself, which the first launch would
 *     overwrite): the first launch computes B and M of segments 1 .. P-2
 *     without outputs, the combine chains the start states, and a third
 *     launch runs segments 1 .. P-1 again from their start states.
 * The outputs equal the one-pass outputs up to rounding.  GDN_SINGLE_PASS
 * disables segmenting.
 * Varlen calls (cu_seqlens != NULL) always run one pass; when they take more
 * blocks than the GPU runs at once and have at most 4096 sequences, a first
 * launch sorts the sequences by length on the device (longest first, into the
 * workspace) and the blocks take them in that order, so that the longest
 * chains do not start last.  The outputs do not depend on the order.
 * With GDN_CHANNEL_GATE (fp32 arithmetic, the chain's products as 3xTF32
 * warp MMAs with fp32 accumulation; any io dtype) and a
 * workspace, a first launch takes every (chunk, head) at once and writes its
 * decayed operands, T = (I + A)^{-1} and the state-independent products
 * W = T diag(b) (K o e^G), Q' = Q o e^G - P W, U~ = T diag(b) V and
 * O~ = P U~ to the workspace; a second walks each (sequence, head, 16-wide
 * dv slice) chain through its chunks with U = U~ - W S, O = scale (Q' S + O~)
 * and the carry.  Without a workspace one launch does all of it per
 * (sequence, head, 32-wide slice).  Both give the same outputs up to
 * rounding.
 *
 * ws/ws_bytes: device workspace of at least gdn_chunk_fwd_workspace(p) bytes,
 * 256-byte aligned, owned by the caller and not read back afterwards.
 * ws == NULL with ws_bytes == 0 is always accepted and selects the one-pass
 * schedule (the one-launch kernel for GDN_CHANNEL_GATE); a non-NULL ws
 * smaller than the need returns GDN_ERR_WORKSPACE, and so does ws == NULL
 * with ws_bytes != 0 when the chosen schedule needs a workspace. */
gdn_status gdn_chunk_fwd(const gdn_fwd_params *p, void *ws, size_t ws_bytes,
                         cudaStream_t stream);

/*
 * gdn_chunk_fwd without a workspace argument, for callers that cannot allocate
 * device memory for it: a plugin inside an engine or framework that owns all
 * device memory through its own pool and forbids direct cudaMalloc (it would
 * bypass the pool's accounting and limits), or code on a latency-critical path
 * that must not call cudaMalloc because that call can synchronise the device.
 * The paper has no counterpart to this entry point; it is this library's own
 * addition.
 *
 * The segmented schedule's scratch is one array compiled into the library:
 * 32 MiB (33554432 bytes) of device memory that every GPU which loads the
 * library holds until the process exits.  A call whose
 * gdn_chunk_fwd_workspace(p) exceeds that returns GDN_ERR_WORKSPACE without
 * launching anything, except a GDN_CHANNEL_GATE call, which then runs the
 * one-launch kernel (no workspace); a call that needs no workspace runs as
 * gdn_chunk_fwd.
 * Nothing is allocated or freed.
 *
 * The first call on each device looks up the array's device address (with
 * that device current) and caches it; make that first call before any stream
 * capture.  All calls share the one array, which keeps the last call's
 * contents (nothing in it needs clearing between calls): calls whose kernels
 * overlap on the GPU, on different streams, race on it.  Otherwise the same
 * contract, results and errors as gdn_chunk_fwd.
 */
gdn_status gdn_chunk_fwd_noalloc(const gdn_fwd_params *p, cudaStream_t stream);

/*
 * Reverse mode of gdn_chunk_fwd: gradients of a loss that depends on the
 * outputs o (through grad_o = dloss/do) and on the final states S_T (through
 * grad_S_T) with respect to q, k, v, a, b and S0.  Per token, with G_t the
 * gradient with respect to S_t (the part flowing back from the later tokens and
 * the final state, plus the readout of token t), x_t = S_{t-1}^T k_t and
 * y_t = G_t^T k_t:
 *     G_t      = dS_t + scale q_t grad_o_t^T
 *     grad_q_t = scale S_t grad_o_t          grad_v_t = b_t y_t
 *     grad_k_t = -a_t b_t (G_t x_t + S_{t-1} y_t) + b_t G_t v_t
 *     grad_a_t = <G_t, S_{t-1}> - b_t y_t . x_t
 *     grad_b_t = y_t . (v_t - a_t x_t)
 *     dS_{t-1} = a_t (G_t - b_t k_t y_t^T)
 * and grad_S0 = dS_0: the derivatives of the factors of the update as written
 * above gdn_fwd_params ("LT2: Linear-Time Looped Transformers", §2).
 *
 * Inputs as in gdn_fwd_params (q, k, v, a, b, S0, cu_seqlens, n_seq, seq_len,
 * total_tokens, H, dk, dv, io_dtype, scale), plus
 *   grad_o      [total_tokens][H][dv]   io_dtype
 *   grad_S_T    [n_seq][H][dk][dv]      fp32, or NULL (no loss term on S_T)
 * Outputs, fp32, overwritten, none overlapping an input:
 *   grad_q, grad_k [total_tokens][H][dk]; grad_v [total_tokens][H][dv];
 *   grad_a, grad_b [total_tokens][H];     grad_S0 [n_seq][H][dk][dv] or NULL.
 * Supported: dk in {64, 128}; dv a multiple of 32, at most 256; flags 0 or
 * GDN_PRECISE (the in-kernel q/k norm has no reverse mode here: differentiate
 * it outside).  fp32 arithmetic on the CUDA cores throughout.
 * flags 0, the chunkwise path: the same relations in the chunked (WY/UT) form
 * of gdn_chunk_fwd, chunks of 64 tokens, in four launches: per chunk the
 * solve T = (I + A)^-1 and the chunk's transition factors; the chunk start
 * states forward and the state gradients backward (one CTA per sequence,
 * head and 32 columns of dv); then every token gradient, one CTA per chunk.
 * It takes log a_t with a_t clamped to 1e-30 and returns grad_a_t =
 * (dloss/dlog a_t) / a_t, so a gate of exactly 0 gets no meaningful grad_a_t
 * (use GDN_PRECISE there).
 * GDN_PRECISE, token by token: one CTA per (sequence, head) chain recomputes
 * the forward states from checkpoints taken every 64 tokens and walks each
 * chunk backwards with the per-token relations above.
 * ws/ws_bytes: device workspace of at least gdn_chunk_bwd_workspace(p) bytes,
 * 256-byte aligned (chunkwise: per chunk and head the factors W, Qh [64][dk]
 * and U~ [64][dv], the decays, the start state and the end-state gradient;
 * token by token: the checkpoints, one chunk of states and the running G of
 * every chain); a missing or short workspace returns GDN_ERR_WORKSPACE.
 */
typedef struct {
    const void *q, *k, *v;
    const float *a, *b;
    const float *S0;
    const void *grad_o;
    const float *grad_S_T;
    float *grad_q, *grad_k, *grad_v, *grad_a, *grad_b, *grad_S0;
    const int32_t *cu_seqlens;
    int n_seq, seq_len, total_tokens, H, dk, dv;
    gdn_dtype io_dtype;
    float scale;
    unsigned flags;
} gdn_bwd_params;

/* Bytes of device workspace gdn_chunk_bwd needs (host only); (size_t)-1 if the
 * parameters are invalid. */
size_t gdn_chunk_bwd_workspace(const gdn_bwd_params *p);

gdn_status gdn_chunk_bwd(const gdn_bwd_params *p, void *ws, size_t ws_bytes,
                         cudaStream_t stream);

/*
 * One decode step: one new token for each of N independent state slots (a slot
 * is one sequence x layer x loop state), H heads each.
 *   q, k [N][H][dk], v [N][H][dv], o [N][H][dv]  io_dtype
 *   a, b [N][H] fp32 (a [N][H][dk] with GDN_CHANNEL_GATE)
 *   S    [N][H][dk][dv] fp32, read and overwritten in place with S_t.
 * flags: GDN_QK_L2NORM, GDN_CHANNEL_GATE as above.  Supported: dk in {64, 128}, dv a multiple of
 * 64 up to 512.  o must not overlap S or the inputs.
 */
gdn_status gdn_decode_step(const void *q, const void *k, const void *v,
                           const float *a, const float *b, float *S, void *o,
                           int N, int H, int dk, int dv, gdn_dtype io_dtype,
                           float scale, unsigned flags, cudaStream_t stream);

/*
 * gdn_decode_step with the looped block's output epilogue, as in
 * gdn_fwd_params: gate [N][H] fp32 logits of the head-wise sigmoid output gate
 * (or NULL), and the loop residual o <- round(o) + rho (.) h_prev with
 * h_prev [N][H*dv] io_dtype and rho [H*dv] fp32 (both or neither; o may be
 * h_prev exactly).  With every epilogue pointer NULL it is gdn_decode_step.
 */
gdn_status gdn_decode_step_looped(const void *q, const void *k, const void *v,
                                  const float *a, const float *b, float *S, void *o,
                                  const float *gate, const void *h_prev, const float *rho,
                                  int N, int H, int dk, int dv, gdn_dtype io_dtype,
                                  float scale, unsigned flags, cudaStream_t stream);

/*
 * Loop residual h_out = h_tilde + rho (.) h_prev, computed in fp32 and rounded
 * to nearest-even in io_dtype.
 *   h_tilde, h_prev, h_out [rows][d] io_dtype; rho [d] fp32.
 * h_out may alias h_tilde or h_prev exactly.  d must be a multiple of 8.
 */
gdn_status loop_residual(const void *h_tilde, const void *h_prev, const float *rho,
                         void *h_out, int64_t rows, int d, gdn_dtype io_dtype,
                         cudaStream_t stream);

/*
 * Sliding-window causal softmax attention, the window mixer of the hybrid LT2
 * loops ("LT2: Linear-Time Looped Transformers", §2: a sliding-window block of
 * window w, whose receptive field grows to T w over T loops; Appendix C: the
 * windowed variants attend to the w - 1 previous tokens and the token itself,
 * none after it).  For query t of a sequence starting at t0, over the keys
 * j in [max(t0, t - w + 1), t]:
 *     o_t = sum_j softmax_j(scale q_t . k_j) v_j
 *
 *   q, k       [total_tokens][H][d]   bf16
 *   v, o       [total_tokens][H][dv]  bf16 (o written; must not overlap q, k, v)
 *   cu_seqlens device int32 [n_seq+1] token offsets, or NULL: n_seq sequences of
 *              seq_len tokens each (total_tokens = n_seq * seq_len).
 *   max_seq_len  with cu_seqlens: no sequence is longer (the grid is sized by
 *              it; a longer sequence records GDN_ERR_INVALID in the device
 *              status word and loses its last queries).  Ignored without.
 *   window     w >= 1 (w >= a sequence's length gives full causal attention).
 *   scale      score scale (1/sqrt(d) is the usual one).
 * Supported: bf16, d = dv = 128, H >= 1.  One launch; tensor cores (tcgen05)
 * for Q K^T and P V.  Async on `stream`; nothing allocated.
 */
typedef struct {
    const void *q, *k, *v;
    void *o;
    const int32_t *cu_seqlens;
    int n_seq, seq_len, max_seq_len, total_tokens, H, d, dv, window;
    gdn_dtype io_dtype;
    float scale;
} swa_params;

gdn_status swa_fwd(const swa_params *p, cudaStream_t stream);

/* Static description of a status code (never NULL). */
const char *gdn_status_string(gdn_status s);

/* Synchronises `stream`, then returns and clears the device status word of the
 * current device (GDN_OK if no kernel recorded an error since the last call). */
gdn_status gdn_get_device_status(cudaStream_t stream);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LOOPED_GDN_H */
