/*
 * kda.h -- C ABI of the B200 (sm_100a) library for the gated delta-rule
 * recurrence with channel-wise decay: KDA, Complex KDA, RDA and GDN-2.
 *
 * The operation (update equations on the Raon-1-mini-preview discussion page,
 * range extension in the "Complex KDA" arXiv abstract).  For each sequence n,
 * head h and token t, with the state S in R^{d_k x d_v} (rows = key channel):
 *
 *   KDA / Complex KDA : S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   RDA               : S_t = (I - e_t k_t k_t^T) Diag(alpha_t) S_{t-1} + w_t k_t v_t^T
 *   GDN-2             : S_t = (I - k_t (b_t (.) k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t (.) v_t)^T
 *   readout           : o_t = S_t^T q_t     (post-update state, no scaling; a
 *                                            caller wanting 1/sqrt(d_k) pre-scales q)
 *
 * KDA range: alpha in (0,1], beta in [0,1].  Complex KDA (KDA_RANGE_EXTENDED):
 * alpha in [-1,1], beta in [0,2].  The kernels never take a logarithm of
 * alpha and never divide by a product of alphas, so negative and zero gates
 * are computed exactly as the recurrence defines them; the range argument
 * only declares the caller's contract.
 *
 * Memory model.  Every tensor pointer is a DEVICE pointer owned by the
 * caller, 16-byte aligned, densely packed in the row-major layouts below.
 * The library never frees caller memory and enqueues all work
 * asynchronously on `stream` (a cudaStream_t; NULL = legacy default stream).
 * Only kda_chunk_fwd allocates device memory: the split form's workspace,
 * stream-ordered and released within the call (kda_chunk_fwd_ws takes it
 * from the caller instead).  Between calls the library keeps only per-device
 * set-up (kernel attributes, SM count, the fixed scratch array of
 * kda_chunk_fwd_noalloc) and each device's failure word (kda_device_status).
 * It is reentrant and thread-safe, with one exception: calls of
 * kda_chunk_fwd_noalloc share one scratch array, so two of them that overlap
 * on the GPU race (see there).  A call returns after the launch:
 * asynchronous kernel faults surface at the caller's next synchronisation, as
 * with any CUDA launch; a kernel that gives up a bounded wait (or, in the
 * split form, finds a chunk's operands missing) records it in the device's
 * failure word, which kda_device_status reads.
 *
 * Entry points.
 *   kda_chunk_fwd, kda_chunk_fwd_ws, kda_chunk_fwd_noalloc
 *                           chunked forward over whole sequences (o, final
 *                           state, optional snapshots every 64 tokens)
 *   kda_chunk_bwd           every gradient of that forward (fp32)
 *   kda_chunk_fwd_rank2     two erase/write sub-steps per token
 *   kda_chunk_bwd_rank2     every gradient of the rank-2 forward (fp32)
 *   kda_decode_step         one token per (sequence, head), state in place
 *   *_workspace_size        bytes of the caller-owned workspace of each call
 *   kda_check_gates, kda_check_seqlens   device checks of the inputs' contracts
 *   kda_device_status       failures the kernels recorded on the device
 *   kda_error_string, kda_last_error_detail, kda_version
 *
 * Errors.  Every entry point validates all arguments on the host before it
 * launches anything; on a bad argument it returns a KDA_ERR_* code and has
 * no side effect.  A failed launch returns KDA_ERR_CUDA (detail in
 * kda_last_error_detail()).  Values that live on the device (gates,
 * cu_seqlens) are checked only on request: KDA_FLAG_VALIDATE_RANGE, or the
 * kda_check_* calls.  Device-side failures are reported by kda_device_status.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Variants: which erase direction a~ and written value m the update uses.
 *   KDA  : a~ = beta k,  m = beta v      g1 = beta [..,H],      g2 = NULL
 *   RDA  : a~ = e k,     m = w v         g1 = e    [..,H],      g2 = w [..,H]
 *   GDN2 : a~ = b (.) k, m = w (.) v     g1 = b    [..,H,d_k],  g2 = w [..,H,d_v]  */
enum kda_variant { KDA_VARIANT_KDA = 0, KDA_VARIANT_RDA = 1, KDA_VARIANT_GDN2 = 2 };

/* Declared gate range (not clamped; kda_check_gates tests inputs against it). */
enum kda_gate_range {
    KDA_RANGE_STANDARD = 0, /* alpha in (0,1], beta/e in [0,1]    (KDA)          */
    KDA_RANGE_EXTENDED = 1  /* alpha in [-1,1], beta/e in [0,2]   (Complex KDA)  */
};

/* Element type of q, k, v, alpha, g1, g2 and o.  States are always fp32. */
enum kda_dtype { KDA_DTYPE_BF16 = 0, KDA_DTYPE_F32 = 1 };

enum kda_status {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad cu_seqlens */
    KDA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (head dims, chunk size) */
    KDA_ERR_RANGE = 3,         /* a gate outside the declared range (KDA_FLAG_VALIDATE_RANGE) */
    KDA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    KDA_ERR_DEVICE_TIMEOUT = 5 /* kda_device_status: a kernel gave up a bounded wait or found
                                  a chunk's operands missing; the affected outputs are undefined */
};

/* Flags. */
/* KDA_FLAG_VALIDATE_RANGE -- before the work is launched, check on the device
 * that every gate lies in the declared range (alpha, and beta / e / GDN-2's b,
 * as kda_check_gates does; NaN fails) and that cu_seqlens keeps its contract
 * (as kda_check_seqlens does), and WAIT for the outcome: the call then
 * synchronises `stream`.  A violation returns KDA_ERR_RANGE (gates) or
 * KDA_ERR_INVALID_ARG (cu_seqlens) and launches nothing.  With
 * KDA_FLAG_GATE_LOGITS only cu_seqlens is checked (logits have no range).
 * Accepted by kda_chunk_fwd, kda_chunk_fwd_ws and kda_decode_step.  Without
 * it no device value is checked: the kernels compute out-of-range gates as
 * the recurrence defines them, and a cu_seqlens that breaks its contract
 * makes them read and write out of bounds. */
#define KDA_FLAG_VALIDATE_RANGE 1u
#define KDA_FLAG_FORCE_SCAN     2u  /* use the token-by-token CUDA scan kernel even where the
                                       tensor-core chunked kernel applies (testing aid) */
#define KDA_FLAG_FORCE_FUSED    4u  /* tensor-core path: force the single fused kernel */
#define KDA_FLAG_FORCE_SPLIT    8u  /* tensor-core path: force the two-kernel path */
/* Input preparation inside the kernels (chunked forward and decode), saving
 * the separate passes over HBM a model would otherwise run first:
 *   KDA_FLAG_GATE_LOGITS -- alpha, g1 and g2 hold logits.  Standard range:
 *       alpha = exp(-softplus(x)) = 1/(1+e^x), beta / e / w / b = sigmoid(y);
 *       extended range: alpha = tanh(x), beta / e / w / b = 2 sigmoid(y).
 *   KDA_FLAG_L2NORM_K -- k_t is replaced by k_t / max(||k_t||_2, 1e-6) per
 *       token and head.
 * Both are computed in fp32 from the stored inputs. */
#define KDA_FLAG_GATE_LOGITS   16u
#define KDA_FLAG_L2NORM_K      32u
/* KDA_FLAG_DEBUG_STALL -- testing aid for the failure path (needs
 * KDA_FLAG_FORCE_SPLIT and the tensor-core path): the chain CTA of
 * (sequence 0, head 0) never loads its first chunk's operands and gives up
 * waiting for them after about 1 ms, so that the bounded-wait expiry runs on
 * demand.  That pair's o is left unwritten and its final state is NaN; every
 * other pair is computed normally; kda_device_status then reports
 * KDA_ERR_DEVICE_TIMEOUT with KDA_DEVICE_WAIT_TIMEOUT.  Nothing faults. */
#define KDA_FLAG_DEBUG_STALL   64u

/* Bits of the device failure word (kda_device_status). */
#define KDA_DEVICE_WAIT_TIMEOUT 1u  /* a bounded wait inside a kernel ran out (about 2 s) */
#define KDA_DEVICE_SLOT_MISSING 2u  /* split form: a chunk slot not written by this call's
                                       preparation kernel */

/*
 * kda_chunk_fwd -- chunked-parallel forward over whole sequences.
 *
 * Shapes (row-major):
 *   q, k, alpha : [B,T,H,d_k]        v, o : [B,T,H,d_v]
 *   g1, g2      : per the variant table above, leading dims [B,T,H]
 *   cu_seqlens  : NULL -> B independent sequences of length T (N = B);
 *                 else int32 DEVICE array of num_seqs+1 non-decreasing offsets
 *                 with cu[0] = 0 and cu[num_seqs] = T, B must be 1, and
 *                 sequence n is tokens [cu[n], cu[n+1]) of the packed batch.
 *                 Each sequence starts from its own initial state ("document
 *                 reset", openarchlab page on GDN/KDA state updates, sec. 3);
 *                 there is no padding inside packed input.
 *   initial_state : [N,H,d_k,d_v] fp32 or NULL (zero state)
 *   final_state   : [N,H,d_k,d_v] fp32 or NULL (not written); may alias
 *                   initial_state (each sequence reads its state before writing it)
 *   o             : [B,T,H,d_v] output, same dtype as q
 * Sizes: B >= 1, T >= 0, H >= 1, d_k and d_v in {16, 32, 64, 128},
 * chunk_size in {16, 32, 64, 128}.  With bf16, d_k = d_v = 128 and
 * chunk_size = 64 the tcgen05 tensor-core chunked path runs (WY/UT form,
 * fp32 accumulation, fp32 state kept on chip); every other accepted case
 * runs the token-by-token fp32 CUDA scan, whose result does not depend on
 * chunk_size.  Results of the two agree to rounding.
 * The tensor-core path has two forms with bit-identical results:
 *   fused -- one kernel, one CTA per (sequence, head) builds each chunk's
 *            operands and runs the state chain; no workspace;
 *   split -- a persistent kernel over all SMs builds every chunk's operands
 *            into a workspace, then one CTA per (sequence, head) runs the
 *            chain.  Its workspace holds about 81 KiB per (chunk, head); here
 *            it is allocated stream-ordered (cudaMallocAsync) on `stream`
 *            and freed on it before the call returns, and if that fails the
 *            fused form runs instead.  kda_chunk_fwd_ws takes a caller-owned
 *            workspace instead.
 * The form is chosen by problem shape unless KDA_FLAG_FORCE_FUSED or
 * KDA_FLAG_FORCE_SPLIT (mutually exclusive) names one.
 * Returns KDA_OK or a KDA_ERR_* code.
 */
int kda_chunk_fwd(int variant, int gate_range, int dtype,
                  int B, int T, int H, int d_k, int d_v,
                  const void *q, const void *k, const void *v, const void *alpha,
                  const void *g1, const void *g2,
                  const int32_t *cu_seqlens, int num_seqs,
                  const float *initial_state, float *final_state,
                  void *o, int chunk_size, unsigned flags, void *stream);

/*
 * kda_chunk_fwd_workspace_size -- bytes of workspace kda_chunk_fwd_ws needs
 * for these sizes and flags: (N + ceil(B*T / 64)) * H * 82944 when the split
 * form would run, N = num_seqs with cu_seqlens (has_cu_seqlens = 1) or B
 * without; 0 when another form runs (scan: dtype, head dims or chunk size;
 * fused: chosen by shape on the current device or forced) and when an
 * argument is out of range.  By shape, the split form is chosen for packed
 * (cu_seqlens) batches and, for B equal-length sequences, when a cost model
 * of measured per-chunk times favours it (for example B*H <= about 0.8x the
 * SM count, or a last partial wave of the fused kernel).
 */
size_t kda_chunk_fwd_workspace_size(int dtype, int B, int T, int H, int d_k, int d_v,
                                    int has_cu_seqlens, int num_seqs, int chunk_size, unsigned flags);

/*
 * kda_chunk_fwd_ws -- kda_chunk_fwd with a caller-owned DEVICE workspace of
 * `workspace_bytes` bytes (16-byte aligned; not read before it is written,
 * contents undefined afterwards; it must stay allocated until the call's
 * work on `stream` has finished).  The split form runs when chosen and the
 * workspace holds at least kda_chunk_fwd_workspace_size(...) bytes;
 * otherwise the fused form runs (KDA_FLAG_FORCE_SPLIT with a NULL or short
 * workspace is KDA_ERR_INVALID_ARG).  Nothing is allocated.
 *
 * chunk_states (optional, NULL = none): fp32 [num_slots][H][d_k][d_v] with
 * num_slots = N + ceil(B*T / 64), receives the state after every 64 tokens
 * of each sequence and after its last token, for prefix caching ("state
 * snapshots", openarchlab page on GDN/KDA state updates, sec. 3): the state
 * after chunk c (tokens [64c, min(64c+64, len))) of sequence n goes to slot
 * n + floor(R_n / 64) + c, R_n its first token's row in the packed [B*T]
 * token order (cu[n], or n*T without cu_seqlens).  Slots that belong to no
 * chunk are not written.  Every path writes them (fused, split, scan); the
 * last chunk's entry equals final_state.  Appending tokens to a cached
 * prefix is a forward call with initial_state = that entry.
 */
int kda_chunk_fwd_ws(int variant, int gate_range, int dtype,
                     int B, int T, int H, int d_k, int d_v,
                     const void *q, const void *k, const void *v, const void *alpha,
                     const void *g1, const void *g2,
                     const int32_t *cu_seqlens, int num_seqs,
                     const float *initial_state, float *final_state, float *chunk_states,
                     void *o, int chunk_size, void *workspace, size_t workspace_bytes,
                     unsigned flags, void *stream);

/*
 * kda_chunk_fwd_noalloc -- the split form of the tensor-core chunked forward
 * for callers that cannot allocate device memory at call time: an engine
 * whose allocator already owns all of HBM, a runtime with a fixed device
 * memory budget, or a latency-critical loop that cannot take cudaMalloc's
 * cost and the device synchronisation it may cause.  The pages have no
 * counterpart; this is a deployment entry point, not part of the method.
 *
 * Arguments and results are those of kda_chunk_fwd with chunk_size 64 and
 * no flags (flags must be 0).  It serves bf16 with d_k = d_v = 128 only
 * (else KDA_ERR_UNSUPPORTED) and allocates nothing: its workspace is a fixed
 * 64 MiB device array inside the library, held by every GPU that loads the
 * library until the process exits.  Problems needing more,
 * (N + ceil(B*T/64)) * H > 809, are rejected with KDA_ERR_UNSUPPORTED.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current) and keeps it for the life of the
 * process; make that first call before any stream capture, and do not call
 * this entry point after cudaDeviceReset on that device (the kept address no
 * longer names the array there).  All calls share the array: calls that overlap on the GPU (other
 * streams, other host threads) race and give wrong results; calls in order
 * on one stream are safe.  The array's earlier contents never leak into a
 * result (each call tags its slots).
 */
int kda_chunk_fwd_noalloc(int variant, int gate_range, int dtype,
                          int B, int T, int H, int d_k, int d_v,
                          const void *q, const void *k, const void *v, const void *alpha,
                          const void *g1, const void *g2,
                          const int32_t *cu_seqlens, int num_seqs,
                          const float *initial_state, float *final_state,
                          void *o, unsigned flags, void *stream);

/*
 * kda_chunk_bwd -- gradients of the forward recurrence (backward pass), for
 * L with dL/do = d_o and dL/dS_final = d_final_state (NULL = 0):
 *   dq, dk, alpha-, g1-, g2-gradients and dL/dS_initial, all fp32, in the
 *   layouts of the corresponding inputs (dg1: beta / e [B,T,H] or GDN-2's b
 *   [B,T,H,d_k]; dg2: w [B,T,H] (RDA) or [B,T,H,d_v] (GDN-2), NULL for KDA;
 *   d_initial_state [N,H,d_k,d_v] or NULL).
 * Inputs as for kda_chunk_fwd (d_o in the input dtype, [B,T,H,d_v]); no
 * flags (the inputs are the recurrence's own: no logits, normalised keys).
 * Defined by the update equations of the Raon-1-mini-preview discussion page
 * (the pages give no gradient formulas; training keeping checkpoints and the
 * chunk/scan intermediates is named on the openarchlab page, section 3).
 * The gradient is that of the exact recurrence, in fp32 arithmetic (adjoint of
 * one step: G_{t-1} = Diag(alpha_t) (I - a~_t k_t^T) (G_t + q_t do_t^T)).  Two
 * launches on `stream`: a token scan stores the fp32 state after every 64
 * tokens and the residual u_t = m_t - S_{t-1}^T Diag(alpha_t) a~_t of every
 * token; then a cluster of d_v/32 CTAs per (sequence, head) replays each
 * chunk from its checkpoint (with the stored u_t: the update alone) and walks
 * it backwards.  Results are deterministic (fixed summation order).
 * workspace: caller-owned, 16-byte aligned, at least
 * kda_chunk_bwd_workspace_size(...) bytes: (N + ceil(B*T/64)) * H * d_k * d_v
 * * 4 for the checkpoints, B * T * H * d_v * 4 for u_t, plus N * H * 16 * d_k
 * * d_v * 4 (N * H * 64 * d_k * d_v * 4 at d_k = 16) for the states kept
 * during the replay.
 * Errors: as kda_chunk_fwd; KDA_ERR_INVALID_ARG also for nonzero flags, a NULL
 * or misaligned gradient pointer (dg2 only for RDA and GDN-2) or a workspace
 * that is NULL, misaligned or too small.
 */
size_t kda_chunk_bwd_workspace_size(int dtype, int B, int T, int H, int d_k, int d_v,
                                    int has_cu_seqlens, int num_seqs);
int kda_chunk_bwd(int variant, int gate_range, int dtype,
                  int B, int T, int H, int d_k, int d_v,
                  const void *q, const void *k, const void *v, const void *alpha,
                  const void *g1, const void *g2,
                  const int32_t *cu_seqlens, int num_seqs, const float *initial_state,
                  const void *d_o, const float *d_final_state,
                  float *dq, float *dk, float *dv, float *dalpha, float *dg1, float *dg2,
                  float *d_initial_state, void *workspace, size_t workspace_bytes,
                  unsigned flags, void *stream);

/*
 * kda_chunk_bwd_rank2 -- gradients of kda_chunk_fwd_rank2 (two erase/write
 * sub-steps per token: the DeltaProduct_2-style composition the "Complex KDA"
 * arXiv abstract names as prior work), for L with dL/do = d_o [B,T,H,d_v] (the
 * inputs' dtype) and dL/dS_final = d_final_state (NULL = 0).
 * Layouts as for kda_chunk_fwd_rank2: q, alpha, d_o and their gradients dq,
 * dalpha per token [B,T,H,.]; k, v, g1, g2 and their gradients dk, dv, dg1,
 * dg2 with the sub-step axis after T ([B,T,2,H,.]); all gradients fp32.
 * A rank-2 step is two rank-1 steps of the same recurrence, the second with
 * alpha = 1 and the readout after it, so the gradient is the rank-1 backward
 * (kda_chunk_bwd, same arithmetic and tolerance) over the 2T sub-tokens with
 * d_o on the second ones, mapped back: dq from the second sub-tokens, dalpha
 * from the first; the k, v and gate gradients are already in the caller's
 * layout.  Caller-owned workspace of kda_chunk_bwd_rank2_workspace_size bytes
 * (16-byte aligned): the expanded q, alpha, d_o, the sub-token dq, dalpha,
 * the doubled offsets and the rank-1 backward's workspace.  No flags.
 * Errors as kda_chunk_bwd; everything is checked before anything is launched.
 */
size_t kda_chunk_bwd_rank2_workspace_size(int dtype, int B, int T, int H, int d_k, int d_v,
                                          int has_cu_seqlens, int num_seqs);
int kda_chunk_bwd_rank2(int variant, int gate_range, int dtype,
                        int B, int T, int H, int d_k, int d_v,
                        const void *q, const void *k, const void *v, const void *alpha,
                        const void *g1, const void *g2,
                        const int32_t *cu_seqlens, int num_seqs, const float *initial_state,
                        const void *d_o, const float *d_final_state,
                        float *dq, float *dk, float *dv, float *dalpha, float *dg1, float *dg2,
                        float *d_initial_state, void *workspace, size_t workspace_bytes,
                        unsigned flags, void *stream);

/*
 * kda_decode_step -- one recurrent step for N sequences (single-token decode;
 * the fixed-size state of the openarchlab page, sec. 1 and 3).
 *
 *   q, k, alpha : [N,H,d_k]     v, o : [N,H,d_v]     g1, g2 : per variant, [N,H](,d)
 *   state       : [N,H,d_k,d_v] fp32, read and overwritten IN PLACE with S_t
 *   o           : [N,H,d_v] = S_t^T q_t, same dtype as q
 * Sizes: N >= 1, H >= 1, d_k and d_v in {16, 32, 64, 128}.
 * The state is streamed once (read, update, write).  Returns KDA_OK or KDA_ERR_*.
 */
int kda_decode_step(int variant, int gate_range, int dtype,
                    int N, int H, int d_k, int d_v,
                    const void *q, const void *k, const void *v, const void *alpha,
                    const void *g1, const void *g2,
                    float *state, void *o, unsigned flags, void *stream);

/*
 * kda_check_gates -- count gates outside the declared range on the device.
 * Checks alpha [n_tok*d_k] against the range's alpha interval and g1 (beta/e,
 * n_tok values; GDN-2 b, n_tok*d_k values, against [0, 2] for the extended
 * range and [0, 1] otherwise).  Writes the count of violations to the device
 * int `d_count` (caller-owned, overwritten).  NaN counts as a violation.
 */
int kda_check_gates(int variant, int gate_range, int dtype, long long n_tok, int d_k,
                    const void *alpha, const void *g1, int *d_count, void *stream);

/*
 * kda_check_seqlens -- check packed-document offsets on the device: counts
 * cu_seqlens[0] != 0, each n < num_seqs with cu_seqlens[n+1] < cu_seqlens[n],
 * and cu_seqlens[num_seqs] != total_tokens (the B*T of the forward call), and
 * writes the count to the device int `d_count` (caller-owned, overwritten).
 * cu_seqlens: int32 DEVICE array of num_seqs + 1 entries.  The forward calls
 * rely on this contract (the "document reset" of the openarchlab page on
 * GDN/KDA state updates, sec. 3); a batch that breaks it must not be passed
 * to them.  Asynchronous on `stream`; never traps.
 */
int kda_check_seqlens(const int32_t *cu_seqlens, int num_seqs, long long total_tokens, int *d_count,
                      void *stream);

/*
 * kda_device_status -- failures the library's kernels recorded on the current
 * device.  Waits for the work queued on `stream`, then reads and clears the
 * device's failure word: KDA_OK when it was clear, else KDA_ERR_DEVICE_TIMEOUT
 * with the KDA_DEVICE_* bits in *bits (when `bits` is not NULL; 0 on
 * KDA_OK).  The word collects failures of every call on the device since the
 * previous query, whatever its stream: synchronise other streams first to
 * attribute theirs.  Failures a kernel records: a bounded mbarrier wait that
 * ran out (about 2 s; only a broken pipeline gets near it; the kernel then
 * drains its copies in flight, writes NaN to the final state of its
 * (sequence, head) and exits), and in the split form a chunk slot that this
 * call's preparation kernel did not complete.  No kernel traps.
 */
int kda_device_status(void *stream, unsigned *bits);

/* Static description of a status code (never NULL). */
const char *kda_error_string(int code);

/* Detail of the last KDA_ERR_CUDA / KDA_ERR_INVALID_ARG on the calling thread. */
const char *kda_last_error_detail(void);

/* Library version: major*10000 + minor*100 + patch. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
