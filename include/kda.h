/*
 * kda.h -- C ABI of libkda: the bounded-decay gated delta rule (the Kimi Delta
 * Attention scan) on NVIDIA B200 (sm_100a).
 *
 * Operations and the passages that define them:
 *
 *   kda_bounded_decay  "Kimi K3: Bounded Decay and Delta Memory", Formula and
 *                      conventions, eq. 5: g = g_min * sigmoid(e^A * z),
 *                      alpha = e^g, per channel, with A a per-head log-scale.
 *   kda_prefill        same page, eq. 1 (fade, correct, read the updated
 *                      state) over whole sequences, returning every output
 *                      and the final state; computed in the chunkwise form of
 *                      the "KDA cheat sheet", Chunkwise parallel form
 *                      (eqs. 3-4). The argument set follows the chunked kernel
 *                      call excerpted on the "Kept memory" page (initial
 *                      state, final state, cu_seqlens).
 *   kda_decode_step    the same recurrence for one new token against a kept
 *                      state that is updated in place ("Kept memory": the
 *                      recurrent form used for one new position with a cache).
 *   kda_prefill_logits, kda_decode_step_logits
 *                      the same two scans fed with the decay logits z: eq. 5
 *                      is evaluated inside the scan kernels.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every call returns a kda_status. KDA_OK is 0. Nothing is launched when a
 *   call returns an error other than KDA_ERR_CUDA; kda_last_error() then holds
 *   a one-line, thread-local description. Nothing throws across the ABI.
 * - Tensor pointers are DEVICE pointers owned by the caller; the library never
 *   allocates device or pinned memory and never frees what it is given (the one
 *   exception is kda_prefill_noalloc's fixed scratch array, which the CUDA
 *   runtime places on a device when that call first runs there). Calls
 *   are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 *   stream); the caller keeps every buffer alive until the work has finished.
 * - Layouts are the contract table's: q, k, alpha/g [B,T,H,K]; v, o [B,T,H,V];
 *   beta [B,T,H]; states [N,H,K,V] (key-by-value: K rows, V columns, V
 *   contiguous, the whole state tensor contiguous). The innermost dimension of
 *   every token tensor is contiguous; its B, T and H dimensions take element
 *   strides (kda_strides), so non-contiguous views such as slices of a fused
 *   projection can be passed directly. A NULL strides pointer means contiguous.
 *   Every row start must be 16-byte aligned (base pointer and strides), else
 *   the call returns KDA_ERR_UNSUPPORTED.
 * - Inputs are never written, except the decode state, which is updated in
 *   place by contract.
 * - No query scaling happens inside the scan (the PaperLeet contract says the
 *   scan performs no query scaling or key normalisation); a caller who wants
 *   D^-1/2 scaling pre-scales q.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* kda_stream_t; /* the same type as cudaStream_t */

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad cu_seqlens size, g_min not < 0 ... */
  KDA_ERR_UNSUPPORTED = 2, /* K, V, dtype or alignment outside the supported set */
  KDA_ERR_CUDA = 3         /* a CUDA launch or runtime call failed; see kda_last_error() */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/* How a decay tensor is given: retention factors alpha in [0,1], or their
 * logarithms g = log(alpha) <= 0. */
typedef enum { KDA_GATE_ALPHA = 0, KDA_GATE_LOG = 1 } kda_gate_kind;

/* Element strides of the B, T and H dimensions of a [B,T,H,D] tensor (or of
 * a [B,T,H] tensor such as beta). For decode tensors ([B,H,D], [B,H]) the t
 * member is ignored. */
typedef struct {
  int64_t b, t, h;
} kda_strides;

typedef struct {
  kda_strides q, k, v, gate, beta, o;
} kda_layout;

/* ---------------------------------------------------------------------------
 * kda_bounded_decay: retention factors from decay logits.
 *
 *   out[b,t,h,c] = alpha = exp(g)      (out_kind == KDA_GATE_ALPHA), or
 *   out[b,t,h,c] = g                   (out_kind == KDA_GATE_LOG),
 *   g = g_min * sigmoid(exp(A_log[h]) * logits[b,t,h,c]).
 *
 * logits  [B,T,H,K], dtype `dtype` (KDA_F32 or KDA_BF16); `out` has the same
 *         shape and dtype (the page: retention matches the logits' dtype).
 * A_log   [H] fp32, the per-head log-scale A.
 * g_min   the lower bound of the log-decay; must be finite and < 0.
 * strides of logits and out: NULL = contiguous.
 * alpha lies in [exp(g_min), 1]; strictly inside for moderate logits, and at
 * an end point only where sigmoid rounds to 0 or 1 in fp32.
 * ------------------------------------------------------------------------- */
int kda_bounded_decay(const void* logits, const kda_strides* logits_strides, kda_dtype dtype,
                      const float* A_log, float g_min, int64_t B, int64_t T, int64_t H, int64_t K,
                      void* out, const kda_strides* out_strides, kda_gate_kind out_kind,
                      kda_stream_t stream);

/* ---------------------------------------------------------------------------
 * kda_softplus_decay: Kimi Linear's unbounded gate, the contrast the
 * bounded-decay page draws (Figure 3(a); "KDA cheat sheet", g_min table):
 *   g = -exp(A_log[h]) * softplus(logits),  softplus(z) = log(1 + e^z),
 * out = exp(g) or g as for kda_bounded_decay, whose arguments, layouts and
 * errors it shares (without g_min). g is unbounded below: alpha can be
 * arbitrarily close to 0.
 * ------------------------------------------------------------------------- */
int kda_softplus_decay(const void* logits, const kda_strides* logits_strides, kda_dtype dtype,
                       const float* A_log, int64_t B, int64_t T, int64_t H, int64_t K,
                       void* out, const kda_strides* out_strides, kda_gate_kind out_kind,
                       kda_stream_t stream);

/* ---------------------------------------------------------------------------
 * kda_prefill_workspace_bytes: bytes of device scratch that let kda_prefill
 * take its two-kernel path for these sizes (0 when no path uses scratch).
 * With bf16 inputs and K = 128, the two-kernel path first computes every
 * chunk's state-independent operands in parallel and stores them in the
 * workspace (about 1 KB per token and head), then runs the recurrence. Given
 * at least this many bytes kda_prefill uses it; given less (or no workspace),
 * it runs the single fused kernel instead, with identical results up to
 * rounding. The caller allocates the workspace; a larger buffer is fine. n_seq
 * is the number of packed sequences (0 without cu_seqlens).
 * ------------------------------------------------------------------------- */
int kda_prefill_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                                int64_t n_seq, kda_dtype dtype, size_t* bytes);

/* ---------------------------------------------------------------------------
 * kda_prefill: the scan over whole sequences.
 *
 * q, k      [B,T,H,K]  dtype `dtype` (KDA_BF16 or KDA_F32; q, k, v share it)
 * v         [B,T,H,V]  dtype `dtype`
 * gate      [B,T,H,K]  fp32 alpha (gate_kind KDA_GATE_ALPHA) or g = log alpha
 *                      (KDA_GATE_LOG), any alpha in [0,1] (g in [-inf, 0]).
 *                      The chunked bf16 kernels factor decay ratios across
 *                      16-token blocks, which stays in range while a block's
 *                      decay on every channel is at least 2^-120 (always so
 *                      for g >= -5, the bounded gate's "KDA cheat sheet"
 *                      range); a block that decays further has its diagonal
 *                      16x16 tiles formed pair by pair from running products
 *                      of alpha instead (slower, exact). alpha below 2^-126,
 *                      alpha = 0 included, is taken as 2^-126: what it leaves
 *                      of the past state is below fp32 resolution.
 * beta      [B,T,H]    fp32 write strength in [0,1]
 * initial_state [N,H,K,V] fp32 or NULL (zeros)
 * final_state   [N,H,K,V] fp32 or NULL (not written). It may be the same
 *               pointer as initial_state (resume in place); partial overlap is
 *               not allowed.
 * cu_seqlens  NULL, or int32 [n_seq+1] device offsets of n_seq packed
 *             sequences along T (B must be 1; offsets non-decreasing from 0
 *             to T; zero-length sequences allowed). N = n_seq then, else N = B.
 * o         [B,T,H,V]  dtype `dtype`, o[t] = S_t^T q_t with S_t the state
 *                      after token t's update.
 * workspace, workspace_bytes: device scratch (see kda_prefill_workspace_bytes);
 *             NULL / 0 selects the single-kernel path. Its contents are
 *             overwritten; concurrent calls must not share one workspace.
 * T == 0 (or a zero-length packed sequence) copies initial_state (or zeros)
 * to final_state. Supported: K, V multiples of 16 in [16, 256].
 * ------------------------------------------------------------------------- */
int kda_prefill(const void* q, const void* k, const void* v, kda_dtype dtype,
                const float* gate, kda_gate_kind gate_kind, const float* beta,
                const float* initial_state, float* final_state,
                const int32_t* cu_seqlens, int64_t n_seq,
                int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                const kda_layout* layout, void* o,
                void* workspace, size_t workspace_bytes, kda_stream_t stream);

/* Input preparation the logits entry points can do inside their kernels
 * (bit flags): the steps the surrounding model applies to q, k and beta
 * ("KDA cheat sheet", How the inputs are produced: q, k = L2Norm(...),
 * beta = Sigmoid(W_beta x)).
 *   KDA_QK_L2NORM    q and k are replaced by x / sqrt(sum_c x_c^2 + 1e-6) over
 *                    the K channels of each (token, head) before use.
 *   KDA_BETA_LOGITS  beta holds logits b; the kernels use sigmoid(b).
 *   KDA_STATE_VK     the states (initial, final, decode) are stored
 *                    value-by-key, [N,H,V,K] with K contiguous (the
 *                    transpose of the default [N,H,K,V]; "Kept memory": the
 *                    production cache keeps S this way).
 *   KDA_GATE_SOFTPLUS the logits feed Kimi Linear's unbounded gate,
 *                    g = -exp(A_log[h]) * softplus(z + dt_bias) (g_min is
 *                    ignored), instead of the bounded one. Its per-token decay
 *                    has no lower bound; the chunked kernels form the diagonal
 *                    16x16 blocks of any block it takes out of range pair by
 *                    pair (see kda_prefill), with or without a workspace. */
#define KDA_QK_L2NORM 1u
#define KDA_BETA_LOGITS 2u
#define KDA_STATE_VK 4u
#define KDA_GATE_SOFTPLUS 8u

/* ---------------------------------------------------------------------------
 * kda_prefill_logits: kda_prefill with the bounded gate applied inside the
 * scan ("Kimi K3: Bounded Decay and Delta Memory", Formula and conventions,
 * eq. 5 feeding eq. 1): the decay input is the logits z instead of alpha or g,
 *   g = g_min * sigmoid(exp(A_log[h]) * z),  alpha = exp(g),
 * evaluated per element while the scan reads it, so g never travels through
 * device memory.
 *
 * logits   [B,T,H,K] fp32, strides in layout->gate (the slot kda_prefill
 *          uses for alpha / g).
 * A_log    [H] fp32 device pointer; g_min finite and < 0
 *          (else KDA_ERR_INVALID_ARG).
 * dt_bias  NULL, or [H,K] fp32 device pointer (contiguous, 16-byte aligned):
 *          a per-(head, channel) bias added to the logits before the gate,
 *          g = g_min * sigmoid(exp(A_log[h]) * (z + dt_bias[h,c])) ("KDA cheat
 *          sheet", How the inputs are produced: z = W_up W_down x + b; the
 *          chunked kernel call on the "Kept memory" page takes it as dt_bias).
 *          The sum z + dt_bias is rounded to fp32 once, as a caller adding it
 *          beforehand would.
 * flags    0, or any of KDA_QK_L2NORM, KDA_BETA_LOGITS, KDA_STATE_VK,
 *          KDA_GATE_SOFTPLUS (unknown bits: KDA_ERR_INVALID_ARG). The chunked bf16 kernels round normalised
 *          q and k to bf16, their operand precision; the fp32 kernel keeps
 *          them in fp32.
 * Every other argument, layout, result, workspace rule and error is
 * kda_prefill's. With flags 0 the result is bit-identical to
 * kda_bounded_decay (on z + dt_bias) with out_kind KDA_GATE_LOG (bf16 inputs)
 * or KDA_GATE_ALPHA (fp32 inputs) followed by kda_prefill on its output: both
 * evaluate the gate with the same device code.
 * ------------------------------------------------------------------------- */
int kda_prefill_logits(const void* q, const void* k, const void* v, kda_dtype dtype,
                       const float* logits, const float* A_log, const float* dt_bias, float g_min,
                       const float* beta, unsigned flags,
                       const float* initial_state, float* final_state,
                       const int32_t* cu_seqlens, int64_t n_seq,
                       int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                       const kda_layout* layout, void* o,
                       void* workspace, size_t workspace_bytes, kda_stream_t stream);

/* ---------------------------------------------------------------------------
 * kda_prefill_noalloc: kda_prefill for callers that cannot allocate device
 * memory. The pages have no counterpart; it is a library convenience.
 *
 * Who needs it: a plain C host that links only libkda and has no CUDA
 * allocator of its own, and a serving loop that must not call cudaMalloc /
 * cudaFree between steps (they synchronise the device). Such callers cannot
 * hand kda_prefill the workspace its two-kernel path wants. This call takes
 * that workspace from a scratch array compiled into the library, one copy per
 * device, of KDA_NOALLOC_SCRATCH_BYTES bytes, and allocates nothing itself.
 *
 * Arguments, layouts, results and errors are kda_prefill's, without the
 * workspace pair. Sizes whose workspace (kda_prefill_workspace_bytes) exceeds
 * KDA_NOALLOC_SCRATCH_BYTES are rejected with KDA_ERR_UNSUPPORTED and a
 * message naming both sizes; nothing is launched then. Sizes that need no
 * workspace (fp32 inputs, K != 128) run as kda_prefill does without one.
 *
 * Setup: the first call on a device (the device current at the call) looks
 * up the scratch's device address once and keeps it; make that first call
 * before any stream capture on that device. The address stays valid for the
 * life of the device's primary context: do not reset the device
 * (cudaDeviceReset) between calls, since the scratch may then sit elsewhere.
 * With lazy module loading (the CUDA default) the array takes device memory
 * only on devices where this call has run; with CUDA_MODULE_LOADING=EAGER it
 * is reserved on every device the library is loaded on.
 *
 * Sharing: every call on a device uses the same scratch. Nothing in it has to
 * start at zero (each call writes all it reads), but calls whose GPU work may
 * overlap -- on different streams, or from host threads with no ordering
 * between them -- race on it; order them on one stream.
 * ------------------------------------------------------------------------- */
#define KDA_NOALLOC_SCRATCH_BYTES ((size_t)128 << 20) /* 128 MiB: 2,032 chunk-heads of 64 tokens */

int kda_prefill_noalloc(const void* q, const void* k, const void* v, kda_dtype dtype,
                        const float* gate, kda_gate_kind gate_kind, const float* beta,
                        const float* initial_state, float* final_state,
                        const int32_t* cu_seqlens, int64_t n_seq,
                        int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                        const kda_layout* layout, void* o, kda_stream_t stream);

/* ---------------------------------------------------------------------------
 * kda_decode_step: one new token per (b, h) against a kept state, in place.
 *
 * q, k [B,H,K]; v, o [B,H,V]  dtype `dtype` (a [B,1,H,D] tensor is passed with
 *                             its b and h strides)
 * gate [B,H,K] fp32 alpha or g; beta [B,H] fp32
 * state [B,H,K,V] fp32, contiguous: read as S_{t-1}, overwritten with S_t.
 *   Sbar = Diag(alpha) S;  delta = v - Sbar^T k;  S = Sbar + beta k delta^T;
 *   o = S^T q.
 * Any alpha in [0,1] is accepted. Supported: K, V multiples of 16 in [16,256].
 * ------------------------------------------------------------------------- */
int kda_decode_step(const void* q, const void* k, const void* v, kda_dtype dtype,
                    const float* gate, kda_gate_kind gate_kind, const float* beta,
                    float* state, int64_t B, int64_t H, int64_t K, int64_t V,
                    const kda_layout* layout, void* o, kda_stream_t stream);

/* ---------------------------------------------------------------------------
 * kda_decode_step_logits: kda_decode_step with the bounded gate (eq. 5)
 * applied inside the step: logits [B,H,K] fp32 (strides in layout->gate),
 * A_log [H] fp32, dt_bias NULL or [H,K] fp32 (as for kda_prefill_logits),
 * g_min finite and < 0. alpha = exp(g_min * sigmoid(exp(A_log[h]) *
 * (z + dt_bias[h,c]))). flags as for kda_prefill_logits (normalised q, k kept
 * in fp32). Everything else is kda_decode_step's; with flags 0 the result is
 * bit-identical to kda_bounded_decay (alpha out) followed by kda_decode_step.
 * ------------------------------------------------------------------------- */
int kda_decode_step_logits(const void* q, const void* k, const void* v, kda_dtype dtype,
                           const float* logits, const float* A_log, const float* dt_bias, float g_min,
                           const float* beta, unsigned flags,
                           float* state, int64_t B, int64_t H, int64_t K, int64_t V,
                           const kda_layout* layout, void* o, kda_stream_t stream);

/* ---------------------------------------------------------------------------
 * kda_scan_backward: gradients of kda_prefill's scan (eq. 1 over whole
 * sequences) with respect to every input. The pages' contract is
 * differentiable ("Kimi K3: Bounded Decay and Delta Memory", contract table);
 * this computes, by the adjoint of the token recurrence,
 *   dq, dk [B,T,H,K], dv [B,T,H,V], dgate [B,T,H,K] (dL/dalpha for
 *   KDA_GATE_ALPHA, dL/dg for KDA_GATE_LOG), dbeta [B,T,H] and
 *   d_initial_state [B,H,K,V] (NULL: not written),
 * given d_o [B,T,H,V] = dL/do and d_final_state [B,H,K,V] = dL/dS_T (NULL:
 * zeros); with cu_seqlens the states are per sequence (below). All gradient tensors are fp32 and contiguous; q, k, v, gate, beta
 * and initial_state are the forward call's inputs (layout strides for q, k, v,
 * gate, beta as in kda_prefill). cu_seqlens (device int32 [n_seq + 1],
 * nullable) packs variable-length sequences as in kda_prefill: B must be 1,
 * the states initial_state, d_final_state and d_initial_state are
 * [n_seq,H,K,V], and gradients of tokens outside [cu[0], cu[n_seq]) are not
 * written; without it n_seq is ignored. Supported: K, V in {16, 32, 64, 128}.
 * The scan is recomputed from checkpoints every 32 tokens: the caller passes
 * a workspace of kda_scan_backward_workspace_bytes for the same B, T, H, K, V
 * and n_seq (0 without cu_seqlens; KDA_ERR_INVALID_ARG if smaller). This is
 * the exact token-by-token adjoint, not a chunked kernel.
 * ------------------------------------------------------------------------- */
int kda_scan_backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V, int64_t n_seq,
                                      size_t* bytes);

int kda_scan_backward(const void* q, const void* k, const void* v, kda_dtype dtype,
                      const float* gate, kda_gate_kind gate_kind, const float* beta,
                      const float* initial_state, const float* d_o, const float* d_final_state,
                      const int32_t* cu_seqlens, int64_t n_seq,
                      int64_t B, int64_t T, int64_t H, int64_t K, int64_t V, const kda_layout* layout,
                      float* dq, float* dk, float* dv, float* dgate, float* dbeta, float* d_initial_state,
                      void* workspace, size_t workspace_bytes, kda_stream_t stream);

/* ---------------------------------------------------------------------------
 * kda_scan_backward_chunked: the same gradients as kda_scan_backward, computed
 * through the chunkwise form ("KDA cheat sheet", chunkwise form, eqs. 3-4) in
 * parallel over 64-token chunks: the forward's split kernels keep the state at
 * every chunk start, one reverse recurrence over chunks gives the gradient of
 * the state at every chunk end, and every other gradient is formed per chunk
 * (per-pair decay ratios, triangular inverse, plain batched products through
 * cuBLAS in fp32 with TF32 tensor cores). Arguments, layouts and outputs as for
 * kda_scan_backward, packed sequences (cu_seqlens, n_seq; B = 1; states per
 * sequence) included. Supported: bf16 q, k, v with K = V = 128
 * (KDA_ERR_UNSUPPORTED otherwise). With KDA_GATE_ALPHA the gate's gradient is
 * formed as dL/dalpha = (dL/dlog alpha) / alpha: its absolute error grows like
 * 1/alpha for small alpha, and it is 0 where alpha = 0; gates near zero take
 * KDA_GATE_LOG or kda_scan_backward. The chunk-start states come from the bf16
 * tensor-core forward, so the gradients carry its rounding (relative RMS errors
 * near 1e-3) where kda_scan_backward's token-level adjoint is exact fp32. The
 * workspace (kda_scan_backward_chunked_workspace_bytes for the same B, T, H, K,
 * V and n_seq, 0 without cu_seqlens; about 880 KB per chunk and head, plus
 * n_seq + 1 chunks per head with cu_seqlens; KDA_ERR_INVALID_ARG if smaller)
 * holds every intermediate. cuBLAS creates its handle (device memory) on the
 * first call on each device and is given a part of the workspace for its own
 * scratch; host threads calling on the same device take turns while a call
 * enqueues its work (the call does not wait for the GPU).
 * ------------------------------------------------------------------------- */
int kda_scan_backward_chunked_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                                              int64_t n_seq, size_t* bytes);

int kda_scan_backward_chunked(const void* q, const void* k, const void* v, kda_dtype dtype,
                              const float* gate, kda_gate_kind gate_kind, const float* beta,
                              const float* initial_state, const float* d_o, const float* d_final_state,
                              const int32_t* cu_seqlens, int64_t n_seq,
                              int64_t B, int64_t T, int64_t H, int64_t K, int64_t V, const kda_layout* layout,
                              float* dq, float* dk, float* dv, float* dgate, float* dbeta, float* d_initial_state,
                              void* workspace, size_t workspace_bytes, kda_stream_t stream);

/* ---------------------------------------------------------------------------
 * kda_bounded_decay_backward: gradients of eq. 5's log-decay
 * g = g_min * sigmoid(exp(A_log[h]) * z) given d_log_decay = dL/dg:
 *   d_logits = dL/dz [B,T,H,K], d_A_log = dL/dA_log [H] (overwritten).
 * All fp32 and contiguous. With kda_scan_backward in KDA_GATE_LOG mode this
 * completes the chain from the logits.
 * ------------------------------------------------------------------------- */
int kda_bounded_decay_backward(const float* logits, const float* A_log, float g_min, const float* d_log_decay,
                               int64_t B, int64_t T, int64_t H, int64_t K, float* d_logits, float* d_A_log,
                               kda_stream_t stream);

/* ---------------------------------------------------------------------------
 * kda_device_status: device-side failure flags, for callers that check them
 * after their work has finished. Every wait inside the library's kernels is
 * bounded (about one second of device time, at most 2^22 polls); a kernel
 * whose wait expires records the event in a device flag and returns instead
 * of hanging. This call synchronises the current device, writes 1 to
 * *timed_out if any such event has been recorded since the last reset (0
 * otherwise), and clears the flag when reset != 0.
 * ------------------------------------------------------------------------- */
int kda_device_status(int* timed_out, int reset);

/* ---------------------------------------------------------------------------
 * kda_selftest_wait_expiry: diagnostics for the failure path above. Launches
 * one single-thread kernel on `stream` that waits on an mbarrier nothing ever
 * arrives on; the wait gives up after its limit (about one second) and
 * records the expiry, which the next kda_device_status reports. Nothing else
 * is touched and the context stays usable.
 * ------------------------------------------------------------------------- */
int kda_selftest_wait_expiry(kda_stream_t stream);

/* Last error of the calling thread ("" when the last call succeeded). */
const char* kda_last_error(void);

/* Library version string. */
const char* kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
