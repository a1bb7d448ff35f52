/*
 * kd.h -- C ABI of the fused chunked top-K KL distillation loss for B200 (sm_100a).
 *
 * The method (offline top-K teacher cache + fused, chunked KL loss) is the one
 * described on these pages, cited below by title and section:
 *   [DD] developersdigest.tech, "Distilling an LLM on One GPU: Offline Top-K
 *        Logits and a Fused Chunked KL Loss", section "The two changes".
 *   [ST] scitechpulse.com, "New distillation trick cuts training memory below
 *        single-GPU limit for large language models".
 *   [AS] andresseo.expert, sections "Offline Top-K: Compute the Teacher Once,
 *        Then Discard It" and "Fused Chunked KL: The Loss That Never Builds the
 *        Full Grid".
 *
 * Conventions shared by every entry point:
 *   - All tensors are dense, row-major, contiguous, in device memory owned by
 *     the caller.  The library never allocates, frees or synchronises (except
 *     kd_read_device_status, which synchronises the given stream).
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy default
 *     stream.  Every call is asynchronous and stream-ordered.
 *   - Host-side argument checks run before any launch; on failure the call
 *     returns a non-zero kd_status and launches nothing.
 *   - Device-side errors (a bad or duplicate cache index, a wait that ran past
 *     its time limit) are recorded in a status word at the start of the
 *     workspace `ws`; read it with kd_read_device_status.  Each call clears the
 *     status word of its workspace when it starts.
 *   - A workspace may not be used by two calls that can run at the same time.
 *   - Device pointers must be 16-byte aligned; `ws` must be 1024-byte aligned.
 *   - Inside one call, consecutive kernels use programmatic dependent launch:
 *     a kernel may start while the one before it finishes, and waits inside
 *     for that kernel's results.  The first kernel of every call is launched
 *     in plain stream order, so a call starts only after all earlier work in
 *     the stream; work launched after a call in plain stream order starts only
 *     after the whole call has completed.
 */
#ifndef KD_H_
#define KD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kd_status {
  KD_OK = 0,
  KD_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, non-positive size, K > V, bad tau ... */
  KD_ERR_UNSUPPORTED = 2,  /* well-formed but outside the supported ranges          */
  KD_ERR_WORKSPACE = 3,    /* ws_bytes smaller than the matching *_workspace_size   */
  KD_ERR_BAD_INDEX = 4,    /* device: a cache index outside [0,V) or repeated in a row */
  KD_ERR_TIMEOUT = 5,      /* device: a pipeline wait exceeded its time limit        */
  KD_ERR_CUDA = 6,         /* a CUDA runtime/driver call failed                      */
  KD_ERR_INTERNAL = 7      /* device: an internal invariant failed (checked only in
                              the debug build of the library, libkd_debug.so)        */
} kd_status;

typedef enum kd_dtype {
  KD_DTYPE_F32 = 0,  /* float32 operands; tensor cores run kind::tf32, fp32 accumulate */
  KD_DTYPE_BF16 = 1  /* bfloat16 operands; tensor cores run kind::f16, fp32 accumulate */
} kd_dtype;

/* Human-readable name of a status code (static storage, never NULL). */
const char* kd_status_string(int status);

/* ABI version: (major << 16) | minor. */
int kd_version(void);

/* ------------------------------------------------------------------------ */
/* Top-K cache build  ([DD] "The two changes"; [AS] "Offline Top-K"):        */
/* the teacher is run once and its top-K tokens per position are cached.    */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace kd_topk_build needs (the device status word and the
 * counter that hands rows to the kernel's thread blocks). */
size_t kd_topk_workspace_size(int64_t T, int64_t V, int K);

/*
 * For every row t of teacher logits `logits` [T, V] (dtype must be
 * KD_DTYPE_BF16), select the K entries ranked by value descending and, among
 * equal values, index ascending; +0 and -0 compare equal and NaN ranks below
 * -inf.  Writes them in that order:
 *   out_vals float32 [T, K]: exact copies of the selected logits;
 *   out_idx  int32   [T, K]: their column indices.
 * Requires 1 <= K <= min(V, 1024), T >= 1, V < 2^31.
 * ws (1024-byte aligned, ws_bytes >= kd_topk_workspace_size) holds the
 * device status word and a row counter, both cleared at the start of the
 * call; only the debug build records anything in the status word
 * (KD_ERR_INTERNAL).  Read it with kd_read_device_status.  Rows go to the
 * kernel's thread blocks in the order they ask for them, so the workspace must
 * not be shared with a build running at the same time; each row's result does
 * not depend on which block computed it.
 */
kd_status kd_topk_build(const void* logits, int dtype, int64_t T, int64_t V, int K,
                        float* out_vals, int32_t* out_idx,
                        void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Fused chunked KL loss  ([DD] "The two changes"; [ST]; [AS] "Fused        */
/* Chunked KL"): per chunk of positions, project hidden states through the  */
/* output head, take the full-vocabulary logsumexp, gather the student      */
/* log-probs at the cached teacher indices, fold KL into the running loss   */
/* and discard the chunk.  The [T, V] logit grid is never materialised.     */
/*                                                                          */
/*   z = h W^T,  a = z / tau,  LSE_t = log sum_v exp(a_tv)                  */
/*   p_t = softmax(t_vals[t,:] / tau)   (renormalised teacher top-K)        */
/*   KL_t = sum_k p_tk (log p_tk - a_{t, t_idx[t,k]} + LSE_t)               */
/*   loss = (1/T) sum_t KL_t                                                */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace kd_fused_kl_fwd / kd_fused_kl_bwd need for these sizes.
 * One workspace of this size serves both calls.  Besides O(T*K) for the
 * prepared cache it holds, independent of T: the backward's dz of two
 * consecutive chunks (2 * min(chunk,T) * V values of the operand dtype; dW is
 * updated once per pair of chunks) and up to four fp32 K-split partials of one
 * chunk's dH. */
size_t kd_fused_kl_workspace_size(int64_t T, int64_t d, int64_t V, int K, int64_t chunk,
                                  int dtype);

/*
 * Forward.
 *   h      [T, d]  dtype     student hidden states
 *   W      [V, d]  dtype     output head (nn.Linear layout, no bias)
 *   t_vals [T, K]  float32   cached teacher logits (any order within a row)
 *   t_idx  [T, K]  int32     their vocabulary indices, distinct within a row
 *   chunk            positions per chunk (bounds the per-launch working set)
 *   temperature      tau > 0, finite; divides teacher and student logits
 * Outputs (device):
 *   loss   float32 scalar    mean KL over the T positions
 *   lse    float32 [T]       LSE_t (keep it for kd_fused_kl_bwd)
 *   kl_rows float32 [T] or NULL   per-position KL_t
 * Requires d % 8 == 0, 1 <= K <= min(V, 1024), chunk >= 1, V < 2^31 - 256,
 * T < 2^40 and min(chunk, T) <= 2^30 (else KD_ERR_UNSUPPORTED).
 * Per-position results (lse, kl_rows) and the loss are bit-identical for every
 * `chunk`.
 */
kd_status kd_fused_kl_fwd(const void* h, const void* W, int dtype,
                          int64_t T, int64_t d, int64_t V,
                          const float* t_vals, const int32_t* t_idx, int K,
                          int64_t chunk, float temperature,
                          float* loss, float* lse, float* kl_rows,
                          void* ws, size_t ws_bytes, void* stream);

/*
 * Backward (recomputes each chunk's projection; [DD] "The two changes": the
 * backward pass recomputes each chunk on the fly).
 *   dz_tv = g / (T tau) * (S_t exp(a_tv - LSE_t) - sum_k p_tk [v == t_idx[t,k]])
 *   dH = dz W          -> dH [T, d], same dtype as h (overwritten)
 *   dW (+)= dz^T h     -> dW [V, d] float32; overwritten when accumulate_dW == 0,
 *                         added to when accumulate_dW != 0
 *   lse        [T] float32 from kd_fused_kl_fwd on the same inputs
 *   grad_loss  device float32 scalar g, or NULL for g = 1
 */
kd_status kd_fused_kl_bwd(const void* h, const void* W, int dtype,
                          int64_t T, int64_t d, int64_t V,
                          const float* t_vals, const int32_t* t_idx, int K,
                          int64_t chunk, float temperature, const float* lse,
                          const float* grad_loss,
                          void* dH, float* dW, int accumulate_dW,
                          void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Variants of the same objective, selected by `flags` (bitwise OR):        */
/* ------------------------------------------------------------------------ */

/* t_vals hold the teacher's log-probabilities from a softmax over the FULL
 * vocabulary (at whatever temperature the teacher was run), not logits.
 * p_tk = exp(t_vals[t,k]) is used as given, with no renormalisation and no
 * temperature, so S_t = sum_k p_tk may be below 1 (the mass of the tokens the
 * cache dropped).  The loss and gradient formulas above hold with this p:
 * KL_t = sum_k p_tk (t_vals[t,k] - a_{t, t_idx[t,k]} + LSE_t), and dz keeps
 * its S_t softmax - p form.  [DD] "The two changes" caches the teacher's top-K
 * entries; this flag reads such a cache as probabilities of the full teacher
 * distribution. */
#define KD_KL_LOGPROB_CACHE 0x1u
/* Multiply the loss and every gradient by tau^2 (the usual temperature
 * compensation of distillation).  kl_rows stays the unscaled KL_t. */
#define KD_KL_TAU_SQUARED 0x2u
#define KD_KL_KNOWN_FLAGS (KD_KL_LOGPROB_CACHE | KD_KL_TAU_SQUARED)

/* kd_fused_kl_fwd / kd_fused_kl_bwd with `flags`; flags == 0 is exactly the
 * plain calls.  Pass the same flags to the forward and to the backward of one
 * step (the backward re-derives p from t_vals).  Unknown bits return
 * KD_ERR_INVALID_ARG and launch nothing. */
kd_status kd_fused_kl_fwd_ex(const void* h, const void* W, int dtype,
                             int64_t T, int64_t d, int64_t V,
                             const float* t_vals, const int32_t* t_idx, int K,
                             int64_t chunk, float temperature, uint32_t flags,
                             float* loss, float* lse, float* kl_rows,
                             void* ws, size_t ws_bytes, void* stream);

kd_status kd_fused_kl_bwd_ex(const void* h, const void* W, int dtype,
                             int64_t T, int64_t d, int64_t V,
                             const float* t_vals, const int32_t* t_idx, int K,
                             int64_t chunk, float temperature, uint32_t flags,
                             const float* lse, const float* grad_loss,
                             void* dH, float* dW, int accumulate_dW,
                             void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Data-parallel shards.  The loss is a mean over positions and every       */
/* position's terms are independent, so a batch of T_total positions can be */
/* split along T over ranks: each rank runs the fused loss on its own rows  */
/* and only the scalar loss and dW (a sum over positions) are summed across */
/* ranks afterwards (an all-reduce; the pages' method runs on one GPU --    */
/* [GX] "Detailed Chronology and Technical Evolution" and [AS] "What a      */
/* Single H200 GPU Can Now Do That Once Required Four Nodes" describe the   */
/* multi-GPU sharding it replaces).                                          */
/* ------------------------------------------------------------------------ */

/*
 * kd_fused_kl_fwd_ex / kd_fused_kl_bwd_ex for T rows that are one shard of a
 * batch of T_total >= T positions: every 1/T of the plain calls becomes
 * 1/T_total.
 *   loss  = (1/T_total) sum over this shard's rows of KL_t (times tau^2 under
 *           KD_KL_TAU_SQUARED), so the shards' losses sum to the batch's loss;
 *   dz_tv = g / (T_total tau) * (...), so dH holds exactly the batch gradient's
 *           rows of this shard and dW this shard's term of the batch's dW (the
 *           sum of the shards' dW is the batch's dW; accumulate_dW may chain
 *           shards on one device).
 * lse and kl_rows are per position and do not depend on T_total.  With
 * T_total == T these are the _ex calls, bit for bit.  T_total < T returns
 * KD_ERR_INVALID_ARG; T_total >= 2^40 returns KD_ERR_UNSUPPORTED.  The
 * workspace is sized for the shard: kd_fused_kl_workspace_size(T, ...).
 */
kd_status kd_fused_kl_fwd_shard(const void* h, const void* W, int dtype,
                                int64_t T, int64_t d, int64_t V,
                                const float* t_vals, const int32_t* t_idx, int K,
                                int64_t chunk, float temperature, uint32_t flags,
                                int64_t T_total,
                                float* loss, float* lse, float* kl_rows,
                                void* ws, size_t ws_bytes, void* stream);

kd_status kd_fused_kl_bwd_shard(const void* h, const void* W, int dtype,
                                int64_t T, int64_t d, int64_t V,
                                const float* t_vals, const int32_t* t_idx, int K,
                                int64_t chunk, float temperature, uint32_t flags,
                                int64_t T_total,
                                const float* lse, const float* grad_loss,
                                void* dH, float* dW, int accumulate_dW,
                                void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then returns the device status recorded in `ws`
 * (KD_OK, KD_ERR_BAD_INDEX, KD_ERR_TIMEOUT or, in the debug build,
 * KD_ERR_INTERNAL), or KD_ERR_CUDA.  Works for the workspaces of both
 * kd_topk_build and the fused loss. */
kd_status kd_read_device_status(const void* ws, void* stream);

/* ------------------------------------------------------------------------ */
/* Failure-detection support.                                               */
/* ------------------------------------------------------------------------ */

/* Time limit, in nanoseconds, of every device-side pipeline wait launched
 * after this call (default 4e9).  On expiry a kernel records KD_ERR_TIMEOUT,
 * waits (with the same limit) for its own copies and MMAs in flight, frees its
 * tensor memory and returns.  limit_ns must be >= 1000. */
kd_status kd_set_wait_limit_ns(uint64_t limit_ns);

/* Launches one block that waits on a barrier nothing ever arrives at, using
 * the same bounded wait as the pipelines, with the given limit.  The kernel
 * returns by itself and records KD_ERR_TIMEOUT in `ws` (ws_bytes >= 1024). */
kd_status kd_debug_wait_probe(void* ws, size_t ws_bytes, uint64_t limit_ns, void* stream);

/* ------------------------------------------------------------------------ */
/* Forward without a caller workspace.  (The pages have no counterpart to   */
/* this entry point; it exists for callers of this library.)                */
/* ------------------------------------------------------------------------ */

/* Size of the scratch array compiled into the library for
 * kd_fused_kl_fwd_noalloc.  Every GPU that loads the library holds this much
 * device memory until the process exits. */
#define KD_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * Same computation, arguments and outputs as kd_fused_kl_fwd, for callers that
 * cannot provide a workspace -- for example a plugin that receives only its
 * input and output pointers, or a program whose device memory all belongs to
 * another framework's pool.  Scratch comes from a fixed array inside the
 * library (1024-byte aligned, like a caller workspace); nothing is allocated.
 *   - The arguments are checked exactly as kd_fused_kl_fwd checks them (same
 *     ranges and status codes) before anything else happens.
 *   - Scratch needed: about 8*T*K + 12*T + 16*min(chunk,T)*ceil(V/256) bytes
 *     plus alignment, computed with overflow checks; when that exceeds
 *     KD_NOALLOC_SCRATCH_BYTES the call returns KD_ERR_WORKSPACE and launches
 *     nothing (e.g. T=32768, K=100, chunk=2048, V=131072 needs about 43 MB and
 *     fits).
 *   - The first call in a CUDA context looks up the array's device address in
 *     that context (cudaGetSymbolAddress, with the device current) and caches
 *     it under the context's unique id; make that first call before any stream
 *     capture.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents (each call rewrites every part it reads): calls that can
 *     overlap on the GPU (other streams, other threads) race and give wrong
 *     results; serialise them.
 *   - Device-side status (bad cache index, timeout) goes to the array's status
 *     word, which this ABI does not expose; use kd_fused_kl_fwd with a
 *     workspace when that check matters.
 */
kd_status kd_fused_kl_fwd_noalloc(const void* h, const void* W, int dtype,
                                  int64_t T, int64_t d, int64_t V,
                                  const float* t_vals, const int32_t* t_idx, int K,
                                  int64_t chunk, float temperature,
                                  float* loss, float* lse, float* kl_rows, void* stream);

/* ------------------------------------------------------------------------ */
/* Measurement support (process-wide state; not thread-safe).              */
/* ------------------------------------------------------------------------ */

/* Number of kernels this library has launched in this process. */
uint64_t kd_launch_count(void);

/* Kinds of tensor-core GEMM launch, for kd_profile_attach's kind_mask. */
#define KD_GEMM_FWD_LSE 1  /* z = h W^T with the logsumexp/gather epilogue      */
#define KD_GEMM_BWD_DZ 2   /* z recomputed with the dz epilogue                 */
#define KD_GEMM_DH 4       /* dH = dz W                                         */
#define KD_GEMM_DW 8       /* dW (+)= dz^T h                                    */

/* While attached, the i-th GEMM launch whose kind is in kind_mask records
 * start_events[i] before and end_events[i] after itself on its stream
 * (cudaEvent_t handles created by the caller with timing enabled), and its
 * kind and FLOP count in kinds[i] / flops[i] (host arrays owned by the caller),
 * for i < capacity.  Launches beyond capacity are not recorded.  The events
 * are recorded as external records, so launches made while their stream is
 * being captured into a CUDA graph put event nodes in the graph, timed again
 * on every replay. */
kd_status kd_profile_attach(void* const* start_events, void* const* end_events, int* kinds,
                            double* flops, int capacity, int kind_mask);

/* Stops recording; returns how many launches were recorded. */
int kd_profile_detach(void);

#ifdef __cplusplus
}
#endif

#endif /* KD_H_ */
