/*
 * flce.h -- C ABI of the fused linear + cross-entropy (FLCE) head for NVIDIA
 * B200 (sm_100a).
 *
 * The operation.  Given hidden states X[N,H] and an LM-head weight W[V,H] (one
 * row per vocabulary entry) and integer targets y[N], the head returns the
 * token-mean cross-entropy of the logits z = X W^T against y, and the
 * gradients of that loss with respect to X and W, without ever holding the
 * N x V logit tensor in device memory:
 *
 *   valid_i = (y_i != ignore_index),       n = sum_i valid_i
 *   lse_i   = log sum_j exp(z_ij)
 *   loss    = (1/n) sum_{valid i} (lse_i - z_{i,y_i})
 *   G_ij    = valid_i (exp(z_ij - lse_i) - [j == y_i]) / n
 *   dX      = G W,      dW = G^T X
 *
 * Sources: "Liger-Kernel: Triton kernels that replace HF training ops",
 * section "What actually gets replaced" (FusedLinearCrossEntropy consumes the
 * hidden states and the LM-head weight and produces the loss directly, the
 * (batch, sequence, vocab) tensor is never allocated, same call signature as
 * the unfused modules); "Liger Kernel explained", section on the
 * cross-entropy head (loss and gradient computed in chunks over the
 * vocabulary, intermediates recomputed instead of stored); "Complete Guide to
 * Liger Kernel", section LigerFusedLinearCrossEntropyLoss (the call takes
 * hidden states, a (vocab_size, hidden_size) weight and labels).  The pages
 * never state the ignore value or the mean's denominator; this library reads
 * them as PyTorch's: targets equal to ignore_index (normally -100) are
 * skipped and the mean runs over the n non-ignored rows.  With n = 0 the
 * loss, dX and dW are all zero.
 *
 * Layouts.  Every matrix is row-major and contiguous.  X, W, dX and dW hold
 * bf16 values (passed as uint16_t bit patterns); y holds int32 targets; the
 * loss is an fp32 scalar.  H must be a multiple of 8 (16-byte rows for the
 * tensor-memory-access engine); X, W, dX and dW must be 16-byte aligned and
 * the workspace 256-byte aligned.
 *
 * Ownership.  All device pointers belong to the caller.  The library never
 * allocates device memory: scratch space is the caller's `workspace`, at least
 * flce_workspace_size(N, H, V) bytes, a size that does not depend on V.  dX
 * and dW are overwritten, not accumulated into.  The library keeps only
 * read-only host caches (device properties, a driver entry point) and, for
 * the host-buffer entry, one copy stream with a few events per device.
 *
 * Errors.  Argument errors are found on the host and returned before anything
 * is launched.  Errors found on the device (a valid target outside [0, V), a
 * bounded wait inside a kernel that ran out) are written to a device status
 * word; the synchronous entry points read it back and return it.  Nothing
 * traps or asserts on the device.
 *
 * Ignored rows.  The work runs in 256-row token tiles, and a tile whose
 * targets are all ignored is skipped.  When ignored rows are scattered, so
 * that packing the valid rows first would fill fewer tiles than the tiles
 * holding any valid row, and the workspace holds the packed-X area (see
 * flce_workspace_size_reorder), the library reorders the token rows on the
 * device (a stable partition, valid rows first): it packs those rows of X
 * into the workspace, runs both passes on them, and writes dX and the per-row
 * losses back in the caller's row order.  The choice changes only the order of
 * floating-point sums, not the result's definition.
 */
#ifndef FLCE_H_
#define FLCE_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FLCE_OK = 0,
  FLCE_ERR_INVALID_ARGUMENT = 1,    /* NULL pointer, non-positive size, size too large */
  FLCE_ERR_UNSUPPORTED = 2,         /* H % 8 != 0, misaligned pointer, device is not sm_100 */
  FLCE_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes < flce_workspace_size(N, H, V) */
  FLCE_ERR_TARGET_OUT_OF_RANGE = 4, /* some y_i != ignore_index lies outside [0, V) */
  FLCE_ERR_TIMEOUT = 5,             /* a bounded wait inside a kernel gave up */
  FLCE_ERR_CUDA = 6                 /* a CUDA runtime call failed */
} flce_status_t;

/* Human-readable name of a status code (static storage). */
const char* flce_status_string(int status);

/* Where the last FLCE_ERR_CUDA returned on this host thread came from: the
 * library's source line of the failing step, the CUDA runtime's error code
 * and its text (static storage).  Any argument may be NULL.  Zero / "no error"
 * when no call on this thread has failed. */
void flce_last_cuda_error(int32_t* line, int32_t* cuda_error, const char** text);

/* Bytes of device workspace one call needs.  The logits are processed one
 * vocabulary chunk of fixed width at a time, so the size depends on N and H
 * only: V is accepted for the caller's convenience and does not change the
 * value.  Returns 0 for invalid sizes. */
size_t flce_workspace_size(int64_t N, int64_t H, int64_t V);

/* Bytes of a workspace that also holds the N x H bf16 area (its byte size
 * rounded up to a multiple of 256) for a packed copy of X, which reordered
 * token rows need (see "Ignored rows"): flce_workspace_size(N, H, V) plus that
 * area, again independent of V.  Entries that take a workspace_bytes argument
 * reorder rows only when given at least this many bytes; with less (but at
 * least flce_workspace_size) they keep the caller's order.  Returns 0 for
 * invalid sizes.  The pages describe no such query; it sizes the library's
 * own row gather. */
size_t flce_workspace_size_reorder(int64_t N, int64_t H);

/* Synchronous forward + backward.
 *   X  [N,H] bf16, device      W  [V,H] bf16, device      y [N] int32, device
 *   loss: HOST float*, receives the token-mean loss
 *   dX [N,H] bf16, device (out)   dW [V,H] bf16, device (out)
 *   workspace: device, >= flce_workspace_size(N, H, V) bytes, 256-B aligned
 *              (this entry never reorders token rows: it has no size argument)
 *   stream: the CUDA stream to run on (0 = legacy default stream)
 * Blocks the calling host thread until the stream has finished the call, then
 * returns FLCE_OK or the first error seen, including device-side errors. */
flce_status_t flce_forward_backward(const uint16_t* X, const uint16_t* W, const int32_t* y,
                                    int64_t N, int64_t H, int64_t V, int32_t ignore_index,
                                    float* loss, uint16_t* dX, uint16_t* dW, void* workspace,
                                    cudaStream_t stream);

/* Asynchronous twin: enqueues the whole computation on `stream` and returns.
 *   d_loss:   DEVICE float*, receives the loss when the stream gets there
 *   d_status: DEVICE int32_t*, receives 0 or a device-side flce_status_t
 *   workspace_bytes: size of `workspace`, at least flce_workspace_size(N, H, V);
 *                    flce_workspace_size_reorder(N, H) or more lets the call
 *                    reorder token rows
 * Host-side argument errors are returned immediately; device-side errors only
 * appear in *d_status.
 * CUDA graphs: the call enqueues only memsets and kernel launches, so it may
 * be captured on `stream` once one call outside a capture has set up the
 * library on this device.  Decisions that depend on the data (skipped token
 * tiles, reordered rows, the mean's count) are taken on the device, so a
 * replay computes the head on whatever the captured buffers hold then. */
flce_status_t flce_forward_backward_async(const uint16_t* X, const uint16_t* W, const int32_t* y,
                                          int64_t N, int64_t H, int64_t V, int32_t ignore_index,
                                          float* d_loss, int32_t* d_status, uint16_t* dX,
                                          uint16_t* dW, void* workspace, size_t workspace_bytes,
                                          cudaStream_t stream);

/* End-to-end entry for callers whose data sits in HOST memory.
 *   h_X, h_W, h_y: host inputs (pinned memory gives full copy bandwidth)
 *   h_loss, h_dX, h_dW: host outputs
 *   d_X, d_W, d_y, d_dX, d_dW, workspace: caller-owned device buffers of the
 *   same shapes (workspace >= flce_workspace_size bytes)
 * Copies the inputs to the device, runs the computation, copies loss, dX and
 * dW back, and waits for the stream.  No allocation happens inside.  The
 * copies overlap the kernels: W goes over in up to 16 pieces on an internal
 * copy stream and pass 1 runs piece by piece as they land; pass 2 runs in up
 * to 16 sections of whole vocabulary chunks, the last one a single chunk, and
 * each section's finished dW rows come back while the next one computes.  Results agree with flce_forward_backward's to
 * rounding (the log-sum-exp partials are merged in another order).  The copy
 * stream and its events are made on first use, one set per device, and kept;
 * host-buffer calls on one device run one at a time. */
flce_status_t flce_forward_backward_host(const uint16_t* h_X, const uint16_t* h_W,
                                         const int32_t* h_y, int64_t N, int64_t H, int64_t V,
                                         int32_t ignore_index, float* h_loss, uint16_t* h_dX,
                                         uint16_t* h_dW, uint16_t* d_X, uint16_t* d_W,
                                         int32_t* d_y, uint16_t* d_dX, uint16_t* d_dW,
                                         void* workspace, size_t workspace_bytes,
                                         cudaStream_t stream);

/* Data-parallel entry whose dW can be reduced while the call still runs.
 * Enqueues the mean-reduced call of flce_forward_backward_ex (d_mean_count:
 * DEVICE int32 or NULL, as there) with the gradient pass split into
 * `sections` launches over consecutive ranges of vocabulary chunks (1 ..
 * 16; at most one per 2048-entry chunk; with several, the last section is
 * the last chunk alone, so that little is left to reduce after the last
 * launch).  After section k the call records
 * section_done[k] (caller-created CUDA events) on `stream`; from then on dW rows
 * [section_rows[k], section_rows[k+1]) are final, so the caller can start
 * reducing them over the data-parallel ranks on another stream (e.g. an NCCL
 * all-reduce after cudaStreamWaitEvent) while the later sections compute.
 * section_rows: HOST int64 [sections + 1], filled before the call returns;
 * sections beyond the number of chunks are empty and complete with the last.
 * Other arguments and results as flce_forward_backward_async; the results
 * are those of an unsplit call (the same sums in the same order).  The split
 * follows from the pages' method: the gradient is computed chunk by chunk
 * over the vocabulary ("Liger Kernel explained", cross-entropy head section),
 * so the dW rows of a chunk are complete when its chunk is. */
flce_status_t flce_forward_backward_sections(const uint16_t* X, const uint16_t* W, const int32_t* y, int64_t N,
                                             int64_t H, int64_t V, int32_t ignore_index, const int32_t* d_mean_count,
                                             float* d_loss, int32_t* d_status, uint16_t* dX, uint16_t* dW,
                                             void* workspace, size_t workspace_bytes, int32_t sections,
                                             cudaEvent_t* section_done, int64_t* section_rows, cudaStream_t stream);

/* Reductions of flce_forward_backward_ex.  All three are one weighted sum over
 * the non-ignored rows, loss = sum_i s_i l_i with l_i = lse_i - z_{i,y_i}, and
 * dX, dW are the gradients of that loss (G_ij = s_i (softmax_ij - [j == y_i])):
 *   MEAN  s_i = 1/n_valid (the default of the other entry points)
 *   SUM   s_i = 1
 *   NONE  s_i = grad_row_scale[i], the caller's upstream gradient of row i's
 *         loss (1 when grad_row_scale is NULL); the per-row losses themselves
 *         come back in row_loss.
 * These are PyTorch's cross_entropy reductions, which a drop-in replacement of
 * the unfused head ("Liger-Kernel: Triton kernels that replace HF training
 * ops", section "What actually gets replaced") has to offer; per-row weights
 * and log-probabilities are also what a fused-linear preference loss builds on. */
typedef enum { FLCE_REDUCTION_MEAN = 0, FLCE_REDUCTION_SUM = 1, FLCE_REDUCTION_NONE = 2 } flce_reduction_t;

/* Asynchronous entry with every option.
 *   reduction:      flce_reduction_t
 *   grad_row_scale: DEVICE float[N] or NULL (used by NONE only)
 *   d_mean_count:   DEVICE int32 or NULL (MEAN only): divide by this count
 *                   instead of this call's n_valid, e.g. the number of valid
 *                   targets over every data-parallel rank, so that the ranks'
 *                   losses and dW add up to those of the whole batch
 *   d_loss:         DEVICE float, receives sum_i s_i l_i
 *   d_row_loss:     DEVICE float[N] or NULL: l_i for valid rows, 0 for ignored rows
 *   d_status:       DEVICE int32, 0 or a device-side flce_status_t
 *   dX, dW:         device outputs; both NULL = forward only (loss and row
 *                   losses, no gradient pass); exactly one NULL is an error
 * Other arguments as flce_forward_backward_async. */
flce_status_t flce_forward_backward_ex(const uint16_t* X, const uint16_t* W, const int32_t* y, int64_t N,
                                       int64_t H, int64_t V, int32_t ignore_index, int32_t reduction,
                                       const float* grad_row_scale, const int32_t* d_mean_count,
                                       float* d_loss, float* d_row_loss, int32_t* d_status, uint16_t* dX,
                                       uint16_t* dW, void* workspace, size_t workspace_bytes,
                                       cudaStream_t stream);

/* Vocabulary-parallel head.  The loss and its gradient are computed in chunks
 * over the vocabulary ("Liger Kernel explained", section on the cross-entropy
 * head), so the chunks can live on different devices: rank r holds W rows
 * [v0, v0 + V_shard) of a V-entry vocabulary as W_shard [V_shard][H], and
 * every rank holds the same X [N][H] and y [N] (whole-vocabulary ids).  A step
 * runs as
 *   1. flce_vp_shard_stats: pass 1 on the shard.  Per row i it writes
 *      d_shard_lse[i] = log sum_{j in shard} exp(z_ij) and d_shard_zy[i] =
 *      z_{i,y_i} when v0 <= y_i < v0 + V_shard, else 0 (device fp32 [N]).
 *   2. the exchange, by the caller (e.g. NCCL all-gather): every rank's two
 *      vectors, stacked as d_all_lse, d_all_zy [shards][N] (shard order free).
 *   3. flce_vp_backward: lse_i = log sum_s exp(all_lse[s][i]) and z_{i,y_i} =
 *      sum_s all_zy[s][i] give the token-mean loss (d_loss, the same on every
 *      rank) and this shard's G; it writes dW_shard [V_shard][H] complete and
 *      this shard's part of dX, dX_part [N][H] = G_shard W_shard.
 *   4. the caller sums dX_part over the ranks (e.g. NCCL all-reduce).
 * Targets are checked against [0, V); out-of-range ones set
 * FLCE_ERR_TARGET_OUT_OF_RANGE in d_status.  d_mean_count works as in
 * flce_forward_backward_ex (mean only).  dX_part and dW_shard may both be NULL
 * in step 3 for the loss alone.  Rows keep the caller's order (no
 * reordering); the workspace needs flce_workspace_size(N, H, 1) bytes. */
flce_status_t flce_vp_shard_stats(const uint16_t* X, const uint16_t* W_shard, const int32_t* y, int64_t N,
                                  int64_t H, int64_t V_shard, int64_t v0, int64_t V, int32_t ignore_index,
                                  float* d_shard_lse, float* d_shard_zy, int32_t* d_status, void* workspace,
                                  size_t workspace_bytes, cudaStream_t stream);
flce_status_t flce_vp_backward(const uint16_t* X, const uint16_t* W_shard, const int32_t* y, int64_t N, int64_t H,
                               int64_t V_shard, int64_t v0, int64_t V, int32_t ignore_index, int32_t shards,
                               const float* d_all_lse, const float* d_all_zy, const int32_t* d_mean_count,
                               float* d_loss, int32_t* d_status, uint16_t* dX_part, uint16_t* dW_shard,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Cross-entropy on a logit tensor the caller already holds, the unfused
 * counterpart of the head ("Complete Guide to Liger Kernel", section
 * LigerCrossEntropyLoss): the same loss, reductions and row losses as
 * flce_forward_backward_ex, with z given instead of X W^T.
 *   logits:  DEVICE bf16 [N][V], row-major
 *   dlogits: DEVICE bf16 [N][V] receiving d loss / d logits, or NULL for a
 *            forward-only call; may be the same pointer as logits (in place)
 *   workspace: DEVICE, >= flce_ce_workspace_size(N, V) bytes (depends on N only),
 *            256-byte aligned
 * Asynchronous; d_loss, d_row_loss, d_status as in flce_forward_backward_ex. */
size_t flce_ce_workspace_size(int64_t N, int64_t V);
flce_status_t flce_cross_entropy(const uint16_t* logits, const int32_t* y, int64_t N, int64_t V,
                                 int32_t ignore_index, int32_t reduction, const float* grad_row_scale,
                                 float* d_loss, float* d_row_loss, int32_t* d_status, uint16_t* dlogits,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Number of targets y_i != ignore_index among y[0..N), written to the DEVICE
 * int32 *d_count when the stream gets there (an exact integer count).  It is
 * the denominator of the token mean; a data-parallel caller all-reduces it
 * over the ranks and passes the sum as d_mean_count of
 * flce_forward_backward_ex, so that every rank's loss and dW are shares of
 * the whole batch's.  y: DEVICE int32 [N].  Asynchronous. */
flce_status_t flce_count_valid(const int32_t* y, int64_t N, int32_t ignore_index, int32_t* d_count,
                               cudaStream_t stream);

/* Pairwise logistic (DPO-form) preference loss on the head's per-row losses.
 * The post-training losses of the library the pages describe ("Liger-Kernel:
 * Triton kernels that replace HF training ops", section "Installation and the
 * one-line patch": ORPO, DPO, CPO, SimPO ... called with the LM-head weight,
 * the hidden states and the targets, returning the loss) build on two things
 * the fused head gives without the logits: each target's log-probability,
 * -l_i (flce_forward_backward_ex with reduction NONE and d_row_loss), and the
 * gradient of a loss of their per-sequence sums (the same entry with
 * grad_row_scale).  This entry is the step between them:
 *   sequence s = token rows [seq_start[s], seq_start[s+1]),
 *   logp_s = -sum of their row losses,
 *   m_k = beta ((logp_c - ref_c) - (logp_r - ref_r)) for pair k with
 *         c = chosen[k], r = rejected[k] (ref_logp NULL: ref = 0),
 *   loss = -(1/P) sum_k log sigmoid(m_k),
 *   grad_logp[s] = d loss / d logp_s,
 *   row_weight[i] = -grad_logp[s] for a row i of sequence s whose target is
 *                   not ignore_index, 0 for every other row: the upstream
 *                   gradient of l_i, to pass as grad_row_scale.
 * Arguments (all DEVICE, caller-owned): d_row_loss fp32 [N], y int32 [N],
 * d_seq_start int32 [S+1] (non-decreasing, within [0, N]), d_chosen and
 * d_rejected int32 [P] (sequence ids in [0, S)), d_ref_logp fp64 [S] or NULL;
 * outputs d_loss fp64 [1], d_logp and d_grad_logp fp64 [S], d_row_weight
 * fp32 [N], d_status int32 [1].  Sums are fp64 in a fixed order, so the result
 * is the same on every call.  Sequence bounds or pair ids out of range set
 * FLCE_ERR_INVALID_ARGUMENT in d_status.  Asynchronous. */
flce_status_t flce_pairwise_logistic(const float* d_row_loss, const int32_t* y, int64_t N, int32_t ignore_index,
                                     const int32_t* d_seq_start, int32_t S, const int32_t* d_chosen,
                                     const int32_t* d_rejected, int32_t P, double beta, const double* d_ref_logp,
                                     double* d_loss, double* d_logp, double* d_grad_logp, float* d_row_weight,
                                     int32_t* d_status, cudaStream_t stream);

/* Allocation-free variant of flce_forward_backward, for callers that cannot
 * allocate device memory: a plug-in or custom operator that is handed only the
 * tensors it works on and has no allocator to ask for scratch, and processes
 * where a framework's memory pool has already reserved nearly all of the GPU,
 * so that a raw cudaMalloc from a library would fail.  The published
 * fused-head method has no counterpart of this entry: it exists only for such
 * callers.
 *
 * Arguments are those of flce_forward_backward minus the workspace (X, W, y,
 * dX, dW on the device; loss on the host; synchronous).  Scratch comes from a
 * fixed array of FLCE_NOALLOC_SCRATCH_BYTES in the library's device module,
 * held on every GPU that loads the library until the process exits.  Sizes
 * whose flce_workspace_size exceeds it are rejected with
 * FLCE_ERR_WORKSPACE_TOO_SMALL before anything runs; token rows are reordered
 * only when flce_workspace_size_reorder fits in it too.
 *
 * The first call on a device looks the array's device address up (a
 * cudaGetSymbolAddress, no allocation); make that first call before any stream
 * capture.  All calls share the one array and it keeps the last call's
 * contents; each call clears the words that must start at zero.  Calls that
 * overlap on the GPU (several streams or host threads at once) race on the
 * array and must be serialised by the caller. */
#define FLCE_NOALLOC_SCRATCH_BYTES (16u << 20)
flce_status_t flce_forward_backward_noalloc(const uint16_t* X, const uint16_t* W, const int32_t* y,
                                            int64_t N, int64_t H, int64_t V, int32_t ignore_index,
                                            float* loss, uint16_t* dX, uint16_t* dW,
                                            cudaStream_t stream);

/* Failure-detection probe.  Launches one thread that waits, each time for at
 * most timeout_ns, on an mbarrier phase that nobody completes and on a global
 * counter that nobody increments, with the same bounded-wait code the
 * kernels use.  d_status: DEVICE int32[3]; afterwards d_status[0] and
 * d_status[1] hold FLCE_ERR_TIMEOUT (the waits gave up instead of hanging)
 * and d_status[2] the untouched counter.  timeout_ns in (0, 1e10]. */
flce_status_t flce_probe_bounded_wait(int64_t timeout_ns, int32_t* d_status, cudaStream_t stream);

/* Failure-detection probe of the GEMM kernels' own waits.  Enqueues one call
 * with the arguments of flce_forward_backward_async, except that every dW
 * item of pass 2 waits for one more finished logit-gradient tile than the
 * queue produces, and every wait inside the kernels is bounded by timeout_ns
 * instead of 2 s.  The starved waits give up, the SM pairs wind down (both
 * CTAs of a pair together) and *d_status receives FLCE_ERR_TIMEOUT; the
 * loss, dX and dW are then undefined.  The device stays usable.
 * timeout_ns in (0, 1e10]. */
flce_status_t flce_probe_pass2_timeout(const uint16_t* X, const uint16_t* W, const int32_t* y,
                                       int64_t N, int64_t H, int64_t V, int32_t ignore_index,
                                       float* d_loss, int32_t* d_status, uint16_t* dX, uint16_t* dW,
                                       void* workspace, size_t workspace_bytes, int64_t timeout_ns,
                                       cudaStream_t stream);

/* Token-row order chosen by the last call that used `workspace` (see
 * "Ignored rows" above), read back once `stream` has finished that call:
 *   *reordered = 1 when the rows were reordered (valid rows first, X packed
 *                in that order, dX scattered back), 0 otherwise
 *   *n_valid   = the number of rows whose target is not ignore_index
 * Synchronises `stream`.  The workspace must be the 256-B aligned buffer the
 * call used; FLCE_ERR_INVALID_ARGUMENT for NULL or misaligned pointers.  The
 * pages describe no such query; it exposes the library's own choice. */
flce_status_t flce_row_order_info(const void* workspace, int32_t* reordered, int32_t* n_valid,
                                  cudaStream_t stream);

/* How a call of these sizes is split into launches (host-only query). */
typedef struct {
  int64_t workspace_bytes; /* same as flce_workspace_size */
  int64_t workspace_reorder_bytes; /* same as flce_workspace_size_reorder */
  int32_t vocab_chunk;     /* vocabulary entries per pass-2 chunk */
  int32_t num_chunks;      /* pass-2 chunks */
  int32_t lse_splits;      /* vocabulary splits of the pass-1 log-sum-exp */
  int32_t launches;        /* kernels launched by one device-buffer call on a
                              workspace of workspace_bytes (one more, the X row
                              packing, on one of workspace_reorder_bytes; the
                              host-buffer entry splits pass 1 per W piece and
                              pass 2 per section of chunks) */
  int32_t num_sms;         /* SMs the persistent kernels are sized for */
} flce_plan_t;
flce_status_t flce_plan(int64_t N, int64_t H, int64_t V, flce_plan_t* out);

/* Per-kernel timing.  While enabled, every launch of the library is bracketed
 * by CUDA events on its stream.  flce_profile_read waits for those events and
 * returns, per kernel kind, the number of launches and their summed device
 * time in milliseconds, then clears the record.  kinds: 0 pass-1 GEMM +
 * online log-sum-exp, 1 combine, 2 pass 2 (logit recompute + G, dW and dX
 * contractions of every vocabulary chunk, one persistent launch), 3 prep
 * (valid rows per 256-row token tile), 4 cross-entropy on given logits (rows
 * pass; its final sum is counted under kind 1), 5 token-row order (see
 * "Ignored rows"), 6 dX row scatter and 7 X row packing (both only do work
 * when the rows were reordered). */
#define FLCE_NUM_KERNEL_KINDS 8
const char* flce_kernel_name(int kind);
flce_status_t flce_profile_enable(int on);
flce_status_t flce_profile_read(int32_t* launches, double* total_ms);

/* Timeline of what the record holds, in the order it was recorded: the
 * launches (kinds as above) and, for the host-buffer entry
 * (flce_forward_backward_host), its copies: kind 8 host to device (X and y
 * on the caller's stream, each W piece on the copy stream), kind 9 device to
 * host (each section's dW rows on the copy stream, then dX and the loss on
 * the caller's stream); flce_kernel_name names them too.  Waits for the
 * recorded events and writes, for the first `capacity` intervals, kinds[i]
 * and their begin and end in milliseconds after the begin of the first
 * interval (HOST arrays of `capacity` entries); *count receives the number
 * recorded, which may exceed capacity.  Clears the record, as
 * flce_profile_read does.  FLCE_ERR_INVALID_ARGUMENT for a NULL pointer or a
 * negative capacity. */
#define FLCE_PROFILE_KIND_H2D 8
#define FLCE_PROFILE_KIND_D2H 9
flce_status_t flce_profile_timeline(int32_t* kinds, double* begin_ms, double* end_ms, int32_t capacity,
                                    int32_t* count);

#ifdef __cplusplus
}
#endif

#endif /* FLCE_H_ */
