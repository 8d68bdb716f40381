/*
 * haste.h -- C ABI of libhaste.so, a B200 (sm_100a) implementation of the HASTE
 * group-shared fixed fan-in output layer for extreme multi-label classification.
 *
 * Source of the operations: "HASTE: Hardware-Aware Dynamic Sparse Training for
 * Large Output Spaces" (summary page):
 *   Methodology 1, Group-Shared Fixed Fan-In Sparsity
 *     - structure: labels are partitioned into groups; all labels of a group share
 *       one sparse set of input-feature indices (the fan-in pattern) and keep
 *       independent weight vectors;
 *     - hardware alignment: a group's input features are gathered into shared
 *       memory once and reused by all labels of the group in a dense tensor-core
 *       product;
 *     - memory efficiency: indices are stored once per group.
 *   Methodology 2, Head-Tail Decomposition: a dense classifier for the few frequent
 *     (head) labels next to the sparse layer for the long tail.
 *
 * Notation: B batch rows, d input features, L tail labels in n_groups groups of G
 * (group g owns labels [g*G, g*G+G)), k fan-in per group, H head labels.
 *   idx [n_groups, k]  int32, each row strictly increasing in [0, d)
 *   X   [B, d]   W [L, k] (W[l, s] multiplies feature idx[l / G, s])
 *   logits, dY [B, L]   dW [L, k]   dX [B, d] (always fp32)
 *   Xh  [B, d]   Wh [H, d]   logits_h, dY_h [B, H]   dWh [H, d]   dXh [B, d] fp32
 * All matrices are contiguous and row-major.
 *
 * Conventions
 *   - Tensor pointers are DEVICE pointers unless a parameter says "host".  The
 *     caller owns every buffer it passes; the library owns only plan objects.
 *   - Workspace is caller-provided; query its size first.  The library keeps no
 *     pointer to it after the call's kernels finish.
 *   - Every compute call is asynchronous on the given stream (a cudaStream_t cast
 *     to void*, NULL = legacy default stream).  Argument errors are returned
 *     synchronously before any launch; launch failures return HASTE_ERR_CUDA.
 *     Nothing throws across the ABI.  haste_last_error() gives a message.
 *   - Device-side bounded waits that run out set a device error word instead of
 *     hanging; haste_device_status() synchronises and reports it.
 *   - Supported by the GPU path: k*elem % 128 == 0 (k % 64 for bf16, k % 32 for
 *     fp32), k <= 256, G % 16 == 0, 16 <= G <= 128, L*elem % 16 == 0, B <= 512;
 *     head: H*elem and d*elem multiples of 16 bytes.  Other shapes return
 *     HASTE_ERR_UNSUPPORTED_SHAPE.
 *   - Results are deterministic: repeated calls give identical bits (fixed-order
 *     reductions, no floating-point atomics).
 */
#ifndef HASTE_H
#define HASTE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct haste_plan_s* haste_plan_t; /* opaque; owned by the library */
typedef void* haste_stream_t;              /* a cudaStream_t */

typedef enum {
  HASTE_OK = 0,
  HASTE_ERR_INVALID_ARG = 1,
  HASTE_ERR_INDEX_UNSORTED_OR_DUP = 2,
  HASTE_ERR_INDEX_OUT_OF_RANGE = 3,
  HASTE_ERR_UNSUPPORTED_SHAPE = 4,
  HASTE_ERR_WORKSPACE = 5,
  HASTE_ERR_CUDA = 6,
  HASTE_ERR_TIMEOUT = 7
} haste_status_t;

typedef enum { HASTE_F32 = 0, HASTE_BF16 = 1 } haste_dtype_t;

/* Sparse positive labels per sample as a device CSR: row_ptr [B+1], ids [nnz],
 * ids branch-local (tail: global id minus H; head: global id), each row sorted
 * ascending without duplicates. */
typedef struct {
  const int32_t* row_ptr;
  const int32_t* ids;
} haste_targets_t;

/* ABI version of this header (bumped on incompatible change). */
int haste_abi_version(void);

/* Thread-local message of the last failing call ("" when none). */
const char* haste_last_error(void);

/* Synchronise the stream and report the device error word: HASTE_OK, or
 * HASTE_ERR_TIMEOUT if a kernel's bounded wait ran out (the word is then
 * cleared), or HASTE_ERR_CUDA. */
haste_status_t haste_device_status(haste_stream_t stream);

/* Self-test of failure detection: launches a kernel whose bounded wait (20 ms)
 * on a barrier that nothing releases runs out.  A following
 * haste_device_status() returns HASTE_ERR_TIMEOUT once, and the context stays
 * usable.  No GPU fault is involved. */
haste_status_t haste_selftest_wait_timeout(haste_stream_t stream);

/* Limit, in ns, of the waits between the warps of the pipelined kernels (a
 * producer waiting for a free ring stage, a consumer for a full one) on the
 * current device, for kernels launched after the call; 0 restores the default of
 * 2 s, larger values are refused (HASTE_ERR_INVALID_ARG).  A wait that runs out
 * sets the device error word and the kernel unwinds: its results are then
 * undefined and haste_device_status() returns HASTE_ERR_TIMEOUT.  Waits for a
 * kernel's own copies or MMAs in flight keep the 2 s limit, so that no kernel
 * exits while they can still write its memory.  Meant for failure-detection
 * tests (a very short limit forces the abort paths); not thread-safe against
 * concurrent launches. */
haste_status_t haste_set_wait_limit_ns(uint64_t ns);

/* Per-kernel timing without a profiler.  Between haste_profile_start() and
 * haste_profile_stop(), every kernel the library launches is bracketed by CUDA
 * events recorded on its launch stream.  haste_profile_stop() waits for those
 * events, writes up to max_entries aggregates {kernel name, launches, summed
 * milliseconds} (names are static strings) in order of first launch, turns
 * recording off and returns the number of distinct kernels (-1 on a CUDA error). */
typedef struct {
  const char* name;
  int32_t launches;
  double total_ms;
} haste_kernel_time_t;
haste_status_t haste_profile_start(void);
int32_t haste_profile_stop(haste_kernel_time_t* out, int32_t max_entries);

/* ------------------------------------------------------------------ plan --- */

/* Host-only core of the plan (no GPU needed): validates idx (host [n_groups*k])
 * and writes the inverse map feature -> (group, slot) into host buffers:
 * inv_off [d+1], inv_off[f] = number of entries whose feature is below f;
 * inv_ent [n_groups*k], the entries e = g*k + s of feature f in ascending g.
 * Validation: the first offending element in row-major order decides: out of
 * [0, d) -> HASTE_ERR_INDEX_OUT_OF_RANGE; not above its predecessor in the row
 * -> HASTE_ERR_INDEX_UNSORTED_OR_DUP.  Source: Methodology 1, structure (shared
 * index set per group) and memory efficiency (indices stored once per group). */
haste_status_t haste_plan_inverse_host(const int32_t* idx, int64_t n_groups, int32_t k, int32_t d,
                                       int32_t* inv_off, int32_t* inv_ent);

/* Build a plan: validate idx (host [n_groups*k]), copy it to the current device
 * and build the inverse map there (the stable counting sort described at
 * haste_plan_inverse_host, on the device; for d above about 57,000 features it
 * is built on the host and copied).  The call returns after the work completes.
 * *out receives the new plan, which belongs
 * to that device: calls made while another device is current are refused with
 * HASTE_ERR_INVALID_ARG.  Source: Methodology 1, structure (one index set I_g
 * shared by the G labels of a group) and memory efficiency (indices stored once
 * per group, not once per label). */
haste_status_t haste_plan(haste_plan_t* out, const int32_t* idx, int64_t n_groups, int32_t G, int32_t k,
                          int32_t d, haste_stream_t stream);

/* Rewire the fan-in sets of some groups, for dynamic sparse training (the
 * HASTE page's title: the index sets change during training; how they change is
 * the caller's rule): the index rows of the n_changed groups listed in groups
 * (host, ascending, distinct, in [0, n_groups)) become rows (host
 * [n_changed * k], each row strictly increasing in [0, d)), and the inverse map
 * is rebuilt on the device.  Only the changed rows cross PCIe.  Validation as
 * haste_plan (HASTE_ERR_INDEX_* for a bad row, HASTE_ERR_INVALID_ARG for bad
 * group ids) happens before anything changes.  The update is ordered on
 * `stream`: later calls on that stream see the new sets; work on other streams
 * that uses the plan must be ordered by the caller.  The host arrays may be
 * reused when the call returns.  A plan whose inverse map was built on the host
 * (very large d) returns HASTE_ERR_UNSUPPORTED_SHAPE.  n_changed = 0 is a no-op.
 * The weights of a rewired group keep their slots: the caller resets or carries
 * over W and dW rows of the changed groups as its rule says. */
haste_status_t haste_plan_update(haste_plan_t plan, const int32_t* groups, int64_t n_changed, const int32_t* rows,
                                 haste_stream_t stream);

/* Free a plan's device and host memory (synchronous).  NULL is accepted. */
haste_status_t haste_plan_destroy(haste_plan_t plan);

/* Index store of the plan: index_bytes = 4*n_groups*k (one int32 per group and
 * slot, against 4*L*k for per-label fan-in); inverse_bytes = 4*(d+1+n_groups*k).
 * Source: Methodology 1, memory efficiency (the saving of storing the fan-in
 * indices per group). */
haste_status_t haste_plan_info(haste_plan_t plan, int64_t* index_bytes, int64_t* inverse_bytes);

/* Copy the plan's DEVICE arrays back to host buffers (synchronous): idx
 * [n_groups*k], inv_off [d+1], inv_ent [n_groups*k].  Any pointer may be NULL.
 * For bit-exact checks of the plan (Methodology 1, structure and memory
 * efficiency). */
haste_status_t haste_plan_export(haste_plan_t plan, int32_t* idx, int32_t* inv_off, int32_t* inv_ent);

/* Workspace bytes that every sparse-tail call below needs at batch B (0 for a
 * NULL plan, B <= 0 or a plan of another device).  The workspace holds X^T, the
 * dX pass's partial sums and the fused step's gradient buffer: the staging that
 * Methodology 1's gather-once, dense-product scheme needs on this GPU. */
size_t haste_workspace_size(haste_plan_t plan, int32_t B, haste_dtype_t dtype);

/* ------------------------------------------------------------- sparse tail --- */

/* Forward: logits[b, g*G+j] = sum_s X[b, idx[g,s]] * W[g*G+j, s]  (fp32
 * accumulation on the tensor cores; logits in the input dtype).
 * Source: Methodology 1 (gather-once, dense tensor-core product per group). */
haste_status_t haste_forward(haste_plan_t plan, int32_t B, haste_dtype_t dtype, const void* X, const void* W,
                             void* logits, void* ws, size_t ws_bytes, haste_stream_t stream);

/* dW[g*G+j, s] = sum_b dY[b, g*G+j] * X[b, idx[g,s]], dW in the input dtype.
 * Source: Methodology 1 (the gathered inputs X[:, I_g] are shared by the G labels
 * of a group, so dW_g = dY_g^T . X[:, I_g] is one dense product per group) and
 * Experimental results (the backward pass's speed-up over per-label fan-in). */
haste_status_t haste_backward_dw(haste_plan_t plan, int32_t B, haste_dtype_t dtype, const void* X,
                                 const void* dY, void* dW, void* ws, size_t ws_bytes, haste_stream_t stream);

/* dX[b, f] (+)= sum over the (g, s) with idx[g,s] == f, in ascending g, of
 * sum_j dY[b, g*G+j] * W[g*G+j, s]; fp32 output.  accumulate = 0 overwrites dX,
 * 1 adds into it.  Features in no group receive exactly 0.  Source: Methodology 1
 * (a group's G labels scatter into the same k features I_g, so its contribution
 * dY_g . W_g lands in dX[:, I_g]) and Experimental results (backward speed-up). */
haste_status_t haste_backward_dx(haste_plan_t plan, int32_t B, haste_dtype_t dtype, const void* W,
                                 const void* dY, float* dX, int accumulate, void* ws, size_t ws_bytes,
                                 haste_stream_t stream);

/* dX like haste_backward_dx, for callers that must not allocate device memory:
 * no workspace argument, and the call makes no cudaMalloc, cudaFree or other
 * allocating call.  Such callers include code running under a framework whose
 * caching allocator has reserved the device memory (a raw cudaMalloc can fail or
 * fragment that pool), hooks that run inside another library's call path, and
 * loops that are not allowed to allocate at all.  The paper has no counterpart;
 * this is a deployment variant of the dX reduction.
 *   Scratch: a file-scope static device array of 16 MiB (16777216 bytes) holds
 *   the reduction's per-chunk partials; every GPU that loads the library keeps it
 *   until the process exits.  The partials are fully rewritten by each call, so
 *   nothing in it needs clearing.  All calls share this one array: calls whose
 *   kernels overlap on the GPU (other streams, other host threads) race on it and
 *   give wrong results; serialise them.
 *   Limit: d * roundup(B, 128) * 4 must not exceed 16 MiB (one chunk of
 *   partials); larger shapes return HASTE_ERR_UNSUPPORTED_SHAPE with a message.
 *   Fewer group chunks may be used than in haste_backward_dx, so the two can
 *   differ in the rounding of the chunk sums (both are deterministic).
 *   Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call before
 *   any stream capture. */
haste_status_t haste_backward_dx_noalloc(haste_plan_t plan, int32_t B, haste_dtype_t dtype, const void* W,
                                         const void* dY, float* dX, int accumulate, haste_stream_t stream);

/* Fused tail training step (logits never reach global memory), the forward and
 * backward of Methodology 1 with the loss in between (Experimental results: the
 * forward and backward speed-ups, and the training-memory saving):
 *   z = forward(X, W);  y[b,l] = 1 iff l is in tail_pos row b;
 *   dY = grad_scale * (sigmoid(z) - y)   (rounded to the input dtype);
 *   *loss = grad_scale * sum_{b,l} (softplus(z) - z*y)   (if loss != NULL, device fp32);
 *   dW from dY as haste_backward_dw; dX (+)= from dY as haste_backward_dx.
 * The loss is binary cross-entropy with logits summed over labels; grad_scale is
 * normally 1/B.  (The page names no loss; BCE against sparse positives is this
 * library's reading of the multi-label problem statement.) */
haste_status_t haste_bce_step(haste_plan_t plan, int32_t B, haste_dtype_t dtype, const void* X, const void* W,
                              haste_targets_t tail_pos, float grad_scale, float* loss, void* dW, float* dX,
                              int accumulate, void* ws, size_t ws_bytes, haste_stream_t stream);

/* Fused tail training step with the optimizer update fused into it: as
 * haste_bce_step, but instead of writing dW the step kernel updates each group's
 * weights while its dW is still on chip (SGD with heavy-ball momentum):
 *   M' = momentum * M + dW   (M' = dW when momentum == 0),
 *   W_out = W - lr * M'.
 * W is read, not written: the dX pass of the same call still needs it, so W_out
 * must be a different buffer (callers alternate two weight buffers).  M [L, k]
 * holds the momentum in W's dtype and is updated in place; it may be NULL when
 * momentum == 0; start it at zero.  dX and the loss are those of haste_bce_step
 * (computed with W).  Compared with haste_bce_step followed by a separate
 * update, the dW write and the update pass's reads of W and dW never happen.
 * Supported: bf16, G in {16, 32, 64}, k in {64, 128}, B <= 256; other shapes
 * return HASTE_ERR_UNSUPPORTED_SHAPE.  Source: Methodology 1 (the per-group dW
 * product) and the training loop of Experimental results (training memory);
 * the page names no optimizer, plain SGD with momentum is this library's
 * choice. */
haste_status_t haste_bce_step_sgd(haste_plan_t plan, int32_t B, haste_dtype_t dtype, const void* X, const void* W,
                                  haste_targets_t tail_pos, float grad_scale, float* loss, float lr, float momentum,
                                  void* M, void* W_out, float* dX, int accumulate, void* ws, size_t ws_bytes,
                                  haste_stream_t stream);

/* ----------------------------------------------------- top-k scoring --- */

/* Workspace bytes of haste_topk at (B, n_buckets, kp). */
size_t haste_topk_workspace_size(haste_plan_t plan, int32_t B, haste_dtype_t dtype, int32_t n_buckets, int32_t kp);

/* Two-stage top-k scoring of the tail logits, for inference (P@k).
 * Scores: logits[b, l] = X[b, I_g] . W[l, :] as haste_forward (Methodology 1 of
 * the HASTE summary page); they are ranked inside the forward epilogue and never
 * written to memory.  Selection: "A Faster Generalized Two-Stage Approximate
 * Top-K" (summary page, Methodology): stage 1 splits the labels into n_buckets
 * buckets of whole groups, bucket j = the labels of groups
 * [j*n_groups/n_buckets, (j+1)*n_groups/n_buckets), and keeps the kp best logits
 * of each bucket per sample; stage 2 returns the k best of the n_buckets*kp
 * survivors.  kp = k gives the exact top k; kp < k may miss labels that share a
 * bucket with kp better ones.  Rank order: larger logit first, equal logits by
 * smaller label id.
 *   X        device [B, d] bf16;  W device [L, k] bf16
 *   out_val  device [B, k] fp32, rank order;  out_id device [B, k] int32 tail ids
 * Supported: bf16, G in {16, 32, 64}, k of the plan in {64, 128}, B <= 256,
 * kp in {1, 2, 4, 8}, 1 <= n_buckets <= n_groups, 1 <= k <= min(64, n_buckets*kp).
 * Other arguments return HASTE_ERR_INVALID_ARG or HASTE_ERR_UNSUPPORTED_SHAPE.
 * Stage 1 runs one CTA per bucket (n_buckets = the number of SMs uses the whole
 * GPU).  The dense head's logits are not included. */
haste_status_t haste_topk(haste_plan_t plan, int32_t B, haste_dtype_t dtype, const void* X, const void* W,
                          int32_t k, int32_t kp, int32_t n_buckets, float* out_val, int32_t* out_id, void* ws,
                          size_t ws_bytes, haste_stream_t stream);

/* -------------------------------------------------------------- dense head --- */

/* Workspace bytes of the head calls at (B, H, d). */
size_t haste_head_workspace_size(int32_t B, int32_t H, int32_t d, haste_dtype_t dtype);

/* logits_h = Xh . Wh^T.  pos == NULL: logits_or_dY receives the logits.
 * pos != NULL: it receives dY_h = grad_scale * (sigmoid(z) - y) and, if loss !=
 * NULL, *loss = grad_scale * sum BCE (device fp32).  Source: Methodology 2. */
haste_status_t haste_head_forward(int32_t B, int32_t H, int32_t d, haste_dtype_t dtype, const void* Xh,
                                  const void* Wh, void* logits_or_dY, const haste_targets_t* pos, float grad_scale,
                                  float* loss, void* ws, size_t ws_bytes, haste_stream_t stream);

/* dWh = dY_h^T . Xh (input dtype) and dXh = dY_h . Wh (fp32). */
haste_status_t haste_head_backward(int32_t B, int32_t H, int32_t d, haste_dtype_t dtype, const void* Xh,
                                   const void* Wh, const void* dY_h, void* dWh, float* dXh, void* ws,
                                   size_t ws_bytes, haste_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HASTE_H */
