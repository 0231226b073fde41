/*
 * moe.h -- C ABI of libmoe: the Mixtral top-2-of-8 sparse-MoE SwiGLU feed-forward
 * layer on one NVIDIA B200 (sm_100a).
 *
 * The layer (notion notes "Mixtral of Experts", "Sparse gating" eq. G(x) and
 * "Implementation" eq. y; crackai "Mixtral of Experts", "Top-2 Routing in Detail"):
 *     l      = x . W_g                              router logits, [T, E]
 *     G(x)   = Softmax(TopK(l)), K = 2              logits outside the top 2 -> -inf
 *     E_e(x) = W2[e] (silu(W1[e] x) * (W3[e] x))    SwiGLU expert (atlas "Mixtral",
 *                                                   "Design overview": inner dim h)
 *     y      = sum_e G(x)_e E_e(x) = w1 E_{i1}(x) + w2 E_{i2}(x)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Ownership: the caller owns every buffer.  The library never allocates, frees
 *   or synchronises on these calls; all scratch lives in the caller's workspace.
 *   All entry points are stateless and may be called from several host threads.
 * - Pointers are DEVICE pointers (cudaMalloc or equivalent) unless stated
 *   otherwise, 16-byte aligned, tensors dense and row-major.  Outputs must not
 *   alias inputs.  Every pointer must belong to the device current on the calling
 *   thread, and `stream` to that device: the kernels launch on the current device.
 * - Execution: work is queued on `stream` and runs asynchronously.  Argument
 *   errors are returned before anything is queued.  A failed launch returns
 *   MOE_ERR_CUDA.  Errors found on the device (a pipeline wait that ran out of
 *   time) are recorded in the workspace status word; read it with
 *   moe_device_status().
 * - dtype: MOE_BF16 (bfloat16 activations and weights, fp32 accumulation on tensor
 *   cores) or MOE_F32 (fp32 everywhere, CUDA cores, no TF32).
 * - Supported shapes: k == 2; 2 <= E <= 32 (moe_expert_ffn, which routes nothing,
 *   also takes E == 1); d and h multiples of 8; T >= 0 (T == 0 is a no-op returning
 *   MOE_OK); T <= 2^29, and E*d, E*h below 2^31 (32-bit row coordinates).  Inputs
 *   must be finite.
 * - Routing: experts are ranked by (logit descending, index ascending), so ties go
 *   to the lower index; logits are accumulated in fp64 from the exact products of
 *   the inputs.  Slot 0 holds the larger logit.  w1 = 1/(1+exp(l_i2-l_i1)) is
 *   computed in fp64 and rounded once to float; w2 = 1 - w1 in float.
 * - Grouping: the (token, slot) pairs are stably sorted by expert over the
 *   flattened index f = t*k + j; group e owns rows offsets[e] .. offsets[e+1]-1 in
 *   ascending token order.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative or inconsistent size */
    MOE_ERR_UNSUPPORTED = 2, /* k != 2, E outside [2, 32], d or h not a multiple of 8 */
    MOE_ERR_WORKSPACE = 3,   /* ws_bytes smaller than moe_workspace_bytes() */
    MOE_ERR_CUDA = 4,        /* a CUDA call or kernel launch failed */
    MOE_ERR_TIMEOUT = 5      /* a device-side pipeline wait gave up (moe_device_status) */
} moe_status;

/* Device status flags, OR-ed into the workspace status word. */
#define MOE_DEV_FLAG_TIMEOUT 0x1u

/* Bytes of workspace that moe_layer_forward needs for this shape (a 1 KiB-aligned
 * layout of routing results, permutation, gathered rows x_perm, the SwiGLU
 * activations H, the fp32 expert outputs and, for batches of at most 128 tokens, the
 * fp32 partial sums of the split-K down projection).  It also covers moe_permute and
 * moe_expert_ffn.  The size never decreases with T: a workspace sized for T serves
 * every batch of at most T tokens (same d, h, E, k, dt).  Zero the workspace once
 * before its first use: it holds a status word and dependency counters that every
 * completed call leaves at zero.  After a call that ended in MOE_ERR_TIMEOUT (or set
 * MOE_DEV_FLAG_TIMEOUT), the counters may be left non-zero: zero the whole
 * workspace again before reusing it.  Returns 0 for unsupported arguments. */
size_t moe_workspace_bytes(int T, int d, int h, int E, int k, moe_dtype dt);

/* Router + top-2 + softmax of the two kept logits.
 * crackai "Mixtral of Experts", "Top-2 Routing in Detail" (gate_logits = x . W_gate);
 * notion notes, "Sparse gating" eq. G(x).
 *   x        [T, d]  dt          tokens
 *   Wg       [d, E]  dt          router weights
 *   topk_idx [T, k]  int32 out   chosen experts, slot 0 = larger logit
 *   topk_w   [T, k]  float out   their gate weights (sum exactly 1 in float) */
moe_status moe_route(const void *x, const void *Wg, int T, int d, int E, int k,
                     moe_dtype dt, int32_t *topk_idx, float *topk_w,
                     cudaStream_t stream);

/* Group token rows by expert: histogram, exclusive scan, stable ranks, row gather.
 * ml-canon "52 Mixtral", "Questions worth asking" (gather and scatter tokens);
 * notion notes, "Expert Parallelism" (outputs returned to the token's location).
 *   topk_idx   [T, k]     int32 in
 *   x          [T, d]     dt in
 *   offsets    [E + 1]    int32 out   group e = rows offsets[e] .. offsets[e+1]-1
 *   perm_token [T*k]      int32 out   source token of each grouped row
 *   inv_perm   [T, k]     int32 out   grouped row holding pair (t, j)
 *   x_perm     [T*k, d]   dt out      x_perm[r] = x[perm_token[r]]
 *   ws, ws_bytes                       workspace (>= moe_workspace_bytes)
 * topk_idx entries must lie in [0, E) and differ within a token. */
moe_status moe_permute(const int32_t *topk_idx, const void *x, int T, int d, int E,
                       int k, moe_dtype dt, int32_t *offsets, int32_t *perm_token,
                       int32_t *inv_perm, void *x_perm, void *ws, size_t ws_bytes,
                       cudaStream_t stream);

/* Per-expert SwiGLU FFN over the grouped rows (notion notes, "Implementation":
 * SwiGLU expert function; atlas "Mixtral", "Design overview").
 *   x_perm  [rows, d]   dt in        rows grouped by expert
 *   offsets [E + 1]     int32 in     device copy; offsets[E] must equal rows
 *   W1, W3  [E, h, d]   dt in        gate and up projections (d contiguous)
 *   W2      [E, d, h]   dt in        down projection (h contiguous)
 *   y_perm  [rows, d]   float out    Y_r = W2[e](silu(W1[e] x_r) * W3[e] x_r)
 *   ws, ws_bytes                      workspace (holds H [rows, h])
 * bf16 runs on tcgen05 tensor cores (fp32 accumulation in tensor memory; H is
 * rounded once to bf16); f32 runs on CUDA cores in fp32.  rows must be even (pad with
 * a row outside every group; output rows outside every group are unspecified);
 * 1 <= E <= 32.  ws_bytes: at least moe_workspace_bytes(rows / 2, d, h, max(E, 2), 2,
 * dt). */
moe_status moe_expert_ffn(const void *x_perm, const int32_t *offsets, const void *W1,
                          const void *W3, const void *W2, int rows, int d, int h,
                          int E, moe_dtype dt, float *y_perm, void *ws,
                          size_t ws_bytes, cudaStream_t stream);

/* Weighted un-permute: y[t] = w[t,0] Y[inv[t,0]] + w[t,1] Y[inv[t,1]] in fp32,
 * rounded once to dt.  crackai "Mixtral of Experts", "Top-2 Routing in Detail"
 * (y = w_1 Expert_{i1}(x) + w_2 Expert_{i2}(x)); notion notes, eq. y.
 *   y_perm   [T*k, d] float in;  inv_perm [T, k] int32 in;  topk_w [T, k] float in
 *   y        [T, d]   dt out */
moe_status moe_combine(const float *y_perm, const int32_t *inv_perm,
                       const float *topk_w, int T, int d, int k, moe_dtype dt, void *y,
                       cudaStream_t stream);

/* moe_expert_ffn for callers that cannot allocate device memory -- for example an
 * op inside an inference engine that owns all device allocations and gives its
 * ops no allocator, or a serving loop that must not allocate once it is running.
 * It takes no workspace: its scratch (the SwiGLU activations H [rows, h] and a
 * status word) lives in a library-owned __device__ array of
 * MOE_STATIC_SCRATCH_BYTES bytes that every GPU loading the library keeps until
 * the process exits.  No counterpart in the paper: it exists only for such callers.
 *   Arguments, layouts and results are those of moe_expert_ffn, minus ws/ws_bytes.
 *   Limit: rows * h * sizeof(dt) <= MOE_STATIC_SCRATCH_BYTES - 256, else
 *   MOE_ERR_WORKSPACE is returned and nothing is queued (8 MiB: 292 grouped rows
 *   of a bf16 Mixtral expert with h = 14336, i.e. up to 146 tokens).
 *   The first call on a device, with that device current, looks up the array's
 *   device address (cudaGetSymbolAddress) and caches it; make that first call
 *   before any stream capture on the device.  The cached address belongs to the
 *   device's primary context: after cudaDeviceReset it is stale, so do not call
 *   this entry point on a device that the process has reset.
 *   Device-side wait timeouts set a status word inside the library's array, which
 *   no caller can read: they are reported (as MOE_ERR_TIMEOUT) only when the
 *   MOE_DEBUG_SYNC=1 setting makes each call synchronise and check that word.
 *   All calls share the one array, which keeps the previous call's contents; each
 *   call clears the status word itself.  Calls whose work overlaps on the GPU
 *   (other streams, other threads) race on the array: serialise them.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
#define MOE_STATIC_SCRATCH_BYTES ((size_t)8 << 20)
moe_status moe_expert_ffn_static(const void *x_perm, const int32_t *offsets,
                                 const void *W1, const void *W3, const void *W2, int rows,
                                 int d, int h, int E, moe_dtype dt, float *y_perm,
                                 cudaStream_t stream);

/* The whole layer: route -> permute -> expert FFN -> combine, queued on `stream`
 * with no host synchronisation (group sizes stay on the device).
 *   x [T, d], Wg [d, E], W1/W3 [E, h, d], W2 [E, d, h] in dt;  y [T, d] out in dt. */
moe_status moe_layer_forward(const void *x, const void *Wg, const void *W1,
                             const void *W3, const void *W2, int T, int d, int h,
                             int E, int k, moe_dtype dt, void *y, void *ws,
                             size_t ws_bytes, cudaStream_t stream);

/* The layer with an opt-in per-expert capacity (token dropping).  ml-canon "52
 * Mixtral", "Questions worth asking": a capacity factor caps the tokens each expert
 * takes.  Each expert keeps the first `capacity` of its (token, slot) pairs in the
 * grouping order (ascending token, then slot); a dropped pair's expert output is
 * not computed and contributes nothing to y, and the other gate weight of that
 * token is not renormalised.  capacity < 0 means no limit (= moe_layer_forward); a
 * capacity factor f corresponds to capacity = ceil(f * T * k / E).  Other
 * arguments as moe_layer_forward. */
moe_status moe_layer_forward_capacity(const void *x, const void *Wg, const void *W1,
                                      const void *W3, const void *W2, int T, int d, int h,
                                      int E, int k, moe_dtype dt, int capacity, void *y,
                                      void *ws, size_t ws_bytes, cudaStream_t stream);

/* moe_layer_forward that also records up to five caller-created events on `stream`
 * between its stages, for timing them without a profiler:
 *   events[0] before the router, events[1] after the permutation (before the
 *   expert FFN), events[2] after the first FFN kernel (GEMM1 + SwiGLU; for batches
 *   of at most 128 tokens, where one fused kernel runs both GEMMs, after it),
 *   events[3] after the expert FFN, events[4] after the combine.
 * n_events may be 0..5; events beyond n_events, and null handles, are not recorded. */
moe_status moe_layer_forward_events(const void *x, const void *Wg, const void *W1,
                                    const void *W3, const void *W2, int T, int d, int h,
                                    int E, int k, moe_dtype dt, void *y, void *ws,
                                    size_t ws_bytes, cudaEvent_t *events, int n_events,
                                    cudaStream_t stream);

/* Synchronise `stream`, read the workspace status word into *flags (host
 * pointer; MOE_DEV_FLAG_* bits), then clear it.  Returns MOE_ERR_TIMEOUT if the
 * timeout flag was set, MOE_OK otherwise.  Diagnostic call: it synchronises.  After
 * a timeout, zero the whole workspace before its next use (the dependency counters
 * of an interrupted call may be non-zero). */
moe_status moe_device_status(void *ws, size_t ws_bytes, uint32_t *flags,
                             cudaStream_t stream);

/* Self-test of the device-side failure detection (no counterpart in the paper; it
 * checks this library's safety mechanism).  Runs, on `stream`, the same bounded
 * waits the pipelines use -- an mbarrier wait and a device-counter wait -- against
 * a barrier and a counter that nothing completes, with a limit of `limit_seconds`
 * (0 < limit <= 10).  Both waits must give up: outcome[0] (barrier) and outcome[1]
 * (counter) are set to 2 ("gave up") or 1 ("completed", a failure of the test), and
 * MOE_DEV_FLAG_TIMEOUT is raised in the workspace status word, where
 * moe_device_status() reports it.  Nothing hangs, traps or faults; the context
 * stays usable.  Synchronises `stream`.  ws: a workspace of >= 2 KiB (as from
 * moe_workspace_bytes); outcome: host array of 2. */
moe_status moe_selftest_wait_timeout(void *ws, size_t ws_bytes, double limit_seconds,
                                     uint32_t *outcome, cudaStream_t stream);

/* Bytes of backward workspace moe_layer_backward needs for these sizes (0 for an
 * unsupported shape: the backward pass is built for bf16 layers with h % 64 == 0).
 * It includes 2 * (2T) * h fp32 values for the pre-activations moe_layer_forward_train
 * keeps. */
size_t moe_backward_workspace_bytes(int T, int d, int h, int E, int k, moe_dtype dt);

/* moe_layer_forward for training: the same layer, the same y and forward workspace,
 * and in addition the pre-activations a = x W1_e^T and b = x W3_e^T of every grouped
 * row kept in fp32 in bwd_ws (the GEMM1 epilogue writes them next to H).  A
 * moe_layer_backward call with the same fwd_ws and bwd_ws (and capacity < 0) then
 * computes du and dv from them element by element instead of recomputing a and b with
 * a second GEMM1.  From T = 512 on the backward's recompute runs the same GEMM as the
 * forward, so the gradients are bit-identical to the recomputing path by construction;
 * below, a and b come from the forward's own kernels (weight streaming up to 128
 * tokens, single-SM tiles above), which sum over d in the same 16-wide tensor-core
 * steps and the same order as the backward's recompute (bit-identical gradients in
 * every case measured on B200), though the two are separate kernels and only rounding
 * (fp32 accumulation, then a bf16 store of du and dv) could tell them apart.  Any later
 * forward call on fwd_ws
 * (moe_layer_forward), and the two-launch small-batch form this call falls back to on
 * a device that cannot co-schedule the fused launch, record that nothing was kept, and
 * the backward recomputes.  Costs 4 * (2T) * h * 2 bytes of extra writes in the
 * forward.  dt must be MOE_BF16 and h % 64 == 0 (MOE_ERR_UNSUPPORTED otherwise);
 * bwd_ws_bytes >= moe_backward_workspace_bytes (MOE_ERR_WORKSPACE otherwise).  T == 0
 * queues nothing and returns MOE_OK. */
moe_status moe_layer_forward_train(const void *x, const void *Wg, const void *W1,
                                   const void *W3, const void *W2, int T, int d, int h, int E,
                                   int k, moe_dtype dt, void *y, void *ws, size_t ws_bytes,
                                   void *bwd_ws, size_t bwd_ws_bytes, cudaStream_t stream);

/* Gradients of the layer, for training.  crackai "Mixtral of Experts", "Key
 * Takeaways": routing is learned jointly with the model.  The pages print no backward
 * formulas; this is the exact derivative of moe_layer_forward (or, with capacity >= 0,
 * moe_layer_forward_capacity) with the top-2 choice held fixed: for an upstream
 * gradient dy of L with respect to y it returns dL/dx, dL/dWg, dL/dW1, dL/dW3 and
 * dL/dW2.  The gate weights w1 = sigma(l_i1 - l_i2), w2 = 1 - w1 pass the gradient
 * to the two chosen logits only; a pair dropped by the capacity passes nothing.
 *
 * Arguments: x, Wg, W1, W3, W2 and T, d, h, E, k, dt exactly as given to the forward
 * call; dy bf16 [T, d].  fwd_ws: the workspace of that forward call, unchanged since
 * (it holds the routing, the permutation, the gathered rows, H and the expert
 * outputs).  Outputs (caller-owned, device): dx bf16 [T, d]; dWg, dW1, dW3, dW2 fp32
 * with the shapes of Wg [d, E], W1/W3 [E, h, d] and W2 [E, d, h] (overwritten, not
 * accumulated; an expert that received no rows gets zeros).  bwd_ws: device scratch
 * of moe_backward_workspace_bytes bytes; its status word (offset 0) collects device
 * flags like the forward's.  Only dt == MOE_BF16 and h % 64 == 0 are supported
 * (MOE_ERR_UNSUPPORTED otherwise).  Queued on `stream`; argument errors return before
 * anything is queued. */
moe_status moe_layer_backward(const void *x, const void *Wg, const void *W1, const void *W3,
                              const void *W2, const void *dy, int T, int d, int h, int E, int k,
                              moe_dtype dt, int capacity, void *dx, float *dWg, float *dW1,
                              float *dW3, float *dW2, const void *fwd_ws, size_t fwd_ws_bytes,
                              void *bwd_ws, size_t bwd_ws_bytes, cudaStream_t stream);

/* moe_layer_backward with caller-created events recorded on `stream` before its first
 * launch and after each stage: [0] start, [1] dY/dw/logit gradients, [2] dH, [3] du/dv,
 * [4] dX, [5] dx, [6] dW2, [7] dW1/dW3, [8] dWg.  Null handles (or n_events <= i) are
 * skipped.  For timing the stages (bench.py). */
moe_status moe_layer_backward_events(const void *x, const void *Wg, const void *W1,
                                     const void *W3, const void *W2, const void *dy, int T, int d,
                                     int h, int E, int k, moe_dtype dt, int capacity, void *dx,
                                     float *dWg, float *dW1, float *dW3, float *dW2,
                                     const void *fwd_ws, size_t fwd_ws_bytes, void *bwd_ws,
                                     size_t bwd_ws_bytes, cudaEvent_t *events, int n_events,
                                     cudaStream_t stream);

/* Static description of a status code. */
const char *moe_status_string(moe_status st);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
