/*
 * lags.h - C ABI of the B200 LAGS sparsification library (liblags.so).
 *
 * The operation is the data-parallel hot path of LAGS-SGD, as described by
 * "Layer-wise Adaptive Gradient Sparsification for Distributed Deep Learning
 * with Convergence Guarantees" (nubint.ai review; abstract and section
 * "proposed method"): every worker, for every layer independently, adds its
 * error-compensation residual to the scaled gradient, keeps the k entries of
 * largest magnitude of that layer, sends them as (index, value) pairs and
 * keeps the remainder as its next residual; the workers' sparse sets are then
 * summed into the averaged dense update of sparsified synchronous SGD, which
 * is applied to the weights.
 *
 * Exact arithmetic (the pages give no formula; these are the readings the
 * library implements and tests bit for bit against its CPU oracle):
 *   acc_i      = fl32(residual_i + fl32(lr * grad_i))         (two roundings)
 *   k_l        = min(d_l, max(1, ceil(fl64(rho_l * d_l))))   (rho_l a double)
 *   selection  = the k_l largest |acc| of the layer; equal magnitudes are
 *                ordered by the lower index; +0 and -0 tie; +-inf are largest
 *   picks      = (global index, acc) of the selected entries, ascending index
 *   residual_i = +0.0f where picked, acc_i elsewhere
 *   dense_j    = fl32( (((+0 + v_0j) + v_1j) + ... + v_(P-1)j) / P ), workers
 *                in order 0..P-1, absent picks contributing nothing
 *   weights_j  = fl32(weights_j - dense_j)
 * NaN inputs are not supported (a NaN magnitude orders above +inf).
 *
 * Conventions shared by every call:
 *   - "device" pointers are CUDA device memory of the current device; "host"
 *     pointers are ordinary host memory read during the call only.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every compute call only enqueues work on that stream: it never
 *     allocates, never synchronises and returns before the work runs.  Work on
 *     one plan must be issued in stream order (one stream, or events).
 *   - Argument errors are reported by the return value before anything is
 *     enqueued.  Errors a kernel detects are recorded in the plan's device
 *     status word and read with lags_status_poll().
 *   - The library owns only the plan's host-side tables.  All device memory
 *     (inputs, outputs and the plan workspace) belongs to the caller.
 */
#ifndef LAGS_H
#define LAGS_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LAGS_API __attribute__((visibility("default")))
#else
#define LAGS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct lags_plan lags_plan; /* opaque; created and destroyed by the caller */

typedef enum {
  LAGS_OK = 0,
  LAGS_ERR_INVALID_ARG = 1,        /* null pointer, size or count out of range */
  LAGS_ERR_ALIGNMENT = 2,          /* a device pointer is not aligned as required */
  LAGS_ERR_CUDA = 3,               /* a CUDA runtime call or launch failed */
  LAGS_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not sm_100 (B200) */
  LAGS_ERR_WORKSPACE = 5,          /* workspace missing or smaller than required */
  LAGS_ERR_BAD_PICKS = 6,          /* (status word) pick lists not ascending/in layer */
  LAGS_ERR_TIMEOUT = 7,            /* (status word) a kernel's bounded wait gave up */
  LAGS_ERR_INTERNAL = 8,           /* (status word) a kernel failed a self-check */
  LAGS_ERR_WRONG_DEVICE = 9        /* the current device is not the plan's */
} lags_status;

/* Largest number of simulated workers one plan accepts. */
#define LAGS_MAX_WORKERS 256

/* Largest N (elements per worker buffer) a plan accepts: indices are uint32,
 * and the kernels' index arithmetic (a tile's 16-byte groups, a grid's
 * threads past the end) stays below 2^32 with this much headroom. */
#define LAGS_MAX_ELEMENTS 4294901760ull /* 2^32 - 65536 */

/* Bits of the device status word returned by lags_status_poll(). */
#define LAGS_FLAG_BAD_PICKS 0x1u /* lags_aggregate saw an unsorted or out-of-layer index */
#define LAGS_FLAG_TIMEOUT 0x4u   /* the selection's bounded wait on its own bulk copies gave
                                    up; the selection then read its candidates from global
                                    memory, and its picks may be incomplete */
#define LAGS_FLAG_INTERNAL 0x2u  /* a selection kernel failed a self-check (a library bug);
                                    the write it guarded was skipped */

/*
 * lags_plan_create - describe one flattened gradient buffer.
 *   layer_sizes  host, [num_layers] int64: d_l > 0, layers stored back to back
 *                in this order; N = sum d_l must be <= LAGS_MAX_ELEMENTS.
 *   densities    host, [num_layers] double: rho_l in (0, 1]; k_l follows the
 *                rule above (rho_l = 1 or k_l = d_l sends the layer densely).
 *   num_workers  P, 1 <= P <= LAGS_MAX_WORKERS.
 *   out_plan     host, receives the plan.
 * Host only: computes k_l, the layer and tile tables and the workspace size.
 * Returns LAGS_ERR_INVALID_ARG on any bad argument (nothing is created).
 */
LAGS_API lags_status lags_plan_create(const int64_t* layer_sizes, const double* densities,
                             int32_t num_layers, int32_t num_workers, lags_plan** out_plan);

/*
 * lags_plan_create_range - a plan for layers [layer_begin, layer_end) of the
 * model that layer_sizes/densities describe (all num_layers of them), for
 * layer-wise pipelining: LAGS ("Layer-wise Adaptive Gradient Sparsification
 * ..." review, "proposed method") sparsifies and sends each layer as soon as
 * the backward pass has produced it, instead of after the whole pass.
 *   - Element indices stay those of the whole model: grads, residuals,
 *     dense_out and weights are the whole model's buffers and the emitted
 *     indices are global.  Calls on the plan read and write only the range's
 *     elements [offset of layer_begin, N) and its own pick lists.
 *   - The plan's layers are numbered from 0 (= model layer layer_begin) in
 *     lags_plan_layer; its pick lists are [P][K] with K the range's picks.
 *   - lags_plan_info reports N = one past the range's last element (buffers
 *     must hold at least N elements) and that K.
 *   - Each layer is selected, aggregated and applied exactly as by a plan of
 *     the whole model, so the plans of a partition of the layers together
 *     give bit for bit the results of one whole-model plan.
 * Other arguments and errors as lags_plan_create; also LAGS_ERR_INVALID_ARG
 * unless 0 <= layer_begin < layer_end <= num_layers.
 */
LAGS_API lags_status lags_plan_create_range(const int64_t* layer_sizes, const double* densities,
                                            int32_t num_layers, int32_t num_workers,
                                            int32_t layer_begin, int32_t layer_end,
                                            lags_plan** out_plan);

/* Frees the host tables.  The workspace stays the caller's. */
LAGS_API lags_status lags_plan_destroy(lags_plan* plan);

/*
 * lags_plan_info - sizes of the plan (any output pointer may be NULL).
 *   N                elements per worker buffer
 *   K                picks per worker (sum of k_l); out_idx/out_val are [P][K]
 *   workspace_bytes  device bytes lags_plan_set_workspace() needs
 */
LAGS_API lags_status lags_plan_info(const lags_plan* plan, int64_t* N, int64_t* K,
                           size_t* workspace_bytes);

/*
 * lags_plan_aggregate_workspace_bytes - the smaller workspace that serves a
 * plan used only to aggregate (lags_aggregate, lags_aggregate_apply,
 * lags_status_poll), e.g. the job-wide plan of a data-parallel rank that
 * sparsifies its own workers with another plan.  It leaves out the selection's
 * candidate slots, most of the full workspace.  Host only.
 *   bytes  host, receives the size (<= workspace_bytes of lags_plan_info).
 */
LAGS_API lags_status lags_plan_aggregate_workspace_bytes(const lags_plan* plan, size_t* bytes);

/*
 * lags_plan_layer - placement of layer l: its first element in a worker buffer
 * (offset), its pick count k_l and the first slot of its picks in a worker's
 * pick list (pick_offset).  Picks of layer l occupy
 * out[p*K + pick_offset .. p*K + pick_offset + k_l).
 */
LAGS_API lags_status lags_plan_layer(const lags_plan* plan, int32_t l, int64_t* offset, int64_t* k,
                            int64_t* pick_offset);

/*
 * lags_plan_set_workspace - bind caller-owned device memory to the plan and
 * upload the plan's tables into it (enqueued on `stream`; the host tables are
 * owned by the plan, so nothing has to outlive the call on the caller side).
 *   workspace  device, 256-byte aligned, >= workspace_bytes of lags_plan_info
 *              (full plan), or >= lags_plan_aggregate_workspace_bytes (the plan
 *              then only aggregates: lags_sparsify returns LAGS_ERR_WORKSPACE).
 * Also checks that the current device is an sm_100 part and makes it the
 * plan's device: later calls on the plan return LAGS_ERR_WRONG_DEVICE, before
 * enqueuing anything, when another device is current.  Call it again after
 * freeing or moving the workspace.  Not for use inside stream capture.
 */
LAGS_API lags_status lags_plan_set_workspace(lags_plan* plan, void* workspace, size_t bytes,
                                    void* stream);

/*
 * lags_sparsify - error feedback and layer-wise top-k for all P workers.
 *   grads      host array of P device pointers, each a float[N] gradient
 *              buffer (16-byte aligned); read only.
 *   residuals  host array of P device pointers, each a float[N] residual
 *              buffer (16-byte aligned); read, then overwritten with the new
 *              residual.  Buffers of different workers must not overlap.
 *   lr         learning rate (fp32).
 *   out_idx    device uint32[P*K] (4-byte aligned): worker p's picks at
 *              [p*K, (p+1)*K), layer by layer, ascending global index.
 *   out_val    device float[P*K]: acc at those indices.
 * The pointer arrays are copied into the launch arguments, so they need not
 * outlive the call.  Enqueues a few kernels on `stream`.
 */
LAGS_API lags_status lags_sparsify(lags_plan* plan, const float* const* grads, float* const* residuals,
                          float lr, uint32_t* out_idx, float* out_val, void* stream);

/*
 * lags_aggregate - dense averaged update from P workers' pick lists.
 *   idx, val   device [P*K] in the layout lags_sparsify writes (each layer's
 *              indices ascending and inside the layer; otherwise the status
 *              word gets LAGS_FLAG_BAD_PICKS and dense_out is unspecified).
 *   dense_out  device float[N], 16-byte aligned; fully overwritten.
 * Uses the plan workspace; order it after lags_sparsify on the same stream
 * when it consumes that call's output.
 */
LAGS_API lags_status lags_aggregate(lags_plan* plan, const uint32_t* idx, const float* val,
                           float* dense_out, void* stream);

/*
 * lags_aggregate_apply - lags_aggregate followed by lags_apply without a
 * pass over the whole update: dense_out is written exactly as lags_aggregate
 * writes it and weights end exactly as lags_apply leaves them, but only the
 * picked positions of weights are read and written (entries no worker picked
 * keep their weight, since w - (+0) == w) and dense_out is not read back.
 *   weights    device float[N], 16-byte aligned, updated in place.
 * Other arguments, layout and errors: as lags_aggregate.
 */
LAGS_API lags_status lags_aggregate_apply(lags_plan* plan, const uint32_t* idx, const float* val,
                                          float* dense_out, float* weights, void* stream);

/*
 * lags_apply - weights <- weights - dense_out over the plan's elements
 * (0 .. N-1, or the range of a lags_plan_create_range plan).
 *   weights    device float[N], 16-byte aligned, updated in place.
 *   dense_out  device float[N], 16-byte aligned.
 */
LAGS_API lags_status lags_apply(const lags_plan* plan, float* weights, const float* dense_out,
                       void* stream);

/*
 * lags_status_poll - synchronise `stream`, read and clear the plan's device
 * status word.  The word collects the flags of every call on the plan since
 * the last poll.
 *   flags              host, receives LAGS_FLAG_* bits (may be NULL)
 *   exact_fallbacks    host, receives how many (worker, layer) segments since
 *                      the last poll were selected by the exhaustive path
 *                      because the sampled candidate threshold did not hold
 *                      (results are exact either way; may be NULL)
 * Returns, when a flag is set: LAGS_ERR_TIMEOUT (LAGS_FLAG_TIMEOUT: picks may
 * be incomplete), else LAGS_ERR_INTERNAL (LAGS_FLAG_INTERNAL: a library bug),
 * else LAGS_ERR_BAD_PICKS; otherwise LAGS_OK.  The outputs are written in
 * every case.  LAGS_ERR_CUDA if the copy fails.
 */
LAGS_API lags_status lags_status_poll(lags_plan* plan, uint32_t* flags, uint32_t* exact_fallbacks,
                             void* stream);

/*
 * lags_sparsify_static - lags_sparsify for callers that cannot allocate device
 * memory (code running inside an allocator or memory-pool callback, runtimes
 * that own every device allocation, hosts that forbid cudaMalloc after
 * start-up).  The pages have no counterpart: it is a deployment variant, not
 * part of the method.  Arguments and results are those of lags_sparsify, and
 * the plan needs no workspace: the scratch lives in a 16 MiB array with static
 * storage in the library, present on every GPU that loads it until exit.
 *   - Returns LAGS_ERR_WORKSPACE, before enqueuing anything, when the plan's
 *     workspace_bytes exceed 16 MiB.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating routine.
 *   - All calls share the array, which keeps the last call's contents; each
 *     call uploads its plan's tables and clears what must start at zero.
 *     Calls whose work overlaps on the GPU race on it.
 *   - The first call on a device (of this function or of
 *     lags_static_status_poll) resolves the array's address there and
 *     configures the kernels.  Under CUDA's lazy module loading (the default)
 *     that first call is also when the driver loads the array's code and
 *     reserves its 16 MiB on the device, so make it at start-up: outside any
 *     context that must not allocate, and before any stream capture.
 *   - Its status words live in the same array, at a fixed place, and collect
 *     the flags of every call on the device until lags_static_status_poll
 *     reads and clears them (lags_status_poll does not see them).
 */
LAGS_API lags_status lags_sparsify_static(lags_plan* plan, const float* const* grads,
                                          float* const* residuals, float lr, uint32_t* out_idx,
                                          float* out_val, void* stream);

/*
 * lags_static_status_poll - lags_status_poll for lags_sparsify_static: copy the
 * status words of the static array of the current device into host memory
 * (synchronising `stream`), then clear them.  Allocates nothing.
 *   flags, exact_fallbacks   as lags_status_poll (either may be NULL).
 * Returns as lags_status_poll.
 */
LAGS_API lags_status lags_static_status_poll(uint32_t* flags, uint32_t* exact_fallbacks,
                                             void* stream);

/*
 * lags_plan_set_events - timing instrumentation.  When `before` and `after`
 * (cudaEvent_t passed as void*, created by the caller) are both non-NULL, each
 * later lags_sparsify on this plan records `before` on its stream just before
 * it launches the fused error-feedback pass and `after` just after it, so
 * cudaEventElapsedTime(before, after) is that kernel's device time.  Pass
 * NULL, NULL to stop.  The events stay the caller's.  Inside stream capture
 * the records are captured as external event nodes, so every replay of the
 * graph records them again.
 */
LAGS_API lags_status lags_plan_set_events(lags_plan* plan, void* before, void* after);

/*
 * lags_plan_set_stage_wait_limit - failure-injection knob for tests of the
 * timeout path.  The selection kernel stages a layer's candidates in shared
 * memory with bulk copies and polls their completion barrier at most
 * `polls` times (default LAGS_STAGE_WAIT_POLLS) before it gives up, sets
 * LAGS_FLAG_TIMEOUT and selects from global memory instead; it then still
 * waits (up to the default limit) for its copies before it exits.  0 makes
 * every staged selection give up at once: the status poll then reports the
 * timeout, while the picks of layers without overflowed candidate tiles stay
 * exact.  Takes effect from the next lags_sparsify on the plan.
 */
#define LAGS_STAGE_WAIT_POLLS 4194304u
LAGS_API lags_status lags_plan_set_stage_wait_limit(lags_plan* plan, uint32_t polls);

/*
 * lags_plan_set_index_wait_limit - failure-injection knob for the second
 * bounded wait of the selections that stage candidate values only: after the
 * emission they bulk-copy the candidate indices over their stage and poll
 * that copy's completion at most `polls` times (default
 * LAGS_STAGE_WAIT_POLLS).  On timeout they set LAGS_FLAG_TIMEOUT and read
 * each pick's index from global memory instead (the same index, so every
 * output stays exact), then still wait (up to the default limit) for the
 * copies before they exit.  Takes effect from the next lags_sparsify.
 */
LAGS_API lags_status lags_plan_set_index_wait_limit(lags_plan* plan, uint32_t polls);

/*
 * lags_adaptive_densities - per-layer densities from each layer's
 * communication-to-computation ratio ("Layer-wise Adaptive Gradient
 * Sparsification ..." review, "proposed method": each layer's sparsification
 * ratio is set by its communication-to-computation ratio so that its
 * communication hides behind computation).  Host only, no device.
 *   layer_sizes       host, [num_layers] d_l > 0, in forward order.
 *   backward_seconds  host, [num_layers] t_l >= 0: backward time of each layer.
 *   alpha, beta       message model: a layer sending k picks takes
 *                     alpha + beta * 8 * k seconds (alpha, beta >= 0).
 *   rho_min           smallest density, in (0, 1].
 *   out_densities     host, [num_layers] rho_l in [rho_min, 1].
 * Rule: backward produces layers L-1 .. 0; layer l's gradient exists at
 * R_l = sum_{j >= l} t_j, its message starts at max(R_l, end of the previous
 * message) and must end by R_0 (the end of the backward pass).  Layer l gets
 * the largest rho in [rho_min, 1] with k_l = ceil(rho d_l) meeting that
 * deadline (rho_min when none does); messages go out in production order.
 */
LAGS_API lags_status lags_adaptive_densities(const int64_t* layer_sizes,
                                             const double* backward_seconds, int32_t num_layers,
                                             double alpha, double beta, double rho_min,
                                             double* out_densities);

/*
 * lags_merge_layers - cut the layers into buckets of consecutive layers, one
 * message per bucket, so that the last message ends as early as possible
 * (merged-gradient wait-free backpropagation, "MG-WFBP: Efficient Data
 * Communication for Distributed Synchronous SGD Algorithms" review, "proposed
 * method": small per-layer messages are merged to save start-up costs, the
 * merge is optimal for the iteration time, found by dynamic programming in
 * O(L^2) once before training).  Host only, no device.
 *   message_bytes     host, [num_layers] bytes >= 0 each layer sends (for
 *                     LAGS: 8 * k_l * workers per rank).
 *   backward_seconds  host, [num_layers] t_l >= 0: backward time of each layer.
 *   alpha, beta       message model: B bytes in one message take
 *                     alpha + beta * B seconds (alpha, beta >= 0).
 *   out_bucket_first  host, [num_layers]: receives the first layer of every
 *                     bucket, ascending; bucket b is layers
 *                     [first[b], first[b+1]) (the last ends at num_layers).
 *   out_num_buckets   host, receives the bucket count.
 *   out_end_seconds   host, receives the end of the last message (may be NULL).
 * Model: backward produces layers L-1 .. 0; layer l exists at
 * R_l = sum_{j >= l} t_j; a bucket's message starts once its first layer is
 * produced and the previous message has ended; messages go out in production
 * order.  Among cuts with the same end time the planner prefers longer
 * buckets, starting from the last layers.
 */
LAGS_API lags_status lags_merge_layers(const int64_t* message_bytes,
                                       const double* backward_seconds, int32_t num_layers,
                                       double alpha, double beta, int32_t* out_bucket_first,
                                       int32_t* out_num_buckets, double* out_end_seconds);

/*
 * lags_dense_sum - first half of one dense S-SGD step, the baseline LAGS-SGD
 * is compared with ("Layer-wise Adaptive Gradient Sparsification ..." review,
 * main findings: every worker sends its whole gradient, the averaged gradient
 * updates the model):
 *   sum_out_j = fl32( ((+0 + fl32(lr g_0j)) + fl32(lr g_1j)) + ... ),
 * workers in order 0..num_workers-1.  This is the sum a LAGS step with every
 * density 1 and zero residuals forms, so lags_dense_sum + lags_dense_finish
 * give that step's dense update bit for bit.  With several ranks, the caller
 * all-reduces the ranks' sums between the two calls (the all-reduce adds the
 * ranks' sums in its own order).
 *   grads        host array of num_workers device pointers, each a float[N]
 *                gradient (16-byte aligned); read only.
 *   num_workers  1 .. LAGS_MAX_WORKERS.
 *   N            elements per buffer, >= 1.
 *   sum_out      device float[N], 16-byte aligned; fully overwritten.
 * No plan or workspace is involved.
 */
LAGS_API lags_status lags_dense_sum(const float* const* grads, int32_t num_workers, int64_t N,
                                    float lr, float* sum_out, void* stream);

/*
 * lags_dense_finish - second half of the dense S-SGD step:
 *   dense_out_j = fl32(sum_j / num_workers_total)   (a true IEEE division)
 *   weights_j   = fl32(weights_j - dense_out_j)     (skipped if weights is NULL)
 *   sum, dense_out, weights  device float[N], 16-byte aligned.
 */
LAGS_API lags_status lags_dense_finish(const float* sum, int64_t N, int32_t num_workers_total,
                                       float* dense_out, float* weights, void* stream);

/*
 * lags_plan_kernel_launches - how many kernels one lags_sparsify, one
 * lags_aggregate_apply and one lags_apply call enqueue for this plan (any
 * output pointer may be NULL); lags_aggregate enqueues one fewer than
 * lags_aggregate_apply.
 */
LAGS_API lags_status lags_plan_kernel_launches(const lags_plan* plan, int32_t* sparsify,
                                               int32_t* aggregate, int32_t* apply);

/* Static, human-readable text for a status code. */
LAGS_API const char* lags_error_string(lags_status status);

#ifdef __cplusplus
}
#endif

#endif /* LAGS_H */
