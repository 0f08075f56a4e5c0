/*
 * topk_ef.h -- C ABI of the B200 Top-k + error-feedback sparsifier and the
 * gTop-k merge of sparse (index, value) sets.
 *
 * What the calls compute (sources are web pages, cited by title and section):
 *
 *  - One error-feedback step ("Sparsified SGD with Memory", abstract: send the
 *    top-k entries and keep the accumulated error in memory; "The Convergence
 *    of Sparsified Gradient Methods", abstract: transmit a subset by
 *    magnitude, accumulate the rest locally):
 *        acc[i]      = fmaf(lr, grad[i], residual[i])      (one fp32 rounding)
 *        S           = the k indices of largest |acc|, ties to the lower index
 *        out         = (i, acc[i]) for i in S, ascending i
 *        residual[i] = +0.0f for i in S, acc[i] otherwise
 *    |x| order is the order of bits(x) & 0x7FFFFFFF as an unsigned integer
 *    (-0 == +0; NaN above +Inf).
 *
 *  - The gTop-k merge ("A Distributed Synchronous SGD Algorithm with Global
 *    Top-k Sparsification for Low Bandwidth Networks", ABSTRACT: the global
 *    top-k largest absolute values from P workers; method section: a
 *    tournament in O(log P) rounds).  Round r = 0, 1, ... while 2^r < P: every
 *    worker i that is a multiple of 2^(r+1) with i + 2^r < P replaces its set
 *    by the top min(k, |U|) of U = S_i (+) S_{i+2^r}, the union with one fp32
 *    add (round to nearest even) at common indices.  A worker without a
 *    partner in a round keeps its set.  The result is the top min(k, |S_0|)
 *    of S_0, ascending index.
 *
 * Conventions shared by every call:
 *  - Pointers marked "device" are CUDA device pointers on the current device;
 *    pointers marked "host" are host memory read before the call returns.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    compute call is asynchronous on that stream and returns once its work
 *    is enqueued.
 *  - The caller owns every buffer, including the workspace `ws`
 *    (device memory, at least the size the matching *_workspace_bytes call
 *    returns, 256-byte aligned).  Calls on the same workspace must be ordered
 *    (same stream, or synchronised); the library allocates no memory and
 *    keeps nothing between calls except inside `ws`.  A workspace needs no
 *    initialisation: its contents before the first call (zeros, garbage, a
 *    workspace last used with other sizes) never change a result.
 *  - fp32 arrays must be 4-byte aligned; 16-byte aligned grad/residual take
 *    the vectorised path, other alignments a scalar path with identical
 *    results.
 *  - Results are deterministic and bit-identical from run to run.
 *
 * Return codes.  The return value covers argument checks and launch errors;
 * problems found on the device (a bounded wait that gave up, malformed merge
 * input) are recorded in the workspace and read back with
 * topk_ef_last_device_status().  No call traps, asserts on the device or
 * waits without bound.
 */
#ifndef TOPK_EF_H
#define TOPK_EF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TOPK_EF_OK 0
/* null pointer, n < 0, k < 0, k > n, n > 2^31 - 1, T < 1, P < 1, k_in > n,
   offsets not starting at 0 or decreasing, misaligned fp32 pointer */
#define TOPK_EF_ERR_INVALID_ARG (-1)
/* ws_bytes smaller than the matching *_workspace_bytes() */
#define TOPK_EF_ERR_WORKSPACE (-2)
/* a CUDA launch or runtime call failed; topk_ef_last_cuda_error() has it */
#define TOPK_EF_ERR_CUDA (-3)
/* device: a bounded spin-wait gave up (outputs are undefined) */
#define TOPK_EF_ERR_DEVICE_TIMEOUT (-4)
/* device: merge input rows not strictly ascending or indices outside [0, n) */
#define TOPK_EF_ERR_BAD_INPUT (-5)
/* device: an internal count did not add up (outputs are undefined) */
#define TOPK_EF_ERR_INTERNAL (-6)

/* ---------------------------------------------------------------- compress */

/* Workspace bytes for topk_ef_compress on n elements with k kept.
   Returns 0 for invalid (n, k). */
size_t topk_ef_workspace_bytes(int64_t n, int64_t k);

/*
 * One error-feedback step on a flat fp32 tensor.
 *   grad      device, fp32[n], read only; must not overlap residual or outputs
 *   residual  device, fp32[n]; in: the memory, out: acc with the k sent slots
 *             set to +0.0f
 *   n         0 <= n <= 2^31 - 1 (indices are int32)
 *   lr        scale applied to grad inside the single fmaf
 *   k         0 <= k <= n
 *   out_idx   device, int32[k], ascending indices of the sent entries
 *   out_val   device, fp32[k], acc at those indices (signed)
 *   ws        device workspace of ws_bytes >= topk_ef_workspace_bytes(n, k)
 *
 * The compress keeps, in `ws`, the threshold of the previous call made with
 * the same residual pointer, n, k and lr ("Sparsified SGD with Memory",
 * abstract: the memory carries over from step to step, and so does the
 * magnitude of what is sent): a prefilter only, the result is exact whatever
 * it holds.  A tensor small enough for one wave of blocks (n <= 148 * 16,384
 * on a 148-SM device) takes one kernel launch; its workspace holds 8 n bytes
 * of candidate lists besides.  The launch's parameters are the same from
 * call to call apart from a host-issued call number, and the kernel keeps
 * its own call counter in `ws`, so a call captured in a CUDA graph may be
 * replayed.
 */
int topk_ef_compress(const float* grad, float* residual, int64_t n, float lr,
                     int64_t k, int32_t* out_idx, float* out_val, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * topk_ef_compress_static: the same error-feedback step as topk_ef_compress,
 * for callers that cannot allocate device memory, and so cannot provide the
 * workspace: for instance code that runs inside a host program whose
 * framework owns all device memory and forbids other allocations, or a
 * latency-critical path where a cudaMalloc (which can synchronise the device)
 * is not acceptable.  The pages have no counterpart of this entry point.
 *
 * The scratch it uses in place of `ws` is a fixed array of
 * TOPK_EF_STATIC_SCRATCH_BYTES (32 MiB) inside the library's device module:
 * every GPU on which the library is used holds it until the process exits.
 * It allocates nothing itself: no cudaMalloc, cudaFree or allocating library
 * routine.  The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and keeps it; make that
 * first call before any stream capture.  Sizes whose workspace
 * (topk_ef_workspace_bytes(n, k)) exceeds the array are rejected with
 * TOPK_EF_ERR_WORKSPACE (32 MiB holds, e.g., n = 25.6M at k = 1% or
 * n = 150M at k = 0.1%).  All calls share the one array and each call resets
 * the state it needs at its start, so it keeps no result between calls; two
 * calls whose GPU work overlaps (different streams, or different host threads
 * without ordering) race on it and must not be issued.
 *   Arguments and results: exactly those of topk_ef_compress, without ws and
 *   ws_bytes.
 */
#define TOPK_EF_STATIC_SCRATCH_BYTES ((size_t)32 << 20)
int topk_ef_compress_static(const float* grad, float* residual, int64_t n, float lr,
                            int64_t k, int32_t* out_idx, float* out_val,
                            void* stream);

/*
 * Device-side status of the last topk_ef_compress_static call on the current
 * device, the counterpart of topk_ef_last_device_status(ws, stream) for the
 * library's scratch array (which the caller has no address of): synchronises
 * `stream` and returns TOPK_EF_OK, TOPK_EF_ERR_DEVICE_TIMEOUT or
 * TOPK_EF_ERR_INTERNAL (TOPK_EF_ERR_CUDA if the read-back failed).  Check it
 * before using the outputs of a call that may have hit a bounded wait.  The
 * device address of the array is looked up once per device and kept; after
 * cudaDeviceReset it is stale (as is every other device pointer of the
 * process), and neither call may be used again.
 */
int topk_ef_static_last_device_status(void* stream);

/* ------------------------------------------------------- hard threshold */

/* Workspace bytes for topk_ef_threshold on n elements; 0 for invalid n. */
size_t topk_ef_threshold_workspace_bytes(int64_t n);

/*
 * One error-feedback step of the hard-threshold sparsifier ("Rethinking
 * gradient sparsification as total error minimization", abstract: the
 * variant of Top-k whose k is set by a constant hard threshold, analysed
 * under error feedback):
 *     acc = fmaf(lr, grad, residual);
 *     the entries with key(acc) >= key(threshold) pass (|acc| at least
 *     |threshold|; NaN above +Inf, as in topk_ef_compress; a NaN threshold
 *     passes only NaNs);
 *     the first min(count, max_out) passing entries in ascending index order
 *     are sent; the others stay in memory.
 *   grad, residual, n, lr  as in topk_ef_compress
 *   threshold  compared by magnitude (its sign is ignored)
 *   max_out    >= 0: capacity of out_idx / out_val
 *   out_idx    device, int32[max_out]: ascending indices of the sent entries;
 *              slots from min(count, max_out) on are not written
 *   out_val    device, fp32[max_out]: acc at those indices
 *   out_count  device, int64 (8-byte aligned): count, the number of entries
 *              that passed (may exceed max_out)
 *   ws         device workspace of >= topk_ef_threshold_workspace_bytes(n)
 * Errors: TOPK_EF_ERR_INVALID_ARG (n out of range, max_out < 0, null or
 * misaligned pointers), TOPK_EF_ERR_WORKSPACE, TOPK_EF_ERR_CUDA.
 */
int topk_ef_threshold(const float* grad, float* residual, int64_t n, float lr,
                      float threshold, int64_t max_out, int32_t* out_idx,
                      float* out_val, int64_t* out_count, void* ws,
                      size_t ws_bytes, void* stream);

/* Workspace bytes for topk_ef_compress_batched with the same (offsets, k, T).
   offsets and k are host arrays.  Returns 0 for invalid arguments. */
size_t topk_ef_batched_workspace_bytes(const int64_t* offsets,
                                       const int64_t* k, int32_t T);

/*
 * One error-feedback step on each of T tensors stored back to back in one
 * flat bucket (per-tensor k; the tensors are independent problems).
 *   grad, residual  device, fp32[offsets[T]]; tensor l is
 *                   [offsets[l], offsets[l+1]); residual updated in place
 *   offsets         host, int64[T+1], offsets[0] = 0, non-decreasing,
 *                   offsets[T] <= 2^31 - 1
 *   k               host, int64[T], 0 <= k[l] <= offsets[l+1] - offsets[l]
 *   T               number of tensors, >= 1
 *   out_idx         device, int32[sum k]; tensor l's entries start at
 *                   sum_{j<l} k[j] and hold indices LOCAL to tensor l,
 *                   ascending
 *   out_val         device, fp32[sum k], matching acc values
 *   ws              device workspace of ws_bytes >=
 *                   topk_ef_batched_workspace_bytes(offsets, k, T)
 */
int topk_ef_compress_batched(const float* grad, float* residual,
                             const int64_t* offsets, const int64_t* k,
                             int32_t T, float lr, int32_t* out_idx,
                             float* out_val, void* ws, size_t ws_bytes,
                             void* stream);

/* ------------------------------------------------------------------ merge */

/* Workspace bytes for gtopk_merge with P sets of k_in entries keeping k.
   Returns 0 for invalid arguments. */
size_t gtopk_merge_workspace_bytes(int32_t P, int64_t k_in, int64_t k);

/*
 * gTop-k tournament over P sparse sets (P workers simulated on one GPU).
 *   in_idx     device, int32[P][k_in], each row strictly ascending, values in
 *              [0, n) (checked on the device: TOPK_EF_ERR_BAD_INPUT)
 *   in_val     device, fp32[P][k_in]
 *   P          number of workers, 1 <= P <= 512
 *   k_in       entries per input set, 0 <= k_in <= n
 *   k          entries kept per round and in the result, k >= 0
 *   n          index bound
 *   out_idx    device, int32[k]; the result in ascending index order; slots
 *              past the result length hold -1
 *   out_val    device, fp32[k]; the summed values; slots past the length 0
 *   out_count  device, int32[1]; the result length min(k, |S_0|)
 *   ws         device workspace of ws_bytes >=
 *              gtopk_merge_workspace_bytes(P, k_in, k)
 */
int gtopk_merge(const int32_t* in_idx, const float* in_val, int32_t P,
                int64_t k_in, int64_t k, int64_t n, int32_t* out_idx,
                float* out_val, int32_t* out_count, void* ws, size_t ws_bytes,
                void* stream);

/* ---------------------------------------------------------------- status */

/* ------------------------------------------- after the gTop-k merge */

/* Workspace bytes for gtopk_residual_return (a status block). */
size_t gtopk_residual_return_workspace_bytes(void);

/*
 * Residual return after gTop-k: only the global set updates the model ("A
 * Distributed Synchronous SGD Algorithm with Global Top-k Sparsification
 * for Low Bandwidth Networks", ABSTRACT), so each worker puts back into its
 * memory the values it sent whose index is not in the global set (error
 * feedback: what is not transmitted accumulates locally, "The Convergence of
 * Sparsified Gradient Methods", abstract):
 *     for every worker p and sent (i, v) with i not in global_idx:
 *         residual[p][i] = residual[p][i] + v          (one fp32 add)
 *   sent_idx    device, int32[P][k_sent], each row strictly ascending in [0, n)
 *               (the sets the workers sent, as given to gtopk_merge)
 *   sent_val    device, fp32[P][k_sent]
 *   global_idx  device, int32[k_global], strictly ascending in [0, n) (the
 *               first out_count indices gtopk_merge returned)
 *   residual    device, fp32[P][n], row p is worker p's memory
 *   ws          device workspace of >= gtopk_residual_return_workspace_bytes()
 * Malformed rows or global list: TOPK_EF_ERR_BAD_INPUT through
 * topk_ef_last_device_status(ws); no memory outside residual is written.
 * Errors: TOPK_EF_ERR_INVALID_ARG (P < 1, sizes out of range, null or
 * misaligned pointers), TOPK_EF_ERR_WORKSPACE, TOPK_EF_ERR_CUDA.
 */
int gtopk_residual_return(const int32_t* sent_idx, const float* sent_val,
                          int32_t P, int64_t k_sent, const int32_t* global_idx,
                          int64_t k_global, float* residual, int64_t n,
                          void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes for topk_allgather_sum; 0 for invalid sizes
   (1 <= P <= 256, 0 <= k_in <= n <= 2^31 - 1). */
size_t topk_allgather_workspace_bytes(int32_t P, int64_t k_in, int64_t n);

/*
 * Top-k aggregation by AllGather, the O(kP) method the gTop-k review
 * measures its merge against ("A Distributed Synchronous SGD Algorithm with
 * Global Top-k Sparsification for Low Bandwidth Networks", ABSTRACT: current
 * methods use AllGather to accumulate the sparse gradients), on one GPU:
 * every worker's set is gathered and summed into a dense gradient in rank
 * order,
 *     out[i] = +0.0f;  for p = 0..P-1, for (i, v) in set p: out[i] += v
 * (one fp32 add each, in that order).
 *   in_idx   device, int32[P][k_in], rows strictly ascending in [0, n)
 *   in_val   device, fp32[P][k_in]
 *   out      device, fp32[n], written in full
 *   ws       device workspace of >= topk_allgather_workspace_bytes(P, k_in, n)
 * Malformed rows: TOPK_EF_ERR_BAD_INPUT through topk_ef_last_device_status;
 * no memory outside out is written.
 */
int topk_allgather_sum(const int32_t* in_idx, const float* in_val, int32_t P,
                       int64_t k_in, int64_t n, float* out, void* ws,
                       size_t ws_bytes, void* stream);

/* Synchronises `stream` and returns the device-side status of the last call
   that used `ws`: TOPK_EF_OK, TOPK_EF_ERR_DEVICE_TIMEOUT,
   TOPK_EF_ERR_BAD_INPUT or TOPK_EF_ERR_INTERNAL (or TOPK_EF_ERR_CUDA if the
   read-back failed). */
int topk_ef_last_device_status(const void* ws, void* stream);

/* The cudaError_t of the last TOPK_EF_ERR_CUDA returned on this thread. */
int topk_ef_last_cuda_error(void);

/* Human-readable name of a return code (static string). */
const char* topk_ef_status_string(int status);

/*
 * Diagnostics of the last compress call on `ws` (synchronises `stream`):
 *   info[0]  path taken: 0 = candidate prefilter, 1 = full rescan fallback
 *            (a small tensor: 1 = the previous call's threshold did not
 *            decide the top k, so every block ran the exact select)
 *   info[1]  candidates kept by the prefilter
 *   info[2]  candidate capacity of the workspace
 *   info[3]  kernels launched by that call
 *   info[4]  1 if the k-th key's relative digit-1 bin of some tensor held
 *            more candidates than its entry list, so the select kernel took
 *            the exact-count exchange (one more grid barrier); else 0
 *   info[5]  reserved (0)
 * `info` is host memory of 6 int64.  Returns a status code.
 */
int topk_ef_path_info(const void* ws, void* stream, int64_t* info);

/*
 * Diagnostics of the last compress call on `ws` (synchronises `stream`), in
 * nanoseconds; -1 for a step that did not run.  `ns` is host memory of 20
 * int64.  ns[0..7]: block 0 of the select kernel, from the kernel's start:
 *   candidate path: ns[4] offset look-back done, ns[5] gather done,
 *     ns[1] first grid barrier, ns[2] second grid barrier, ns[3] barrier of
 *     the exact-count exchange (only when a bin overflowed its entry list),
 *     ns[6] emission starts, ns[7] end;
 *   rescan fallback: ns[1] gather barrier, ns[3..5] the barriers after
 *     digit passes 1..3, ns[6] the count barrier, ns[7] end.
 * ns[8..10]: the sampling block of the first tensor, from its start: samples
 * loaded, first histogram level resolved, end.
 * ns[11..14], over all blocks and from the moment the first block of the
 * streaming pass got past its wait on the setup kernel: the last streaming
 * block done, the first select (or threshold) block started, block 0 of that
 * kernel started, its last block done; then, latest over the blocks of that
 * kernel: block started, output offset known (candidate path), candidates
 * gathered, arrived at the barrier after the entry lists.  ns[19] is
 * reserved (-1).
 */
int topk_ef_phase_times(const void* ws, void* stream, int64_t* ns);

/*
 * Test hook, process wide: bit 0 forces the full rescan fallback of the
 * compress calls; bit 1 forces the prefilter threshold of every tensor to 0
 * (every element a candidate, which overflows the candidate capacity for
 * large tensors and so also ends in the fallback); bit 2 makes the grid-wide
 * exchange of a single-tensor compress call wait for one block more than
 * the grid has, so that its bounded wait runs out (after about a second) and
 * the call records TOPK_EF_ERR_DEVICE_TIMEOUT, with undefined outputs; bits
 * 3..5, when 1, 2, 3 or 4, make the rounds of gtopk_merge that one thread-block
 * cluster per pair can hold use clusters of 16, 14, 12 or 8 CTAs wherever
 * that size can run (else the size is chosen per round as usual).  0
 * restores normal behaviour.  Returns the previous flags.  The flags are
 * process-wide state read by every call in the process (the library's only
 * state outside the caller's workspace besides the tracing record and the
 * scratch array of topk_ef_compress_static): set them only in tests, with no
 * other calls in flight.
 */
int topk_ef_set_test_flags(int flags);

/*
 * Tracing, process wide, for one thread at a time: while enabled, every
 * kernel a compute call launches is bracketed by two CUDA events recorded on
 * the call's stream (the library owns the events, created on the device that
 * is current when tracing is enabled).  Up to 4096 launches are recorded;
 * later ones are not.
 *   topk_ef_trace_enable(1|0)   switch on / off (either clears the record)
 *   topk_ef_trace_read(ms, names, max, &count)
 *       waits for the recorded launches, writes the duration in milliseconds
 *       (host float[max]) and kernel name (host const char*[max], static
 *       strings) of the first min(max, recorded) of them, sets *count to that
 *       number and clears the record.
 *   topk_ef_trace_only(name, every)    record only the launches of the
 *       kernel with this name (as topk_ef_trace_read reports it, e.g.
 *       "stream_kernel"), and of those the 1st, (every+1)-th, ... after
 *       tracing was enabled, so that the other launches keep running back to
 *       back; NULL or "" selects every kernel again.  The string is copied.
 *       every < 1: TOPK_EF_ERR_INVALID_ARG.
 */
int topk_ef_trace_enable(int on);
int topk_ef_trace_read(float* ms, const char** names, int max_entries, int* count);
int topk_ef_trace_only(const char* kernel_name, int every);

#ifdef __cplusplus
}
#endif

#endif /* TOPK_EF_H */
