/*
 * km.h -- C ABI of the B200 (sm_100a) exact Lloyd K-Means library (libkm.so).
 *
 * The method is the one described in "Flash-KMeans: Fast and Memory-Efficient
 * Exact K-Means":
 *   - §2.1 FlashAssign: the nearest-centroid assignment computed by fusing the
 *     distance tile ||x||^2 - 2 x.c + ||c||^2 with an online per-row argmin,
 *     so no N x K distance matrix is ever written to device memory;
 *   - §2.2 Sort-Inverse Update: the centroid update formed by sorting the
 *     assignment vector (an explicit inverse map from cluster to points) and
 *     reducing contiguous same-cluster segments on chip, instead of scattering
 *     every point into its cluster with atomics;
 *   - §2.3 Chunked Stream Overlap: points held in host memory are streamed in
 *     chunks, with copies overlapping compute.
 * §2 states that the mathematics of standard Lloyd K-Means is unchanged, so
 * every entry point computes exact Lloyd iterations (up to floating-point
 * rounding of the stated precisions).
 *
 * Conventions shared by all entry points
 * --------------------------------------
 *  - Pointers are DEVICE pointers owned by the caller unless a parameter says
 *    "host".  The library never allocates or frees device memory: all scratch
 *    comes from the caller's `workspace` (size from km_workspace_size).
 *    Workspace base must be 256-byte aligned (cudaMalloc/torch allocations are).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Unless stated,
 *    work is enqueued asynchronously and the call returns without waiting.
 *  - Layouts are row-major and contiguous.  B >= 1 independent problems are
 *    stacked: instance b owns X + b*N*D, C + b*K*D, idx + b*N, counts + b*K.
 *  - dtype: KM_BF16 (X and centroid operands in bfloat16; the distance dot
 *    products run on the tensor cores with float32 accumulation) or KM_F32
 *    (float32 inputs; dot products use a three-term TF32 split, hi*hi + hi*lo
 *    + lo*hi, on the tensor cores, which keeps float32-level accuracy).
 *  - Centroid outputs are float32.  Assignments are int32 in [0, K).
 *  - Ties: the lowest centroid index wins an exact tie.  The device compares
 *    distances with the column in their 5 lowest mantissa bits, so distances
 *    within 2^-18 relative also count as tied; identical centroid rows tie
 *    exactly, at distance 0 too.  A cluster with no member keeps its previous
 *    centroid (the pages fix neither rule; these are the plain readings).
 *  - Supported shapes: D % 8 == 0; bf16: 8 <= D <= 256; f32: 8 <= D <= 64;
 *    1 <= K <= min(N, 1 << 20); N < 2^31.  Others return KM_ERR_UNSUPPORTED
 *    or KM_ERR_INVALID_ARG before anything is launched.
 *  - Inputs containing NaN or Inf give unspecified (but memory-safe) results.
 *  - Every wait inside a kernel is bounded in time; a wait that runs out sets
 *    a status word in the workspace and the kernel returns early.  Read it with
 *    km_workspace_status().  Entry points that synchronise (km_fit_host,
 *    km_workspace_status) report it as KM_ERR_TIMEOUT.
 *  - Errors: a non-zero km_status; km_last_error() gives a message for the
 *    calling thread.
 *  - Calls on distinct workspaces may run concurrently; calls sharing one
 *    workspace must be ordered (same stream or synchronised).
 *  - Environment (read once per process): KM_WAIT_LIMIT_NS sets the bound of
 *    every in-kernel wait (default 2e9 ns); KM_ASSIGN_FORM=single|pair picks
 *    the assignment kernel's form: one CTA per 128-point tile or two-SM CTA
 *    pairs on 256-point tiles (the default wherever the centroid tile is 128
 *    or 256 wide).  Both forms meet the same
 *    accuracy rules; the objective's float64 summation order follows the
 *    form's tiling and the number of assignment CTAs the device holds at
 *    once, so its last bits may differ between forms and between GPUs
 *    (assignments and centroids do not).
 *    KM_ASSIGN_TILE=pair,BN,XB,CS (read at every call) forces the whole
 *    assignment tiling; see km_plan_describe.
 *  - Fault injection (testing the error paths; nothing is done to the GPU):
 *    KM_FAULT=<point>[:<n>] in the environment, read at the entry of every
 *    call, makes the n-th occurrence (default 1) of that point inside the
 *    call fail before it is issued: "alloc" (creating the copy stream or an
 *    event of km_fit_host, or an event of km_fit_profile / km_fit_timed),
 *    "h2d" (a host-to-device chunk copy of km_fit_host) or "launch" (a
 *    kernel launch).  The call returns KM_ERR_INJECTED after the clean-up a
 *    real failure of that step gets: work already enqueued completes, the
 *    call's own streams and events are released (km_fit_host synchronises
 *    first), and the context stays usable.
 *  - Launch chaining: within one call, a kernel that directly follows another
 *    of this library's kernels on the stream is launched with programmatic
 *    stream serialization (it may become resident while its predecessor
 *    drains and waits on the device, griddepcontrol.wait, before touching
 *    shared data).  The first kernel of every call, and any kernel after a
 *    memset, copy, event or plain launch, is stream-ordered as usual, so
 *    calls compose with any other work on the stream.  Results do not depend
 *    on it; KM_PDL=0 in the environment (read at every launch) turns it off.
 */
#ifndef KM_H_
#define KM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KM_VERSION 1

typedef enum km_status {
  KM_OK = 0,
  KM_ERR_INVALID_ARG = 1, /* null required pointer, bad size, misaligned pointer */
  KM_ERR_UNSUPPORTED = 2, /* valid request the library cannot serve (shape, device) */
  KM_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  KM_ERR_WORKSPACE = 4,   /* workspace null or smaller than km_workspace_size() */
  KM_ERR_TIMEOUT = 5,     /* a bounded in-kernel wait ran out */
  KM_ERR_INJECTED = 6     /* a failure made on purpose by KM_FAULT (testing only) */
} km_status;

typedef enum km_dtype { KM_F32 = 0, KM_BF16 = 1 } km_dtype;

typedef enum km_op {
  KM_OP_ASSIGN = 0,  /* km_assign */
  KM_OP_UPDATE = 1,  /* km_update */
  KM_OP_FIT = 2,     /* km_fit */
  KM_OP_FIT_HOST = 3, /* km_fit_host (uses chunk_rows) */
  KM_OP_ARGSORT = 4   /* km_argsort (D and dtype ignored) */
} km_op;

/* Library version (KM_VERSION of the build). */
int km_version(void);

/* Static string for a km_status value. */
const char* km_status_string(int status);

/* Message describing the last failure on the calling thread ("" if none). */
const char* km_last_error(void);

/*
 * Bytes of workspace the operation needs for this shape (0 if the shape is
 * invalid or unsupported; km_last_error() says why).  The size is O(B*N + K*D)
 * (plus 2*chunk_rows*D elements for KM_OP_FIT_HOST); never O(N*K).
 */
size_t km_workspace_size(int op, int B, int64_t N, int D, int K, int dtype, int64_t chunk_rows);

/*
 * Synchronise `stream`, read and clear the workspace status word.
 * Returns KM_OK, or KM_ERR_TIMEOUT if a kernel that used this workspace gave
 * up on a bounded wait since the status was last cleared.
 */
int km_workspace_status(void* workspace, void* stream);

/*
 * FlashAssign (Flash-KMeans §2.1): for every point i of every instance,
 *   idx[i]     = argmin_k ||x_i - c_k||^2   (lowest k on exact ties)
 *   mindist[i] = max(0, ||x_i||^2 - 2 x_i.c_idx + ||c_idx||^2)
 * computed tile by tile with an online argmin; the N x K distances never
 * reach device memory.
 *   X        [B][N][D] dtype, device, read only.
 *   C        [B][K][D] dtype, device, read only.
 *   idx      [B][N] int32, device, written.
 *   mindist  [B][N] float, device, written; may be NULL.
 *   objective [B] double, device, written (sum of mindist per instance, in a
 *            fixed order); may be NULL.
 * X and C (bf16) must be 16-byte aligned.
 */
int km_assign(const void* X, const void* C, int B, int64_t N, int D, int K, int dtype,
              int32_t* idx, float* mindist, double* objective,
              void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sort-Inverse Update (Flash-KMeans §2.2): new centroids as member means.
 * The assignment vector is argsorted by a device radix sort (stable, so the
 * order is deterministic), same-cluster runs of the sorted order are summed on
 * chip in float32, and only run boundaries are combined across thread blocks,
 * in a fixed order (no atomics on centroid sums; results are bitwise
 * reproducible run to run).
 *   X       [B][N][D] dtype, device, read only.
 *   idx     [B][N] int32 in [0, K), device, read only (values outside [0,K)
 *           are undefined behaviour).
 *   C       [B][K][D] float, device, in: previous centroids (kept for empty
 *           clusters), out: updated centroids.
 *   counts  [B][K] int32, device, written: members per cluster; may be NULL.
 */
int km_update(const void* X, const int32_t* idx, int B, int64_t N, int D, int K, int dtype,
              float* C, int32_t* counts,
              void* workspace, size_t workspace_bytes, void* stream);

/*
 * The explicit inverse map of the Sort-Inverse Update (Flash-KMeans §2.2:
 * argsort of the assignment vector so that each cluster's points become a
 * contiguous run).  Stable: points of one cluster keep increasing index, so
 * the permutation is unique.
 *   idx    [N] int32 in [0, K), device, read only (out-of-range ids are
 *          clamped into [0, K); they are not valid input).
 *   perm   [N] int32, device, written: point indices ordered by cluster.
 *   start  [K+1] int32, device, written: start[k] = first position of
 *          cluster k in perm, start[K] = N (so count_k = start[k+1]-start[k]);
 *          may be NULL.
 * Workspace: km_workspace_size(KM_OP_ARGSORT, 1, N, 0, K, 0, 0).
 */
int km_argsort(const int32_t* idx, int64_t N, int K, int32_t* perm, int32_t* start,
               void* workspace, size_t workspace_bytes, void* stream);

/*
 * `iters` Lloyd iterations (assign then update) from the initial centroids C0.
 * Iteration t (1-based) assigns under C_{t-1}; objective_hist[b*iters + t-1]
 * is the sum of squared distances of that assignment.  After the call
 * C_out = C_iters, idx_out = the assignment of iteration `iters`, and
 * counts_out = its cluster sizes.  In bf16 mode the centroids are kept in
 * float32 and a bfloat16 copy (round to nearest even) feeds the next
 * assignment.
 *   X              [B][N][D] dtype, device.
 *   C0             [B][K][D] dtype, device (may alias nothing written).
 *   C_out          [B][K][D] float, device, written.
 *   idx_out        [B][N] int32, device, written; may be NULL.
 *   counts_out     [B][K] int32, device, written; may be NULL.
 *   objective_hist [B][iters] double, DEVICE, written; may be NULL.
 */
int km_fit(const void* X, const void* C0, int B, int64_t N, int D, int K, int dtype, int iters,
           float* C_out, int32_t* idx_out, int32_t* counts_out, double* objective_hist,
           void* workspace, size_t workspace_bytes, void* stream);

/*
 * km_fit with per-iteration phase timing, for profiling: CUDA events are
 * recorded on `stream` right before and after the assignment kernel and after
 * the update of every iteration.  Synchronous (waits for the stream).
 *   phase_ms  [2*iters + 1] float, HOST, written: for iteration t,
 *             phase_ms[2t] = milliseconds of the assignment kernel and
 *             phase_ms[2t+1] = milliseconds of the whole update (argsort,
 *             segmented sums, finalise); phase_ms[2*iters] = milliseconds from
 *             the start of the first assignment to the end of the last update
 *             (the iterations alone, without the one-time operand preparation).
 * Other arguments as km_fit.
 */
int km_fit_profile(const void* X, const void* C0, int B, int64_t N, int D, int K, int dtype, int iters,
                   float* C_out, int32_t* idx_out, int32_t* counts_out, double* objective_hist,
                   void* workspace, size_t workspace_bytes, void* stream, float* phase_ms);

/*
 * km_fit with the device time of its iterations: one CUDA event is recorded
 * on `stream` right before the first assignment and one after the last
 * update, nothing between them, so consecutive kernels chain exactly as in
 * km_fit (programmatic dependent launch lets each kernel of an iteration
 * become resident while the previous one drains).  Synchronous.
 *   iters_ms  float, HOST, written: milliseconds from the start of the first
 *             assignment to the end of the last update.
 * Other arguments as km_fit.
 */
int km_fit_timed(const void* X, const void* C0, int B, int64_t N, int D, int K, int dtype, int iters,
                 float* C_out, int32_t* idx_out, int32_t* counts_out, double* objective_hist,
                 void* workspace, size_t workspace_bytes, void* stream, float* iters_ms);

/*
 * A fit captured once as a CUDA graph and then replayed.  For shapes whose
 * kernels run for microseconds, launching them one by one from the host
 * costs about as much as running them; a graph launch enqueues the whole
 * fit at once.
 *   km_fit_graph_create records what km_fit would enqueue with these
 *     arguments (stream capture on a private stream: nothing runs, no
 *     caller stream is used) on the current device.  With timed != 0 (and
 *     iters > 0) the graph also records two events around its iterations,
 *     as km_fit_timed does.  *graph receives the handle (NULL on failure).
 *   km_fit_graph_launch enqueues one complete fit on `stream` (any stream of
 *     the creating device, which must be current): every launch starts again
 *     from C0 and writes the same outputs km_fit would.  The graph holds the
 *     argument pointers, not the data: the buffers must stay allocated until
 *     km_fit_graph_destroy, and their contents may change between launches.
 *     Asynchronous; launches of one graph run one after another.
 *   km_fit_graph_elapsed waits for the last launch and writes the
 *     milliseconds of its iterations (timed graphs only).
 *   km_fit_graph_destroy releases the graph (after its launches complete;
 *     NULL is accepted).
 * Switches read at launch time by km_fit (KM_PDL, KM_ASSIGN_FORM,
 * KM_ASSIGN_TILE, KM_FAULT) are read once, at creation.  Arguments and
 * errors of create as km_fit; km_launch_count counts the graph's kernels at
 * every launch, not at creation.
 */
typedef struct km_fit_graph_t* km_fit_graph;
int km_fit_graph_create(km_fit_graph* graph, const void* X, const void* C0, int B, int64_t N, int D, int K,
                        int dtype, int iters, float* C_out, int32_t* idx_out, int32_t* counts_out,
                        double* objective_hist, void* workspace, size_t workspace_bytes, int timed);
int km_fit_graph_launch(km_fit_graph graph, void* stream);
int km_fit_graph_elapsed(km_fit_graph graph, float* iters_ms);
int km_fit_graph_destroy(km_fit_graph graph);

/*
 * Number of kernels this library has enqueued in this process since it was
 * loaded (all entry points, all threads).  For accounting in benchmarks.
 */
uint64_t km_launch_count(void);

/*
 * km_fit for one instance whose points live in HOST memory (Flash-KMeans §2.3
 * Chunked Stream Overlap, out-of-core execution).  Each iteration streams X to
 * the device in chunks of `chunk_rows` rows through two device buffers: the
 * copy of chunk c+1 runs on a library-owned copy stream while chunk c is
 * assigned, sorted and reduced on `stream`.  Per-cluster sums are accumulated
 * across chunks in float64, in chunk order.
 *   X_host         [N][D] dtype, HOST, page-locked (cudaHostAlloc or
 *                  cudaHostRegister); read only.
 *   C0, C_out, idx_out, counts_out: as km_fit (device).
 *   objective_hist [iters] double, HOST, written; may be NULL.
 * This call is synchronous: it returns after all work finished, and reports a
 * kernel timeout as KM_ERR_TIMEOUT.
 */
int km_fit_host(const void* X_host, const void* C0, int64_t N, int D, int K, int dtype, int iters,
                int64_t chunk_rows, float* C_out, int32_t* idx_out, int32_t* counts_out,
                double* objective_hist, void* workspace, size_t workspace_bytes, void* stream);

/*
 * A source of point rows for km_fit_source: returns a pointer to the rows
 * [row0, row0 + rows) of the point set (rows x D elements of the fit's
 * dtype, row-major) in page-locked host memory.  `slot` is 0 or 1: the
 * memory returned for a slot must stay valid and unchanged until the library
 * asks for the same slot again (by then the copy out of it has completed),
 * so a source may fill two caller-owned staging buffers in turn, or point
 * into a larger pinned pool.  Return NULL to abort the fit
 * (KM_ERR_INVALID_ARG).  Called on the thread that called km_fit_source.
 */
typedef const void* (*km_chunk_source)(void* user, int64_t row0, int64_t rows, int slot);

/*
 * km_fit_host for point sets that are never held whole in host memory
 * (Flash-KMeans §2.3 Chunked Stream Overlap; §4 Results runs one billion
 * points, beyond the device's memory): the rows come chunk by chunk from
 * `source`, every iteration, in order.  The host asks for chunk c+2 once the
 * copy of chunk c has finished, so filling a staging buffer on the host
 * overlaps the copy and the compute of the chunks before it.  Same
 * arguments, results and workspace (KM_OP_FIT_HOST) as km_fit_host, with
 * `source` and `user` in place of X_host; synchronous.
 */
int km_fit_source(km_chunk_source source, void* user, const void* C0, int64_t N, int D, int K, int dtype, int iters,
                  int64_t chunk_rows, float* C_out, int32_t* idx_out, int32_t* counts_out, double* objective_hist,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * km_assign for callers that cannot allocate device memory.  Some callers
 * own every byte of device memory: a host framework that serves memory only
 * from its own pool and forbids side allocations, or a latency-critical loop
 * that cannot afford cudaMalloc's synchronisation and cost.  They pass inputs
 * and outputs as for km_assign, but no workspace: the scratch comes from one
 * static device array of KM_ASSIGN_STATIC_SCRATCH_BYTES (16 MiB) inside
 * libkm.so, which every GPU that loads the library holds until the process
 * exits.  The paper has no counterpart to this entry point.
 *   - Arguments and results are those of km_assign (same kernels).
 *   - A shape whose km_assign workspace (km_workspace_size(KM_OP_ASSIGN, ...))
 *     exceeds KM_ASSIGN_STATIC_SCRATCH_BYTES is refused with
 *     KM_ERR_UNSUPPORTED before anything is launched (bf16 with D=128 and
 *     K=1024 fits up to about 500 thousand points per call).
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Every call made outside stream capture looks up the array's device
 *     address on the current device (cudaGetSymbolAddress, with that device
 *     current), so a device reset or a re-created context is followed.  A
 *     call made while its stream is capturing uses the address cached by the
 *     last uncaptured call on that device: make the first call on a device
 *     before any stream capture (a captured call with no cached address is
 *     refused with KM_ERR_UNSUPPORTED).
 *   - All calls on one device share the array and it keeps the last call's
 *     contents; each call clears what must start at zero.  Calls that may
 *     overlap on the GPU (different streams, other threads) race on it: order
 *     them, or use km_assign with separate workspaces.
 */
#define KM_ASSIGN_STATIC_SCRATCH_BYTES ((size_t)16 << 20)
int km_assign_static(const void* X, const void* C, int B, int64_t N, int D, int K, int dtype,
                     int32_t* idx, float* mindist, double* objective, void* stream);

/*
 * Test hook for the bounded-wait machinery: launches one CTA that waits on a
 * shared-memory barrier that nothing ever arrives on, with the given limit in
 * nanoseconds (at most 10^9).  The kernel gives up, sets the workspace status
 * word and returns, leaving the context usable.  Synchronous.  Returns the
 * status km_workspace_status() then reports (KM_ERR_TIMEOUT when it works).
 */
int km_selftest_timeout(void* workspace, size_t workspace_bytes, int64_t limit_ns, void* stream);

/*
 * Data-parallel building blocks (a point set sharded by rows over several
 * devices or processes; the Lloyd iteration of Flash-KMeans §2 Methodology
 * with one exchange per iteration):
 *   km_update_accumulate: the Sort-Inverse Update of this shard (argsort,
 *     segmented sums, ordered combine) added into float64 sums [K][D] and
 *     float64 counts [K] (both zeroed first if zero_first); deterministic.
 *     Counts are float64 so that sums, counts and the objective can sit in
 *     one float64 buffer and be added across ranks by one all-reduce; they
 *     are exact integers below 2^53.  One instance; workspace as km_update
 *     (op KM_OP_UPDATE, B = 1).
 *   km_finalize_sums: C = sums / counts where counts > 0, else C is kept
 *     (C in/out float [K][D]); C_lp [K][D] (dtype; may be NULL) receives the
 *     copy the next km_assign takes (bf16 round-to-nearest-even, or float);
 *     counts_out int32 [K] may be NULL.
 * Between the two, the caller adds the shards' sums and counts (an
 * all-reduce); every rank then finalises the same sums to the same C.
 */
int km_update_accumulate(const void* X, const int32_t* idx, int64_t N, int D, int K, int dtype, double* sums,
                         double* counts, int zero_first, void* workspace, size_t workspace_bytes, void* stream);
int km_finalize_sums(const double* sums, const double* counts, int K, int D, int dtype, float* C, void* C_lp,
                     int32_t* counts_out, void* stream);

/*
 * The tiling the library chooses for a shape (no device needed): out[0..9) =
 * assignment form (0 one CTA per 128-point tile, 1 CTA pairs), centroid tile
 * width BN, point-tile buffers, centroid stages, shared memory bytes of the
 * assignment kernel, K padded to BN, sort passes, sort block size, and the
 * update's form: 0 the sort chain (count, column scan, scatter, segmented
 * sum, finalise), 1 the fused kernel with one CTA per instance (batched
 * problems of at most 8192 points and 1024 clusters).  The
 * choice is a static function of the shape and the shared-memory limit
 * (KM_ASSIGN_FORM and KM_ASSIGN_TILE=pair,BN,XB,CS override it; an override
 * that does not fit is refused).
 */
int km_plan_describe(int op, int B, int64_t N, int D, int K, int dtype, int64_t chunk_rows, int64_t* out);

/*
 * Baselines (not used by the fit).  The two strategies "Flash-KMeans" (§1
 * Problem) says FlashAssign and the Sort-Inverse Update replace, for measuring
 * the method against them on the same device:
 *   km_ablation_assign_materialized: the N x K distance matrix goes through
 *     device memory -- S = X C^T by a library GEMM (cuBLAS, fp32 out) into
 *     the workspace, chunk_rows rows at a time, then an argmin kernel reads S
 *     back: idx / mindist as km_assign (lowest index on exact ties).
 *   km_ablation_update_atomic: every point adds its row to its cluster's sum
 *     with float atomics and counts itself; C = sum / count (an empty cluster
 *     keeps C).  The atomics' order varies, so the last bits of C may differ
 *     from run to run.
 * One instance (B = 1); X [N][D] and C [K][D] in dtype (bf16 or fp32), D a
 * multiple of 8, X 16-byte aligned.  Workspace sizes: which = 0 (assign; at
 * least chunk_rows x K x 4 bytes) or 1 (update).  cuBLAS is loaded at run
 * time (libcublas.so.12); if it cannot be, the assign baseline returns
 * KM_ERR_UNSUPPORTED.
 */
size_t km_ablation_workspace_size(int which, int64_t N, int D, int K, int dtype, int64_t chunk_rows);
int km_ablation_assign_materialized(const void* X, const void* C, int64_t N, int D, int K, int dtype,
                                    int64_t chunk_rows, int32_t* idx, float* mindist, void* workspace,
                                    size_t workspace_bytes, void* stream);
int km_ablation_update_atomic(const void* X, const int32_t* idx, int64_t N, int D, int K, int dtype, float* C,
                              int32_t* counts, void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KM_H_ */
