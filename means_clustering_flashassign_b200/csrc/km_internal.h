// km_internal.h -- host-side plan, workspace layout and kernel launchers
// shared by the translation units of libkm.so.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

namespace km {

constexpr int kDtypeF32 = 0;
constexpr int kDtypeBF16 = 1;

// Rows of points per FlashAssign tile (UMMA M) and warps of that kernel.
constexpr int kTileM = 128;
constexpr int kAssignThreads = 576;  // warp 0 TMA, warp 1 MMA, warps 2..17 epilogue

// Largest problem the single-CTA fused update handles (batched path).
constexpr int kSmallMaxN = 8192;
constexpr int kSmallMaxK = 1024;

// Process-wide count of kernels enqueued by this library (km_launch_count).
// While this thread captures a CUDA graph, its launches are only recorded,
// so they go to the graph's own count (added at every graph launch).
inline std::atomic<uint64_t>& launch_counter() {
  static std::atomic<uint64_t> c{0};
  return c;
}
inline thread_local uint64_t* t_capture_count = nullptr;
inline void count_launch(uint64_t n = 1) {
  if (t_capture_count) *t_capture_count += n;
  else launch_counter().fetch_add(n, std::memory_order_relaxed);
}

// Host-side fault injection, for testing the error paths without faulting a
// GPU.  KM_FAULT=<point>[:<n>] in the environment (read at the entry of every
// call) makes the n-th occurrence (default 1) of that point inside the call
// fail before it is issued: "alloc" (creating a library-owned stream or
// event), "h2d" (a host-to-device chunk copy of the out-of-core fit) or
// "launch" (a kernel launch).  The call then returns KM_ERR_INJECTED after
// the same clean-up as for a real failure of that call.
enum FaultPoint { kFaultAlloc = 0, kFaultH2D = 1, kFaultLaunch = 2 };
void fault_arm_from_env();   // at call entry: parse KM_FAULT, reset the counters
bool fault_hit(int point);   // count one occurrence; true if it must fail
bool fault_fired();          // the current call failed by injection

struct AssignCfg {
  bool pair = false;   // CTA pairs with cta_group::2 UMMAs (256-point tiles)
  int BN = 0;          // centroids per UMMA tile (N of the MMA), 64/128/256
  int XB = 0;          // point-tile buffers (1 or 2)
  int CS = 0;          // centroid-tile stages
  int natoms = 0;      // 128-byte K-atoms per operand row
  int epa = 0;         // elements per atom (64 bf16, 32 fp32)
  size_t smem = 0;     // dynamic shared memory bytes
  int tmem_cols = 0;   // 2 * BN
};

struct SortCfg {
  int passes = 0;
  int bits[2] = {0, 0};
  int shift[2] = {0, 0};
  int W = 8;         // warps per block
  int IPT = 16;      // items per thread
  int T = 0;         // keys per block
  int64_t nblk = 0;  // blocks per pass
  int Rmax = 0;      // largest radix
  int segs[2] = {1, 1};  // segments of blocks each pass's column scan splits the blocks into
};

struct SegCfg {
  int BNS = 0;        // sorted positions per segmented-sum block (seg_block_positions)
  int64_t nchunks = 0;
  int big_span = 8;   // clusters spanning more chunks than this use a whole block in finalize
};

// Programmatic dependent launch for the kernels of one Lloyd iteration: a
// kernel launched this way may become resident while the previous kernel of
// the stream drains, and runs griddepcontrol.wait (pdl_wait) in every thread
// before it reads or writes anything an earlier kernel touches.  KM_PDL=0 in
// the environment launches them with plain stream order instead.
bool pdl_enabled();

// Chaining state of the calling thread's stream.  Only a kernel whose
// immediate predecessor on the stream is one of this library's chained
// kernels gets the programmatic attribute: launch_chained (and the
// assignment launcher) arm the state after enqueueing, and every other
// stream operation -- entry into the library, a memset, a copy, an event, a
// plain kernel launch -- breaks it.
void chain_break();
bool chain_armed();
void chain_arm();

template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                  Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() && chain_armed() ? 1 : 0;
  if (fault_hit(kFaultLaunch)) {
    chain_break();
    return cudaErrorLaunchFailure;
  }
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e == cudaSuccess) chain_arm();
  else chain_break();
  return e;
}

// Sorted positions per segmented-sum block for n positions: the blocks form
// one wave (148 SMs x 4 resident blocks), each a multiple of 256 positions.
constexpr int64_t kSegWaveBlocks = 148 * 4;
inline int64_t seg_block_positions(int64_t n) {
  int64_t p = (n + kSegWaveBlocks - 1) / kSegWaveBlocks;
  p = (p + 255) / 256 * 256;
  return p < 256 ? 256 : p;
}

struct Plan {
  int op = 0, B = 1, D = 0, K = 0, dtype = 0;
  int64_t N = 0;       // points per instance
  int64_t rows = 0;    // points per device pass (N in core; chunk rows out of core)
  int64_t chunk_rows = 0;
  int es = 2;          // bytes per X element
  int Dp = 0;          // fp32: D padded to 32
  int Dop = 0;         // operand row length in elements (bf16: D, fp32: 3 * Dp)
  int Kp = 0;          // K padded to a multiple of BN
  int64_t tiles_per_inst = 0, ntiles = 0;
  bool small_update = false;
  AssignCfg ac;
  SortCfg sc;
  SegCfg gc;
  // workspace offsets (bytes)
  size_t off_hdr = 0, off_xaug = 0, off_caug = 0, off_clp = 0, off_x3 = 0, off_tobj = 0, off_idx = 0;
  size_t off_blkhist = 0, off_blkhist1 = 0, off_total = 0, off_pairs_tmp = 0, off_pairs = 0, off_start = 0;
  size_t off_sums = 0, off_pl = 0, off_pr = 0, off_obj = 0, off_objpart = 0;
  size_t off_dbuf0 = 0, off_dbuf1 = 0, off_acc64 = 0, off_cnt64 = 0, off_objacc = 0;
  size_t off_rk = 0;  // the sort's packed first-pass keys
  size_t total = 0;
};

// Sets the message km_last_error() returns on the calling thread.
void set_last_error(const char* msg);

// Fills `p` for the request; returns 0 or a km_status code (message in *why).
int make_plan(Plan& p, int op, int B, int64_t N, int D, int K, int dtype, int64_t chunk_rows,
              const char** why);

// ------------------------------------------------------------- launchers
// Norm augmentation rows (32 bytes per point, see km_rows.cuh) of `rows`
// points; in f32 mode also the TF32 split operand x3 = [hi | hi | lo]
// (rows x 3*Dp floats).
cudaError_t launch_xprep(const void* X, int dtype, int64_t rows, int D, int Dp, void* xaug, float* x3,
                         cudaStream_t s);

// Centroid operand preparation for B instances of K centroids:
//   src (dtype src_dtype: bf16 or f32) -> optional float32 master copy,
//   -2c operand copy (bf16, or the TF32 split -2 [hi | lo | hi]) and the
//   augmentation rows [B][Kp] holding ||c||^2 of the values the MMA sees;
//   rows K..Kp-1 get the +inf padding row.
cudaError_t launch_cprep(const void* src, int src_dtype, int B, int K, int Kp, int D, int Dp, int dtype,
                         float* master, void* c_op, void* caug, cudaStream_t s);

// FlashAssign over B instances of `rows` points (tcgen05 / TMEM / TMA).
struct AssignArgs {
  const CUtensorMap* xmap;   // host copies, passed by value to the kernel
  const CUtensorMap* xamap;  // point augmentation rows
  const CUtensorMap* cmap;   // -2c operand
  const CUtensorMap* camap;  // centroid augmentation rows (Kp rows)
  int B;
  int64_t rows;
  int K, Kp;
  int32_t* idx;
  float* mindist;
  double* tobj;  // [B * tiles_per_inst][4]: objective partials per 128-point tile and 32-row quarter
  unsigned int* status;
  uint64_t limit_ns;
  int64_t* obj_groups;  // host out (may be null): 4-double groups of partials per instance
  const void* cop = nullptr;  // the centroid operand rows the maps cover (ties at distance 0)
  size_t cop_row_bytes = 0;
};
cudaError_t launch_assign(const Plan& p, const AssignArgs& a, cudaStream_t s);

// Objective of each instance from the assign partials (fixed order);
// groups_per_inst groups of 4 doubles per instance.
cudaError_t launch_objective(const double* tobj, int B, int64_t groups_per_inst, double* out, int out_stride,
                             cudaStream_t s);

// Stable LSD radix sort of one instance's assignment vector; writes perm and
// start[K+1] (start[k] = first sorted position of cluster k).
struct SortArgs {
  const int32_t* keys;  // the assignment vector
  int64_t n;
  int K;
  int32_t* blkhist;     // [nblk][R0] pass-0 block digit counts
  int32_t* blkhist1;    // [nblk][R1] pass-1 block digit counts (two-pass sorts only)
  int32_t* rk;          // [n] or null: the first pass stores each key with its 32-key group rank
                        // and count there, and its scatter then needs no digit ballots
  int32_t* total;       // [segs][Rmax]: digit totals of each column-scan segment
  int2* pairs_tmp;      // [n] (two-pass sorts only)
  int2* pairs;          // [n] sorted (point index, cluster id)
  int32_t* perm;        // [n] sorted point indices, or null
  int32_t* start;       // [K+1]
};
cudaError_t launch_sort(const Plan& p, const SortArgs& a, cudaStream_t s);

// Segmented sums over the sorted order + ordered boundary fix-up + centroid
// finalisation for one instance.
struct SegArgs {
  const void* X;
  int64_t n;
  const int2* pairs;      // sorted (point index, cluster id)
  const int32_t* start;
  float* sums;  // [K][D]
  float* pl;    // [nchunks][D]
  float* pr;    // [nchunks][D]
};
cudaError_t launch_segsum(const Plan& p, const SegArgs& a, cudaStream_t s);

struct FinalizeArgs {
  const int32_t* start;
  const int2* pairs;  // sorted (point, cluster) pairs
  const float* sums;
  const float* pl;
  const float* pr;
  int mode;          // 0: write centroids; 1: accumulate into acc64/cnt64
  float* C;          // [K][D] float master (in: previous, out: new)
  void* c_op;        // operand copy for the next assign (-2c, bf16 or TF32 split)
  void* caug;        // [Kp] augmentation rows
  int32_t* counts;   // [K] or null
  double* acc64;     // [K][D] (mode 1)
  long long* cnt64;  // [K] (mode 1, unless cntf)
  double* cntf;      // [K] (mode 1): float64 counts instead of cnt64, or null
  const double* tobj;
  int64_t ntiles;    // tile partials to reduce into *obj (0: none)
  double* obj;       // objective output (mode 0) or accumulator (mode 1)
  double* objpart;   // [objective_blocks(ntiles)] scratch of the reduction
  unsigned int* objcnt;  // zero on entry; left zero
};
// Blocks of the finalise kernel's objective reduction for `ntiles` 128-point
// tiles (4 partials each, 4096 partials per block).
inline int64_t objective_blocks(int64_t ntiles) { return (ntiles * 4 + 4095) / 4096; }
cudaError_t launch_finalize(const Plan& p, const FinalizeArgs& a, cudaStream_t s);
cudaError_t launch_finalize_sums(int K, int D, int dtype, const double* sums, const double* cnt, float* C,
                                 void* C_lp, int32_t* counts, cudaStream_t s);

// Final step of the out-of-core update: centroids from float64 accumulators.
cudaError_t launch_finalize_acc(const Plan& p, double* acc64, long long* cnt64, float* C, void* c_op, void* caug,
                                int32_t* counts, double* objacc, double* obj_out, cudaStream_t s);

// Fused single-CTA-per-instance update (sort + segmented sums + finalise) for
// B instances with N <= kSmallMaxN, K <= kSmallMaxK.
struct SmallUpdateArgs {
  const void* X;
  const int32_t* idx;
  float* C;
  void* c_op;  // may be null
  void* caug;  // [B][Kp] augmentation rows, may be null
  int32_t* counts;
  const double* tobj;  // may be null
  int64_t tiles_per_inst;
  double* obj;  // [B] with stride obj_stride, may be null
  int obj_stride;
};
cudaError_t launch_small_update(const Plan& p, const SmallUpdateArgs& a, cudaStream_t s);

// Test hook: one CTA waits on a barrier nothing arrives on.
cudaError_t launch_timeout_probe(unsigned int* status, uint64_t limit_ns, cudaStream_t s);

}  // namespace km
