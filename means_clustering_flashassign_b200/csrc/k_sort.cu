// k_sort.cu -- the explicit inverse map of the Sort-Inverse Update
// ("Flash-KMeans: Fast and Memory-Efficient Exact K-Means", §2.2 Sort-Inverse
// Update: argsort the assignment vector so that points of one cluster become
// contiguous).
//
// A stable least-significant-digit radix sort of (key = cluster id, value =
// point index), one or two passes of at most 12 bits.  Per pass:
//   hist     block b counts the digits of its T keys -> blkhist[digit][b]
//   colscan  one warp per digit: exclusive scan over blocks (digit-major
//            order makes the concatenation the stable counting-sort offsets)
//   scatter  each block scans the digit totals, ranks its keys stably with
//            per-warp counters (match.any groups equal digits inside a warp)
//            and writes every element to its final position.
// The sort is deterministic: equal keys keep point order, so the permutation
// is unique and the later float sums always run in the same order.
#include <cstdint>

#include "km_internal.h"

namespace km {

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ int32_t clamp_key(int32_t k, int K) { return k < 0 ? 0 : (k >= K ? K - 1 : k); }

__global__ void k_sort_hist(const int32_t* __restrict__ keys, int64_t n, int T, int shift, int R,
                            int64_t nblk, int32_t* __restrict__ blkhist, int K) {
  extern __shared__ int32_t sh[];
  constexpr int kPer = 16;  // keys per thread (T == blockDim.x * kPer)
  for (int d = threadIdx.x; d < R; d += blockDim.x) sh[d] = 0;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * T;
  const int lane = threadIdx.x & 31;
  int dig[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {  // all loads first, then the counting
    const int64_t i = t0 + static_cast<int64_t>(j) * blockDim.x + threadIdx.x;
    dig[j] = (i < n && j * static_cast<int>(blockDim.x) < T) ? ((clamp_key(keys[i], K) >> shift) & (R - 1)) : -1;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const uint32_t peers = __match_any_sync(0xffffffffu, dig[j]);
    if (dig[j] >= 0 && lane == __ffs(peers) - 1) atomicAdd(&sh[dig[j]], __popc(peers));
  }
  __syncthreads();
  for (int d = threadIdx.x; d < R; d += blockDim.x) blkhist[static_cast<int64_t>(d) * nblk + blockIdx.x] = sh[d];
}

// One warp per digit: in-place exclusive scan of blkhist[d][0..nblk) and the
// digit total.
__global__ void k_sort_colscan(int32_t* __restrict__ blkhist, int R, int64_t nblk, int32_t* __restrict__ total) {
  const int lane = threadIdx.x & 31;
  const int d = static_cast<int>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  if (d >= R) return;
  int32_t* row = blkhist + static_cast<int64_t>(d) * nblk;
  int32_t carry = 0;
  for (int64_t b0 = 0; b0 < nblk; b0 += 32) {
    const int64_t b = b0 + lane;
    const int32_t v = b < nblk ? row[b] : 0;
    int32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (b < nblk) row[b] = carry + x - v;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) total[d] = carry;
}

// Block-wide exclusive scan of total[0..R) into base[0..R) (shared memory):
// contiguous per-thread runs, a warp-shuffle scan of the run sums, then a
// scan of the warp sums by warp 0.  tmp needs blockDim.x / 32 ints.
__device__ void block_exclusive_scan(const int32_t* __restrict__ total, int R, int32_t* base, int32_t* tmp) {
  const int nt = blockDim.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = nt >> 5;
  const int per = (R + nt - 1) / nt;
  const int lo = threadIdx.x * per;
  int32_t s = 0;
  for (int i = lo; i < lo + per && i < R; ++i) s += total[i];
  int32_t x = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int32_t w = lane < nw ? tmp[lane] : 0;
    int32_t v = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane < nw) tmp[lane] = v - w;
  }
  __syncthreads();
  int32_t run = tmp[warp] + x - s;
  for (int i = lo; i < lo + per && i < R; ++i) {
    base[i] = run;
    run += total[i];
  }
  __syncthreads();
}

template <int IPT>
__global__ void k_sort_scatter(const int32_t* __restrict__ keys_in, const int32_t* __restrict__ vals_in, int64_t n,
                               int T, int shift, int R, int64_t nblk, const int32_t* __restrict__ blkhist,
                               const int32_t* __restrict__ total, int32_t* __restrict__ keys_out,
                               int32_t* __restrict__ vals_out, int32_t* __restrict__ start, int K) {
  extern __shared__ int32_t sh[];
  const int W = blockDim.x >> 5;
  int32_t* base = sh;               // [R]
  int32_t* wcnt = sh + R;           // [W][R]
  int32_t* tmp = wcnt + W * R;      // [blockDim.x / 32]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  block_exclusive_scan(total, R, base, tmp);
  if (start && blockIdx.x == 0) {
    // single-pass sorts: the digit is the cluster id, so base[] is start[]
    for (int k = threadIdx.x; k < K; k += blockDim.x) start[k] = base[k];
    if (threadIdx.x == 0) start[K] = static_cast<int32_t>(n);
  }
  for (int i = threadIdx.x; i < W * R; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();

  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * T;
  const int64_t w0 = t0 + static_cast<int64_t>(warp) * (T / W);
  int dig[IPT], rank[IPT];
  int32_t key[IPT];
  const uint32_t ltm = lanemask_lt();
#pragma unroll
  for (int s = 0; s < IPT; ++s) {  // all loads first
    const int64_t i = w0 + s * 32 + lane;
    key[s] = i < n ? clamp_key(keys_in[i], K) : 0;
    dig[s] = i < n ? ((key[s] >> shift) & (R - 1)) : -1;
  }
#pragma unroll
  for (int s = 0; s < IPT; ++s) {
    const int64_t i = w0 + s * 32 + lane;
    const bool v = i < n;
    const uint32_t peers = __match_any_sync(0xffffffffu, dig[s]);
    int before = 0;
    if (v) before = wcnt[warp * R + dig[s]];
    rank[s] = before + __popc(peers & ltm);
    __syncwarp();
    if (v && lane == __ffs(peers) - 1) wcnt[warp * R + dig[s]] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int d = threadIdx.x; d < R; d += blockDim.x) {
    int32_t run = base[d] + blkhist[static_cast<int64_t>(d) * nblk + blockIdx.x];
    for (int w = 0; w < W; ++w) {
      const int32_t c = wcnt[w * R + d];
      wcnt[w * R + d] = run;
      run += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int s = 0; s < IPT; ++s) {
    const int64_t i = w0 + s * 32 + lane;
    if (i < n) {
      const int32_t pos = wcnt[warp * R + dig[s]] + rank[s];
      vals_out[pos] = vals_in ? vals_in[i] : static_cast<int32_t>(i);
      if (keys_out) keys_out[pos] = key[s];
    }
  }
}

// start[k] for every k in [0, K] from sorted keys: each change point i (or
// the ends) writes the starts of all clusters between the two keys.
__global__ void k_bounds(const int32_t* __restrict__ sorted, int64_t n, int K, int32_t* __restrict__ start) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i > n) return;
  const int a = i == 0 ? -1 : clamp_key(sorted[i - 1], K);
  const int c = i == n ? K : clamp_key(sorted[i], K);
  for (int k = a + 1; k <= c; ++k) start[k] = static_cast<int32_t>(i);
}

static size_t scatter_smem(int R, int W, int threads) {
  return (static_cast<size_t>(R) + static_cast<size_t>(W) * R + threads) * 4;
}

cudaError_t launch_sort(const Plan& p, const SortArgs& a, cudaStream_t s) {
  const SortCfg& c = p.sc;
  const int threads = c.W * 32;
  const int64_t nblk = (a.n + c.T - 1) / c.T;
  if (a.n <= 0) return cudaSuccess;
  const int32_t* kin = a.keys;
  const int32_t* vin = nullptr;
  for (int ps = 0; ps < c.passes; ++ps) {
    const int R = 1 << c.bits[ps];
    const bool last = ps == c.passes - 1;
    count_launch(3);  // hist, colscan, scatter
    k_sort_hist<<<static_cast<unsigned>(nblk), 256, R * 4, s>>>(kin, a.n, c.T, c.shift[ps], R, nblk, a.blkhist,
                                                                a.K);
    const int cw = 8;
    k_sort_colscan<<<(R + cw - 1) / cw, cw * 32, 0, s>>>(a.blkhist, R, nblk, a.total);
    // pass 0 of two writes (keys_tmp, vals_tmp); the last pass writes perm
    // and the sorted keys (the segment id of every sorted position).
    int32_t* kout = last ? a.skeys : a.keys_tmp;
    int32_t* vout = last ? a.perm : a.vals_tmp;
    const size_t sm = scatter_smem(R, c.W, threads);
    int32_t* st = (last && c.passes == 1) ? a.start : nullptr;
    cudaError_t e = cudaFuncSetAttribute(k_sort_scatter<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sm));
    if (e != cudaSuccess) return e;
    k_sort_scatter<16><<<static_cast<unsigned>(nblk), threads, sm, s>>>(
        kin, vin, a.n, c.T, c.shift[ps], R, nblk, a.blkhist, a.total, kout, vout, st, a.K);
    kin = kout;
    vin = vout;
  }
  if (c.passes > 1) {
    const int64_t cnt = a.n + 1;
    count_launch();
    k_bounds<<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, s>>>(a.skeys, a.n, a.K, a.start);
  }
  return cudaGetLastError();
}

}  // namespace km
