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
#include "km_ptx.cuh"

namespace km {

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ int32_t clamp_key(int32_t k, int K) { return k < 0 ? 0 : (k >= K ? K - 1 : k); }

// Digit counts of each block's T keys, block-major: blkhist[b][d].
// Pass 0 reads the assignment vector, later passes the (point, key) pairs.
template <bool PAIRS>
__global__ void __launch_bounds__(256) k_sort_hist(const int32_t* __restrict__ keys, const int2* __restrict__ pairs,
                                                   int64_t n, int T, int shift, int R, int32_t* __restrict__ blkhist,
                                                   int K) {
  extern __shared__ int32_t sh[];
  constexpr int kPer = 16;  // keys per thread (T == blockDim.x * kPer)
  for (int d = threadIdx.x; d < R; d += blockDim.x) sh[d] = 0;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * T;
  int dig[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {  // all loads first, then the counting
    const int64_t i = t0 + static_cast<int64_t>(j) * blockDim.x + threadIdx.x;
    int key = 0;
    if (i < n) key = PAIRS ? pairs[i].y : clamp_key(keys[i], K);
    dig[j] = i < n ? ((key >> shift) & (R - 1)) : -1;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPer; ++j)
    if (dig[j] >= 0) atomicAdd(&sh[dig[j]], 1);
  __syncthreads();
  int32_t* out = blkhist + static_cast<int64_t>(blockIdx.x) * R;
  for (int d = threadIdx.x; d < R; d += blockDim.x) out[d] = sh[d];
}

// In-place exclusive scan of blkhist[0..nblk)[d] over the blocks, and the
// digit totals.  A block takes 32 digits (one per lane, so every load is
// coalesced) and splits the block range among its 32 warps: each warp sums
// its part, the parts are scanned in shared memory, and each warp rewrites
// its part as running prefixes.  (Up to 8K blocks the parts are at most 8
// rows: one batch of loads per warp.)
constexpr int kColscanWarps = 32;
__global__ void __launch_bounds__(kColscanWarps * 32) k_sort_colscan(int32_t* __restrict__ blkhist, int R,
                                                                     int64_t nblk, int32_t* __restrict__ total) {
  __shared__ int32_t part[kColscanWarps][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int d = blockIdx.x * 32 + lane;
  const bool ok = d < R;
  const int64_t seg = (nblk + kColscanWarps - 1) / kColscanWarps;
  const int64_t b0 = warp * seg < nblk ? warp * seg : nblk;
  const int64_t b1 = b0 + seg < nblk ? b0 + seg : nblk;
  constexpr int CH = 8;
  int32_t s = 0;
  for (int64_t b = b0; b < b1; b += CH) {
    int32_t v[CH];
#pragma unroll
    for (int u = 0; u < CH; ++u) v[u] = (ok && b + u < b1) ? blkhist[(b + u) * R + d] : 0;
#pragma unroll
    for (int u = 0; u < CH; ++u) s += v[u];
  }
  part[warp][lane] = s;
  __syncthreads();
  int32_t run = 0;
  for (int w = 0; w < warp; ++w) run += part[w][lane];
  if (warp == kColscanWarps - 1 && ok) total[d] = run + s;
  for (int64_t b = b0; b < b1; b += CH) {
    int32_t v[CH];
#pragma unroll
    for (int u = 0; u < CH; ++u) v[u] = (ok && b + u < b1) ? blkhist[(b + u) * R + d] : 0;
#pragma unroll
    for (int u = 0; u < CH; ++u) {
      if (ok && b + u < b1) blkhist[(b + u) * R + d] = run;
      run += v[u];
    }
  }
}

// Block-wide exclusive scan of total[0..R) into base[0..R) (shared memory;
// base may alias total): contiguous per-thread runs, a warp-shuffle scan of
// the run sums, then a scan of the warp sums by warp 0.  tmp needs
// blockDim.x / 32 ints.
__device__ void block_exclusive_scan(const int32_t* total, int R, int32_t* base, int32_t* tmp) {
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
    const int32_t t = total[i];
    base[i] = run;
    run += t;
  }
  __syncthreads();
}

// Stable scatter of one pass: per-warp counters rank equal digits in point
// order (match_digit groups equal digits inside a warp step).  The block first
// places its elements in digit order in shared memory, then writes them out
// in that order, so elements of one digit leave as one contiguous run at
// base[d] + (earlier blocks' d).  Writes one 8-byte (point, key) pair per
// element, and optionally the bare point index (perm_out) on the last pass.
template <int IPT, bool PAIRS>
__global__ void k_sort_scatter(const int32_t* __restrict__ keys_in, const int2* __restrict__ pairs_in, int64_t n,
                               int T, int shift, int R, int32_t* __restrict__ blkhist,
                               const int32_t* __restrict__ total, int2* __restrict__ pairs_out,
                               int32_t* __restrict__ perm_out, int32_t* __restrict__ start, int K) {
  extern __shared__ int32_t sh[];
  const int W = blockDim.x >> 5;
  int2* stage = reinterpret_cast<int2*>(sh);   // [T]
  int32_t* base = sh + 2 * T;                  // [R]  global start of each digit in this block
  int32_t* lstart = base + R;                  // [R]  block-local start of each digit
  int32_t* wcnt = lstart + R;                  // [W][R]
  int32_t* tmp = wcnt + W * R;                 // [blockDim.x / 32]
  int32_t* bo = tmp + (blockDim.x >> 5);       // [R]  earlier blocks' count of each digit
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* boff = blkhist + static_cast<int64_t>(blockIdx.x) * R;
  int bits = 0;
  while ((1 << bits) < R) ++bits;

  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * T;
  const int64_t w0 = t0 + static_cast<int64_t>(warp) * (T / W);
  int dig[IPT], rank[IPT];
  int32_t key[IPT], val[IPT];
  const uint32_t ltm = lanemask_lt();
#pragma unroll
  for (int s = 0; s < IPT; ++s) {  // all loads first
    const int64_t i = w0 + s * 32 + lane;
    if (PAIRS) {
      const int2 pk = i < n ? pairs_in[i] : make_int2(0, 0);
      val[s] = pk.x;
      key[s] = pk.y;
    } else {
      val[s] = static_cast<int32_t>(i);
      key[s] = i < n ? clamp_key(keys_in[i], K) : 0;
    }
    dig[s] = i < n ? ((key[s] >> shift) & (R - 1)) : -1;
  }
  // While the keys are in flight: the digit totals and this block's offsets
  // into shared memory, per-warp counters zeroed; then the digit bases.
  for (int d = threadIdx.x; d < R; d += blockDim.x) {
    base[d] = total[d];
    bo[d] = boff[d];
  }
  for (int i = threadIdx.x; i < W * R; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  block_exclusive_scan(base, R, base, tmp);
  if (start && blockIdx.x == 0) {
    // single-pass sorts: the digit is the cluster id, so base[] is start[]
    for (int k = threadIdx.x; k < K; k += blockDim.x) start[k] = base[k];
    if (threadIdx.x == 0) start[K] = static_cast<int32_t>(n);
  }
#pragma unroll
  for (int s = 0; s < IPT; ++s) {
    const int64_t i = w0 + s * 32 + lane;
    const bool v = i < n;
    const uint32_t peers = match_digit(dig[s], bits, v);
    int before = 0;
    if (v) before = wcnt[warp * R + dig[s]];
    rank[s] = before + __popc(peers & ltm);
    __syncwarp();
    if (v && lane == __ffs(peers) - 1) wcnt[warp * R + dig[s]] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per digit: block count -> block-local starts (scan over digits), then
  // warp offsets inside the digit's local run
  for (int d = threadIdx.x; d < R; d += blockDim.x) {
    int32_t c = 0;
    for (int w = 0; w < W; ++w) c += wcnt[w * R + d];
    lstart[d] = c;
  }
  __syncthreads();
  block_exclusive_scan(lstart, R, lstart, tmp);
  for (int d = threadIdx.x; d < R; d += blockDim.x) {
    int32_t run = lstart[d];
    for (int w = 0; w < W; ++w) {
      const int32_t c = wcnt[w * R + d];
      wcnt[w * R + d] = run;
      run += c;
    }
    base[d] += bo[d] - lstart[d];  // global position = base[d] + local position
    boff[d] = 0;  // leave the counts zeroed for the next accumulation
  }
  __syncthreads();
#pragma unroll
  for (int s = 0; s < IPT; ++s) {
    if (dig[s] >= 0) stage[wcnt[warp * R + dig[s]] + rank[s]] = make_int2(val[s], key[s]);
  }
  __syncthreads();
  const int nvalid = static_cast<int>((n - t0) < T ? (n - t0) : T);
  for (int i = threadIdx.x; i < nvalid; i += blockDim.x) {
    const int2 pk = stage[i];
    const int64_t pos = static_cast<int64_t>(base[(pk.y >> shift) & (R - 1)]) + i;
    // Counts accumulated elsewhere (the assignment kernel) agree with these
    // keys unless that kernel gave up on a bounded wait; stay in bounds then.
    if (pos < 0 || pos >= n) continue;
    pairs_out[pos] = pk;
    if (perm_out) perm_out[pos] = pk.x;
  }
}

// start[k] for every k in [0, K] from the sorted pairs: each change point i
// (or the ends) writes the starts of all clusters between the two keys.
__global__ void k_bounds(const int2* __restrict__ sorted, int64_t n, int K, int32_t* __restrict__ start) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i > n) return;
  const int a = i == 0 ? -1 : clamp_key(sorted[i - 1].y, K);
  const int c = i == n ? K : clamp_key(sorted[i].y, K);
  for (int k = a + 1; k <= c; ++k) start[k] = static_cast<int32_t>(i);
}

static size_t scatter_smem(int R, int W, int threads, int T) {
  return (2 * static_cast<size_t>(T) + 3 * static_cast<size_t>(R) + static_cast<size_t>(W) * R + threads) * 4;
}

cudaError_t launch_sort(const Plan& p, const SortArgs& a, cudaStream_t s) {
  const SortCfg& c = p.sc;
  const int threads = c.W * 32;
  const int64_t nblk = (a.n + c.T - 1) / c.T;
  if (a.n <= 0) return cudaSuccess;
  for (int ps = 0; ps < c.passes; ++ps) {
    const int R = 1 << c.bits[ps];
    const bool last = ps == c.passes - 1;
    const bool pairs_in = ps > 0;
    int32_t* bh = ps == 0 ? a.blkhist : a.blkhist1;
    count_launch(ps == 0 && a.hist0_ready ? 2 : 3);  // [hist,] colscan, scatter
    if (pairs_in)
      k_sort_hist<true><<<static_cast<unsigned>(nblk), 256, R * 4, s>>>(nullptr, a.pairs_tmp, a.n, c.T, c.shift[ps],
                                                                        R, bh, a.K);
    else if (!a.hist0_ready)
      k_sort_hist<false><<<static_cast<unsigned>(nblk), 256, R * 4, s>>>(a.keys, nullptr, a.n, c.T, c.shift[ps], R,
                                                                         bh, a.K);
    k_sort_colscan<<<(R + 31) / 32, kColscanWarps * 32, 0, s>>>(bh, R, nblk, a.total);
    // pass 0 of two writes pairs_tmp; the last pass writes the sorted pairs
    // (and perm when asked for).
    int2* out = last ? a.pairs : a.pairs_tmp;
    int32_t* perm = last ? a.perm : nullptr;
    const size_t sm = scatter_smem(R, c.W, threads, c.T);
    int32_t* st = (last && c.passes == 1) ? a.start : nullptr;
    cudaError_t e;
    if (pairs_in) {
      e = cudaFuncSetAttribute(k_sort_scatter<16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(sm));
      if (e != cudaSuccess) return e;
      k_sort_scatter<16, true><<<static_cast<unsigned>(nblk), threads, sm, s>>>(
          nullptr, a.pairs_tmp, a.n, c.T, c.shift[ps], R, bh, a.total, out, perm, st, a.K);
    } else {
      e = cudaFuncSetAttribute(k_sort_scatter<16, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(sm));
      if (e != cudaSuccess) return e;
      k_sort_scatter<16, false><<<static_cast<unsigned>(nblk), threads, sm, s>>>(
          a.keys, nullptr, a.n, c.T, c.shift[ps], R, bh, a.total, out, perm, st, a.K);
    }
  }
  if (c.passes > 1) {
    const int64_t cnt = a.n + 1;
    count_launch();
    k_bounds<<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, s>>>(a.pairs, a.n, a.K, a.start);
  }
  return cudaGetLastError();
}

}  // namespace km
