// k_sort.cu -- the explicit inverse map of the Sort-Inverse Update
// ("Flash-KMeans: Fast and Memory-Efficient Exact K-Means", §2.2 Sort-Inverse
// Update: argsort the assignment vector so that points of one cluster become
// contiguous).
//
// A stable least-significant-digit radix sort of (key = cluster id, value =
// point index), one or two passes of at most 12 bits.  Per pass:
//   count    block b counts the digits of its T keys -> blkhist[b][digit],
//            per 32-key group with ballots (one shared-memory add per
//            distinct digit of a group, so a hot digit does not serialise);
//            on the first pass it also stores each key with its rank and
//            count among the equal digits of its group, for the scatter
//   colscan  one lane per digit: exclusive scan over the blocks of each
//            digit's counts, plus the digit totals (digit-major order of the
//            runs makes the concatenation the stable counting-sort offsets)
//   scatter  each block ranks its keys stably with per-warp counters
//            (equal digits inside a warp step grouped by ballots, or taken
//            from the ranks the count kernel stored), scans the digit
//            totals and its own digit counts, and writes every element to
//            its final position.
// Cluster starts: a one-pass sort's digit is the cluster id, so the scatter
// writes start[]; a two-pass sort finds them in the sorted keys (k_bounds).
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

constexpr int kSortThreads = 256;
constexpr int kSortWarps = kSortThreads / 32;

// Digit counts of each block's T keys, block-major blkhist[b][d].  The
// block's 32 warps take STEPS = T / 1024 steps of 32 consecutive keys each
// (all loads issued first).  The lanes of a step with equal digits are found
// with one ballot per digit bit, each lane keeping the lanes whose bit agrees
// with its own; the lowest of them adds their number to the block's count.
// With rk: rk[i] = key | rank << 20 | (count - 1) << 25, the key's rank
// among the equal digits of its aligned 32-key group and their number, as
// the scatter ranks them (on a pass over pairs the key bits are 0: that
// scatter reads the key from the pair).
constexpr int kCountThreads = 1024;
template <int STEPS, bool PAIRS>
__global__ void __launch_bounds__(kCountThreads) k_sort_count(const int32_t* __restrict__ keys,
                                                              const int2* __restrict__ pairs, int64_t n, int shift,
                                                              int R, int bits, int32_t* __restrict__ blkhist,
                                                              int32_t* __restrict__ rk, int K) {
  constexpr int T = kCountThreads * STEPS;
  extern __shared__ int32_t sh[];
  pdl_trigger();
  for (int d = threadIdx.x; d < R; d += kCountThreads) sh[d] = 0;
  pdl_wait();
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t w0 = static_cast<int64_t>(blockIdx.x) * T + static_cast<int64_t>(warp) * (32 * STEPS);
  int32_t key[STEPS];
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    const int64_t i = w0 + 32 * s + lane;
    key[s] = i < n ? (PAIRS ? pairs[i].y : clamp_key(keys[i], K)) : 0;
  }
  const uint32_t lt = lanemask_lt();
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    const int64_t i = w0 + 32 * s + lane;
    const bool valid = i < n;
    const int dig = (key[s] >> shift) & (R - 1);
    const uint32_t dz = valid ? static_cast<uint32_t>(dig) : 0u;
    uint32_t peers = __ballot_sync(0xffffffffu, valid);
    auto narrow = [&](int bit) {
      const uint32_t b = (dz >> bit) & 1u;
      const uint32_t bb = __ballot_sync(0xffffffffu, b != 0u);
      peers &= ~(bb ^ (0u - b));
    };
    int bit = 0;
    for (; bit + 4 <= bits; bit += 4) {
      narrow(bit);
      narrow(bit + 1);
      narrow(bit + 2);
      narrow(bit + 3);
    }
    for (; bit < bits; ++bit) narrow(bit);
    if (!valid) continue;
    const int rank = __popc(peers & lt), cnt = __popc(peers);
    if (rank == 0) atomicAdd(&sh[dig], cnt);
    if (rk) rk[i] = (PAIRS ? 0 : key[s]) | (rank << 20) | ((cnt - 1) << 25);
  }
  __syncthreads();
  int32_t* out = blkhist + static_cast<int64_t>(blockIdx.x) * R;
  for (int d = threadIdx.x; d < R; d += kCountThreads) out[d] = sh[d];
}

// In-place exclusive scan of blkhist[0..nblk)[d] over the blocks (within
// segments of blocks, see k_sort_colscan), and the digit totals of each
// segment.  Each warp sums its part of the segment, the parts are scanned in
// shared memory, and each warp rewrites its part as running prefixes.
constexpr int kColscanWarps = 32;

// The block counts are scanned in S segments of consecutive sort blocks, so
// that few digits still spread over many CTAs: CTA (g, s) takes digits
// [32 g, 32 g + 32) (one per lane, every load coalesced) and the blocks of
// segment s, split among its 32 warps; it rewrites them in place as prefixes
// within the segment and stores the segment's digit totals in segtot[s][d].
// The scatter adds the totals of the earlier segments (and sums all of them
// for the digit totals).
__global__ void __launch_bounds__(kColscanWarps * 32) k_sort_colscan(int32_t* __restrict__ blkhist, int R,
                                                                     int64_t nblk, int S,
                                                                     int32_t* __restrict__ segtot) {
  __shared__ int32_t part[kColscanWarps][32];
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int groups = (R + 31) / 32;
  const int g = static_cast<int>(blockIdx.x) % groups, sg = static_cast<int>(blockIdx.x) / groups;
  const int d = g * 32 + lane;
  const bool ok = d < R;
  const int64_t L = (nblk + S - 1) / S;
  const int64_t r0 = sg * L < nblk ? sg * L : nblk;
  const int64_t r1 = r0 + L < nblk ? r0 + L : nblk;
  const int64_t seg = (r1 - r0 + kColscanWarps - 1) / kColscanWarps;
  const int64_t b0 = r0 + warp * seg < r1 ? r0 + warp * seg : r1;
  const int64_t b1 = b0 + seg < r1 ? b0 + seg : r1;
  // The first KEEP rows of the warp's part stay in registers for the second
  // pass (all of it up to 512 blocks); rows beyond are read again.
  constexpr int KEEP = 16, CH = 8;
  int32_t keep[KEEP];
#pragma unroll
  for (int u = 0; u < KEEP; ++u) keep[u] = (ok && b0 + u < b1) ? blkhist[(b0 + u) * R + d] : 0;
  int32_t s = 0;
  for (int64_t b = b0 + KEEP; b < b1; b += CH) {
    int32_t v[CH];
#pragma unroll
    for (int u = 0; u < CH; ++u) v[u] = (ok && b + u < b1) ? blkhist[(b + u) * R + d] : 0;
#pragma unroll
    for (int u = 0; u < CH; ++u) s += v[u];
  }
#pragma unroll
  for (int u = 0; u < KEEP; ++u) s += keep[u];
  part[warp][lane] = s;
  __syncthreads();
  int32_t run = 0;
#pragma unroll
  for (int w = 0; w < kColscanWarps; ++w)
    if (w < warp) run += part[w][lane];
  if (warp == kColscanWarps - 1 && ok) segtot[static_cast<int64_t>(sg) * R + d] = run + s;
#pragma unroll
  for (int u = 0; u < KEEP; ++u) {
    if (ok && b0 + u < b1) blkhist[(b0 + u) * R + d] = run;
    run += keep[u];
  }
  for (int64_t b = b0 + KEEP; b < b1; b += CH) {
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

// RPT consecutive ints (RPT = 1, 2 or a multiple of 4; p aligned to them).
template <int RPT>
__device__ __forceinline__ void ld_run(const int32_t* p, int32_t (&v)[RPT]) {
  if constexpr (RPT % 4 == 0) {
#pragma unroll
    for (int q = 0; q < RPT / 4; ++q) {
      const int4 x = reinterpret_cast<const int4*>(p)[q];
      v[4 * q] = x.x;
      v[4 * q + 1] = x.y;
      v[4 * q + 2] = x.z;
      v[4 * q + 3] = x.w;
    }
  } else if constexpr (RPT == 2) {
    const int2 x = *reinterpret_cast<const int2*>(p);
    v[0] = x.x;
    v[1] = x.y;
  } else {
    v[0] = p[0];
  }
}

// ld_run from device memory through L2 only (ld.global.cg): for arrays an
// earlier kernel of the same chained sequence may have read into this SM's
// L1 before a later kernel rewrote them (see k_sort_scatter).
template <int RPT>
__device__ __forceinline__ void ld_run_l2(const int32_t* p, int32_t (&v)[RPT]) {
  if constexpr (RPT % 4 == 0) {
#pragma unroll
    for (int q = 0; q < RPT / 4; ++q) {
      const int4 x = __ldcg(reinterpret_cast<const int4*>(p) + q);
      v[4 * q] = x.x;
      v[4 * q + 1] = x.y;
      v[4 * q + 2] = x.z;
      v[4 * q + 3] = x.w;
    }
  } else if constexpr (RPT == 2) {
    const int2 x = __ldcg(reinterpret_cast<const int2*>(p));
    v[0] = x.x;
    v[1] = x.y;
  } else {
    v[0] = __ldcg(p);
  }
}

template <int RPT>
__device__ __forceinline__ void st_run(int32_t* p, const int32_t (&v)[RPT]) {
  if constexpr (RPT % 4 == 0) {
#pragma unroll
    for (int q = 0; q < RPT / 4; ++q)
      reinterpret_cast<int4*>(p)[q] = make_int4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  } else if constexpr (RPT == 2) {
    *reinterpret_cast<int2*>(p) = make_int2(v[0], v[1]);
  } else {
    p[0] = v[0];
  }
}

// Exclusive scan over the block's threads of two values per thread at once;
// red holds 2 x kSortWarps ints.  Ends with the block synchronised.
__device__ __forceinline__ void block_scan_pair(int32_t a, int32_t b, int32_t& ea, int32_t& eb, int32_t* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t x = a, y = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t u = __shfl_up_sync(0xffffffffu, x, o);
    const int32_t v = __shfl_up_sync(0xffffffffu, y, o);
    if (lane >= o) {
      x += u;
      y += v;
    }
  }
  if (lane == 31) {
    red[warp] = x;
    red[kSortWarps + warp] = y;
  }
  __syncthreads();
  int32_t pa = 0, pb = 0;
#pragma unroll
  for (int w = 0; w < kSortWarps; ++w)
    if (w < warp) {
      pa += red[w];
      pb += red[kSortWarps + w];
    }
  ea = pa + x - a;
  eb = pb + y - b;
}

// Stable scatter of one pass, one block per T = 256 * IPT keys.  Warp w
// takes keys [w T/8, (w+1) T/8) of the block in IPT steps of 32; per-warp
// counters rank equal digits in point order (match_digit groups equal digits
// of one step; every step's groups are found before the counter chain, so
// the chain is one shared load and one store per step).  Thread t owns the
// RPT digits [t RPT, (t+1) RPT): it scans the digit totals and the block's
// counts of them (one two-value block scan), turns the per-warp counts into
// warp offsets inside the digit's block-local run, and keeps the digit's
// global position minus its local start.  The block then places its keys in
// digit order in shared memory and writes them out in that order, so the
// elements of one digit leave as one contiguous run.  Writes one 8-byte
// (point, key) pair per element, and optionally the bare point index
// (perm_out) on the last pass.
// Resident blocks per SM the register budget is sized for: what the shared
// memory (2T + 9R ints) admits, 1 to 4.
template <int IPT, int RPT, bool PAIRS, bool PRE>
__global__ void __launch_bounds__(kSortThreads, RPT >= 16 ? 1 : (IPT <= 8 && RPT < 8 ? 4 : 2)) k_sort_scatter(
    const int32_t* __restrict__ keys_in, const int2* __restrict__ pairs_in, int64_t n, int shift, int R, int bits,
    int32_t* __restrict__ blkhist, const int32_t* __restrict__ segtot, int S, int64_t L,
    int2* __restrict__ pairs_out, int32_t* __restrict__ perm_out, int32_t* __restrict__ start, int K) {
  constexpr int W = kSortWarps;
  constexpr int T = kSortThreads * IPT;
  extern __shared__ __align__(16) int32_t sh[];
  int2* stage = reinterpret_cast<int2*>(sh);  // [T]
  int32_t* wcnt = sh + 2 * T;                 // [W][R]
  int32_t* gpos = wcnt + W * R;               // [R] global position of the digit's run minus its local start
  int32_t* red = gpos + R;                    // [2][W]
  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d0 = tid * RPT;
  const bool owner = d0 < R;
  if (owner) {
    const int32_t z[RPT] = {};
#pragma unroll
    for (int w = 0; w < W; ++w) st_run<RPT>(wcnt + w * R + d0, z);
  }
  {
    // While the previous kernel drains: pull this block's keys into L2.
    const int64_t first = static_cast<int64_t>(blockIdx.x) * T;
    const int64_t line = first + static_cast<int64_t>(tid) * (PAIRS ? 16 : 32);
    if (tid < T / (PAIRS ? 16 : 32) && line < n) {
      if (PAIRS) prefetch_l2(pairs_in + line);
      else prefetch_l2(keys_in + line);
    }
  }
  pdl_wait();

  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * T;
  const int64_t w0 = t0 + static_cast<int64_t>(warp) * (T / W);
  // step s of this lane holds point w0 + 32 s + lane (valid while < n); its
  // digit is computed from the key where needed
  const int64_t nw = n - w0 - lane;  // steps s with 32 s < nw are valid
  auto valid = [&](int s) { return 32 * s < nw; };
  auto digit = [&](int32_t k) { return (k >> shift) & (R - 1); };
  int32_t key[IPT], val[PAIRS ? IPT : 1];
  // PRE: the key word (keys_in) also holds the point's rank among the equal
  // digits of its 32-point group (bits 20..24) and the group's count of that
  // digit minus one (bits 25..29), as the count kernel found them; over
  // pairs only those bits are used.  The rank array, like the digit totals,
  // is rewritten by the second pass after the first pass's scatter read it,
  // and a chained kernel can become resident while its predecessors still
  // run: reading such arrays through the non-coherent L1 path returned the
  // first pass's lines in the second pass (repeated fits stopped being
  // bit-identical), so they are read through L2 (ld.global.cg).
  uint32_t pre[PRE ? IPT : 1];
#pragma unroll
  for (int s = 0; s < IPT; ++s) {  // all loads first
    const int64_t i = w0 + s * 32 + lane;
    if constexpr (PAIRS) {
      const int2 pk = i < n ? pairs_in[i] : make_int2(0, 0);
      val[s] = pk.x;
      key[s] = pk.y;
      if constexpr (PRE) pre[s] = i < n ? static_cast<uint32_t>(__ldcg(keys_in + i)) >> 20 : 0u;
    } else if constexpr (PRE) {
      const int32_t w = i < n ? __ldcg(keys_in + i) : 0;
      key[s] = clamp_key(w & 0xFFFFF, K);
      pre[s] = static_cast<uint32_t>(w) >> 20;
    } else {
      key[s] = i < n ? clamp_key(keys_in[i], K) : 0;
    }
  }
  int32_t* boff = blkhist + static_cast<int64_t>(blockIdx.x) * R;
  // digit totals (all segments) and this block's offsets (its prefix inside
  // its segment plus the totals of the earlier segments)
  int32_t tot[RPT] = {}, bo[RPT] = {};
  if (owner) {
    ld_run_l2<RPT>(boff + d0, bo);
    const int sb = static_cast<int>(static_cast<int64_t>(blockIdx.x) / L);
    for (int s2 = 0; s2 < S; ++s2) {
      int32_t v[RPT];
      ld_run_l2<RPT>(segtot + static_cast<int64_t>(s2) * R + d0, v);
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        tot[j] += v[j];
        if (s2 < sb) bo[j] += v[j];
      }
    }
  }
  // digit bits: R = 256 RPT exactly when RPT > 1; at most 8 when RPT == 1
  constexpr int NB = RPT == 1 ? 8 : RPT == 2 ? 9 : RPT == 4 ? 10 : RPT == 8 ? 11 : 12;
  // per step: this lane's rank among the step's lanes of equal digit, and
  // (on the group's first lane) the group's size
  uint32_t gr[IPT], gn[IPT];
  if constexpr (PRE) {
#pragma unroll
    for (int s = 0; s < IPT; ++s) {
      gr[s] = pre[s] & 31u;
      gn[s] = ((pre[s] >> 5) & 31u) + 1u;
    }
  } else {
    const uint32_t ltm = lanemask_lt();
#pragma unroll
    for (int s = 0; s < IPT; ++s) {
      const uint32_t peers = match_digit<NB>(digit(key[s]), bits, valid(s));
      gr[s] = __popc(peers & ltm);
      gn[s] = __popc(peers);
    }
  }
  __syncthreads();  // counters zeroed

  int32_t rank[IPT];
#pragma unroll
  for (int s = 0; s < IPT; ++s) {
    const bool v = valid(s);
    int32_t* cp = wcnt + warp * R + digit(key[s]);
    const int32_t before = v ? *cp : 0;
    rank[s] = before + static_cast<int32_t>(gr[s]);
    __syncwarp();
    if (v && gr[s] == 0) *cp = before + static_cast<int32_t>(gn[s]);
    __syncwarp();
  }
  __syncthreads();

  // block count of each owned digit, then both scans over the digits
  int32_t cnt[RPT] = {};
  if (owner) {
#pragma unroll
    for (int w = 0; w < W; ++w) {
      int32_t c[RPT];
      ld_run<RPT>(wcnt + w * R + d0, c);
#pragma unroll
      for (int j = 0; j < RPT; ++j) cnt[j] += c[j];
    }
  }
  int32_t sT = 0, sC = 0;
#pragma unroll
  for (int j = 0; j < RPT; ++j) {
    sT += tot[j];
    sC += cnt[j];
  }
  int32_t eT, eC;
  block_scan_pair(sT, sC, eT, eC, red);
  if (owner) {
    int32_t dbase = eT, lstart = eC;
    int32_t gp[RPT];
    int32_t run[RPT];
#pragma unroll
    for (int j = 0; j < RPT; ++j) {
      // single-pass sorts: the digit is the cluster id, so the digit base is start[]
      if (start && blockIdx.x == 0 && d0 + j < K) start[d0 + j] = dbase;
      gp[j] = dbase + bo[j] - lstart;
      run[j] = lstart;
      dbase += tot[j];
      lstart += cnt[j];
    }
    st_run<RPT>(gpos + d0, gp);
#pragma unroll
    for (int w = 0; w < W; ++w) {
      int32_t c[RPT];
      ld_run<RPT>(wcnt + w * R + d0, c);
      st_run<RPT>(wcnt + w * R + d0, run);
#pragma unroll
      for (int j = 0; j < RPT; ++j) run[j] += c[j];
    }
  }
  if (start && blockIdx.x == 0 && tid == 0) start[K] = static_cast<int32_t>(n);
  __syncthreads();
  // all slot lookups, then all stores (they do not wait on each other)
#pragma unroll
  for (int s = 0; s < IPT; ++s) rank[s] = valid(s) ? wcnt[warp * R + digit(key[s])] + rank[s] : -1;
#pragma unroll
  for (int s = 0; s < IPT; ++s) {
    const int32_t pt = PAIRS ? val[PAIRS ? s : 0] : static_cast<int32_t>(w0 + s * 32 + lane);
    // ranks are below T; the check keeps the stage safe whatever the counts
    if (rank[s] >= 0 && rank[s] < T) stage[rank[s]] = make_int2(pt, key[s]);
  }
  __syncthreads();
  const int64_t left = n - t0;
  const int nvalid = static_cast<int>(left < T ? left : T);
  // staged elements in order, then their run positions, then the stores
  int2 pk[IPT];
  int32_t gp[IPT];
#pragma unroll
  for (int s = 0; s < IPT; ++s) pk[s] = s * kSortThreads + tid < nvalid ? stage[s * kSortThreads + tid] : make_int2(0, 0);
#pragma unroll
  for (int s = 0; s < IPT; ++s) gp[s] = gpos[digit(pk[s].y)];
#pragma unroll
  for (int s = 0; s < IPT; ++s) {
    const int i = s * kSortThreads + tid;
    const int64_t pos = static_cast<int64_t>(gp[s]) + i;
    // positions lie in [0, n) when the counts match the keys; checked anyway
    if (i < nvalid && pos >= 0 && pos < n) {
      pairs_out[pos] = pk[s];
      if (perm_out) perm_out[pos] = pk[s].x;
    }
  }
}

// start[k] for every k in [0, K] from the sorted pairs: each change point i
// (or the ends) writes the starts of all clusters between the two keys.
// A thread covers kBoundsPer consecutive positions (two 16-byte loads).
constexpr int kBoundsPer = 4;
__global__ void k_bounds(const int2* __restrict__ sorted, int64_t n, int K, int32_t* __restrict__ start) {
  pdl_trigger();
  pdl_wait();
  const int64_t i0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * kBoundsPer;
  if (i0 > n) return;
  int key[kBoundsPer];
  if (i0 + kBoundsPer <= n) {
    const int4* q = reinterpret_cast<const int4*>(sorted + i0);  // 32-byte aligned: i0 is a multiple of 4
    const int4 u = q[0], w = q[1];
    key[0] = u.y;
    key[1] = u.w;
    key[2] = w.y;
    key[3] = w.w;
  } else {
#pragma unroll
    for (int j = 0; j < kBoundsPer; ++j) key[j] = i0 + j < n ? sorted[i0 + j].y : K;
  }
  int a = i0 == 0 ? -1 : clamp_key(sorted[i0 - 1].y, K);
#pragma unroll
  for (int j = 0; j < kBoundsPer; ++j) {
    const int64_t i = i0 + j;
    if (i > n) break;
    const int c = i == n ? K : clamp_key(key[j], K);
    for (int k = a + 1; k <= c; ++k) start[k] = static_cast<int32_t>(i);
    a = c;
  }
}

// Digits per scatter thread for radix R: R / 256, at least 1.
static int scatter_rpt(int R) { return R <= kSortThreads ? 1 : R / kSortThreads; }

static size_t scatter_smem(int R, int T) {
  return (2 * static_cast<size_t>(T) + static_cast<size_t>(kSortWarps + 1) * R + 2 * kSortWarps) * 4;
}

template <int IPT, int RPT, bool PAIRS, bool PRE>
static cudaError_t launch_scatter_t(int64_t nblk, size_t sm, cudaStream_t s, const int32_t* keys, const int2* pin,
                                    int64_t n, int shift, int R, int bits, int32_t* bh, const int32_t* total,
                                    int S, int64_t L, int2* out, int32_t* perm, int32_t* st, int K) {
  auto kern = k_sort_scatter<IPT, RPT, PAIRS, PRE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
  if (e != cudaSuccess) return e;
  return launch_chained(kern, dim3(static_cast<unsigned>(nblk)), dim3(kSortThreads), sm, s, keys, pin, n, shift, R,
                        bits, bh, total, S, L, out, perm, st, K);
}

template <int IPT, bool PAIRS, bool PRE>
static cudaError_t launch_scatter_r(int rpt, int64_t nblk, size_t sm, cudaStream_t s, const int32_t* keys,
                                    const int2* pin, int64_t n, int shift, int R, int bits, int32_t* bh,
                                    const int32_t* total, int S, int64_t L, int2* out, int32_t* perm, int32_t* st,
                                    int K) {
  switch (rpt) {
    case 1: return launch_scatter_t<IPT, 1, PAIRS, PRE>(nblk, sm, s, keys, pin, n, shift, R, bits, bh, total, S, L, out, perm, st, K);
    case 2: return launch_scatter_t<IPT, 2, PAIRS, PRE>(nblk, sm, s, keys, pin, n, shift, R, bits, bh, total, S, L, out, perm, st, K);
    case 4: return launch_scatter_t<IPT, 4, PAIRS, PRE>(nblk, sm, s, keys, pin, n, shift, R, bits, bh, total, S, L, out, perm, st, K);
    case 8: return launch_scatter_t<IPT, 8, PAIRS, PRE>(nblk, sm, s, keys, pin, n, shift, R, bits, bh, total, S, L, out, perm, st, K);
    case 16: return launch_scatter_t<IPT, 16, PAIRS, PRE>(nblk, sm, s, keys, pin, n, shift, R, bits, bh, total, S, L, out, perm, st, K);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_sort(const Plan& p, const SortArgs& a, cudaStream_t s) {
  const SortCfg& c = p.sc;
  const int64_t nblk = (a.n + c.T - 1) / c.T;
  if (a.n <= 0) return cudaSuccess;
  if (c.T != kSortThreads * c.IPT || (c.IPT != 8 && c.IPT != 16)) return cudaErrorInvalidValue;
  cudaError_t e;
  for (int ps = 0; ps < c.passes; ++ps) {
    const int bits = c.bits[ps];
    const int R = 1 << bits;
    const bool last = ps == c.passes - 1;
    const bool pairs_in = ps > 0;
    int32_t* bh = ps == 0 ? a.blkhist : a.blkhist1;
    count_launch(3);  // count, colscan, scatter
    const dim3 hgrid(static_cast<unsigned>(nblk));
    int32_t* rk = a.rk;
    // T = 4096 or 2048 keys per block: 4 or 2 steps per warp of 1024 threads
    if (c.IPT == 16)
      e = pairs_in ? launch_chained(k_sort_count<4, true>, hgrid, dim3(kCountThreads), R * 4, s, nullptr,
                                    a.pairs_tmp, a.n, c.shift[ps], R, bits, bh, rk, a.K)
                   : launch_chained(k_sort_count<4, false>, hgrid, dim3(kCountThreads), R * 4, s, a.keys, nullptr,
                                    a.n, c.shift[ps], R, bits, bh, rk, a.K);
    else
      e = pairs_in ? launch_chained(k_sort_count<2, true>, hgrid, dim3(kCountThreads), R * 4, s, nullptr,
                                    a.pairs_tmp, a.n, c.shift[ps], R, bits, bh, rk, a.K)
                   : launch_chained(k_sort_count<2, false>, hgrid, dim3(kCountThreads), R * 4, s, a.keys, nullptr,
                                    a.n, c.shift[ps], R, bits, bh, rk, a.K);
    if (e != cudaSuccess) return e;
    const int S = c.segs[ps];
    const int64_t L = (nblk + S - 1) / S;
    e = launch_chained(k_sort_colscan, dim3((R + 31) / 32 * S), dim3(kColscanWarps * 32), 0, s, bh, R, nblk, S,
                       a.total);
    if (e != cudaSuccess) return e;
    // pass 0 of two writes pairs_tmp; the last pass writes the sorted pairs
    // (and perm when asked for).
    int2* out = last ? a.pairs : a.pairs_tmp;
    int32_t* perm = last ? a.perm : nullptr;
    const size_t sm = scatter_smem(R, c.T);
    int32_t* st = (last && c.passes == 1) ? a.start : nullptr;
    const int rpt = scatter_rpt(R);
    if (pairs_in && rk)
      e = c.IPT == 16 ? launch_scatter_r<16, true, true>(rpt, nblk, sm, s, rk, a.pairs_tmp, a.n, c.shift[ps], R,
                                                         bits, bh, a.total, S, L, out, perm, st, a.K)
                      : launch_scatter_r<8, true, true>(rpt, nblk, sm, s, rk, a.pairs_tmp, a.n, c.shift[ps], R,
                                                        bits, bh, a.total, S, L, out, perm, st, a.K);
    else if (pairs_in)
      e = c.IPT == 16 ? launch_scatter_r<16, true, false>(rpt, nblk, sm, s, nullptr, a.pairs_tmp, a.n, c.shift[ps], R,
                                                          bits, bh, a.total, S, L, out, perm, st, a.K)
                      : launch_scatter_r<8, true, false>(rpt, nblk, sm, s, nullptr, a.pairs_tmp, a.n, c.shift[ps], R,
                                                         bits, bh, a.total, S, L, out, perm, st, a.K);
    else if (rk)
      e = c.IPT == 16 ? launch_scatter_r<16, false, true>(rpt, nblk, sm, s, rk, nullptr, a.n, c.shift[ps], R, bits,
                                                          bh, a.total, S, L, out, perm, st, a.K)
                      : launch_scatter_r<8, false, true>(rpt, nblk, sm, s, rk, nullptr, a.n, c.shift[ps], R, bits,
                                                         bh, a.total, S, L, out, perm, st, a.K);
    else
      e = c.IPT == 16 ? launch_scatter_r<16, false, false>(rpt, nblk, sm, s, a.keys, nullptr, a.n, c.shift[ps], R,
                                                           bits, bh, a.total, S, L, out, perm, st, a.K)
                      : launch_scatter_r<8, false, false>(rpt, nblk, sm, s, a.keys, nullptr, a.n, c.shift[ps], R,
                                                          bits, bh, a.total, S, L, out, perm, st, a.K);
    if (e != cudaSuccess) return e;
  }
  if (c.passes > 1) {
    const int64_t cnt = (a.n + 1 + kBoundsPer - 1) / kBoundsPer;  // threads
    count_launch();
    e = launch_chained(k_bounds, dim3(static_cast<unsigned>((cnt + 255) / 256)), dim3(256), 0, s, a.pairs, a.n, a.K,
                       a.start);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace km
