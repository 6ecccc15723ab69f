// k_update.cu -- segmented reduction of the Sort-Inverse Update ("Flash-KMeans:
// Fast and Memory-Efficient Exact K-Means", §2.2 Sort-Inverse Update).
//
// After the argsort, points of one cluster occupy a contiguous run of sorted
// positions.  Thread blocks take fixed chunks of sorted positions, gather the
// point rows (one coalesced 16-byte load per lane) and sum each run in float32
// registers.  Runs that lie inside one warp's range are final at once; a run
// cut by a warp or block edge leaves a partial that is combined in the fixed
// order of the cut positions.  The pages let thread blocks add their boundary
// partials with atomics; here the combination is atomic-free and ordered, so
// the result is bitwise reproducible, with the same O((K + N/B_N) d) boundary
// writes (§2.2, "原子操作优化").
#include <cuda_bf16.h>
#include <math_constants.h>

#include "km_internal.h"
#include "km_ptx.cuh"
#include "km_rows.cuh"

namespace km {

// --------------------------------------------------------- row gathering
// Lanes are grouped: LPR lanes (16 bytes each) cover one point row; the
// warp reads 32/LPR rows per step.
template <int LPR>
struct RowGeom {
  static constexpr int RPS = 32 / LPR;                    // rows per step
  static constexpr int STEPS = LPR < 8 ? LPR : 8;          // steps (16-byte loads per lane) per batch
  static constexpr int BATCH = STEPS * RPS;               // rows per batch (<= 32)
};

template <bool BF16>
__device__ __forceinline__ void add16(float (&acc)[8], const uint4 v) {
  if constexpr (BF16) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += __uint_as_float(w[i] << 16);
      acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
    }
  } else {
    acc[0] += __uint_as_float(v.x);
    acc[1] += __uint_as_float(v.y);
    acc[2] += __uint_as_float(v.z);
    acc[3] += __uint_as_float(v.w);
  }
}

// Store a lane's column sums (lanes < LPR) to dst[0..D) floats, scaled.
template <int LPR, bool BF16>
__device__ __forceinline__ void store_row(float* dst, int row_bytes, int lane, const float (&acc)[8], float scale) {
  const int cl = lane;
  if (lane >= LPR || cl * 16 >= row_bytes) return;
  if constexpr (BF16) {
    float4* d4 = reinterpret_cast<float4*>(dst + cl * 8);
    d4[0] = make_float4(acc[0] * scale, acc[1] * scale, acc[2] * scale, acc[3] * scale);
    d4[1] = make_float4(acc[4] * scale, acc[5] * scale, acc[6] * scale, acc[7] * scale);
  } else {
    reinterpret_cast<float4*>(dst + cl * 4)[0] =
        make_float4(acc[0] * scale, acc[1] * scale, acc[2] * scale, acc[3] * scale);
  }
}

// One warp sums the runs of sorted positions [q0, q1) using the sorted keys:
// the cluster of every position is known, so run starts are found with a
// warp ballot on key changes and the row ids / keys of the next batch are
// prefetched while the current batch is summed.  Runs inside the range go to
// `final_store(k, acc)`; a run continuing past the left edge goes to slot 0,
// one continuing only past the right edge to slot 1 (cluster ids in slot_k,
// -1 when unused, vectors in slot_v[2][D]).
__device__ __forceinline__ int clamp_id(int v, int64_t hi) {
  return v < 0 ? 0 : (v >= hi ? static_cast<int>(hi - 1) : v);
}

template <int LPR, bool BF16, bool RS, bool PF, class FinalStore>
__device__ __forceinline__ void warp_range_sums_keyed(const uint8_t* __restrict__ X, int row_bytes, int D, int K,
                                                      const int2* __restrict__ pairs, int64_t n, int64_t q0,
                                                      int64_t q1, int lane, int* slot_k, float* slot_v,
                                                      FinalStore final_store) {
  using G = RowGeom<LPR>;
  if (lane == 0) { slot_k[0] = -1; slot_k[1] = -1; }
  if (q0 >= q1) return;
  const int sub = lane / LPR;
  const int cl = lane % LPR;
  const bool active = cl * 16 < row_bytes;
  // ids are clamped (memory safety only: valid pairs are always in range)
  const int kfirst = clamp_id(pairs[q0].y, K);
  const bool left_cont = q0 > 0 && clamp_id(pairs[q0 - 1].y, K) == kfirst;
  const int klast = clamp_id(pairs[q1 - 1].y, K);
  const bool right_cont = q1 < n && clamp_id(pairs[q1].y, K) == klast;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  int open_k = kfirst;
  bool open_left = left_cont;
  // RS (reduce-scatter): the row groups' partial sums are halved across
  // lanes each round instead of all-reduced, so every lane ends with its own
  // NV of the VPL columns and the per-cluster tail runs on all 32 lanes.
  constexpr int VPL = BF16 ? 8 : 4;  // columns per lane's 16 bytes
  constexpr bool kRS = RS && (32 / LPR) <= VPL;
  auto flush = [&](bool right) {
    if constexpr (kRS) {
      constexpr int NV = VPL / (32 / LPR);
      int off = 0;
      int len = VPL;
#pragma unroll
      for (int o = LPR; o < 32; o <<= 1) {
        const int half = len >> 1;
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < VPL / 2; ++i) {
          if (i < half) {
            const float a = acc[i], b = acc[half + i];
            const float keep = up ? b : a;
            acc[i] = keep + __shfl_xor_sync(0xffffffffu, up ? a : b, o);
          }
        }
        if (up) off += half;
        len = half;
      }
      const int col0 = cl * VPL + off;  // this lane's NV columns start here
      if (!open_left && !right) {
        final_store(open_k, acc, col0, NV, active);
      } else {
        const int slot = open_left ? 0 : 1;
        if (active)
#pragma unroll
          for (int i = 0; i < NV; ++i) slot_v[slot * D + col0 + i] = acc[i];
        if (lane == 0) slot_k[slot] = open_k;
      }
    } else {
#pragma unroll
      for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
      if (!open_left && !right) {
        if constexpr (RS) final_store(open_k, acc, cl * VPL, VPL, active && lane < LPR);
        else final_store(open_k, acc);
      } else {
        const int slot = open_left ? 0 : 1;
        store_row<LPR, BF16>(slot_v + slot * D, row_bytes, lane, acc, 1.f);
        if (lane == 0) slot_k[slot] = open_k;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  };
  const bool in_batch = lane < G::BATCH;
  int2 pv = (in_batch && q0 + lane < q1) ? pairs[q0 + lane] : make_int2(-1, -1);
  for (int64_t p = q0; p < q1; p += G::BATCH) {
    // ids are clamped into range: memory safety if an aborted kernel left
    // the pairs incomplete (no effect on valid input)
    const int cur_p = clamp_id(pv.x, n), cur_k = pv.y < 0 ? -1 : clamp_id(pv.y, K);
    const int64_t pn = p + G::BATCH;
    pv = (in_batch && pn + lane < q1) ? pairs[pn + lane] : make_int2(-1, -1);
    const int nb = q1 - p < G::BATCH ? static_cast<int>(q1 - p) : G::BATCH;
    int prevk = __shfl_up_sync(0xffffffffu, cur_k, 1);
    if (lane == 0) prevk = open_k;
    const uint32_t starts = __ballot_sync(0xffffffffu, lane < nb && cur_k != prevk);
    // every row of the batch in one round trip ...
    uint4 buf[G::STEPS];
#pragma unroll
    for (int s = 0; s < G::STEPS; ++s) {
      const int slot = s * G::RPS + sub;
      const int r = __shfl_sync(0xffffffffu, cur_p, slot);
      if (slot < nb && active)
        buf[s] = __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(r) * row_bytes + cl * 16));
      else
        buf[s] = make_uint4(0u, 0u, 0u, 0u);
    }
    // PF: the next batch's rows are pulled into L2 (hints, one per 128-byte
    // line, each lane its own next position) while this batch is summed,
    // so its loads wait on L2 rather than on DRAM
    if constexpr (PF) {
      if (in_batch && pn + lane < q1) {
        const uint8_t* nrow = X + static_cast<int64_t>(clamp_id(pv.x, n)) * row_bytes;
        for (int off = 0; off < row_bytes; off += 128) prefetch_l2(nrow + off);
      }
    }
    // ... then the runs inside it are split from registers
    if (starts == 0u) {
#pragma unroll
      for (int s = 0; s < G::STEPS; ++s) add16<BF16>(acc, buf[s]);
    } else {
      int a = 0;
      while (a < nb) {
        if ((starts >> a) & 1u) {
          flush(false);
          open_k = __shfl_sync(0xffffffffu, cur_k, a);
          open_left = false;
        }
        const uint32_t later = a + 1 < 32 ? (starts >> (a + 1)) << (a + 1) : 0u;
        const int e = later ? __ffs(later) - 1 : nb;
#pragma unroll
        for (int s = 0; s < G::STEPS; ++s) {
          const int slot = s * G::RPS + sub;
          if (slot >= a && slot < e) add16<BF16>(acc, buf[s]);
        }
        a = e;
      }
    }
  }
  flush(right_cont);
}

// ------------------------------------------------------------ big path
// One wave of blocks; block c owns sorted positions [c*P, (c+1)*P), split in
// 8 contiguous warp ranges.  Each warp sums its range; then the block
// combines the runs cut at warp edges in position order: runs inside the
// block's range become final sums, a run continuing past its left edge goes
// to pl[c], one continuing only past its right edge to pr[c].
template <int LPR, bool BF16>
__global__ void __launch_bounds__(256, 4) k_segsum(const uint8_t* __restrict__ X, int64_t n, int D, int row_bytes,
                                                   const int2* __restrict__ pairs, int K,
                                                   const int32_t* __restrict__ start, int64_t P,
                                                   float* __restrict__ sums, float* __restrict__ pl,
                                                   float* __restrict__ pr) {
  extern __shared__ float sm[];
  pdl_trigger();
  pdl_wait();
  constexpr int W = 8;
  int* slot_k = reinterpret_cast<int*>(sm);          // [W][2]
  float* slot_v = sm + 2 * W;                         // [W][2][D]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t c = blockIdx.x;
  const int64_t p0 = c * P;
  const int64_t p1 = p0 + P < n ? p0 + P : n;
  const int64_t Lw = P / W;
  const int64_t q0 = p0 + warp * Lw < p1 ? p0 + warp * Lw : p1;
  const int64_t q1 = q0 + Lw < p1 ? q0 + Lw : p1;
  warp_range_sums_keyed<LPR, BF16, false, false>(X, row_bytes, D, K, pairs, n, q0, q1, lane, slot_k + 2 * warp,
                                   slot_v + 2 * warp * D, [&](int k, const float (&acc)[8]) {
                                     store_row<LPR, BF16>(sums + static_cast<int64_t>(k) * D, row_bytes, lane, acc,
                                                          1.f);
                                   });
  __syncthreads();
  // Ordered combine of the cut runs, one thread per column.
  for (int j = threadIdx.x; j < D; j += blockDim.x) {
    int open = -1;
    float a = 0.f;
    auto flush = [&](int k, float v) {
      const int64_t s0 = start[k], s1 = start[k + 1];
      if (s0 >= p0 && s1 <= p1) sums[static_cast<int64_t>(k) * D + j] = v;
      else if (s0 < p0) pl[c * D + j] = v;
      else pr[c * D + j] = v;
    };
    for (int w = 0; w < W; ++w) {
      for (int sl = 0; sl < 2; ++sl) {
        const int k = slot_k[2 * w + sl];
        if (k < 0) continue;
        const float v = slot_v[(2 * w + sl) * D + j];
        if (k == open) {
          a += v;
        } else {
          if (open >= 0) flush(open, a);
          open = k;
          a = v;
        }
      }
    }
    if (open >= 0) flush(open, a);
  }
}

template <int LPR>
static cudaError_t launch_segsum_t(const Plan& p, const SegArgs& a, cudaStream_t s) {
  const int row_bytes = p.D * p.es;
  const int64_t P = seg_block_positions(a.n);
  const int64_t nch = (a.n + P - 1) / P;
  const size_t sm = (2 * 8 + 2 * 8 * static_cast<size_t>(p.D)) * 4;
  count_launch();
  auto kern = p.dtype == kDtypeBF16 ? k_segsum<LPR, true> : k_segsum<LPR, false>;
  return launch_chained(kern, dim3(static_cast<unsigned>(nch)), dim3(256), sm, s,
                        static_cast<const uint8_t*>(a.X), a.n, p.D, row_bytes, a.pairs, p.K, a.start, P, a.sums,
                        a.pl, a.pr);
}

static int lanes_per_row(int row_bytes) {
  int v = (row_bytes + 15) / 16, l = 1;
  while (l < v) l <<= 1;
  return l;
}

cudaError_t launch_segsum(const Plan& p, const SegArgs& a, cudaStream_t s) {
  if (a.n <= 0) return cudaSuccess;
  switch (lanes_per_row(p.D * p.es)) {
    case 1: return launch_segsum_t<1>(p, a, s);
    case 2: return launch_segsum_t<2>(p, a, s);
    case 4: return launch_segsum_t<4>(p, a, s);
    case 8: return launch_segsum_t<8>(p, a, s);
    case 16: return launch_segsum_t<16>(p, a, s);
    case 32: return launch_segsum_t<32>(p, a, s);
    default: return cudaErrorInvalidValue;
  }
}

// --------------------------------------------------------------- finalize
// Largest number of segmented-sum chunk boundaries a cluster may cross and
// still be finalised by one warp (more: a whole block).
constexpr int kBigSpan = 8;

struct FinK {
  int K, D, Dp, dtype, BNS, big_span;
  int64_t n, nwarp_blocks;
  const int32_t* start;
  const int2* pairs;
  const float* sums;
  const float* pl;
  const float* pr;
  int mode;
  float* C;
  void* c_op;
  uint8_t* caug;
  int32_t* counts;
  double* acc64;
  long long* cnt64;
  double* cntf;  // mode 1: float64 counts instead of cnt64 (data-parallel sums), or null
  const double* tobj;
  int64_t ntiles;
  double* obj;
  int nobj;                // objective blocks (the grid's last nobj blocks; 0: no objective)
  double* objpart;         // [nobj] block sums
  unsigned int* objcnt;    // blocks done (zero at entry; the last block resets it)
};

// Objective partials per block of the finalise kernel: each block sums a
// fixed range of this many assignment partials.
constexpr int kObjPerBlock = 4096;

// Block j of nobj: the objective of this pass from the assignment's
// per-tile partials in a fixed order -- block j sums partials
// [j*kObjPerBlock, (j+1)*kObjPerBlock) (thread-strided, then a fixed tree),
// and the last block to finish sums the nobj block sums the same way.  The
// order depends only on the number of partials, never on which CTA computed
// which tile, so the objective is bitwise reproducible across grids.
__device__ void objective_block(const FinK& f, int j, double* red) {
  const int tid = threadIdx.x;
  const int64_t total = f.ntiles * 4;
  const int64_t lo = static_cast<int64_t>(j) * kObjPerBlock;
  const int64_t hi = lo + kObjPerBlock < total ? lo + kObjPerBlock : total;
  __shared__ int is_last;
  auto block_sum = [&](double v) {
    red[tid] = v;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
      if (tid < w) red[tid] += red[tid + w];
      __syncthreads();
    }
    return red[0];
  };
  double s = 0.0;
  for (int64_t i = lo + tid; i < hi; i += blockDim.x) s += f.tobj[i];
  const double bs = block_sum(s);
  if (tid == 0) {
    f.objpart[j] = bs;
    __threadfence();
    is_last = atomicAdd(f.objcnt, 1u) == static_cast<unsigned>(f.nobj - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  s = 0.0;
  for (int i = tid; i < f.nobj; i += blockDim.x) s += __ldcg(f.objpart + i);
  __syncthreads();  // red is reused
  const double tot = block_sum(s);
  if (tid == 0) {
    if (f.mode == 0) *f.obj = tot;
    else *f.obj += tot;
    *f.objcnt = 0u;
  }
}

__device__ __forceinline__ void* op_row(const FinK& f, int k) {
  if (!f.c_op) return nullptr;
  if (f.dtype == kDtypeBF16) return reinterpret_cast<__nv_bfloat16*>(f.c_op) + static_cast<int64_t>(k) * f.D;
  return reinterpret_cast<float*>(f.c_op) + static_cast<int64_t>(k) * 3 * f.Dp;
}

// Operand row (-2c in bf16, or the TF32 split) and ||c||^2 of a centroid held
// in registers: v[i] = c[lane + 32 i] (D <= 256).
__device__ __forceinline__ float emit_operand_regs(const float (&v)[8], int D, int Dp, int dtype, void* row,
                                                   int lane) {
  float s = 0.f;
  if (dtype == kDtypeBF16) {
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(row);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = lane + 32 * i;
      if (j < D) {
        const float f = __bfloat162float(__float2bfloat16_rn(v[i]));
        if (o) o[j] = __float2bfloat16_rn(-2.f * f);
        s = fmaf(f, f, s);
      }
    }
  } else {
    float* o = reinterpret_cast<float*>(row);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int j = lane + 32 * i;
      if (j < Dp) {
        const float val = j < D ? v[i] : 0.f;
        if (o) {
          const float hi = tf32_round(val);
          const float lo = tf32_round(val - hi);
          o[j] = -2.f * hi;
          o[Dp + j] = -2.f * lo;
          o[2 * Dp + j] = -2.f * hi;
        }
        s = fmaf(val, val, s);
      }
    }
  }
  return warp_sum_f(s);
}

// Finalise cluster k, run by one warp.  sum[i] holds the member sum of column
// lane + 32 i (ignored when cnt == 0).  Mode 0: centroid = sum / count (or
// keep the previous one), operand copy, augmentation row, count.  Mode 1:
// add the sum and count to the float64 accumulators.
__device__ void finish_cluster(const FinK& f, int k, int64_t cnt, float (&sum)[8], int lane) {
  float* crow = f.C + static_cast<int64_t>(k) * f.D;
  if (f.mode == 0) {
    if (cnt > 0) {
      const float fc = static_cast<float>(cnt);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int j = lane + 32 * i;
        if (j < f.D) {
          sum[i] = sum[i] / fc;
          crow[j] = sum[i];
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int j = lane + 32 * i;
        sum[i] = j < f.D ? crow[j] : 0.f;
      }
    }
    const float s = emit_operand_regs(sum, f.D, f.Dp, f.dtype, op_row(f, k), lane);
    if (lane == 0) {
      if (f.caug) write_aug_row(f.caug + static_cast<int64_t>(k) * kAugBytes, f.dtype, s, 1);
      if (f.counts) f.counts[k] = static_cast<int32_t>(cnt);
    }
  } else if (cnt > 0) {
    double* arow = f.acc64 + static_cast<int64_t>(k) * f.D;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = lane + 32 * i;
      if (j < f.D) arow[j] += static_cast<double>(sum[i]);
    }
    if (lane == 0) {
      if (f.cntf) f.cntf[k] += static_cast<double>(cnt);
      else f.cnt64[k] += cnt;
    }
  }
}

__global__ void __launch_bounds__(512) k_finalize(const FinK f) {
  extern __shared__ float fsm[];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (static_cast<int>(blockIdx.x) >= static_cast<int>(gridDim.x) - f.nobj) {
    // the last nobj blocks: objective of this pass (fixed-order reduction)
    objective_block(f, static_cast<int>(blockIdx.x) - (static_cast<int>(gridDim.x) - f.nobj),
                    reinterpret_cast<double*>(fsm));
    return;
  }
  if (blockIdx.x < f.nwarp_blocks) {
    const int k = static_cast<int>(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (k >= f.K) return;
    // The whole-block sum row is loaded together with the segment bounds (it
    // is the answer for every cluster inside one segmented-sum block).
    float w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = lane + 32 * i;
      w[i] = j < f.D ? f.sums[static_cast<int64_t>(k) * f.D + j] : 0.f;
    }
    const int64_t s0 = f.start[k], s1 = f.start[k + 1], cnt = s1 - s0;
    float v[8];
    if (cnt > 0) {
      const int64_t ca = s0 / f.BNS, cb = (s1 - 1) / f.BNS;
      if (cb - ca > f.big_span) return;  // handled by a whole block below
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int j = lane + 32 * i;
        v[i] = 0.f;
        if (j < f.D) {
          if (ca == cb) {
            v[i] = w[i];
          } else {
            // the pieces (right end of chunk ca, left ends of ca+1..cb) are
            // loaded together, then added in chunk order
            float pc[kBigSpan + 1];
#pragma unroll
            for (int q = 0; q <= kBigSpan; ++q)
              pc[q] = ca + q <= cb ? (q == 0 ? f.pr : f.pl)[(ca + q) * f.D + j] : 0.f;
            float a = pc[0];
#pragma unroll
            for (int q = 1; q <= kBigSpan; ++q)
              if (ca + q <= cb) a += pc[q];
            v[i] = a;
          }
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    finish_cluster(f, k, cnt, v, lane);
    return;
  }
  // Big clusters: block i owns the cluster containing position i*G (G =
  // big_span*BNS) if that is the first multiple of G inside the cluster.
  const int64_t G = static_cast<int64_t>(f.big_span) * f.BNS;
  const int64_t P = (static_cast<int64_t>(blockIdx.x) - f.nwarp_blocks) * G;
  if (P >= f.n) return;
  const int k = clamp_id(f.pairs[P].y, f.K);
  const int64_t s0 = f.start[k], s1 = f.start[k + 1];
  const int64_t ca = s0 / f.BNS, cb = (s1 - 1) / f.BNS;
  if (cb - ca <= f.big_span) return;
  if ((s0 + G - 1) / G != P / G) return;
  // column groups of 4 floats x slices of the chunk range
  const int groups = f.D / 4;
  const int slices = blockDim.x / groups;
  const int tg = threadIdx.x % groups, sl = threadIdx.x / groups;
  float* part = fsm;                       // [slices][D]
  float* srow = fsm + slices * f.D;        // [D]
  if (sl < slices) {
    const int64_t nc = cb - ca + 1;
    const int64_t per = (nc + slices - 1) / slices;
    const int64_t c0 = ca + sl * per;
    const int64_t c1 = c0 + per - 1 < cb ? c0 + per - 1 : cb;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t c = c0; c <= c1; ++c) {
      const float* src = (c == ca ? f.pr : f.pl) + c * f.D + tg * 4;
      const float4 v = *reinterpret_cast<const float4*>(src);
      a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
    }
    reinterpret_cast<float4*>(part + sl * f.D)[tg] = a;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < f.D; j += blockDim.x) {
    float a = 0.f;
    for (int s2 = 0; s2 < slices; ++s2) a += part[s2 * f.D + j];
    srow[j] = a;
  }
  __syncthreads();
  if (warp == 0) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = lane + 32 * i;
      v[i] = j < f.D ? srow[j] : 0.f;
    }
    finish_cluster(f, k, s1 - s0, v, lane);
  }
}

cudaError_t launch_finalize(const Plan& p, const FinalizeArgs& a, cudaStream_t s) {
  FinK f{};
  f.K = p.K;
  f.D = p.D;
  f.Dp = p.Dp;
  f.dtype = p.dtype;
  f.BNS = static_cast<int>(seg_block_positions(p.rows));
  f.big_span = p.gc.big_span < kBigSpan ? p.gc.big_span : kBigSpan;
  f.n = p.rows;
  f.start = a.start;
  f.pairs = a.pairs;
  f.sums = a.sums;
  f.pl = a.pl;
  f.pr = a.pr;
  f.mode = a.mode;
  f.C = a.C;
  f.c_op = a.c_op;
  f.caug = static_cast<uint8_t*>(a.caug);
  f.counts = a.counts;
  f.acc64 = a.acc64;
  f.cnt64 = a.cnt64;
  f.cntf = a.cntf;
  f.tobj = a.tobj;
  f.ntiles = a.ntiles;
  f.obj = a.obj;
  f.nobj = a.ntiles > 0 ? static_cast<int>((a.ntiles * 4 + kObjPerBlock - 1) / kObjPerBlock) : 0;
  f.objpart = a.objpart;
  f.objcnt = a.objcnt;
  const int threads = 512;
  f.nwarp_blocks = (p.K + 15) / 16;
  const int64_t G = static_cast<int64_t>(p.gc.big_span) * f.BNS;
  const int64_t nbig = (p.rows + G - 1) / G;
  // objective blocks: 512 doubles (1024 floats); warp blocks: 16 warp rows;
  // big-cluster blocks: slices x D partial rows + one summed row.
  const size_t fl_warp = 1024 + 16 * static_cast<size_t>(p.D);
  const size_t fl_big = 2048 + 2 * static_cast<size_t>(p.D);
  const size_t sm = 4 * (fl_warp > fl_big ? fl_warp : fl_big);
  cudaError_t e = cudaFuncSetAttribute(k_finalize, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sm));
  if (e != cudaSuccess) return e;
  count_launch();
  return launch_chained(k_finalize, dim3(static_cast<unsigned>(f.nwarp_blocks + nbig + f.nobj)), dim3(threads), sm, s,
                        f);
}

// Out-of-core: float64 accumulators -> centroids; resets the accumulators.
__global__ void k_finalize_acc(int K, int D, int Dp, int dtype, double* acc64, long long* cnt64, float* C,
                               void* c_op, uint8_t* caug, int32_t* counts, double* objacc, double* obj_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.x * (blockDim.x >> 5) + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (obj_out) *obj_out = *objacc;
    *objacc = 0.0;
  }
  if (k >= K) return;
  const long long cnt = cnt64[k];
  float* crow = C + static_cast<int64_t>(k) * D;
  double* arow = acc64 + static_cast<int64_t>(k) * D;
  if (cnt > 0)
    for (int j = lane; j < D; j += 32) crow[j] = static_cast<float>(arow[j] / static_cast<double>(cnt));
  for (int j = lane; j < D; j += 32) arow[j] = 0.0;
  __syncwarp();
  void* orow = nullptr;
  if (c_op)
    orow = dtype == kDtypeBF16 ? static_cast<void*>(reinterpret_cast<__nv_bfloat16*>(c_op) + static_cast<int64_t>(k) * D)
                               : static_cast<void*>(reinterpret_cast<float*>(c_op) + static_cast<int64_t>(k) * 3 * Dp);
  const float s = emit_operand_row([&](int j) { return crow[j]; }, D, Dp, dtype, orow, lane);
  if (lane == 0) {
    if (caug) write_aug_row(caug + static_cast<int64_t>(k) * kAugBytes, dtype, s, 1);
    if (counts) counts[k] = static_cast<int32_t>(cnt);
    cnt64[k] = 0;
  }
}

// Centroids from float64 sums and counts accumulated elsewhere (e.g. added
// up across the ranks of a data-parallel fit; counts are float64, exact
// integers below 2^53): C = sum / count where count > 0, else C is kept;
// C_lp is the dtype copy the next assignment takes (bf16
// round-to-nearest-even or the float values); counts as int32.
__global__ void k_finalize_sums(const double* __restrict__ sums, const double* __restrict__ cnt, int K, int D,
                                int dtype, float* C, void* C_lp, int32_t* counts) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= static_cast<int64_t>(K) * D) return;
  const int k = static_cast<int>(e / D);
  const double n = cnt[k];
  float c = C[e];
  if (n > 0.0) {
    c = static_cast<float>(sums[e] / n);
    C[e] = c;
  }
  if (C_lp) {
    if (dtype == kDtypeBF16) static_cast<__nv_bfloat16*>(C_lp)[e] = __float2bfloat16_rn(c);
    else static_cast<float*>(C_lp)[e] = c;
  }
  if (counts && e - static_cast<int64_t>(k) * D == 0) counts[k] = static_cast<int32_t>(n);
}

cudaError_t launch_finalize_sums(int K, int D, int dtype, const double* sums, const double* cnt, float* C,
                                 void* C_lp, int32_t* counts, cudaStream_t s) {
  chain_break();  // plain launch: the next kernel must not chain to it
  const int64_t e = static_cast<int64_t>(K) * D;
  if (fault_hit(kFaultLaunch)) return cudaErrorLaunchFailure;
  count_launch();
  k_finalize_sums<<<static_cast<unsigned>((e + 255) / 256), 256, 0, s>>>(sums, cnt, K, D, dtype, C, C_lp, counts);
  return cudaGetLastError();
}

cudaError_t launch_finalize_acc(const Plan& p, double* acc64, long long* cnt64, float* C, void* c_op, void* caug,
                                int32_t* counts, double* objacc, double* obj_out, cudaStream_t s) {
  chain_break();  // plain launch: the next kernel must not chain to it
  const int threads = 256;
  const int blocks = (p.K + 7) / 8;
  if (fault_hit(kFaultLaunch)) return cudaErrorLaunchFailure;
  count_launch();
  k_finalize_acc<<<blocks, threads, 0, s>>>(p.K, p.D, p.Dp, p.dtype, acc64, cnt64, C, c_op, static_cast<uint8_t*>(caug), counts, objacc,
                                            obj_out);
  return cudaGetLastError();
}

// ------------------------------------------------- fused small-problem path
// One CTA per instance: stable counting sort of its assignment vector in
// shared memory, segmented sums over the sorted order, ordered combine of
// warp-boundary runs, centroids, operand copy, norms, counts and objective.
struct SmallK {
  int B, K, Kp, D, Dp, dtype;
  int64_t N;
  int row_bytes;
  const uint8_t* X;
  const int32_t* idx;
  float* C;
  void* c_op;
  uint8_t* caug;
  int32_t* counts;
  const double* tobj;
  int64_t tiles_per_inst;
  double* obj;
  int obj_stride;
};

__device__ __forceinline__ void* op_row_of(const SmallK& p, int64_t grow) {
  if (!p.c_op) return nullptr;
  if (p.dtype == kDtypeBF16) return reinterpret_cast<__nv_bfloat16*>(p.c_op) + grow * p.D;
  return reinterpret_cast<float*>(p.c_op) + grow * 3 * p.Dp;
}

__device__ __forceinline__ uint32_t lanemask_lt_u() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Exclusive scan of v[0..256) in place (256 threads): warp shuffles, then
// the 8 warp totals.
__device__ __forceinline__ void scan256_exclusive(int32_t* v, int32_t* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int32_t x0 = v[threadIdx.x];
  int32_t x = x0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t run = 0;
    for (int w = 0; w < 8; ++w) { const int32_t t = wsum[w]; wsum[w] = run; run += t; }
  }
  __syncthreads();
  v[threadIdx.x] = wsum[warp] + x - x0;
  __syncthreads();
}

static_assert(kSmallMaxN <= 65536 && kSmallMaxK <= 65536, "key and rank are packed in 16 bits each");

template <int LPR, bool BF16>
__global__ void __launch_bounds__(256) k_small_update(const SmallK p) {
  extern __shared__ __align__(16) int32_t ssm[];
  pdl_trigger();
  pdl_wait();
  constexpr int W = 8;
  const int N = static_cast<int>(p.N), K = p.K, D = p.D;
  // 16-byte aligned pieces first: slot vectors, the double reduction buffer,
  // the sorted pairs, then the integer arrays.  kr[i] packs point i's key
  // (low 16 bits; K <= kSmallMaxK) and its rank among equal keys of its warp
  // range (high 16 bits; N <= kSmallMaxN).
  float* slot_v = reinterpret_cast<float*>(ssm);                      // [W][2][D]
  double* red = reinterpret_cast<double*>(slot_v + 2 * W * D);        // [256]
  int2* pairs = reinterpret_cast<int2*>(red + 256);                   // [N] sorted (point, cluster)
  uint32_t* kr = reinterpret_cast<uint32_t*>(pairs + N);              // [N]
  int32_t* wcnt = reinterpret_cast<int32_t*>(kr + N);                 // [W][K]
  int32_t* start = wcnt + W * K;       // [K+1]
  int32_t* tmp = start + K + 1;        // [256]
  int* slot_k = tmp + 256;             // [W][2]
  int32_t* wsum = slot_k + 2 * W;      // [8]
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* gidx = p.idx + static_cast<int64_t>(b) * N;
  const uint8_t* X = p.X + static_cast<int64_t>(b) * N * p.row_bytes;
  float* C = p.C + static_cast<int64_t>(b) * K * D;
  int bits = 0;
  while ((1 << bits) < K) ++bits;

  for (int i0 = 0; i0 < N; i0 += 8 * 256) {  // eight loads in flight per thread
    int32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * 256 + threadIdx.x;
      v[u] = i < N ? gidx[i] : 0;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * 256 + threadIdx.x;
      // ids outside [0, K) are clamped (memory safety only)
      if (i < N) kr[i] = static_cast<uint32_t>(v[u] < 0 ? 0 : (v[u] >= K ? K - 1 : v[u]));
    }
  }
  for (int i = threadIdx.x; i < W * K; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  // stable ranks inside each warp's contiguous range (equal keys of a warp
  // step found with one ballot per key bit)
  const int Lw = ((N + W - 1) / W + 31) / 32 * 32;
  const uint32_t ltm = lanemask_lt_u();
  for (int i0 = warp * Lw; i0 < (warp + 1) * Lw && i0 < N; i0 += 32) {
    const int i = i0 + lane;
    const bool v = i < N && i < (warp + 1) * Lw;
    const int d = v ? static_cast<int>(kr[i]) : -1;
    const uint32_t peers = match_digit<10>(d, bits, v);  // K <= kSmallMaxK = 1024
    int before = 0;
    if (v) before = wcnt[warp * K + d];
    if (v) kr[i] = static_cast<uint32_t>(d) | (static_cast<uint32_t>(before + __popc(peers & ltm)) << 16);
    __syncwarp();
    if (v && lane == __ffs(peers) - 1) wcnt[warp * K + d] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per-cluster warp prefixes, then cluster starts
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    int run = 0;
    for (int w = 0; w < W; ++w) {
      const int c = wcnt[w * K + k];
      wcnt[w * K + k] = run;
      run += c;
    }
    start[k] = run;  // total, scanned below
  }
  __syncthreads();
  {
    const int per = (K + 255) / 256;
    const int lo = threadIdx.x * per;
    int sum = 0;
    for (int i = lo; i < lo + per && i < K; ++i) sum += start[i];
    tmp[threadIdx.x] = sum;
    __syncthreads();
    scan256_exclusive(tmp, wsum);
    int run = tmp[threadIdx.x];
    for (int i = lo; i < lo + per && i < K; ++i) { const int v = start[i]; start[i] = run; run += v; }
    if (threadIdx.x == 0) start[K] = N;
  }
  __syncthreads();
  // scatter into sorted (point, cluster) pairs
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const int key = static_cast<int>(kr[i] & 0xffffu), rank = static_cast<int>(kr[i] >> 16);
    pairs[start[key] + wcnt[(i / Lw) * K + key] + rank] = make_int2(i, key);
  }
  __syncthreads();
  // segmented sums over the sorted pairs: runs inside a warp range become
  // centroids directly
  const int L = (N + W - 1) / W;
  const int q0 = warp * L < N ? warp * L : N;
  const int q1 = q0 + L < N ? q0 + L : N;
  warp_range_sums_keyed<LPR, BF16, true, true>(
      X, p.row_bytes, D, K, pairs, N, q0, q1, lane, slot_k + 2 * warp, slot_v + 2 * warp * D,
      [&](int k, const float (&v)[8], int col0, int nv, bool writer) {
        // mean = sum x (1 / count): one division per cluster (within 1.5 ulp of
        // sum / count; this tail is the kernel's issue bottleneck).  Each lane
        // holds nv columns from col0 (all lanes distinct when reduce-scattered).
        const float inv = 1.f / static_cast<float>(start[k + 1] - start[k]);
        const int64_t grow = static_cast<int64_t>(b) * K + k;
        void* orow = op_row_of(p, grow);
        float* crow = C + static_cast<int64_t>(k) * D;
        float s = 0.f;
        if constexpr (BF16) {
          if (nv == 1) {  // 8 row groups (16-column rows): one column per lane, any offset
            if (writer) {
              const float q = v[0] * inv;
              crow[col0] = q;
              const __nv_bfloat16 h = __float2bfloat16_rn(q);
              const float f = __bfloat162float(h);
              s = f * f;
              if (orow) static_cast<__nv_bfloat16*>(orow)[col0] = __float2bfloat16_rn(-2.f * f);
            }
          } else {
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            // nv is even here and so is col0: the pair stores are aligned
            if (i < nv && writer) {
              const float q0v = v[i] * inv, q1v = v[i + 1] * inv;
              *reinterpret_cast<float2*>(crow + col0 + i) = make_float2(q0v, q1v);
              // round the pair to bf16, square the rounded values, scale by -2 in
              // bf16 (exact: a power of two)
              const __nv_bfloat162 h = __floats2bfloat162_rn(q0v, q1v);
              const float2 f = __bfloat1622float2(h);
              s = fmaf(f.y, f.y, fmaf(f.x, f.x, s));
              if (orow)
                *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(orow) + col0 + i) =
                    __hmul2(h, __float2bfloat162_rn(-2.f));
            }
          }
          }
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (i < nv && writer) {
              const float q = v[i] * inv;
              crow[col0 + i] = q;
              s = fmaf(q, q, s);
              if (orow) {
                float* o = static_cast<float*>(orow);
                const float hi = tf32_round(q), lo = tf32_round(q - hi);
                o[col0 + i] = -2.f * hi;
                o[p.Dp + col0 + i] = -2.f * lo;
                o[2 * p.Dp + col0 + i] = -2.f * hi;
              }
            }
          }
        }
        s = warp_sum_f(s);
        if (lane == 0 && p.caug) write_aug_row(p.caug + (static_cast<int64_t>(b) * p.Kp + k) * kAugBytes, p.dtype, s, 1);
      });
  __syncthreads();
  int* cut_list = tmp;  // clusters finished by the combine below (at most 2W)
  if (threadIdx.x == 0) tmp[255] = 0;
  __syncthreads();
  for (int j = threadIdx.x; j < D; j += blockDim.x) {
    int open = -1;
    float a = 0.f;
    auto flush = [&](int k, float v) {
      C[static_cast<int64_t>(k) * D + j] = v / static_cast<float>(start[k + 1] - start[k]);
      if (j == 0) cut_list[tmp[255]++] = k;
    };
    for (int w = 0; w < W; ++w)
      for (int sl = 0; sl < 2; ++sl) {
        const int k = slot_k[2 * w + sl];
        if (k < 0) continue;
        const float v = slot_v[(2 * w + sl) * D + j];
        if (k == open) {
          a += v;
        } else {
          if (open >= 0) flush(open, a);
          open = k;
          a = v;
        }
      }
    if (open >= 0) flush(open, a);
  }
  __syncthreads();
  // operand and norm rows of the clusters the combine finished (the others
  // were written from registers; empty clusters keep C and their rows)
  const int ncut = tmp[255];
  for (int c = warp; c < ncut; c += W) {
    const int k = cut_list[c];
    const float* crow = C + static_cast<int64_t>(k) * D;
    const int64_t grow = static_cast<int64_t>(b) * K + k;
    const float sq = emit_operand_row([&](int j) { return crow[j]; }, D, p.Dp, p.dtype, op_row_of(p, grow), lane);
    if (lane == 0 && p.caug) write_aug_row(p.caug + (static_cast<int64_t>(b) * p.Kp + k) * kAugBytes, p.dtype, sq, 1);
  }
  if (p.counts)
    for (int k = threadIdx.x; k < K; k += blockDim.x) p.counts[static_cast<int64_t>(b) * K + k] = start[k + 1] - start[k];
  if (p.tobj && p.obj) {
    const double* t = p.tobj + static_cast<int64_t>(b) * p.tiles_per_inst * 4;
    double sd = 0.0;
    for (int64_t i = threadIdx.x; i < p.tiles_per_inst * 4; i += blockDim.x) sd += t[i];
    red[threadIdx.x] = sd;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
      if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
      __syncthreads();
    }
    if (threadIdx.x == 0) p.obj[static_cast<int64_t>(b) * p.obj_stride] = red[0];
  }
}

size_t small_update_smem(int64_t N, int K, int D) {
  const int W = 8;
  const size_t floats = 2 * static_cast<size_t>(W) * D;                                   // slot vectors
  const size_t ints = 3 * static_cast<size_t>(N) + static_cast<size_t>(W) * K + K + 1 + 256 + 2 * W + 8;
  return floats * 4 + 256 * 8 + ints * 4 + 16;
}

template <int LPR>
static cudaError_t launch_small_t(const Plan& p, const SmallUpdateArgs& a, cudaStream_t s) {
  SmallK k{};
  k.B = p.B;
  k.K = p.K;
  k.Kp = p.Kp;
  k.D = p.D;
  k.Dp = p.Dp;
  k.dtype = p.dtype;
  k.N = p.N;
  k.row_bytes = p.D * p.es;
  k.X = static_cast<const uint8_t*>(a.X);
  k.idx = a.idx;
  k.C = a.C;
  k.c_op = a.c_op;
  k.caug = static_cast<uint8_t*>(a.caug);
  k.counts = a.counts;
  k.tobj = a.tobj;
  k.tiles_per_inst = a.tiles_per_inst;
  k.obj = a.obj;
  k.obj_stride = a.obj_stride;
  const size_t sm = small_update_smem(p.N, p.K, p.D);
  count_launch();
  cudaError_t e;
  if (p.dtype == kDtypeBF16) {
    e = cudaFuncSetAttribute(k_small_update<LPR, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sm));
    if (e != cudaSuccess) return e;
    e = launch_chained(k_small_update<LPR, true>, dim3(p.B), dim3(256), sm, s, k);
  } else {
    e = cudaFuncSetAttribute(k_small_update<LPR, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sm));
    if (e != cudaSuccess) return e;
    e = launch_chained(k_small_update<LPR, false>, dim3(p.B), dim3(256), sm, s, k);
  }
  return e;
}

cudaError_t launch_small_update(const Plan& p, const SmallUpdateArgs& a, cudaStream_t s) {
  switch (lanes_per_row(p.D * p.es)) {
    case 1: return launch_small_t<1>(p, a, s);
    case 2: return launch_small_t<2>(p, a, s);
    case 4: return launch_small_t<4>(p, a, s);
    case 8: return launch_small_t<8>(p, a, s);
    case 16: return launch_small_t<16>(p, a, s);
    case 32: return launch_small_t<32>(p, a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace km
