// k_assign.cu -- FlashAssign on sm_100a ("Flash-KMeans: Fast and
// Memory-Efficient Exact K-Means", §2.1 FlashAssign).
//
// For a tile of 128 points the kernel streams every centroid tile through the
// tensor cores and keeps, per point, the running minimum of
//     score_k = ||c_k||^2 - 2 x.c_k
// and its index (the §2.1 online argmin: each point carries its current best
// distance and cluster id, each new tile's local minimum is merged into it).
// The N x K scores live only in tensor memory; device memory sees X once, the
// centroid tiles (from L2) and the N-long outputs, i.e. O(Nd + Kd) traffic
// instead of O(NK) (§2.1, "效果").
//
// Structure: persistent CTAs (one per SM) with warp-specialised roles
//   warp 0      TMA producer: point tile (resident for the whole centroid
//               sweep, double buffered across tiles), centroid tiles through a
//               ring of stages (the §2.1 "异步预取" double-buffered prefetch),
//               and the matching ||c||^2 slices through a separate ring;
//   warp 1      tcgen05.mma issuer (one thread): M=128 x N=BN x K=16 (bf16)
//               or K=8 (tf32) steps into a double-buffered TMEM accumulator;
//   warps 2..9  epilogue: tcgen05.ld of the accumulator, score = cn - 2*acc,
//               per-lane argmin with the lowest index winning exact ties; two
//               warps per TMEM lane quarter split the BN columns in halves and
//               merge at the end of the point tile.
// Every wait is an mbarrier wait bounded in time (see km_ptx.cuh).
#include <cuda_bf16.h>
#include <math_constants.h>

#include "km_internal.h"
#include "km_ptx.cuh"

namespace km {

struct AssignK {
  int B;
  int64_t rows;
  int K, Kp, natoms, XB, CS, nct;
  int64_t tiles_per_inst, ntiles;
  const float* xn;
  const float* cn;
  int32_t* idx;
  float* mindist;
  double* tobj;
  int obj_per_cta;  // 1: tobj[cta][4] sums over the CTA's tiles in order; 0: tobj[tile][4]
  unsigned int* status;
  uint64_t limit_ns;
};

constexpr int kAtomBytesPerRow = 128;
constexpr int kXAtomBytes = kTileM * kAtomBytesPerRow;  // 16 KB per point-tile atom

template <int BN>
__host__ __device__ constexpr size_t assign_smem_bytes(int natoms, int XB, int CS) {
  return 1024 /* alignment slack */ + static_cast<size_t>(XB) * natoms * kXAtomBytes +
         static_cast<size_t>(CS) * natoms * BN * kAtomBytesPerRow + kCnStages * BN * 4 + kTileM * 8 +
         32 * 8 /* barriers */ + 16;
}

template <int BN, bool TF32>
__global__ void __launch_bounds__(kAssignThreads, 1)
    k_assign(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap cmap, const AssignK p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int natoms = p.natoms;
  const int XB = p.XB, CS = p.CS;
  uint8_t* xs = base;
  uint8_t* cs = xs + static_cast<size_t>(XB) * natoms * kXAtomBytes;
  float* cns = reinterpret_cast<float*>(cs + static_cast<size_t>(CS) * natoms * BN * kAtomBytesPerRow);
  float* mval = cns + kCnStages * BN;
  int* midx = reinterpret_cast<int*>(mval + kTileM);
  uint64_t* bars = reinterpret_cast<uint64_t*>(midx + kTileM);
  uint64_t* x_full = bars + 0;    // [2]
  uint64_t* x_empty = bars + 2;   // [2]
  uint64_t* c_full = bars + 4;    // [4]
  uint64_t* c_empty = bars + 8;   // [4]
  uint64_t* n_full = bars + 12;   // [4]
  uint64_t* n_empty = bars + 16;  // [4]
  uint64_t* a_full = bars + 20;   // [2]
  uint64_t* a_empty = bars + 22;  // [2]
  uint64_t* m_full = bars + 24;
  uint64_t* m_empty = bars + 25;
  uint64_t* drain = bars + 26;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr uint32_t kTmemCols = 2 * BN;
  constexpr int kHalf = BN / 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], 1);
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 8);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&c_full[i], 1);
      mbar_init(&c_empty[i], 1);
      mbar_init(&n_full[i], 1);
      mbar_init(&n_empty[i], 8);
    }
    mbar_init(m_full, kTileM);
    mbar_init(m_empty, kTileM);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const WaitGuard g{p.status, abort_flag, p.limit_ns};
  const int nct = p.nct;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      prefetch_tensormap(&xmap);
      prefetch_tensormap(&cmap);
      int xb = 0, cst = 0, ns = 0;
      uint32_t xph = 0, cph = 0, nph = 0;
      int x_iss[2] = {-1, -1}, c_iss[4] = {-1, -1, -1, -1}, n_iss[4] = {-1, -1, -1, -1};
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < p.ntiles; t += gridDim.x) {
        const int b = static_cast<int>(t / p.tiles_per_inst);
        const int rt = static_cast<int>(t - static_cast<int64_t>(b) * p.tiles_per_inst);
        if (!mbar_wait(&x_empty[xb], xph ^ 1u, g)) { ok = false; break; }
        mbar_arrive_expect_tx(&x_full[xb], static_cast<uint32_t>(natoms) * kXAtomBytes);
        for (int a = 0; a < natoms; ++a)
          tma_load_3d(xs + (static_cast<size_t>(xb) * natoms + a) * kXAtomBytes, &xmap,
                      a * (TF32 ? 32 : 64), rt * kTileM, b, &x_full[xb]);
        x_iss[xb] = static_cast<int>(xph);
        if (++xb == XB) { xb = 0; xph ^= 1u; }
        for (int j = 0; j < nct; ++j) {
          if (!mbar_wait(&c_empty[cst], cph ^ 1u, g)) { ok = false; break; }
          mbar_arrive_expect_tx(&c_full[cst], static_cast<uint32_t>(natoms) * BN * kAtomBytesPerRow);
          for (int a = 0; a < natoms; ++a)
            tma_load_3d(cs + (static_cast<size_t>(cst) * natoms + a) * BN * kAtomBytesPerRow, &cmap,
                        a * (TF32 ? 32 : 64), j * BN, b, &c_full[cst]);
          c_iss[cst] = static_cast<int>(cph);
          if (++cst == CS) { cst = 0; cph ^= 1u; }
          if (!mbar_wait(&n_empty[ns], nph ^ 1u, g)) { ok = false; break; }
          mbar_arrive_expect_tx(&n_full[ns], BN * 4);
          bulk_load(cns + ns * BN, p.cn + static_cast<int64_t>(b) * p.Kp + static_cast<int64_t>(j) * BN, BN * 4,
                    &n_full[ns]);
          n_iss[ns] = static_cast<int>(nph);
          if (++ns == kCnStages) { ns = 0; nph ^= 1u; }
        }
      }
      if (!ok) {
        // Let copies already in flight land before the CTA can exit.
        WaitGuard g2 = g;
        volatile int never = 0;
        g2.abort_flag = &never;
        for (int i = 0; i < XB; ++i) if (x_iss[i] >= 0) mbar_wait(&x_full[i], static_cast<uint32_t>(x_iss[i]), g2);
        for (int i = 0; i < CS; ++i) if (c_iss[i] >= 0) mbar_wait(&c_full[i], static_cast<uint32_t>(c_iss[i]), g2);
        for (int i = 0; i < kCnStages; ++i)
          if (n_iss[i] >= 0) mbar_wait(&n_full[i], static_cast<uint32_t>(n_iss[i]), g2);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = umma_idesc(TF32, kTileM, BN);
      constexpr int kSteps = 4;  // 32-byte K steps per 128-byte atom
      int xb = 0, cst = 0, ab = 0;
      uint32_t xph = 0, cph = 0, aph = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < p.ntiles; t += gridDim.x) {
        if (!mbar_wait(&x_full[xb], xph, g)) { ok = false; break; }
        const uint32_t xaddr = smem_addr(xs + static_cast<size_t>(xb) * natoms * kXAtomBytes);
        for (int j = 0; j < nct; ++j) {
          if (!mbar_wait(&c_full[cst], cph, g)) { ok = false; break; }
          if (!mbar_wait(&a_empty[ab], aph ^ 1u, g)) { ok = false; break; }
          tc_fence_after();
          const uint32_t caddr = smem_addr(cs + static_cast<size_t>(cst) * natoms * BN * kAtomBytesPerRow);
          const uint32_t dtm = tmem_base + static_cast<uint32_t>(ab * BN);
          for (int a = 0; a < natoms; ++a) {
#pragma unroll
            for (int s = 0; s < kSteps; ++s) {
              const uint64_t ad = sw128_kmajor_desc(xaddr + a * kXAtomBytes + s * 32);
              const uint64_t bd = sw128_kmajor_desc(caddr + a * BN * kAtomBytesPerRow + s * 32);
              umma_ss<TF32>(dtm, ad, bd, idesc, (a | s) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&c_empty[cst]);
          umma_commit(&a_full[ab]);
          if (++cst == CS) { cst = 0; cph ^= 1u; }
          if (++ab == 2) { ab = 0; aph ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&x_empty[xb]);
        if (++xb == XB) { xb = 0; xph ^= 1u; }
      }
      // Wait for every MMA this thread issued before TMEM can be released.
      umma_commit(drain);
      WaitGuard g2 = g;
      volatile int never = 0;
      g2.abort_flag = &never;
      mbar_wait(drain, 0u, g2);
    }
  } else {
    // -------------------------------------------------- epilogue warps
    const int ew = warp - 2;
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    const int h = ew >> 2;    // column half of each accumulator tile
    const int r_local = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    int ab = 0, ns = 0;
    uint32_t aph = 0, nph = 0, mph = 0;
    bool ok = true;
    double cta_obj = 0.0;
    for (int64_t t = blockIdx.x; ok && t < p.ntiles; t += gridDim.x) {
      const int b = static_cast<int>(t / p.tiles_per_inst);
      const int64_t rt = t - static_cast<int64_t>(b) * p.tiles_per_inst;
      const int64_t row = rt * kTileM + r_local;
      const bool valid = row < p.rows;
      float best = CUDART_INF_F;
      int bk = 0;
      for (int j = 0; j < nct; ++j) {
        if (!mbar_wait(&a_full[ab], aph, g) || !mbar_wait(&n_full[ns], nph, g)) { ok = false; break; }
        tc_fence_after();
        const float* cnp = cns + ns * BN + h * kHalf;
        float lb[4] = {CUDART_INF_F, CUDART_INF_F, CUDART_INF_F, CUDART_INF_F};
        int li[4] = {0, 0, 0, 0};
#pragma unroll
        for (int c = 0; c < kHalf / 32; ++c) {
          float v[32];
          tmem_ld32(tmem_base + lane_off + static_cast<uint32_t>(ab * BN + h * kHalf + c * 32), v);
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const float4 c4 = *reinterpret_cast<const float4*>(cnp + c * 32 + i4 * 4);
            const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float s = fmaf(-2.f, v[i4 * 4 + u], cv[u]);
              const bool pr = s < lb[u];
              lb[u] = pr ? s : lb[u];
              li[u] = pr ? (c * 32 + i4 * 4 + u) : li[u];
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&a_empty[ab]);
          mbar_arrive(&n_empty[ns]);
        }
        const int kbase = j * BN + h * kHalf;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int k = kbase + li[u];
          if (lb[u] < best || (lb[u] == best && k < bk)) {
            best = lb[u];
            bk = k;
          }
        }
        if (++ab == 2) { ab = 0; aph ^= 1u; }
        if (++ns == kCnStages) { ns = 0; nph ^= 1u; }
      }
      if (!ok) break;
      // merge the two column halves of this point tile
      if (h == 1) {
        if (!mbar_wait(m_empty, mph ^ 1u, g)) { ok = false; break; }
        mval[r_local] = best;
        midx[r_local] = bk;
        mbar_arrive(m_full);
      } else {
        if (!mbar_wait(m_full, mph, g)) { ok = false; break; }
        const float ob = mval[r_local];
        const int ok_ = midx[r_local];
        mbar_arrive(m_empty);
        if (ob < best || (ob == best && ok_ < bk)) {
          best = ob;
          bk = ok_;
        }
        float md = 0.f;
        if (valid) {
          const int64_t o = static_cast<int64_t>(b) * p.rows + row;
          md = fmaxf(0.f, p.xn[o] + best);
          p.idx[o] = bk;
          if (p.mindist) p.mindist[o] = md;
        }
        double ds = static_cast<double>(md);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
        if (p.obj_per_cta) cta_obj += ds;
        else if (lane == 0 && p.tobj) p.tobj[t * 4 + q] = ds;
      }
      mph ^= 1u;
    }
    if (h == 0 && p.obj_per_cta && lane == 0 && p.tobj) p.tobj[static_cast<int64_t>(blockIdx.x) * 4 + q] = cta_obj;
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int BN, bool TF32>
static cudaError_t launch_t(const Plan& pl, const AssignArgs& a, cudaStream_t s) {
  AssignK k{};
  k.B = a.B;
  k.rows = a.rows;
  k.K = a.K;
  k.Kp = a.Kp;
  k.natoms = pl.ac.natoms;
  k.XB = pl.ac.XB;
  k.CS = pl.ac.CS;
  k.nct = a.Kp / BN;
  k.tiles_per_inst = (a.rows + kTileM - 1) / kTileM;
  k.ntiles = k.tiles_per_inst * a.B;
  k.xn = a.xn;
  k.cn = a.cn;
  k.idx = a.idx;
  k.mindist = a.mindist;
  k.tobj = a.tobj;
  k.obj_per_cta = a.B == 1 ? 1 : 0;
  k.status = a.status;
  k.limit_ns = a.limit_ns;
  const size_t smem = assign_smem_bytes<BN>(k.natoms, k.XB, k.CS);
  cudaError_t e = cudaFuncSetAttribute(k_assign<BN, TF32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = k.ntiles < nsm ? k.ntiles : nsm;
  if (a.obj_groups) *a.obj_groups = k.obj_per_cta ? grid : k.tiles_per_inst;
  if (grid <= 0) return cudaSuccess;
  count_launch();
  k_assign<BN, TF32><<<static_cast<unsigned>(grid), kAssignThreads, smem, s>>>(*a.xmap, *a.cmap, k);
  return cudaGetLastError();
}

size_t assign_smem_for(int BN, int natoms, int XB, int CS) {
  switch (BN) {
    case 256: return assign_smem_bytes<256>(natoms, XB, CS);
    case 128: return assign_smem_bytes<128>(natoms, XB, CS);
    default: return assign_smem_bytes<64>(natoms, XB, CS);
  }
}

cudaError_t launch_assign(const Plan& p, const AssignArgs& a, cudaStream_t s) {
  const bool tf32 = p.dtype == kDtypeF32;
  switch (p.ac.BN) {
    case 256: return tf32 ? launch_t<256, true>(p, a, s) : launch_t<256, false>(p, a, s);
    case 128: return tf32 ? launch_t<128, true>(p, a, s) : launch_t<128, false>(p, a, s);
    case 64: return tf32 ? launch_t<64, true>(p, a, s) : launch_t<64, false>(p, a, s);
    default: return cudaErrorInvalidValue;
  }
}

// ------------------------------------------------------- timeout self-test
__global__ void k_timeout_probe(unsigned int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitGuard g{status, reinterpret_cast<volatile int*>(&abort_flag), limit_ns};
    mbar_wait(&bar, 0u, g);  // nothing arrives: runs out after limit_ns
  }
  __syncthreads();
}

cudaError_t launch_timeout_probe(unsigned int* status, uint64_t limit_ns, cudaStream_t s) {
  count_launch();
  k_timeout_probe<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace km
