// k_assign.cu -- FlashAssign on sm_100a ("Flash-KMeans: Fast and
// Memory-Efficient Exact K-Means", §2.1 FlashAssign).
//
// For a tile of 128 points the kernel streams every centroid tile through the
// tensor cores and keeps, per point, the running minimum distance and its
// centroid index (the §2.1 online argmin: each point carries its current best
// distance and cluster id; each new tile's local minimum is merged into it).
// The N x K distances live only in tensor memory; device memory sees X once,
// the centroid tiles (from L2) and the N-long outputs, i.e. O(Nd + Kd)
// traffic instead of O(NK) (§2.1, "效果").
//
// The tensor cores produce the whole distance, not just the cross term: the
// operands carry one extra 32-byte K-slice (km_rows.cuh, "norm augmentation")
// so that one UMMA chain accumulates
//     ||x||^2 + ||c||^2 - 2 x.c        (centroid operand holds -2c)
// and the epilogue is a pure argmin.  Per score it forms a key -- the float
// bits with the 5 low mantissa bits replaced by the column inside its
// 32-column chunk -- and reduces keys with 3-input float minimum; a chunk's
// winner is merged into the running best only on a strictly smaller
// distance, and the column quarters of a tile merge lowest index first on
// equal distances, so equal scores go to the lowest index -- except inside
// one chunk when they are negative, where a larger column makes a more
// negative key.  Equal negative scores mean a zero distance (a point on a
// centroid; the expanded form lands a few ulps either side of 0) to two or
// more identical centroid rows, which the tensor cores score bit for bit
// alike.  So a point whose best ends at or below zero takes the lowest
// centroid of its winning chunk whose operand row equals the winner's (a
// rare pass in which the warp compares up to 31 rows at once).  The lowest
// index wins exact ties.  (Distances closer than 2^-18 relative also compare equal; that is
// far inside the parity rule's near-tie band.)
//
// Structure: persistent CTAs (one per SM), warp-specialised:
//   warp 0       TMA producer: point tile + its augmentation (resident for the
//                whole centroid sweep, double buffered across tiles), centroid
//                tiles + augmentation through a ring of stages (the §2.1
//                asynchronous double-buffered prefetch);
//   warp 1       tcgen05.mma issuer (one thread): M=128 x N=BN x K=16 (bf16)
//                or K=8 (tf32) steps into a double-buffered TMEM accumulator;
//   warps 2..17  epilogue: 4 warps per TMEM lane quarter, each owning a
//                quarter of the BN columns; tcgen05.ld, key, min tree; the
//                four column quarters merge at the end of the point tile.
// Pair variant (PAIR=true): two CTAs of a cluster on an SM pair cooperate on
// 256-point tiles with cta_group::2 UMMAs (M=256): each CTA holds its 128
// points and half of every centroid tile, the lead CTA issues the MMAs, and
// each CTA's TMEM receives the distances of its own 128 points for the whole
// centroid tile.  Per SM this halves the centroid bytes streamed from L2 and
// read from shared memory, which leaves room for 4 centroid stages.
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
  int64_t tiles_per_inst, ntiles;  // tiles of TM points (256 for pairs, else 128)
  int64_t tiles128_per_inst;       // 128-point tiles per instance (per-tile objective layout)
  int32_t* idx;
  float* mindist;
  double* tobj;     // [B * tiles128_per_inst][4]: per 128-point tile, one sum per 32-row quarter
  uint32_t zero;    // always 0; keeps the epilogue's column constants in registers
  const uint8_t* cop;  // centroid operand rows (-2c), K per instance, cop_rb bytes each
  int64_t cop_rb;
  unsigned int* status;
  uint64_t limit_ns;
};

constexpr int kAtomBytesPerRow = 128;
constexpr int kXAtomBytes = kTileM * kAtomBytesPerRow;  // 16 KB per point-tile atom
constexpr int kAugRowBytes = 32;
constexpr int kEpiWarps = 16;
constexpr int kMaxXB = 8;  // point-tile buffers at most

__host__ __device__ constexpr size_t x_buf_bytes(int natoms) {
  return static_cast<size_t>(natoms) * kXAtomBytes + kTileM * kAugRowBytes;
}
__host__ __device__ constexpr size_t c_stage_bytes(int natoms, int rows) {
  return static_cast<size_t>(natoms) * rows * kAtomBytesPerRow + static_cast<size_t>(rows) * kAugRowBytes;
}

// BN centroids per MMA; a CTA of a pair holds BN/2 of them per stage.
template <int BN, bool PAIR>
__host__ __device__ constexpr size_t assign_smem_bytes(int natoms, int XB, int CS) {
  return 1024 /* alignment slack */ + XB * x_buf_bytes(natoms) + CS * c_stage_bytes(natoms, PAIR ? BN / 2 : BN) +
         3 * kTileM * 8 /* merge slots */ + 40 * 8 /* barriers */ + 16;
}

// Shared-memory descriptor for the 32-byte augmentation slice (K-major,
// 32-byte swizzle: rows of 32 bytes, 8-row groups 256 bytes apart).
__device__ __forceinline__ uint64_t sw32_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(256u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(6u) << 61;
  return d;
}

__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Start loading CW (16 or 32) consecutive TMEM columns of this thread's lane.
// The registers are valid only after tmem_ld_wait on the same array.
template <int CW>
__device__ __forceinline__ void tmem_ld_issue(uint32_t taddr, uint32_t (&r)[CW]);

template <>
__device__ __forceinline__ void tmem_ld_issue<32>(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

template <>
__device__ __forceinline__ void tmem_ld_issue<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// Wait for this thread's outstanding TMEM loads.  The registers of `r` pass
// through the statement, so no use of them can be scheduled before it.
template <int CW>
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[CW]);

template <>
__device__ __forceinline__ void tmem_ld_wait<32>(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

template <>
__device__ __forceinline__ void tmem_ld_wait<16>(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}

// Minimum key of CW scores: key = score bits with the low 5 bits replaced by
// the column index i in [0, CW) (mask == ~31 in a register, i an
// immediate), one three-input bitwise operation per score, reduced with
// 3-input minima.  With CLAMP the score is first raised to +0 (an integer
// maximum with 0: a negative float is a negative signed integer).
template <int CW, bool CLAMP>
__device__ __forceinline__ uint32_t chunk_min_key(const uint32_t (&v)[CW], uint32_t mask) {
  float k[CW];
#pragma unroll
  for (int i = 0; i < CW; ++i) {
    const uint32_t s = CLAMP ? static_cast<uint32_t>(max(static_cast<int32_t>(v[i]), 0)) : v[i];
    k[i] = __uint_as_float((s & mask) | static_cast<uint32_t>(i));
  }
  constexpr int L1 = CW / 3 + (CW % 3);  // CW=32: 10 triples + 2 singles; CW=16: 5 triples + 1 single
  float a[L1];
#pragma unroll
  for (int i = 0; i < CW / 3; ++i) a[i] = fmin3(k[3 * i], k[3 * i + 1], k[3 * i + 2]);
#pragma unroll
  for (int i = 0; i < CW % 3; ++i) a[CW / 3 + i] = k[3 * (CW / 3) + i];
  constexpr int L2 = L1 / 3 + (L1 % 3);
  float b[L2];
#pragma unroll
  for (int i = 0; i < L1 / 3; ++i) b[i] = fmin3(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
#pragma unroll
  for (int i = 0; i < L1 % 3; ++i) b[L1 / 3 + i] = a[3 * (L1 / 3) + i];
  float m = b[0];
  int i = 1;
#pragma unroll
  for (; i + 1 < L2; i += 2) m = fmin3(m, b[i], b[i + 1]);
  if (i < L2) m = fminf(m, b[i]);
  return __float_as_uint(m);
}

// Lowest centroid index in k's 32-column chunk whose operand row (rb
// bytes, a multiple of 16) equals row k's; rows holds the instance's rows.
// The whole warp takes part: lane c compares row (k & ~31) + c for the
// columns below k, so the candidates are read in one parallel round rather
// than one after another.  Runs only for points at distance 0.
__device__ __forceinline__ int lowest_copy(const uint8_t* rows, int64_t rb, int k, int lane) {
  const int c0 = k & ~31;
  bool eq = lane < (k & 31);
  if (eq) {
    const uint4* rk = reinterpret_cast<const uint4*>(rows + k * rb);
    const uint4* rc = reinterpret_cast<const uint4*>(rows + (c0 + lane) * rb);
    const int n16 = static_cast<int>(rb / 16);
    for (int i = 0; i < n16; ++i) {
      const uint4 u = rc[i], w = rk[i];
      if (u.x != w.x || u.y != w.y || u.z != w.z || u.w != w.w) {
        eq = false;
        break;
      }
    }
  }
  const unsigned m = __ballot_sync(0xffffffffu, eq);
  return m ? c0 + __ffs(m) - 1 : k;
}

// The warp's points at distance 0 (the zero set) take the lowest identical
// centroid row, one warp-wide comparison each.  This runs rarely.  The
// CTA-pair kernels call it out of line (inlined, it costs their hot loop
// two registers); the single-CTA kernels inline it (out of line, they
// spill).
__device__ __forceinline__ int zero_distance_ties_body(const uint8_t* rows, int64_t rb, int bk, bool zero, int lane) {
  for (unsigned need = __ballot_sync(0xffffffffu, zero); need; need &= need - 1) {
    const int src = __ffs(need) - 1;
    const int kk = lowest_copy(rows, rb, __shfl_sync(0xffffffffu, bk, src), lane);
    if (lane == src) bk = kk;
  }
  return bk;
}
__device__ __noinline__ int zero_distance_ties_call(const uint8_t* rows, int64_t rb, int bk, bool zero, int lane) {
  return zero_distance_ties_body(rows, rb, bk, zero, lane);
}
template <bool OUT_OF_LINE>
__device__ __forceinline__ int zero_distance_ties(const uint8_t* rows, int64_t rb, int bk, bool zero, int lane) {
  if constexpr (OUT_OF_LINE) return zero_distance_ties_call(rows, rb, bk, zero, lane);
  else return zero_distance_ties_body(rows, rb, bk, zero, lane);
}

// Point-tile position (instance b, tile rt inside it) of the one-tile
// kernels, advanced by counting: they take contiguous runs of tiles per CTA
// (or a single instance), and a 64-bit division per point tile, with only
// the few K-steps of one centroid tile behind it, was a large share of
// their instructions.  The other kernels divide once per point tile,
// amortised over its centroid tiles.
struct TileCount {
  int b;
  int64_t rt;
  __device__ __forceinline__ TileCount(int64_t t0, int64_t tpi, int B) : b(0), rt(t0) {
    if (B > 1) {
      b = static_cast<int>(t0 / tpi);
      rt = t0 - static_cast<int64_t>(b) * tpi;
    }
  }
  // to the next tile of this CTA (B > 1 implies step 1 in these kernels)
  __device__ __forceinline__ void advance(int64_t step, int64_t tpi, int B) {
    if (B == 1) {
      rt += step;
    } else if (++rt == tpi) {
      rt = 0;
      ++b;
    }
  }
};

// ONE_CT: one centroid tile per point tile (K <= BN), kept resident per
// instance (see the producer and the MMA issuer).
template <int BN, bool TF32, bool PAIR, bool ONE_CT>
__global__ void __launch_bounds__(kAssignThreads, 1)
    k_assign(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap xamap,
             const __grid_constant__ CUtensorMap cmap, const __grid_constant__ CUtensorMap camap, const AssignK p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int HB = PAIR ? BN / 2 : BN;       // centroid rows of a stage held by this CTA
  constexpr int TM = PAIR ? 2 * kTileM : kTileM;  // points per tile of the (pair of) CTA(s)
  const int natoms = p.natoms;
  const int XB = p.XB, CS = p.CS;
  const size_t xbb = x_buf_bytes(natoms), csb = c_stage_bytes(natoms, HB);
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int64_t unit = PAIR ? blockIdx.x / 2 : blockIdx.x;     // this CTA's (pair's) index
  const int64_t nunits = PAIR ? gridDim.x / 2 : gridDim.x;
  // Tile order of this CTA (pair).  Batched problems with one centroid tile
  // per point tile take a contiguous run of tiles, so consecutive tiles
  // belong to the same instance and its centroid tile stays resident (see
  // below); otherwise tiles are dealt round robin, which keeps the CTAs'
  // point-tile reads close together in memory (measured faster for one
  // large instance).
  const bool contig = ONE_CT && p.B > 1;
  const int64_t t_first = contig ? unit * p.ntiles / nunits : unit;
  const int64_t t_end = contig ? (unit + 1) * p.ntiles / nunits : p.ntiles;
  const int64_t t_step = contig ? 1 : nunits;
  uint8_t* xs = base;
  uint8_t* cs = xs + XB * xbb;
  float* mval = reinterpret_cast<float*>(cs + CS * csb);  // [3][128]
  int* midx = reinterpret_cast<int*>(mval + 3 * kTileM);  // [3][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(midx + 3 * kTileM);
  uint64_t* x_full = bars + 0;    // [kMaxXB]
  uint64_t* x_empty = bars + 8;   // [kMaxXB]
  uint64_t* c_full = bars + 16;   // [4]
  uint64_t* c_empty = bars + 20;  // [4]
  uint64_t* a_full = bars + 24;   // [2]
  uint64_t* a_empty = bars + 26;  // [2]
  uint64_t* m_full = bars + 28;
  uint64_t* m_empty = bars + 29;
  uint64_t* drain = bars + 30;
  uint64_t* g_full = bars + 31;   // [2] one-tile merge inside epilogue group g
  uint64_t* g_empty = bars + 33;  // [2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 36);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr uint32_t kTmemCols = 2 * BN;
  constexpr int kHalf = BN / 2;                // columns per epilogue warp per tile
  constexpr int CW = kHalf < 32 ? kHalf : 32;  // columns per TMEM load
  constexpr int kChunks = kHalf / CW;
  constexpr int kElem = TF32 ? 32 : 64;      // elements per 128-byte atom row

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxXB; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a_full[i], 1);
      // one epilogue group (half the epilogue warps) reads each accumulator
      // buffer; for pairs both CTAs' groups release the lead's barrier
      mbar_init(&a_empty[i], PAIR ? kEpiWarps : kEpiWarps / 2);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&c_full[i], 1);
      mbar_init(&c_empty[i], 1);
    }
    mbar_init(m_full, 3 * kTileM);
    mbar_init(m_empty, kTileM);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&g_full[i], kTileM);
      mbar_init(&g_empty[i], kTileM);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_holder, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // peers' barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // Everything above touched only this CTA's (pair's) shared memory and
  // TMEM; from here on the centroid operands, the sort counts and the
  // objective partials are shared with the previous kernels.  (This kernel
  // does not signal launch_dependents: the next one becomes resident only as
  // its CTAs exit, which measured faster than letting it in at the start.)
  pdl_wait();
  const WaitGuard g{p.status, abort_flag, p.limit_ns};
  const int nct = p.nct;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      prefetch_tensormap(&xmap);
      prefetch_tensormap(&xamap);
      prefetch_tensormap(&cmap);
      prefetch_tensormap(&camap);
      int xb = 0, cst = 0;
      uint32_t xph = 0, cph = 0;
      int x_iss[kMaxXB], c_iss[4] = {-1, -1, -1, -1};
      for (int i = 0; i < kMaxXB; ++i) x_iss[i] = -1;
      int64_t b_loaded = -1;
      bool ok = true;
      // Loads of a pair complete on the lead CTA's barriers; only the lead
      // posts the expected bytes (both CTAs' share).
      auto load = [&](void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
        if constexpr (PAIR) tma_load_3d_pair(dst, map, x, y, z, mapa_shared(smem_addr(bar), 0));
        else tma_load_3d(dst, map, x, y, z, bar);
      };
      TileCount tcn(t_first, p.tiles_per_inst, p.B);
      for (int64_t t = t_first; ok && t < t_end; t += t_step) {
        const int b = ONE_CT ? tcn.b : static_cast<int>(t / p.tiles_per_inst);
        const int rt = ONE_CT ? static_cast<int>(tcn.rt) : static_cast<int>(t - static_cast<int64_t>(b) * p.tiles_per_inst);
        if constexpr (ONE_CT) tcn.advance(t_step, p.tiles_per_inst, p.B);
        const int row0 = rt * TM + static_cast<int>(rank) * kTileM;
        if (!mbar_wait(&x_empty[xb], xph ^ 1u, g)) { ok = false; break; }
        uint8_t* xdst = xs + xb * xbb;
        if (leader) mbar_arrive_expect_tx(&x_full[xb], static_cast<uint32_t>((PAIR ? 2 : 1) * xbb));
        for (int a = 0; a < natoms; ++a) load(xdst + a * kXAtomBytes, &xmap, a * kElem, row0, b, &x_full[xb]);
        load(xdst + natoms * kXAtomBytes, &xamap, 0, row0, b, &x_full[xb]);
        x_iss[xb] = static_cast<int>(xph);
        if (++xb == XB) { xb = 0; xph ^= 1u; }
        // One centroid tile per point tile: it stays resident while the
        // instance does not change (the MMA issuer releases the stage then).
        if constexpr (ONE_CT) {
          if (b == b_loaded) continue;
          b_loaded = b;
        }
        for (int j = 0; j < nct; ++j) {
          if (!mbar_wait(&c_empty[cst], cph ^ 1u, g)) { ok = false; break; }
          uint8_t* cdst = cs + cst * csb;
          const int crow0 = j * BN + static_cast<int>(rank) * HB;
          if (leader) mbar_arrive_expect_tx(&c_full[cst], static_cast<uint32_t>((PAIR ? 2 : 1) * csb));
          for (int a = 0; a < natoms; ++a)
            load(cdst + static_cast<size_t>(a) * HB * kAtomBytesPerRow, &cmap, a * kElem, crow0, b, &c_full[cst]);
          load(cdst + static_cast<size_t>(natoms) * HB * kAtomBytesPerRow, &camap, 0, crow0, b, &c_full[cst]);
          c_iss[cst] = static_cast<int>(cph);
          if (++cst == CS) { cst = 0; cph ^= 1u; }
        }
      }
      if (!ok) {
        // Let copies already in flight land before the CTA can exit.
        if (PAIR && !leader) {
          // this CTA's copies complete on the lead's barriers: give them time
          const uint64_t t0 = global_timer_ns();
          while (global_timer_ns() - t0 < 200000) {
          }
        } else {
          WaitGuard g2 = g;
          volatile int never = 0;
          g2.abort_flag = &never;
          for (int i = 0; i < XB; ++i)
            if (x_iss[i] >= 0) mbar_wait(&x_full[i], static_cast<uint32_t>(x_iss[i]), g2);
          for (int i = 0; i < CS; ++i)
            if (c_iss[i] >= 0) mbar_wait(&c_full[i], static_cast<uint32_t>(c_iss[i]), g2);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = umma_idesc(TF32, TM, BN);
      constexpr int kSteps = 4;  // 32-byte K steps per 128-byte atom
      auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t acc) {
        if constexpr (PAIR) umma_ss_pair<TF32>(d, ad, bd, idesc, acc);
        else umma_ss<TF32>(d, ad, bd, idesc, acc);
      };
      auto commit = [&](uint64_t* bar) {  // arrives on the barrier in every CTA of the pair
        if constexpr (PAIR) umma_commit_pair(bar, 0x3);
        else umma_commit(bar);
      };
      int xb = 0, cst = 0, ab = 0;
      uint32_t xph = 0, cph = 0, aph = 0;
      bool ok = true;
      int64_t b_cur = -1;
      TileCount tcn(t_first, p.tiles_per_inst, p.B);
      for (int64_t t = t_first; ok && t < t_end; t += t_step) {
        if (!mbar_wait(&x_full[xb], xph, g)) { ok = false; break; }
        const uint32_t xaddr = smem_addr(xs + xb * xbb);
        bool keep = false;  // stage cst already holds this instance's tile
        if constexpr (ONE_CT) {
          const int64_t b = tcn.b;
          tcn.advance(t_step, p.tiles_per_inst, p.B);
          keep = b == b_cur;
          if (!keep && b_cur >= 0) {  // leave the previous instance's stage
            commit(&c_empty[cst]);
            if (++cst == CS) { cst = 0; cph ^= 1u; }
          }
          b_cur = b;
        }
        for (int j = 0; j < nct; ++j) {
          if (!keep && !mbar_wait(&c_full[cst], cph, g)) { ok = false; break; }
          if (!mbar_wait(&a_empty[ab], aph ^ 1u, g)) { ok = false; break; }
          tc_fence_after();
          const uint32_t caddr = smem_addr(cs + cst * csb);
          const uint32_t dtm = tmem_base + static_cast<uint32_t>(ab * BN);
          for (int a = 0; a < natoms; ++a) {
#pragma unroll
            for (int s = 0; s < kSteps; ++s) {
              const uint64_t ad = sw128_kmajor_desc(xaddr + a * kXAtomBytes + s * 32);
              const uint64_t bd = sw128_kmajor_desc(caddr + a * HB * kAtomBytesPerRow + s * 32);
              mma(dtm, ad, bd, (a | s) != 0 ? 1u : 0u);
            }
          }
          mma(dtm, sw32_kmajor_desc(xaddr + natoms * kXAtomBytes),
              sw32_kmajor_desc(caddr + natoms * HB * kAtomBytesPerRow), 1u);
          if constexpr (!ONE_CT) {
            commit(&c_empty[cst]);
            if (++cst == CS) { cst = 0; cph ^= 1u; }
          }
          commit(&a_full[ab]);
          if (++ab == 2) { ab = 0; aph ^= 1u; }
        }
        if (!ok) break;
        commit(&x_empty[xb]);
        if (++xb == XB) { xb = 0; xph ^= 1u; }
      }
      // Wait for every MMA this thread issued before TMEM can be released.
      if constexpr (PAIR) umma_commit_pair(drain, 0x1);
      else umma_commit(drain);
      WaitGuard g2 = g;
      volatile int never = 0;
      g2.abort_flag = &never;
      mbar_wait(drain, 0u, g2);
    }
  } else {
    // -------------------------------------------------- epilogue warps
    // Two groups of 8 warps; group g reads accumulator buffer g, i.e. every
    // other centroid tile, so each group has two MMA tiles' time per tile and
    // the groups' bursts of work interleave.  Within a group, 2 warps per TMEM
    // lane quarter each take half of the tile's columns, in CW-column chunks
    // whose TMEM loads run one chunk ahead of the reduction.
    const int ew = warp - 2;
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int grp = ew >> 3;           // accumulator buffer this warp reads
    const int half = (ew >> 2) & 1;    // column half of each accumulator tile
    const int h = grp * 2 + half;      // partial-result slot of the merge
    const int r_local = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t aph = 0, mph = 0, gph = 0;
    bool ok = true;
    const uint32_t kmask = ~31u + p.zero;
    const uint32_t a_empty_lead = PAIR ? mapa_shared(smem_addr(&a_empty[grp]), 0) : 0u;
    int64_t ct0 = 0;  // centroid tiles this CTA processed before the current point tile
    TileCount tcn(t_first, p.tiles_per_inst, p.B);
    for (int64_t t = t_first; ok && t < t_end; t += t_step, ct0 += nct) {
      const int b = ONE_CT ? tcn.b : static_cast<int>(t / p.tiles_per_inst);
      const int64_t rt = ONE_CT ? tcn.rt : t - static_cast<int64_t>(b) * p.tiles_per_inst;
      if constexpr (ONE_CT) tcn.advance(t_step, p.tiles_per_inst, p.B);
      const int64_t row = rt * TM + static_cast<int64_t>(rank) * kTileM + r_local;
      const bool valid = row < p.rows;
      float best = CUDART_INF_F;
      int bk = 0;
      for (int j = static_cast<int>((ct0 + grp) & 1); j < nct; j += 2) {
        // the MMA issuer alternates buffers per centroid tile: tile ct0 + j uses buffer (ct0 + j) & 1 == grp
        if (!mbar_wait(&a_full[grp], aph, g)) { ok = false; break; }
        tc_fence_after();
        const uint32_t col0 = tmem_base + lane_off + static_cast<uint32_t>(grp * BN + half * kHalf);
        uint32_t v[2][CW];
        tmem_ld_issue<CW>(col0, v[0]);
        tmem_ld_wait<CW>(v[0]);
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          if (c + 1 < kChunks) tmem_ld_issue<CW>(col0 + static_cast<uint32_t>((c + 1) * CW), v[(c + 1) & 1]);
          const uint32_t m = chunk_min_key<CW, false>(v[c & 1], kmask);
          const float mv = __uint_as_float(m & ~31u);
          if (mv < best) {
            best = mv;
            bk = j * BN + half * kHalf + c * CW + static_cast<int>(m & 31u);
          }
          if (c + 1 < kChunks) tmem_ld_wait<CW>(v[(c + 1) & 1]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR && !leader) mbar_arrive_cluster(a_empty_lead);
          else mbar_arrive(&a_empty[grp]);
        }
        aph ^= 1u;
      }
      if (!ok) break;
      // the point tile's result: argmin index, distance, sort counts, objective
      auto emit = [&]() {
        float md = 0.f;
        if (p.cop && __any_sync(0xffffffffu, valid && best <= 0.f))
          bk = zero_distance_ties<PAIR>(p.cop + static_cast<int64_t>(b) * p.K * p.cop_rb, p.cop_rb, bk,
                                        valid && best <= 0.f, lane);
        if (valid) {
          const int64_t o = static_cast<int64_t>(b) * p.rows + row;
          md = fmaxf(0.f, best);
          p.idx[o] = bk;
          if (p.mindist) p.mindist[o] = md;
        }
        double ds = static_cast<double>(md);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
        // objective partial of this 32-row quarter of the 128-point tile: the
        // slot depends on the tile index only, so the later fixed-order
        // reduction does not depend on how tiles were dealt to CTAs
        if (lane == 0 && p.tobj) {
          const int64_t tile128 = rt * (TM / kTileM) + rank;
          if (tile128 * kTileM < p.rows) p.tobj[(static_cast<int64_t>(b) * p.tiles128_per_inst + tile128) * 4 + q] = ds;
        }
      };
      auto better = [&](float ov, int oi) {
        if (ov < best || (ov == best && oi < bk)) {
          best = ov;
          bk = oi;
        }
      };
      if constexpr (ONE_CT) {
        // One accumulator tile per point tile: the owning group's two column
        // halves merge through the group's own slots; the other group skips
        // the tile, so the two groups never wait for each other.
        if (((ct0 + grp) & 1) != 0) continue;
        if (half != 0) {
          if (!mbar_wait(&g_empty[grp], gph ^ 1u, g)) { ok = false; break; }
          mval[grp * kTileM + r_local] = best;
          midx[grp * kTileM + r_local] = bk;
          mbar_arrive(&g_full[grp]);
        } else {
          if (!mbar_wait(&g_full[grp], gph, g)) { ok = false; break; }
          better(mval[grp * kTileM + r_local], midx[grp * kTileM + r_local]);
          mbar_arrive(&g_empty[grp]);
          emit();
        }
        gph ^= 1u;
        continue;
      }
      // merge the four column quarters of this point tile
      if (h != 0) {
        if (!mbar_wait(m_empty, mph ^ 1u, g)) { ok = false; break; }
        mval[(h - 1) * kTileM + r_local] = best;
        midx[(h - 1) * kTileM + r_local] = bk;
        mbar_arrive(m_full);
      } else {
        if (!mbar_wait(m_full, mph, g)) { ok = false; break; }
#pragma unroll
        for (int hh = 0; hh < 3; ++hh) better(mval[hh * kTileM + r_local], midx[hh * kTileM + r_local]);
        mbar_arrive(m_empty);
        emit();
      }
      mph ^= 1u;
    }
  }

  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // the lead's MMAs no longer read this CTA's shared memory
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int BN, bool TF32, bool PAIR, bool ONE_CT>
static cudaError_t launch_t(const Plan& pl, const AssignArgs& a, cudaStream_t s) {
  constexpr int TM = PAIR ? 2 * kTileM : kTileM;
  AssignK k{};
  k.B = a.B;
  k.rows = a.rows;
  k.K = a.K;
  k.Kp = a.Kp;
  k.natoms = pl.ac.natoms;
  k.XB = pl.ac.XB;
  k.CS = pl.ac.CS;
  k.nct = a.Kp / BN;
  k.tiles_per_inst = (a.rows + TM - 1) / TM;
  k.tiles128_per_inst = (a.rows + kTileM - 1) / kTileM;
  k.ntiles = k.tiles_per_inst * a.B;
  k.idx = a.idx;
  k.mindist = a.mindist;
  k.tobj = a.tobj;
  k.zero = 0;
  k.cop = static_cast<const uint8_t*>(a.cop);
  k.cop_rb = static_cast<int64_t>(a.cop_row_bytes);
  k.status = a.status;
  k.limit_ns = a.limit_ns;
  const size_t smem = assign_smem_bytes<BN, PAIR>(k.natoms, k.XB, k.CS);
  cudaError_t e = cudaFuncSetAttribute(k_assign<BN, TF32, PAIR, ONE_CT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  // one CTA (or CTA pair) per SM (pair), never more than there are tiles;
  // pairs: as many as can be resident at once (clusters must fit in a GPC)
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  int64_t units = nsm;
  if constexpr (PAIR) {
    cfg.blockDim = dim3(kAssignThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(nsm / 2 * 2));
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, k_assign<BN, TF32, true, ONE_CT>, &cfg) != cudaSuccess ||
        clusters < 1)
      clusters = nsm / 2;
    units = clusters;
  }
  const int64_t active = k.ntiles < units ? k.ntiles : units;
  const int64_t grid = PAIR ? 2 * active : active;
  if (a.obj_groups) *a.obj_groups = k.tiles128_per_inst;
  if (grid <= 0) return cudaSuccess;
  if (fault_hit(kFaultLaunch)) {
    chain_break();
    return cudaErrorLaunchFailure;
  }
  count_launch();
  cudaLaunchConfig_t lc{};
  lc.gridDim = dim3(static_cast<unsigned>(grid));
  lc.blockDim = dim3(kAssignThreads);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute la[2];
  int na = 0;
  if constexpr (PAIR) {
    la[na].id = cudaLaunchAttributeClusterDimension;
    la[na].val.clusterDim.x = 2;
    la[na].val.clusterDim.y = 1;
    la[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl_enabled() && chain_armed()) {
    la[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    la[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  lc.attrs = la;
  lc.numAttrs = na;
  e = cudaLaunchKernelEx(&lc, k_assign<BN, TF32, PAIR, ONE_CT>, *a.xmap, *a.xamap, *a.cmap, *a.camap, k);
  if (e == cudaSuccess) chain_arm();
  else chain_break();
  return e;
}

size_t assign_smem_for(int BN, int natoms, int XB, int CS, bool pair) {
  switch (BN) {
    case 256: return pair ? assign_smem_bytes<256, true>(natoms, XB, CS) : assign_smem_bytes<256, false>(natoms, XB, CS);
    case 128: return pair ? assign_smem_bytes<128, true>(natoms, XB, CS) : assign_smem_bytes<128, false>(natoms, XB, CS);
    default: return assign_smem_bytes<64, false>(natoms, XB, CS);
  }
}

template <int BN, bool TF32, bool PAIR>
static cudaError_t launch_ct(const Plan& p, const AssignArgs& a, cudaStream_t s) {
  return a.Kp == BN ? launch_t<BN, TF32, PAIR, true>(p, a, s) : launch_t<BN, TF32, PAIR, false>(p, a, s);
}

cudaError_t launch_assign(const Plan& p, const AssignArgs& a, cudaStream_t s) {
  const bool tf32 = p.dtype == kDtypeF32;
  if (p.ac.pair) {
    switch (p.ac.BN) {
      case 256: return tf32 ? launch_ct<256, true, true>(p, a, s) : launch_ct<256, false, true>(p, a, s);
      case 128: return tf32 ? launch_ct<128, true, true>(p, a, s) : launch_ct<128, false, true>(p, a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (p.ac.BN) {
    case 256: return tf32 ? launch_ct<256, true, false>(p, a, s) : launch_ct<256, false, false>(p, a, s);
    case 128: return tf32 ? launch_ct<128, true, false>(p, a, s) : launch_ct<128, false, false>(p, a, s);
    case 64: return tf32 ? launch_ct<64, true, false>(p, a, s) : launch_ct<64, false, false>(p, a, s);
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
  chain_break();  // plain launch: the next kernel must not chain to it
  if (fault_hit(kFaultLaunch)) return cudaErrorLaunchFailure;
  count_launch();
  k_timeout_probe<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace km
