// km_api.cu -- the C ABI of libkm.so (declared in include/km.h): argument
// validation, the shape plan, workspace carving, TMA descriptors and the
// launch sequences of FlashAssign, the Sort-Inverse Update, full Lloyd fits
// and the out-of-core chunk stream ("Flash-KMeans: Fast and Memory-Efficient
// Exact K-Means", §2.1-§2.3).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <functional>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/km.h"
#include "km_internal.h"

namespace km {
size_t assign_smem_for(int BN, int natoms, int XB, int CS, bool pair);
size_t ablation_assign_ws(int64_t chunk_rows, int K);
size_t ablation_update_ws(int D, int K);
int ablation_assign(const void* X, const void* C, int64_t N, int D, int K, int dtype, int64_t chunk_rows,
                    int32_t* idx, float* mindist, void* ws, cudaStream_t s);
int ablation_update(const void* X, const int32_t* idx, int64_t N, int D, int K, int dtype, float* C,
                    int32_t* counts, void* ws, cudaStream_t s);
size_t small_update_smem(int64_t N, int K, int D);

bool pdl_enabled() {
  const char* e = getenv("KM_PDL");
  return !(e && strcmp(e, "0") == 0);
}

static thread_local bool t_chain = false;
void chain_break() { t_chain = false; }
bool chain_armed() { return t_chain; }
void chain_arm() { t_chain = true; }

// Fault injection state of the calling thread (one call at a time).
struct FaultState {
  int point = -1;      // FaultPoint to fail, -1 = none
  int64_t at = 0;      // 1-based occurrence that fails
  int64_t seen[3] = {0, 0, 0};
  bool fired = false;
};
static thread_local FaultState t_fault;

void fault_arm_from_env() {
  t_fault = FaultState{};
  const char* e = getenv("KM_FAULT");
  if (!e || !*e) return;
  static const char* names[3] = {"alloc", "h2d", "launch"};
  for (int i = 0; i < 3; ++i) {
    const size_t n = strlen(names[i]);
    if (strncmp(e, names[i], n) == 0 && (e[n] == 0 || e[n] == ':')) {
      t_fault.point = i;
      t_fault.at = e[n] == ':' ? strtoll(e + n + 1, nullptr, 10) : 1;
      if (t_fault.at < 1) t_fault.point = -1;
    }
  }
}

bool fault_hit(int point) {
  if (t_fault.point != point) return false;
  if (++t_fault.seen[point] != t_fault.at) return false;
  t_fault.fired = true;
  return true;
}

bool fault_fired() { return t_fault.fired; }
}  // namespace km

using namespace km;

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  // a failure that the host-side injector caused (KM_FAULT) reports as such
  if (code == KM_ERR_CUDA && fault_fired()) {
    code = KM_ERR_INJECTED;
    g_err = std::string("injected fault (KM_FAULT): ") + buf;
  }
  return code;
}

#define KM_CUDA(call)                                                                        \
  do {                                                                                       \
    cudaError_t e_ = (call);                                                                 \
    if (e_ != cudaSuccess)                                                                   \
      return fail(KM_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), __FILE__, __LINE__); \
  } while (0)

constexpr size_t kAlign = 256;
constexpr int64_t kMaxHostIters = 1 << 16;
constexpr int kSmemLimit = 232448;  // 227 KB per block on sm_100

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

uint64_t wait_limit_ns() {
  static uint64_t v = [] {
    const char* e = getenv("KM_WAIT_LIMIT_NS");
    uint64_t d = 2000000000ull;
    if (e && *e) d = strtoull(e, nullptr, 10);
    return d;
  }();
  return v;
}

// Form of the assignment kernel: -1 = default (by shape), 0 = one CTA per
// 128-point tile, 1 = CTA pairs.  Set by KM_ASSIGN_FORM=single|pair.
int assign_form() {
  static int v = [] {
    const char* e = getenv("KM_ASSIGN_FORM");
    if (e && strcmp(e, "single") == 0) return 0;
    if (e && strcmp(e, "pair") == 0) return 1;
    return -1;
  }();
  return v;
}  // -1 = chosen by shape (pairs where BN >= 128)

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D tensor map over [B][rows][inner] with a (box_inner x box_rows x 1) box;
// swizzle_bytes 128 or 32 (the box's inner extent in bytes); out-of-range
// rows/columns read as zero.
int encode_map(CUtensorMap* m, const void* ptr, bool f32, int64_t inner, int64_t rows, int B, int box_rows,
               int swizzle_bytes = 128) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return fail(KM_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int es = f32 ? 4 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner * es), static_cast<cuuint64_t>(inner * es * rows)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(swizzle_bytes / es), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return KM_OK;
}

// Augmentation rows: 32 bytes per row (16 bf16 or 8 fp32), 32-byte swizzle.
int encode_aug_map(CUtensorMap* m, const void* ptr, bool f32, int64_t rows, int B, int box_rows) {
  return encode_map(m, ptr, f32, f32 ? 8 : 16, rows, B, box_rows, 32);
}

int check_device() {
  int dev = 0, major = 0, minor = 0;
  KM_CUDA(cudaGetDevice(&dev));
  KM_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  KM_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  if (major != 10 || minor != 0)
    return fail(KM_ERR_UNSUPPORTED, "device is sm_%d%d; this library is built for sm_100a only", major, minor);
  return KM_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

int ceil_log2(int k) {
  int b = 0;
  while ((1 << b) < k) ++b;
  return b;
}

}  // namespace

namespace km {

void set_last_error(const char* msg) { g_err = msg ? msg : ""; }

int make_plan(Plan& p, int op, int B, int64_t N, int D, int K, int dtype, int64_t chunk_rows, const char** why) {
  static thread_local char msg[256];
  auto bad = [&](int code, const char* fmt, auto... a) {
    snprintf(msg, sizeof(msg), fmt, a...);
    *why = msg;
    return code;
  };
  if (op < KM_OP_ASSIGN || op > KM_OP_ARGSORT) return bad(KM_ERR_INVALID_ARG, "unknown op %d", op);
  if (op == KM_OP_ARGSORT) {  // shape-independent of D and dtype
    D = 8;
    dtype = KM_BF16;
    B = 1;
  }
  if (dtype != KM_F32 && dtype != KM_BF16) return bad(KM_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (B < 1 || N < 1 || K < 1) return bad(KM_ERR_INVALID_ARG, "need B >= 1, N >= 1, K >= 1 (B=%d N=%lld K=%d)", B,
                                          static_cast<long long>(N), K);
  if (K > N) return bad(KM_ERR_INVALID_ARG, "K=%d exceeds N=%lld", K, static_cast<long long>(N));
  if (K > (1 << 20)) return bad(KM_ERR_UNSUPPORTED, "K=%d above 2^20", K);
  if (N >= (int64_t(1) << 31)) return bad(KM_ERR_UNSUPPORTED, "N=%lld must be below 2^31", static_cast<long long>(N));
  if (D % 8 != 0) return bad(KM_ERR_UNSUPPORTED, "D=%d must be a multiple of 8", D);
  if (dtype == KM_BF16 && (D < 8 || D > 256)) return bad(KM_ERR_UNSUPPORTED, "bf16 needs 8 <= D <= 256 (D=%d)", D);
  if (dtype == KM_F32 && (D < 8 || D > 64)) return bad(KM_ERR_UNSUPPORTED, "f32 needs 8 <= D <= 64 (D=%d)", D);
  if (op == KM_OP_FIT_HOST && B != 1) return bad(KM_ERR_INVALID_ARG, "%s", "host-resident fits take one instance");
  p = Plan{};
  p.op = op;
  p.B = B;
  p.N = N;
  p.D = D;
  p.K = K;
  p.dtype = dtype;
  p.es = dtype == KM_BF16 ? 2 : 4;
  p.Dp = (D + 31) / 32 * 32;
  p.Dop = dtype == KM_BF16 ? D : 3 * p.Dp;
  if (op == KM_OP_FIT_HOST) {
    if (chunk_rows < 1) return bad(KM_ERR_INVALID_ARG, "%s", "chunk_rows must be >= 1");
    p.chunk_rows = chunk_rows < N ? chunk_rows : N;
    p.rows = p.chunk_rows;
  } else {
    p.rows = N;
  }
  // ---- FlashAssign tile configuration: widest centroid tile that fits
  AssignCfg& ac = p.ac;
  ac.epa = 128 / p.es;
  ac.natoms = (p.Dop * p.es + 127) / 128;
  int bn0 = K <= 64 ? 64 : (K <= 128 ? 128 : 256);
  bool found = false;
  // CTA pairs (cta_group::2) for centroid tiles of 128 or 256 when a point
  // tile meets several centroid tiles, else one CTA per 128-point tile;
  // KM_ASSIGN_FORM=single|pair forces the form.  A sweep of every tiling
  // that fits (bench.py --tile-sweep) measured pairs 1-2 % ahead on
  // 1M x 1024 x 128 and level on 4M x 16384 x 128, and the single form 6 %
  // ahead when K fits one centroid tile (512 x 4096 x 64, K = 256) and the
  // single form keeps its full rings (4 point buffers, 3 centroid stages).
  const int form = assign_form();
  const bool single_one_ct =
      K <= bn0 && assign_smem_for(bn0, ac.natoms, 4, 3, false) <= static_cast<size_t>(kSmemLimit);
  const int pair_first = form == 0 ? 0 : (form == 1 ? 1 : (single_one_ct ? 0 : 1));
  for (int pair = pair_first; pair >= 0 && !found; --pair) {
    if (form == 1 && !pair && bn0 >= 128) continue;
    for (int bn = bn0; bn >= 64 && !found; bn /= 2) {
      if (pair && bn < 128) continue;
      // One centroid tile per point tile (K <= BN): it stays resident per
      // instance and the point tiles (one short tile of MMA time each) get a
      // 4-deep ring with 3 centroid stages (deeper point rings measured
      // slower).  Otherwise two point buffers and the deepest centroid ring.
      const bool one_ct = K <= bn;
      const int xb_hi = one_ct ? 4 : 2;
      for (int xb = xb_hi; xb >= 1 && !found; --xb) {
        for (int cs = one_ct ? 3 : 4; cs >= 2 && !found; --cs) {
          const size_t sm = assign_smem_for(bn, ac.natoms, xb, cs, pair != 0);
          if (sm <= static_cast<size_t>(kSmemLimit)) {
            ac.pair = pair != 0;
            ac.BN = bn;
            ac.XB = xb;
            ac.CS = cs;
            ac.smem = sm;
            found = true;
          }
        }
      }
    }
  }
  if (!found) return bad(KM_ERR_UNSUPPORTED, "no FlashAssign tiling fits shared memory for D=%d", D);
  // Explicit tiling (measurement of the chooser against a sweep):
  // KM_ASSIGN_TILE=pair,BN,XB,CS, e.g. "0,256,2,2"; refused if it does not fit.
  if (const char* e = getenv("KM_ASSIGN_TILE")) {
    int fp = 0, fb = 0, fx = 0, fc = 0;
    if (sscanf(e, "%d,%d,%d,%d", &fp, &fb, &fx, &fc) != 4)
      return bad(KM_ERR_INVALID_ARG, "KM_ASSIGN_TILE='%s' is not pair,BN,XB,CS", e);
    const bool bn_ok = fb == 64 || fb == 128 || fb == 256;
    if (!bn_ok || (fp && fb < 128) || fx < 1 || fx > 8 || fc < 2 || fc > 4)
      return bad(KM_ERR_UNSUPPORTED, "KM_ASSIGN_TILE='%s' is not a supported tiling for K=%d", e, K);
    const size_t sm = assign_smem_for(fb, ac.natoms, fx, fc, fp != 0);
    if (sm > static_cast<size_t>(kSmemLimit)) return bad(KM_ERR_UNSUPPORTED, "KM_ASSIGN_TILE='%s' needs %zu bytes of shared memory", e, sm);
    ac.pair = fp != 0;
    ac.BN = fb;
    ac.XB = fx;
    ac.CS = fc;
    ac.smem = sm;
  }
  ac.tmem_cols = 2 * ac.BN;
  p.Kp = (K + ac.BN - 1) / ac.BN * ac.BN;
  p.tiles_per_inst = (p.rows + kTileM - 1) / kTileM;
  p.ntiles = p.tiles_per_inst * B;
  // ---- update configuration
  p.small_update = B > 1 && N <= kSmallMaxN && K <= kSmallMaxK &&
                   small_update_smem(N, K, D) <= static_cast<size_t>(kSmemLimit) && op != KM_OP_FIT_HOST;
  SortCfg& sc = p.sc;
  const int bits = ceil_log2(K) < 1 ? 1 : ceil_log2(K);
  if (bits <= 12) {
    sc.passes = 1;
    sc.bits[0] = bits;
  } else {
    sc.passes = 2;
    sc.bits[0] = bits / 2;
    sc.bits[1] = bits - bits / 2;
    sc.shift[1] = sc.bits[0];
  }
  sc.W = 8;
  // Keys per scatter block: 4096 when those blocks fill the 148 SMs with one
  // to two resident blocks each (one wave at 2 per SM), else 2048 (4 per SM):
  // measured faster for 16K and 4M points, slower for 1M.
  {
    const int64_t b4k = (p.rows + 4095) / 4096;
    sc.IPT = b4k >= 148 && b4k <= 2 * 148 ? 16 : 8;
  }
  sc.T = sc.W * 32 * sc.IPT;
  sc.nblk = (p.rows + sc.T - 1) / sc.T;
  sc.Rmax = 1 << (sc.bits[0] > sc.bits[1] ? sc.bits[0] : sc.bits[1]);
  // Column-scan segments: about 96 CTAs (32 digits each) when there are few
  // digits and many blocks, at most 16 segments of at least 32 blocks.
  for (int ps = 0; ps < sc.passes; ++ps) {
    const int groups = ((1 << sc.bits[ps]) + 31) / 32;
    int S = (96 + groups - 1) / groups;
    const int64_t byrows = sc.nblk / 32;
    if (S > byrows) S = static_cast<int>(byrows);
    if (S > 16) S = 16;
    sc.segs[ps] = S < 1 ? 1 : S;
  }
  const int segmax = sc.segs[0] > sc.segs[1] ? sc.segs[0] : sc.segs[1];
  SegCfg& gc = p.gc;
  gc.BNS = static_cast<int>(seg_block_positions(p.rows));
  gc.nchunks = (p.rows + gc.BNS - 1) / gc.BNS;
  gc.big_span = 8;
  // ---- workspace layout
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes);
    return o;
  };
  const int64_t BR = static_cast<int64_t>(B) * p.rows;
  p.off_hdr = take(kAlign);
  if (op == KM_OP_ARGSORT) {
    p.off_blkhist = take(sizeof(int32_t) * (static_cast<size_t>(1) << sc.bits[0]) * sc.nblk);
    if (sc.passes > 1) p.off_blkhist1 = take(sizeof(int32_t) * (static_cast<size_t>(1) << sc.bits[1]) * sc.nblk);
    p.off_total = take(sizeof(int32_t) * sc.Rmax * segmax);
    if (sc.passes > 1) p.off_pairs_tmp = take(sizeof(int2) * p.rows);
    p.off_pairs = take(sizeof(int2) * p.rows);
    p.off_start = take(sizeof(int32_t) * (K + 1));
    p.off_rk = take(sizeof(int32_t) * static_cast<size_t>(p.rows));
    p.total = off;
    return KM_OK;
  }
  p.off_xaug = take(32 * static_cast<size_t>(BR));
  p.off_caug = take(32 * static_cast<size_t>(B) * p.Kp);
  p.off_clp = take(static_cast<size_t>(B) * K * p.Dop * (dtype == KM_BF16 ? 2 : 4));
  if (dtype == KM_F32) p.off_x3 = take(sizeof(float) * BR * 3 * p.Dp);
  // per-tile partials, or one group per assignment CTA (at most one per SM)
  p.off_tobj = take(sizeof(double) * 4 * static_cast<size_t>(p.ntiles > 256 ? p.ntiles : 256));
  if (op == KM_OP_FIT || op == KM_OP_FIT_HOST) p.off_idx = take(sizeof(int32_t) * BR);
  p.off_obj = take(sizeof(double) * (op == KM_OP_FIT_HOST ? kMaxHostIters : B));
  p.off_objpart = take(sizeof(double) * static_cast<size_t>(objective_blocks(p.tiles_per_inst) + 1));
  if (op != KM_OP_ASSIGN && !p.small_update) {
    p.off_blkhist = take(sizeof(int32_t) * (static_cast<size_t>(1) << sc.bits[0]) * sc.nblk);
    if (sc.passes > 1) p.off_blkhist1 = take(sizeof(int32_t) * (static_cast<size_t>(1) << sc.bits[1]) * sc.nblk);
    p.off_total = take(sizeof(int32_t) * sc.Rmax * segmax);
    if (sc.passes > 1) p.off_pairs_tmp = take(sizeof(int2) * p.rows);
    p.off_pairs = take(sizeof(int2) * p.rows);
    p.off_start = take(sizeof(int32_t) * (K + 1));
    p.off_sums = take(sizeof(float) * static_cast<size_t>(K) * D);
    p.off_pl = take(sizeof(float) * gc.nchunks * D);
    p.off_pr = take(sizeof(float) * gc.nchunks * D);
  }
  if ((op == KM_OP_FIT || op == KM_OP_FIT_HOST) && !p.small_update) {
    p.off_rk = take(sizeof(int32_t) * static_cast<size_t>(p.rows));
  }
  if (op == KM_OP_FIT_HOST) {
    p.off_dbuf0 = take(static_cast<size_t>(p.chunk_rows) * D * p.es);
    p.off_dbuf1 = take(static_cast<size_t>(p.chunk_rows) * D * p.es);
    p.off_acc64 = take(sizeof(double) * static_cast<size_t>(K) * D);
    p.off_cnt64 = take(sizeof(long long) * K);
    p.off_objacc = take(sizeof(double));
  }
  p.total = off;
  return KM_OK;
}

}  // namespace km

namespace {

// Set while an entry point that already armed the injector (and may have
// counted occurrences, e.g. its event creation) calls a shared helper.
thread_local bool t_fault_keep = false;

struct Ctx {
  Plan p;
  void* ws;
  cudaStream_t s;
  unsigned int* status() const { return at<unsigned int>(ws, p.off_hdr); }
  // header word 1: blocks done of the finalise kernel's objective reduction
  unsigned int* objcnt() const { return at<unsigned int>(ws, p.off_hdr) + 1; }
};

int prepare(Ctx& c, int op, int B, int64_t N, int D, int K, int dtype, int64_t chunk_rows, void* ws,
            size_t ws_bytes, void* stream) {
  const char* why = "";
  if (!t_fault_keep) fault_arm_from_env();
  int r = make_plan(c.p, op, B, N, D, K, dtype, chunk_rows, &why);
  if (r != KM_OK) return fail(r, "%s", why);
  if (!ws) return fail(KM_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % kAlign) return fail(KM_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < c.p.total)
    return fail(KM_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, c.p.total);
  r = check_device();
  if (r != KM_OK) return r;
  c.ws = ws;
  c.s = static_cast<cudaStream_t>(stream);
  chain_break();
  return KM_OK;
}

// Update of one instance through the multi-kernel path.
int update_instance(const Ctx& c, const void* Xb, const int32_t* idxb, int64_t n, float* Cb, void* c_opb, void* caugb,
                    int32_t* countsb, const double* tobjb, int64_t ntiles, double* obj, int mode,
                    double* acc_ext = nullptr, double* cnt_ext = nullptr, int32_t* rk = nullptr) {
  const Plan& p = c.p;
  SortArgs sa{idxb,
              n,
              p.K,
              at<int32_t>(c.ws, p.off_blkhist),
              p.sc.passes > 1 ? at<int32_t>(c.ws, p.off_blkhist1) : nullptr,
              rk,
              at<int32_t>(c.ws, p.off_total),
              p.sc.passes > 1 ? at<int2>(c.ws, p.off_pairs_tmp) : nullptr,
              at<int2>(c.ws, p.off_pairs),
              nullptr,
              at<int32_t>(c.ws, p.off_start)};
  KM_CUDA(launch_sort(p, sa, c.s));
  SegArgs ga{Xb, n, sa.pairs, sa.start, at<float>(c.ws, p.off_sums), at<float>(c.ws, p.off_pl),
             at<float>(c.ws, p.off_pr)};
  KM_CUDA(launch_segsum(p, ga, c.s));
  FinalizeArgs fa{};
  fa.start = sa.start;
  fa.pairs = sa.pairs;
  fa.sums = ga.sums;
  fa.pl = ga.pl;
  fa.pr = ga.pr;
  fa.mode = mode;
  fa.C = Cb;
  fa.c_op = c_opb;
  fa.caug = caugb;
  fa.counts = countsb;
  fa.acc64 = mode == 1 ? (acc_ext ? acc_ext : at<double>(c.ws, p.off_acc64)) : nullptr;
  fa.cnt64 = mode == 1 && !cnt_ext ? at<long long>(c.ws, p.off_cnt64) : nullptr;
  fa.cntf = mode == 1 ? cnt_ext : nullptr;
  fa.tobj = tobjb;
  fa.ntiles = obj ? ntiles : 0;
  fa.obj = obj;
  fa.objpart = at<double>(c.ws, p.off_objpart);
  fa.objcnt = c.objcnt();
  Plan pp = p;
  pp.rows = n;
  KM_CUDA(launch_finalize(pp, fa, c.s));
  return KM_OK;
}

// Centroid rows per TMA box: a CTA of a pair loads half of each centroid tile.
int cbox(const Plan& p) { return p.ac.pair ? p.ac.BN / 2 : p.ac.BN; }

size_t op_row_bytes(const Plan& p) { return static_cast<size_t>(p.Dop) * (p.dtype == KM_BF16 ? 2 : 4); }

}  // namespace

extern "C" {

int km_version(void) { return KM_VERSION; }

uint64_t km_launch_count(void) { return km::launch_counter().load(std::memory_order_relaxed); }

const char* km_status_string(int status) {
  switch (status) {
    case KM_OK: return "ok";
    case KM_ERR_INVALID_ARG: return "invalid argument";
    case KM_ERR_UNSUPPORTED: return "unsupported";
    case KM_ERR_CUDA: return "cuda error";
    case KM_ERR_WORKSPACE: return "workspace too small or misaligned";
    case KM_ERR_TIMEOUT: return "bounded in-kernel wait ran out";
    case KM_ERR_INJECTED: return "injected fault";
    default: return "unknown status";
  }
}

const char* km_last_error(void) { return g_err.c_str(); }

size_t km_workspace_size(int op, int B, int64_t N, int D, int K, int dtype, int64_t chunk_rows) {
  Plan p;
  const char* why = "";
  if (make_plan(p, op, B, N, D, K, dtype, chunk_rows, &why) != KM_OK) {
    g_err = why;
    return 0;
  }
  return p.total;
}

int km_workspace_status(void* workspace, void* stream) {
  if (!workspace) return fail(KM_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int v = 0;
  KM_CUDA(cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, s));
  chain_break();
  KM_CUDA(cudaStreamSynchronize(s));
  KM_CUDA(cudaMemsetAsync(workspace, 0, sizeof(v), s));
  chain_break();
  KM_CUDA(cudaStreamSynchronize(s));
  if (v) return fail(KM_ERR_TIMEOUT, "a kernel gave up on a bounded wait (status 0x%x)", v);
  return KM_OK;
}

int km_assign(const void* X, const void* C, int B, int64_t N, int D, int K, int dtype, int32_t* idx, float* mindist,
              double* objective, void* workspace, size_t workspace_bytes, void* stream) {
  g_err.clear();
  if (!X || !C || !idx) return fail(KM_ERR_INVALID_ARG, "X, C and idx are required");
  if (!aligned16(X) || !aligned16(C)) return fail(KM_ERR_INVALID_ARG, "X and C must be 16-byte aligned");
  Ctx c;
  int r = prepare(c, KM_OP_ASSIGN, B, N, D, K, dtype, 0, workspace, workspace_bytes, stream);
  if (r != KM_OK) return r;
  const Plan& p = c.p;
  void* xaug = at<void>(c.ws, p.off_xaug);
  void* caug = at<void>(c.ws, p.off_caug);
  void* clp = at<void>(c.ws, p.off_clp);
  const bool f32 = dtype == KM_F32;
  KM_CUDA(cudaMemsetAsync(c.status(), 0, sizeof(unsigned int), c.s));
  chain_break();
  float* x3 = f32 ? at<float>(c.ws, p.off_x3) : nullptr;
  KM_CUDA(launch_xprep(X, dtype, static_cast<int64_t>(B) * N, D, p.Dp, xaug, x3, c.s));
  KM_CUDA(launch_cprep(C, dtype, B, K, p.Kp, D, p.Dp, dtype, nullptr, clp, caug, c.s));
  CUtensorMap xmap, xamap, cmap, camap;
  if ((r = encode_map(&xmap, f32 ? static_cast<const void*>(x3) : X, f32, p.Dop, N, B, kTileM)) != KM_OK) return r;
  if ((r = encode_aug_map(&xamap, xaug, f32, N, B, kTileM)) != KM_OK) return r;
  if ((r = encode_map(&cmap, clp, f32, p.Dop, K, B, cbox(p))) != KM_OK) return r;
  if ((r = encode_aug_map(&camap, caug, f32, p.Kp, B, cbox(p))) != KM_OK) return r;
  double* tobj = at<double>(c.ws, p.off_tobj);
  int64_t groups = 0;
  AssignArgs a{&xmap, &xamap, &cmap, &camap, B, N, K, p.Kp, idx, mindist, tobj, c.status(), wait_limit_ns(),
               &groups};
  a.cop = clp;
  a.cop_row_bytes = op_row_bytes(p);
  KM_CUDA(launch_assign(p, a, c.s));
  if (objective) KM_CUDA(launch_objective(tobj, B, groups, objective, 1, c.s));
  return KM_OK;
}

int km_update(const void* X, const int32_t* idx, int B, int64_t N, int D, int K, int dtype, float* C, int32_t* counts,
              void* workspace, size_t workspace_bytes, void* stream) {
  g_err.clear();
  if (!X || !idx || !C) return fail(KM_ERR_INVALID_ARG, "X, idx and C are required");
  if (!aligned16(X) || !aligned16(C)) return fail(KM_ERR_INVALID_ARG, "X and C must be 16-byte aligned");
  Ctx c;
  int r = prepare(c, KM_OP_UPDATE, B, N, D, K, dtype, 0, workspace, workspace_bytes, stream);
  if (r != KM_OK) return r;
  const Plan& p = c.p;
  if (p.small_update) {
    SmallUpdateArgs a{X, idx, C, nullptr, nullptr, counts, nullptr, 0, nullptr, 0};
    KM_CUDA(launch_small_update(p, a, c.s));
    return KM_OK;
  }
  const size_t xstride = static_cast<size_t>(N) * D * p.es;
  for (int b = 0; b < B; ++b) {
    r = update_instance(c, static_cast<const uint8_t*>(X) + b * xstride, idx + static_cast<int64_t>(b) * N, N,
                        C + static_cast<int64_t>(b) * K * D, nullptr, nullptr,
                        counts ? counts + static_cast<int64_t>(b) * K : nullptr, nullptr, 0, nullptr, 0);
    if (r != KM_OK) return r;
  }
  return KM_OK;
}

// ev: events recorded around every phase (per_phase) or around the whole
// loop; ext_events: as event-record nodes of a graph being captured.
static int fit_impl(const void* X, const void* C0, int B, int64_t N, int D, int K, int dtype, int iters,
                    float* C_out, int32_t* idx_out, int32_t* counts_out, double* objective_hist, void* workspace,
                    size_t workspace_bytes, void* stream, cudaEvent_t* ev, bool per_phase = true,
                    bool ext_events = false) {
  const unsigned rec_flags = ext_events ? cudaEventRecordExternal : cudaEventRecordDefault;
  if (!X || !C0 || !C_out) return fail(KM_ERR_INVALID_ARG, "X, C0 and C_out are required");
  if (iters < 0) return fail(KM_ERR_INVALID_ARG, "iters must be >= 0");
  if (!aligned16(X) || !aligned16(C0) || !aligned16(C_out))
    return fail(KM_ERR_INVALID_ARG, "X, C0 and C_out must be 16-byte aligned");
  Ctx c;
  int r = prepare(c, KM_OP_FIT, B, N, D, K, dtype, 0, workspace, workspace_bytes, stream);
  if (r != KM_OK) return r;
  const Plan& p = c.p;
  void* xaug = at<void>(c.ws, p.off_xaug);
  uint8_t* caug = at<uint8_t>(c.ws, p.off_caug);
  void* clp = at<void>(c.ws, p.off_clp);
  double* tobj = at<double>(c.ws, p.off_tobj);
  int32_t* idx = idx_out ? idx_out : at<int32_t>(c.ws, p.off_idx);
  double* objs = at<double>(c.ws, p.off_obj);
  const bool f32 = dtype == KM_F32;
  KM_CUDA(cudaMemsetAsync(c.status(), 0, 2 * sizeof(unsigned int), c.s));  // status, objective counter
  chain_break();
  float* x3 = f32 ? at<float>(c.ws, p.off_x3) : nullptr;
  KM_CUDA(launch_xprep(X, dtype, static_cast<int64_t>(B) * N, D, p.Dp, xaug, x3, c.s));
  CUtensorMap xmap, xamap, cmap, camap;
  if ((r = encode_map(&xmap, f32 ? static_cast<const void*>(x3) : X, f32, p.Dop, N, B, kTileM)) != KM_OK) return r;
  if ((r = encode_aug_map(&xamap, xaug, f32, N, B, kTileM)) != KM_OK) return r;
  if ((r = encode_map(&cmap, clp, f32, p.Dop, K, B, cbox(p))) != KM_OK) return r;
  if ((r = encode_aug_map(&camap, caug, f32, p.Kp, B, cbox(p))) != KM_OK) return r;
  KM_CUDA(launch_cprep(C0, dtype, B, K, p.Kp, D, p.Dp, dtype, C_out, clp, caug, c.s));
  const size_t xstride = static_cast<size_t>(N) * D * p.es;
  const size_t opstride = static_cast<size_t>(K) * op_row_bytes(p);
  // The sort's count kernel hands its scatter each point's key with its
  // rank inside its 32-point group
  int32_t* rk = p.small_update ? nullptr : at<int32_t>(c.ws, p.off_rk);
  for (int t = 0; t < iters; ++t) {
    int64_t groups = 0;
    AssignArgs a{&xmap, &xamap, &cmap, &camap, B, N, K, p.Kp, idx, nullptr, tobj, c.status(), wait_limit_ns(),
                 &groups, clp, op_row_bytes(p)};
    if (ev && (per_phase || t == 0)) {
      KM_CUDA(cudaEventRecordWithFlags(ev[per_phase ? 3 * t : 0], c.s, rec_flags));
      chain_break();
    }
    KM_CUDA(launch_assign(p, a, c.s));
    if (ev && per_phase) {
      KM_CUDA(cudaEventRecordWithFlags(ev[3 * t + 1], c.s, rec_flags));
      chain_break();
    }
    if (p.small_update) {
      SmallUpdateArgs u{X,    idx,       C_out, clp, caug, counts_out, tobj, p.tiles_per_inst,
                        objective_hist ? objective_hist + t : objs, objective_hist ? iters : 1};
      KM_CUDA(launch_small_update(p, u, c.s));
    } else {
      for (int b = 0; b < B; ++b) {
        double* ob = objective_hist ? objective_hist + static_cast<int64_t>(b) * iters + t : objs + b;
        r = update_instance(c, static_cast<const uint8_t*>(X) + b * xstride, idx + static_cast<int64_t>(b) * N, N,
                            C_out + static_cast<int64_t>(b) * K * D, static_cast<uint8_t*>(clp) + b * opstride,
                            caug + static_cast<int64_t>(b) * p.Kp * 32,
                            counts_out ? counts_out + static_cast<int64_t>(b) * K : nullptr,
                            tobj + static_cast<int64_t>(b) * groups * 4, groups, ob, 0, nullptr, nullptr,
                            rk);
        if (r != KM_OK) return r;
      }
    }
    if (ev && (per_phase || t == iters - 1)) {
      KM_CUDA(cudaEventRecordWithFlags(ev[per_phase ? 3 * t + 2 : 1], c.s, rec_flags));
      chain_break();
    }
  }
  return KM_OK;
}

int km_fit(const void* X, const void* C0, int B, int64_t N, int D, int K, int dtype, int iters, float* C_out,
           int32_t* idx_out, int32_t* counts_out, double* objective_hist, void* workspace, size_t workspace_bytes,
           void* stream) {
  g_err.clear();
  return fit_impl(X, C0, B, N, D, K, dtype, iters, C_out, idx_out, counts_out, objective_hist, workspace,
                  workspace_bytes, stream, nullptr);
}

int km_fit_profile(const void* X, const void* C0, int B, int64_t N, int D, int K, int dtype, int iters,
                   float* C_out, int32_t* idx_out, int32_t* counts_out, double* objective_hist, void* workspace,
                   size_t workspace_bytes, void* stream, float* phase_ms) {
  g_err.clear();
  if (!phase_ms) return fail(KM_ERR_INVALID_ARG, "phase_ms is required");
  if (iters < 0) return fail(KM_ERR_INVALID_ARG, "iters must be >= 0");
  fault_arm_from_env();
  std::vector<cudaEvent_t> ev(3 * static_cast<size_t>(iters), nullptr);
  auto destroy = [&]() {
    for (auto e : ev)
      if (e) cudaEventDestroy(e);
  };
  for (auto& e : ev) {
    if (fault_hit(kFaultAlloc) || cudaEventCreate(&e) != cudaSuccess) {
      destroy();
      return fail(KM_ERR_CUDA, "cudaEventCreate failed");
    }
  }
  t_fault_keep = true;
  int r = fit_impl(X, C0, B, N, D, K, dtype, iters, C_out, idx_out, counts_out, objective_hist, workspace,
                   workspace_bytes, stream, iters > 0 ? ev.data() : nullptr);
  t_fault_keep = false;
  if (r == KM_OK && cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    r = fail(KM_ERR_CUDA, "stream synchronisation failed");
  for (int t = 0; r == KM_OK && t < iters; ++t) {
    if (cudaEventElapsedTime(&phase_ms[2 * t], ev[3 * t], ev[3 * t + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&phase_ms[2 * t + 1], ev[3 * t + 1], ev[3 * t + 2]) != cudaSuccess)
      r = fail(KM_ERR_CUDA, "cudaEventElapsedTime failed");
  }
  if (r == KM_OK) {
    phase_ms[2 * static_cast<size_t>(iters)] = 0.f;
    if (iters > 0 && cudaEventElapsedTime(&phase_ms[2 * static_cast<size_t>(iters)], ev[0],
                                          ev[3 * static_cast<size_t>(iters) - 1]) != cudaSuccess)
      r = fail(KM_ERR_CUDA, "cudaEventElapsedTime failed");
  }
  destroy();
  return r;
}

int km_fit_timed(const void* X, const void* C0, int B, int64_t N, int D, int K, int dtype, int iters, float* C_out,
                 int32_t* idx_out, int32_t* counts_out, double* objective_hist, void* workspace,
                 size_t workspace_bytes, void* stream, float* iters_ms) {
  g_err.clear();
  if (!iters_ms) return fail(KM_ERR_INVALID_ARG, "iters_ms is required");
  if (iters < 0) return fail(KM_ERR_INVALID_ARG, "iters must be >= 0");
  fault_arm_from_env();
  cudaEvent_t ev[2] = {nullptr, nullptr};
  for (auto& e : ev)
    if (fault_hit(kFaultAlloc) || cudaEventCreate(&e) != cudaSuccess) {
      for (auto x : ev)
        if (x) cudaEventDestroy(x);
      return fail(KM_ERR_CUDA, "cudaEventCreate failed");
    }
  t_fault_keep = true;
  int r = fit_impl(X, C0, B, N, D, K, dtype, iters, C_out, idx_out, counts_out, objective_hist, workspace,
                   workspace_bytes, stream, iters > 0 ? ev : nullptr, false);
  t_fault_keep = false;
  if (r == KM_OK && cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    r = fail(KM_ERR_CUDA, "stream synchronisation failed");
  *iters_ms = 0.f;
  if (r == KM_OK && iters > 0 && cudaEventElapsedTime(iters_ms, ev[0], ev[1]) != cudaSuccess)
    r = fail(KM_ERR_CUDA, "cudaEventElapsedTime failed");
  for (auto e : ev) cudaEventDestroy(e);
  return r;
}

}  // extern "C"

struct km_fit_graph_t {
  cudaGraphExec_t exec = nullptr;
  cudaEvent_t ev[2] = {nullptr, nullptr};
  bool timed = false;
  bool launched = false;
  uint64_t kernels = 0;  // kernels per launch
  int device = -1;
};

extern "C" {

int km_fit_graph_create(km_fit_graph* graph, const void* X, const void* C0, int B, int64_t N, int D, int K,
                        int dtype, int iters, float* C_out, int32_t* idx_out, int32_t* counts_out,
                        double* objective_hist, void* workspace, size_t workspace_bytes, int timed) {
  g_err.clear();
  if (!graph) return fail(KM_ERR_INVALID_ARG, "graph is required");
  *graph = nullptr;
  if (iters < 0) return fail(KM_ERR_INVALID_ARG, "iters must be >= 0");
  fault_arm_from_env();
  auto* g = new km_fit_graph_t();
  g->timed = timed != 0 && iters > 0;
  cudaStream_t cs = nullptr;
  cudaGraph_t gr = nullptr;
  auto cleanup = [&](int code) {
    if (gr) cudaGraphDestroy(gr);
    if (cs) cudaStreamDestroy(cs);
    km_fit_graph_destroy(g);
    return code;
  };
  if (cudaGetDevice(&g->device) != cudaSuccess) return cleanup(fail(KM_ERR_CUDA, "no CUDA device"));
  if (g->timed)
    for (auto& e : g->ev)
      if (fault_hit(kFaultAlloc) || cudaEventCreate(&e) != cudaSuccess)
        return cleanup(fail(KM_ERR_CUDA, "cudaEventCreate failed"));
  // Capture on a private stream: nothing is executed, and no caller stream
  // is involved until a launch.
  if (fault_hit(kFaultAlloc) || cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess)
    return cleanup(fail(KM_ERR_CUDA, "cudaStreamCreate failed"));
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess)
    return cleanup(fail(KM_ERR_CUDA, "cudaStreamBeginCapture failed"));
  t_fault_keep = true;
  t_capture_count = &g->kernels;
  int r = fit_impl(X, C0, B, N, D, K, dtype, iters, C_out, idx_out, counts_out, objective_hist, workspace,
                   workspace_bytes, cs, g->timed ? g->ev : nullptr, false, true);
  t_capture_count = nullptr;
  t_fault_keep = false;
  const cudaError_t ec = cudaStreamEndCapture(cs, &gr);
  if (r != KM_OK) return cleanup(r);
  if (ec != cudaSuccess || !gr) return cleanup(fail(KM_ERR_CUDA, "graph capture failed: %s", cudaGetErrorString(ec)));
  if (cudaGraphInstantiate(&g->exec, gr, 0) != cudaSuccess)
    return cleanup(fail(KM_ERR_CUDA, "cudaGraphInstantiate failed"));
  cudaGraphDestroy(gr);
  gr = nullptr;
  cudaStreamDestroy(cs);
  *graph = g;
  return KM_OK;
}

int km_fit_graph_launch(km_fit_graph graph, void* stream) {
  g_err.clear();
  if (!graph || !graph->exec) return fail(KM_ERR_INVALID_ARG, "graph is NULL or was not created");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != graph->device)
    return fail(KM_ERR_INVALID_ARG, "the current device is not the one the graph was created on");
  if (cudaGraphLaunch(graph->exec, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(KM_ERR_CUDA, "cudaGraphLaunch failed");
  count_launch(graph->kernels);
  graph->launched = true;
  return KM_OK;
}

int km_fit_graph_elapsed(km_fit_graph graph, float* iters_ms) {
  g_err.clear();
  if (!graph || !iters_ms) return fail(KM_ERR_INVALID_ARG, "graph and iters_ms are required");
  if (!graph->timed) return fail(KM_ERR_INVALID_ARG, "the graph was created without timing (or with iters = 0)");
  if (!graph->launched) return fail(KM_ERR_INVALID_ARG, "the graph has not been launched");
  if (cudaEventSynchronize(graph->ev[1]) != cudaSuccess ||
      cudaEventElapsedTime(iters_ms, graph->ev[0], graph->ev[1]) != cudaSuccess)
    return fail(KM_ERR_CUDA, "reading the graph's events failed");
  return KM_OK;
}

int km_fit_graph_destroy(km_fit_graph graph) {
  if (!graph) return KM_OK;
  if (graph->exec) cudaGraphExecDestroy(graph->exec);
  for (auto e : graph->ev)
    if (e) cudaEventDestroy(e);
  delete graph;
  return KM_OK;
}

}  // extern "C"

namespace {

// Rows [r0, r0 + nr) of a streamed point set for staging slot `slot` (0 or
// 1): a pointer to page-locked host memory, or null with *why set.
using ChunkFn = std::function<const void*(int64_t r0, int64_t nr, int slot, const char** why)>;

// The chunked out-of-core fit (Flash-KMeans §2.3 Chunked Stream Overlap):
// each iteration streams the point set to the device in chunks of
// chunk_rows rows through two device buffers, the copy of chunk c+1 on a
// library-owned copy stream overlapping the assignment and update of chunk
// c on `stream`; per-cluster sums accumulate across chunks in float64, in
// chunk order.  With slot_reuse the host memory behind a slot may be
// rewritten by the source: before asking for slot s again the host waits
// until the previous copy out of slot s has completed.
int fit_stream(const ChunkFn& chunk, bool slot_reuse, const void* C0, int64_t N, int D, int K, int dtype,
               int iters, int64_t chunk_rows, float* C_out, int32_t* idx_out, int32_t* counts_out,
               double* objective_hist, void* workspace, size_t workspace_bytes, void* stream) {
  if (iters < 0 || iters > kMaxHostIters) return fail(KM_ERR_INVALID_ARG, "iters must be in [0, %lld]",
                                                      static_cast<long long>(kMaxHostIters));
  if (!aligned16(C0) || !aligned16(C_out)) return fail(KM_ERR_INVALID_ARG, "C0 and C_out must be 16-byte aligned");
  Ctx c;
  int r = prepare(c, KM_OP_FIT_HOST, 1, N, D, K, dtype, chunk_rows, workspace, workspace_bytes, stream);
  if (r != KM_OK) return r;
  const Plan& p = c.p;
  void* xaug = at<void>(c.ws, p.off_xaug);
  void* caug = at<void>(c.ws, p.off_caug);
  void* clp = at<void>(c.ws, p.off_clp);
  double* tobj = at<double>(c.ws, p.off_tobj);
  double* objs = at<double>(c.ws, p.off_obj);
  void* dbuf[2] = {at<void>(c.ws, p.off_dbuf0), at<void>(c.ws, p.off_dbuf1)};
  double* acc64 = at<double>(c.ws, p.off_acc64);
  long long* cnt64 = at<long long>(c.ws, p.off_cnt64);
  double* objacc = at<double>(c.ws, p.off_objacc);
  float* x3 = dtype == KM_F32 ? at<float>(c.ws, p.off_x3) : nullptr;

  cudaStream_t cs = nullptr;
  cudaEvent_t ev_copied[2] = {nullptr, nullptr}, ev_free[2] = {nullptr, nullptr};
  auto cleanup = [&]() {
    for (int i = 0; i < 2; ++i) {
      if (ev_copied[i]) cudaEventDestroy(ev_copied[i]);
      if (ev_free[i]) cudaEventDestroy(ev_free[i]);
    }
    if (cs) cudaStreamDestroy(cs);
  };
  auto run = [&]() -> int {
    if (fault_hit(kFaultAlloc)) return fail(KM_ERR_CUDA, "cudaStreamCreateWithFlags failed");
    KM_CUDA(cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking));
    for (int i = 0; i < 2; ++i) {
      if (fault_hit(kFaultAlloc)) return fail(KM_ERR_CUDA, "cudaEventCreateWithFlags failed");
      KM_CUDA(cudaEventCreateWithFlags(&ev_copied[i], cudaEventDisableTiming));
      if (fault_hit(kFaultAlloc)) return fail(KM_ERR_CUDA, "cudaEventCreateWithFlags failed");
      KM_CUDA(cudaEventCreateWithFlags(&ev_free[i], cudaEventDisableTiming));
    }
    KM_CUDA(cudaMemsetAsync(c.status(), 0, 2 * sizeof(unsigned int), c.s));  // status, objective counter
    chain_break();
    KM_CUDA(cudaMemsetAsync(acc64, 0, sizeof(double) * static_cast<size_t>(K) * D, c.s));
    chain_break();
    KM_CUDA(cudaMemsetAsync(cnt64, 0, sizeof(long long) * K, c.s));
    chain_break();
    KM_CUDA(cudaMemsetAsync(objacc, 0, sizeof(double), c.s));
    chain_break();
    KM_CUDA(launch_cprep(C0, dtype, 1, K, p.Kp, D, p.Dp, dtype, C_out, clp, caug, c.s));
    int32_t* rk = at<int32_t>(c.ws, p.off_rk);
    for (int i = 0; i < 2; ++i) {
      KM_CUDA(cudaEventRecord(ev_free[i], c.s));
      chain_break();
    }
    const bool f32 = dtype == KM_F32;
    CUtensorMap cmap, camap;
    int rr = encode_map(&cmap, clp, f32, p.Dop, K, 1, cbox(p));
    if (rr != KM_OK) return rr;
    if ((rr = encode_aug_map(&camap, caug, f32, p.Kp, 1, cbox(p))) != KM_OK) return rr;
    const int64_t nch = (N + p.chunk_rows - 1) / p.chunk_rows;
    const size_t rowb = static_cast<size_t>(D) * p.es;
    int64_t g = 0;
    for (int t = 0; t < iters; ++t) {
      for (int64_t ch = 0; ch < nch; ++ch, ++g) {
        const int bi = static_cast<int>(g & 1);
        const int64_t r0 = ch * p.chunk_rows;
        const int64_t nr = N - r0 < p.chunk_rows ? N - r0 : p.chunk_rows;
        // the slot's previous copy (chunk g - 2) must be done before the
        // source may write that slot again
        if (slot_reuse && g >= 2) KM_CUDA(cudaEventSynchronize(ev_copied[bi]));
        const char* why = "";
        const void* src = chunk(r0, nr, bi, &why);
        if (!src) return fail(KM_ERR_INVALID_ARG, "rows %lld..%lld: %s", static_cast<long long>(r0),
                              static_cast<long long>(r0 + nr), why);
        KM_CUDA(cudaStreamWaitEvent(cs, ev_free[bi], 0));
        chain_break();
        if (fault_hit(kFaultH2D)) return fail(KM_ERR_CUDA, "cudaMemcpyAsync of chunk %lld failed", (long long)ch);
        KM_CUDA(cudaMemcpyAsync(dbuf[bi], src, nr * rowb, cudaMemcpyHostToDevice, cs));
        chain_break();
        KM_CUDA(cudaEventRecord(ev_copied[bi], cs));
        chain_break();
        KM_CUDA(cudaStreamWaitEvent(c.s, ev_copied[bi], 0));
        chain_break();
        CUtensorMap xmap, xamap;
        KM_CUDA(launch_xprep(dbuf[bi], dtype, nr, D, p.Dp, xaug, x3, c.s));
        rr = encode_map(&xmap, f32 ? static_cast<const void*>(x3) : dbuf[bi], f32, p.Dop, nr, 1, kTileM);
        if (rr != KM_OK) return rr;
        if ((rr = encode_aug_map(&xamap, xaug, f32, nr, 1, kTileM)) != KM_OK) return rr;
        int32_t* idxc = idx_out ? idx_out + r0 : at<int32_t>(c.ws, p.off_idx);
        Plan pc = p;
        pc.rows = nr;
        pc.tiles_per_inst = (nr + kTileM - 1) / kTileM;
        pc.ntiles = pc.tiles_per_inst;
        int64_t groups = 0;
        AssignArgs a{&xmap, &xamap, &cmap,      &camap,          1,       nr,  K,
                     p.Kp,  idxc,   nullptr,    tobj,            c.status(), wait_limit_ns(), &groups,
                     clp,   op_row_bytes(p)};
        KM_CUDA(launch_assign(pc, a, c.s));
        Ctx cc = c;
        cc.p = pc;
        rr = update_instance(cc, dbuf[bi], idxc, nr, C_out, nullptr, nullptr, nullptr, tobj, groups, objacc, 1,
                             nullptr, nullptr, rk);
        if (rr != KM_OK) return rr;
        KM_CUDA(cudaEventRecord(ev_free[bi], c.s));
        chain_break();
      }
      KM_CUDA(launch_finalize_acc(p, acc64, cnt64, C_out, clp, caug, counts_out, objacc, objs + t, c.s));
    }
    KM_CUDA(cudaStreamSynchronize(c.s));
    if (objective_hist && iters > 0)
      KM_CUDA(cudaMemcpy(objective_hist, objs, sizeof(double) * iters, cudaMemcpyDeviceToHost));
    return km_workspace_status(c.ws, c.s);
  };
  r = run();
  if (r != KM_OK) cudaStreamSynchronize(c.s);
  cleanup();
  return r;
}

}  // namespace

extern "C" {

int km_fit_host(const void* X_host, const void* C0, int64_t N, int D, int K, int dtype, int iters, int64_t chunk_rows,
                float* C_out, int32_t* idx_out, int32_t* counts_out, double* objective_hist, void* workspace,
                size_t workspace_bytes, void* stream) {
  g_err.clear();
  if (!X_host || !C0 || !C_out) return fail(KM_ERR_INVALID_ARG, "X_host, C0 and C_out are required");
  cudaPointerAttributes pa;
  const cudaError_t pe = cudaPointerGetAttributes(&pa, X_host);
  if (pe != cudaSuccess || pa.type != cudaMemoryTypeHost) {
    if (pe != cudaSuccess && pe != cudaErrorInvalidValue) {
      const int rc = check_device();
      if (rc != KM_OK) return rc;
    }
    return fail(KM_ERR_INVALID_ARG, "X_host must be page-locked host memory");
  }
  const size_t rowb = static_cast<size_t>(D) * (dtype == KM_BF16 ? 2 : 4);
  const ChunkFn chunk = [&](int64_t r0, int64_t, int, const char**) -> const void* {
    return static_cast<const uint8_t*>(X_host) + r0 * rowb;
  };
  return fit_stream(chunk, false, C0, N, D, K, dtype, iters, chunk_rows, C_out, idx_out, counts_out, objective_hist,
                    workspace, workspace_bytes, stream);
}

int km_fit_source(km_chunk_source source, void* user, const void* C0, int64_t N, int D, int K, int dtype, int iters,
                  int64_t chunk_rows, float* C_out, int32_t* idx_out, int32_t* counts_out, double* objective_hist,
                  void* workspace, size_t workspace_bytes, void* stream) {
  g_err.clear();
  if (!source || !C0 || !C_out) return fail(KM_ERR_INVALID_ARG, "source, C0 and C_out are required");
  const ChunkFn chunk = [&](int64_t r0, int64_t nr, int slot, const char** why) -> const void* {
    const void* ptr = source(user, r0, nr, slot);
    if (!ptr) {
      *why = "the chunk source returned no rows";
      return nullptr;
    }
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, ptr) != cudaSuccess || pa.type != cudaMemoryTypeHost) {
      cudaGetLastError();
      *why = "the chunk source returned memory that is not page-locked host memory";
      return nullptr;
    }
    return ptr;
  };
  return fit_stream(chunk, true, C0, N, D, K, dtype, iters, chunk_rows, C_out, idx_out, counts_out, objective_hist,
                    workspace, workspace_bytes, stream);
}

int km_argsort(const int32_t* idx, int64_t N, int K, int32_t* perm, int32_t* start, void* workspace,
               size_t workspace_bytes, void* stream) {
  g_err.clear();
  if (!idx || !perm) return fail(KM_ERR_INVALID_ARG, "idx and perm are required");
  Ctx c;
  int r = prepare(c, KM_OP_ARGSORT, 1, N, 8, K, KM_BF16, 0, workspace, workspace_bytes, stream);
  if (r != KM_OK) return r;
  const Plan& p = c.p;
  SortArgs sa{idx,
              N,
              K,
              at<int32_t>(c.ws, p.off_blkhist),
              p.sc.passes > 1 ? at<int32_t>(c.ws, p.off_blkhist1) : nullptr,
              at<int32_t>(c.ws, p.off_rk),
              at<int32_t>(c.ws, p.off_total),
              p.sc.passes > 1 ? at<int2>(c.ws, p.off_pairs_tmp) : nullptr,
              at<int2>(c.ws, p.off_pairs),
              perm,
              start ? start : at<int32_t>(c.ws, p.off_start)};
  KM_CUDA(launch_sort(p, sa, c.s));
  return KM_OK;
}

int km_update_accumulate(const void* X, const int32_t* idx, int64_t N, int D, int K, int dtype, double* sums,
                         double* counts, int zero_first, void* workspace, size_t workspace_bytes, void* stream) {
  g_err.clear();
  if (!X || !idx || !sums || !counts) return fail(KM_ERR_INVALID_ARG, "X, idx, sums and counts are required");
  if (!aligned16(X)) return fail(KM_ERR_INVALID_ARG, "X must be 16-byte aligned");
  Ctx c;
  int r = prepare(c, KM_OP_UPDATE, 1, N, D, K, dtype, 0, workspace, workspace_bytes, stream);
  if (r != KM_OK) return r;
  if (zero_first) {
    KM_CUDA(cudaMemsetAsync(sums, 0, sizeof(double) * static_cast<size_t>(K) * D, c.s));
    chain_break();
    KM_CUDA(cudaMemsetAsync(counts, 0, sizeof(double) * K, c.s));
    chain_break();
  }
  return update_instance(c, X, idx, N, nullptr, nullptr, nullptr, nullptr, nullptr, 0, nullptr, 1, sums, counts);
}

int km_finalize_sums(const double* sums, const double* counts, int K, int D, int dtype, float* C, void* C_lp,
                     int32_t* counts_out, void* stream) {
  g_err.clear();
  if (!sums || !counts || !C) return fail(KM_ERR_INVALID_ARG, "sums, counts and C are required");
  if (K < 1 || D < 1) return fail(KM_ERR_INVALID_ARG, "need K >= 1 and D >= 1");
  if (dtype != KM_F32 && dtype != KM_BF16) return fail(KM_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  fault_arm_from_env();
  int r = check_device();
  if (r != KM_OK) return r;
  KM_CUDA(km::launch_finalize_sums(K, D, dtype, sums, counts, C, C_lp, counts_out,
                                   static_cast<cudaStream_t>(stream)));
  return KM_OK;
}

int km_plan_describe(int op, int B, int64_t N, int D, int K, int dtype, int64_t chunk_rows, int64_t* out) {
  g_err.clear();
  if (!out) return fail(KM_ERR_INVALID_ARG, "out is required");
  km::Plan p;
  const char* why = "";
  const int r = km::make_plan(p, op, B, N, D, K, dtype, chunk_rows, &why);
  if (r != KM_OK) return fail(r, "%s", why);
  out[0] = p.ac.pair ? 1 : 0;
  out[1] = p.ac.BN;
  out[2] = p.ac.XB;
  out[3] = p.ac.CS;
  out[4] = static_cast<int64_t>(p.ac.smem);
  out[5] = p.Kp;
  out[6] = p.sc.passes;
  out[7] = p.sc.T;
  out[8] = p.small_update ? 1 : 0;
  return KM_OK;
}

// ------------------------------------------------------------- baselines
namespace {
int ablation_check(const void* X, int64_t N, int D, int K, int dtype) {
  fault_arm_from_env();
  if (!X) return fail(KM_ERR_INVALID_ARG, "X is required");
  if (dtype != KM_F32 && dtype != KM_BF16) return fail(KM_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (N < 1 || K < 1 || K > N) return fail(KM_ERR_INVALID_ARG, "need 1 <= K <= N (N=%lld K=%d)", (long long)N, K);
  if (N >= (int64_t(1) << 31)) return fail(KM_ERR_UNSUPPORTED, "N must be below 2^31");
  if (D < 8 || D % 8 != 0) return fail(KM_ERR_UNSUPPORTED, "D=%d must be a positive multiple of 8", D);
  if (!aligned16(X)) return fail(KM_ERR_INVALID_ARG, "X must be 16-byte aligned");
  return check_device();
}
}  // namespace

size_t km_ablation_workspace_size(int which, int64_t N, int D, int K, int dtype, int64_t chunk_rows) {
  (void)dtype;
  if (N < 1 || K < 1 || D < 8) return 0;
  if (which == 0) {
    if (chunk_rows < 1) return 0;
    return km::ablation_assign_ws(chunk_rows < N ? chunk_rows : N, K);
  }
  if (which == 1) return km::ablation_update_ws(D, K);
  return 0;
}

int km_ablation_assign_materialized(const void* X, const void* C, int64_t N, int D, int K, int dtype,
                                    int64_t chunk_rows, int32_t* idx, float* mindist, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  g_err.clear();
  int r = ablation_check(X, N, D, K, dtype);
  if (r != KM_OK) return r;
  if (!C || !idx) return fail(KM_ERR_INVALID_ARG, "C and idx are required");
  if (chunk_rows < 1) return fail(KM_ERR_INVALID_ARG, "chunk_rows must be >= 1");
  const int64_t cr = chunk_rows < N ? chunk_rows : N;
  if (cr * static_cast<int64_t>(K) >= (int64_t(1) << 31))
    return fail(KM_ERR_UNSUPPORTED, "chunk_rows x K must stay below 2^31 scores");
  if (!workspace || workspace_bytes < km::ablation_assign_ws(cr, K))
    return fail(KM_ERR_WORKSPACE, "workspace needs %zu bytes", km::ablation_assign_ws(cr, K));
  r = km::ablation_assign(X, C, N, D, K, dtype, cr, idx, mindist, workspace, static_cast<cudaStream_t>(stream));
  if (r == KM_ERR_UNSUPPORTED) return fail(r, "cuBLAS (libcublas.so.12) could not be loaded");
  if (r != KM_OK) return fail(r, "materialised-distance assignment failed");
  return KM_OK;
}

int km_ablation_update_atomic(const void* X, const int32_t* idx, int64_t N, int D, int K, int dtype, float* C,
                              int32_t* counts, void* workspace, size_t workspace_bytes, void* stream) {
  g_err.clear();
  int r = ablation_check(X, N, D, K, dtype);
  if (r != KM_OK) return r;
  if (!idx || !C || !counts) return fail(KM_ERR_INVALID_ARG, "idx, C and counts are required");
  if (!workspace || workspace_bytes < km::ablation_update_ws(D, K))
    return fail(KM_ERR_WORKSPACE, "workspace needs %zu bytes", km::ablation_update_ws(D, K));
  r = km::ablation_update(X, idx, N, D, K, dtype, C, counts, workspace, static_cast<cudaStream_t>(stream));
  if (r != KM_OK) return fail(r, "atomic-scatter update failed");
  return KM_OK;
}

int km_selftest_timeout(void* workspace, size_t workspace_bytes, int64_t limit_ns, void* stream) {
  g_err.clear();
  if (!workspace || workspace_bytes < kAlign) return fail(KM_ERR_WORKSPACE, "need at least 256 bytes of workspace");
  if (limit_ns < 1 || limit_ns > 1000000000) return fail(KM_ERR_INVALID_ARG, "limit_ns must be in [1, 1e9]");
  fault_arm_from_env();
  int r = check_device();
  if (r != KM_OK) return r;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  KM_CUDA(cudaMemsetAsync(workspace, 0, sizeof(unsigned int), s));
  chain_break();
  KM_CUDA(launch_timeout_probe(static_cast<unsigned int*>(workspace), static_cast<uint64_t>(limit_ns), s));
  return km_workspace_status(workspace, s);
}

}  // extern "C"
