// k_ablation.cu -- the two strategies that "Flash-KMeans: Fast and
// Memory-Efficient Exact K-Means" (§1 Problem) says the method replaces,
// built as measured baselines.  The fit never uses them.
//
//  (1) Materialised distances (§1: the N x K distance matrix written to and
//      read back from device memory): S = X C^T by a library GEMM (cuBLAS,
//      bf16 or fp32 in, fp32 out) into a [rows][K] buffer, then an argmin
//      kernel that reads S back and forms ||x||^2 + ||c||^2 - 2 S.  Rows are
//      processed in chunks so that S fits the caller's workspace.
//  (2) Atomic-scatter update (§1: every point adds itself to its cluster's
//      sum with atomics, serialising on popular clusters): one 16-byte vector
//      float atomic per row chunk per point, one integer atomic per point for
//      the count, then a divide kernel (an empty cluster keeps its centroid).
//      Float atomics make the sums' rounding order, and so the last bits of
//      the centroids, vary from run to run.
//
// cuBLAS is opened at run time (dlopen) on first use, so the library has no
// link-time dependency on it; without it these entry points report
// KM_ERR_UNSUPPORTED.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <dlfcn.h>
#include <library_types.h>

#include <cfloat>
#include <cstdint>
#include <mutex>

#include "../../include/km.h"
#include "km_internal.h"

namespace km {

namespace {

// cuBLAS entry points used here (types as in its public header).
typedef int (*CublasCreateFn)(void**);
typedef int (*CublasSetStreamFn)(void*, cudaStream_t);
typedef int (*CublasGemmExFn)(void*, int, int, int, int, int, const void*, const void*, cudaDataType, int,
                              const void*, cudaDataType, int, const void*, void*, cudaDataType, int, int, int);
constexpr int kCublasOpN = 0, kCublasOpT = 1;
constexpr int kCublasCompute32F = 68;    // CUBLAS_COMPUTE_32F
constexpr int kCublasGemmDefault = -1;   // CUBLAS_GEMM_DEFAULT

struct Cublas {
  CublasCreateFn create = nullptr;
  CublasSetStreamFn set_stream = nullptr;
  CublasGemmExFn gemm = nullptr;
  void* handle[64] = {};  // one per device
  bool tried = false, ok = false;
};

Cublas& cublas() {
  static Cublas c;
  return c;
}

std::mutex& cublas_mutex() {
  static std::mutex m;
  return m;
}

// Handle for the current device, or null if cuBLAS cannot be used.
void* cublas_handle(int dev) {
  std::lock_guard<std::mutex> lk(cublas_mutex());
  Cublas& c = cublas();
  if (!c.tried) {
    c.tried = true;
    void* h = dlopen("libcublas.so.12", RTLD_NOW | RTLD_GLOBAL);
    if (!h) h = dlopen("libcublas.so", RTLD_NOW | RTLD_GLOBAL);
    if (h) {
      c.create = reinterpret_cast<CublasCreateFn>(dlsym(h, "cublasCreate_v2"));
      c.set_stream = reinterpret_cast<CublasSetStreamFn>(dlsym(h, "cublasSetStream_v2"));
      c.gemm = reinterpret_cast<CublasGemmExFn>(dlsym(h, "cublasGemmEx"));
      c.ok = c.create && c.set_stream && c.gemm;
    }
  }
  if (!c.ok || dev < 0 || dev >= 64) return nullptr;
  if (!c.handle[dev] && c.create(&c.handle[dev]) != 0) c.handle[dev] = nullptr;
  return c.handle[dev];
}

// ||c_k||^2 of the operand values (bf16 or fp32), one warp per centroid.
__global__ void k_ab_cnorm(const void* C, int K, int D, int dtype, float* cn) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= K) return;
  float s = 0.f;
  for (int j = lane; j < D; j += 32) {
    const int64_t e = static_cast<int64_t>(warp) * D + j;
    const float v = dtype == kDtypeBF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(C)[e])
                                        : static_cast<const float*>(C)[e];
    s = fmaf(v, v, s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) cn[warp] = s;
}

// One warp per row of the materialised scores: ||x||^2 from X, then
// d_k = ||x||^2 + cn_k - 2 S_ik over k; argmin with the lowest index on ties.
__global__ void k_ab_argmin(const void* X, const float* __restrict__ S, const float* __restrict__ cn, int64_t rows,
                            int64_t row0, int D, int K, int dtype, int32_t* idx, float* mindist) {
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float xn = 0.f;
  for (int j = lane; j < D; j += 32) {
    const int64_t e = (row0 + r) * D + j;
    const float v = dtype == kDtypeBF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(X)[e])
                                        : static_cast<const float*>(X)[e];
    xn = fmaf(v, v, xn);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) xn += __shfl_xor_sync(0xffffffffu, xn, o);
  const float* srow = S + r * K;
  float best = FLT_MAX;
  int bk = 0;
  for (int k = lane; k < K; k += 32) {
    const float d = xn + cn[k] - 2.f * srow[k];
    if (d < best) {  // ascending k per lane: the first (lowest) index is kept
      best = d;
      bk = k;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int ok = __shfl_xor_sync(0xffffffffu, bk, o);
    if (ob < best || (ob == best && ok < bk)) {
      best = ob;
      bk = ok;
    }
  }
  if (lane == 0) {
    idx[row0 + r] = bk;
    if (mindist) mindist[row0 + r] = fmaxf(0.f, best);
  }
}

// Atomic scatter: thread per (point, 4-column group); float4 atomics on the
// cluster's sum row, plus the point's count from the group-0 thread.
__global__ void k_ab_scatter(const void* X, const int32_t* __restrict__ idx, int64_t N, int D, int K, int dtype,
                             float* sums, int32_t* counts) {
  const int G = D / 4;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= N * G) return;
  const int64_t i = t / G;
  const int g = static_cast<int>(t - i * G);
  int k = idx[i];
  k = k < 0 ? 0 : (k >= K ? K - 1 : k);  // memory safety only
  float4 v;
  if (dtype == kDtypeBF16) {
    const uint2 w = reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(X) + i * D)[g];
    v = make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u), __uint_as_float(w.y << 16),
                    __uint_as_float(w.y & 0xffff0000u));
  } else {
    v = reinterpret_cast<const float4*>(static_cast<const float*>(X) + i * D)[g];
  }
  atomicAdd(reinterpret_cast<float4*>(sums + static_cast<int64_t>(k) * D) + g, v);
  if (g == 0) atomicAdd(counts + k, 1);
}

__global__ void k_ab_divide(const float* __restrict__ sums, const int32_t* __restrict__ counts, int K, int D,
                            float* C) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= static_cast<int64_t>(K) * D) return;
  const int k = static_cast<int>(e / D);
  const int c = counts[k];
  if (c > 0) C[e] = sums[e] / static_cast<float>(c);
}

}  // namespace

size_t ablation_assign_ws(int64_t chunk_rows, int K) {
  // alignment slack, norms rounded up to 64 floats, the chunk's scores
  return 256 + static_cast<size_t>((K + 63) / 64) * 64 * 4 + static_cast<size_t>(chunk_rows) * K * 4;
}

size_t ablation_update_ws(int D, int K) { return 256 + static_cast<size_t>(K) * D * 4; }

int ablation_assign(const void* X, const void* C, int64_t N, int D, int K, int dtype, int64_t chunk_rows,
                    int32_t* idx, float* mindist, void* ws, cudaStream_t s) {
  chain_break();  // plain launch: the next kernel must not chain to it
  int dev = 0;
  cudaGetDevice(&dev);
  void* h = cublas_handle(dev);
  if (!h) return KM_ERR_UNSUPPORTED;
  float* cn = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  float* S = cn + ((K + 63) / 64) * 64;
  if (fault_hit(kFaultLaunch)) return KM_ERR_CUDA;
  count_launch();
  k_ab_cnorm<<<(K * 32 + 255) / 256, 256, 0, s>>>(C, K, D, dtype, cn);
  if (cudaGetLastError() != cudaSuccess) return KM_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lk(cublas_mutex());
    if (cublas().set_stream(h, s) != 0) return KM_ERR_CUDA;
  }
  const cudaDataType in_t = dtype == kDtypeBF16 ? CUDA_R_16BF : CUDA_R_32F;
  const size_t es = dtype == kDtypeBF16 ? 2 : 4;
  const float alpha = 1.f, beta = 0.f;
  for (int64_t r0 = 0; r0 < N; r0 += chunk_rows) {
    const int64_t nr = N - r0 < chunk_rows ? N - r0 : chunk_rows;
    // column-major view: S^T (K x nr) = C^T (K x D) . X^T (D x nr), i.e. the
    // row-major [nr][K] scores
    const void* Xc = static_cast<const uint8_t*>(X) + r0 * D * es;
    int st;
    {
      std::lock_guard<std::mutex> lk(cublas_mutex());
      st = cublas().gemm(h, kCublasOpT, kCublasOpN, K, static_cast<int>(nr), D, &alpha, C, in_t, D, Xc, in_t, D,
                         &beta, S, CUDA_R_32F, K, kCublasCompute32F, kCublasGemmDefault);
    }
    if (st != 0) return KM_ERR_CUDA;
    if (fault_hit(kFaultLaunch)) return KM_ERR_CUDA;
    count_launch();
    const int64_t threads = nr * 32;
    k_ab_argmin<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, s>>>(X, S, cn, nr, r0, D, K, dtype, idx,
                                                                              mindist);
    if (cudaGetLastError() != cudaSuccess) return KM_ERR_CUDA;
  }
  return KM_OK;
}

int ablation_update(const void* X, const int32_t* idx, int64_t N, int D, int K, int dtype, float* C,
                    int32_t* counts, void* ws, cudaStream_t s) {
  chain_break();  // plain launch: the next kernel must not chain to it
  float* sums = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  if (cudaMemsetAsync(sums, 0, static_cast<size_t>(K) * D * 4, s) != cudaSuccess) return KM_ERR_CUDA;
  if (cudaMemsetAsync(counts, 0, static_cast<size_t>(K) * 4, s) != cudaSuccess) return KM_ERR_CUDA;
  const int64_t threads = N * (D / 4);
  if (fault_hit(kFaultLaunch)) return KM_ERR_CUDA;
  count_launch(2);
  k_ab_scatter<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, s>>>(X, idx, N, D, K, dtype, sums, counts);
  const int64_t e = static_cast<int64_t>(K) * D;
  k_ab_divide<<<static_cast<unsigned>((e + 255) / 256), 256, 0, s>>>(sums, counts, K, D, C);
  return cudaGetLastError() == cudaSuccess ? KM_OK : KM_ERR_CUDA;
}

}  // namespace km
