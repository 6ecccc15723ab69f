// k_prep.cu -- operand preparation for FlashAssign (Flash-KMeans §2.1 uses
// precomputed squared norms: the distance is ||x||^2 - 2 x.c + ||c||^2, and
// only the cross term needs the tensor cores).
#include <cuda_bf16.h>
#include <math_constants.h>

#include "km_internal.h"
#include "km_rows.cuh"

namespace km {

// One warp per point row (f32 mode): ||x||^2 into the augmentation row and
// the TF32 split operand [hi | hi | lo] (paired with the centroid split
// -2 [hi | lo | hi] the dot product becomes -2 (hi*hi + hi*lo + lo*hi)).
__global__ void k_xprep(const void* __restrict__ X, int dtype, int64_t rows, int D, int Dp,
                        uint8_t* __restrict__ xaug, float* __restrict__ x3) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (r >= rows) return;
  float s = 0.f;
  if (dtype == kDtypeBF16) {
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(X) + r * D;
    for (int j = lane; j < D; j += 32) {
      float f = __bfloat162float(x[j]);
      s = fmaf(f, f, s);
    }
  } else {
    const float* x = reinterpret_cast<const float*>(X) + r * D;
    float* o = x3 ? x3 + r * (3 * Dp) : nullptr;
    for (int j = lane; j < Dp; j += 32) {
      float v = j < D ? x[j] : 0.f;
      s = fmaf(v, v, s);
      if (o) {
        float hi = tf32_round(v);
        float lo = tf32_round(v - hi);
        o[j] = hi;
        o[Dp + j] = hi;
        o[2 * Dp + j] = lo;
      }
    }
  }
  s = warp_sum_f(s);
  if (lane == 0) write_aug_row(xaug + r * kAugBytes, dtype, s, 0);
}

// bf16 row norms with one 16-byte load per lane: LPR lanes cover a row (LPR a
// power of two with LPR * 16 >= 2 * D), 32 / LPR rows per warp step.
template <int LPR>
__global__ void __launch_bounds__(256) k_xnorm_bf16(const uint8_t* __restrict__ X, int64_t rows, int row_bytes,
                                                    uint8_t* __restrict__ xaug) {
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, cl = lane % LPR;
  constexpr int RPW = 32 / LPR;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t w0 = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  for (int64_t r0 = w0 * RPW; r0 < rows; r0 += warps * RPW) {
    const int64_t r = r0 + sub;
    float s = 0.f;
    if (r < rows && cl * 16 < row_bytes) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(X + r * row_bytes + cl * 16));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
        s = fmaf(lo, lo, s);
        s = fmaf(hi, hi, s);
      }
    }
#pragma unroll
    for (int o = 1; o < LPR; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (r < rows && cl == 0) write_aug_row(xaug + r * kAugBytes, kDtypeBF16, s, 0);
  }
}

cudaError_t launch_xprep(const void* X, int dtype, int64_t rows, int D, int Dp, void* xaug_v, float* x3,
                         cudaStream_t s) {
  chain_break();  // plain launch: the next kernel must not chain to it
  uint8_t* xaug = static_cast<uint8_t*>(xaug_v);
  if (rows <= 0) return cudaSuccess;
  if (dtype == kDtypeBF16) {
    const int row_bytes = 2 * D;
    int lpr = 1;
    while (lpr * 16 < row_bytes) lpr <<= 1;
    int dev = 0, nsm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int64_t need = (rows * lpr + 255) / 256;
    const unsigned grid = static_cast<unsigned>(need < int64_t(nsm) * 8 ? need : int64_t(nsm) * 8);
    const uint8_t* Xb = static_cast<const uint8_t*>(X);
    if (fault_hit(kFaultLaunch)) return cudaErrorLaunchFailure;
    count_launch();
    switch (lpr) {
      case 1: k_xnorm_bf16<1><<<grid, 256, 0, s>>>(Xb, rows, row_bytes, xaug); break;
      case 2: k_xnorm_bf16<2><<<grid, 256, 0, s>>>(Xb, rows, row_bytes, xaug); break;
      case 4: k_xnorm_bf16<4><<<grid, 256, 0, s>>>(Xb, rows, row_bytes, xaug); break;
      case 8: k_xnorm_bf16<8><<<grid, 256, 0, s>>>(Xb, rows, row_bytes, xaug); break;
      case 16: k_xnorm_bf16<16><<<grid, 256, 0, s>>>(Xb, rows, row_bytes, xaug); break;
      default: k_xnorm_bf16<32><<<grid, 256, 0, s>>>(Xb, rows, row_bytes, xaug); break;
    }
    return cudaGetLastError();
  }
  const int threads = 256;
  const int64_t blocks = (rows * 32 + threads - 1) / threads;
  if (fault_hit(kFaultLaunch)) return cudaErrorLaunchFailure;
  count_launch();
  k_xprep<<<static_cast<unsigned>(blocks), threads, 0, s>>>(X, dtype, rows, D, Dp, xaug, x3);
  return cudaGetLastError();
}

// One warp per (instance, centroid row < Kp).
__global__ void k_cprep(const void* __restrict__ src, int src_dtype, int B, int K, int Kp, int D, int Dp,
                        int dtype, float* __restrict__ master, void* __restrict__ c_op, uint8_t* __restrict__ caug) {
  const int lane = threadIdx.x & 31;
  const int64_t g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (g >= static_cast<int64_t>(B) * Kp) return;
  const int b = static_cast<int>(g / Kp);
  const int k = static_cast<int>(g - static_cast<int64_t>(b) * Kp);
  if (k >= K) {
    if (lane == 0) write_aug_row(caug + g * kAugBytes, dtype, 0.f, 2);
    return;
  }
  const int64_t row = static_cast<int64_t>(b) * K + k;
  if (master) {
    for (int j = lane; j < D; j += 32) master[row * D + j] = load_elem(src, src_dtype, row * D + j);
  }
  void* orow = nullptr;
  if (c_op) {
    orow = dtype == kDtypeBF16
               ? static_cast<void*>(reinterpret_cast<__nv_bfloat16*>(c_op) + row * D)
               : static_cast<void*>(reinterpret_cast<float*>(c_op) + row * (3 * Dp));
  }
  float s = emit_operand_row([&](int j) { return load_elem(src, src_dtype, row * D + j); }, D, Dp, dtype, orow,
                             lane);
  if (lane == 0) write_aug_row(caug + g * kAugBytes, dtype, s, 1);
}

cudaError_t launch_cprep(const void* src, int src_dtype, int B, int K, int Kp, int D, int Dp, int dtype,
                         float* master, void* c_op, void* caug, cudaStream_t s) {
  chain_break();  // plain launch: the next kernel must not chain to it
  const int threads = 256;
  const int64_t warps = static_cast<int64_t>(B) * Kp;
  const int64_t blocks = (warps * 32 + threads - 1) / threads;
  if (fault_hit(kFaultLaunch)) return cudaErrorLaunchFailure;
  count_launch();
  k_cprep<<<static_cast<unsigned>(blocks), threads, 0, s>>>(src, src_dtype, B, K, Kp, D, Dp, dtype, master, c_op,
                                                           static_cast<uint8_t*>(caug));
  return cudaGetLastError();
}

// Objective per instance from the FlashAssign tile partials, in a fixed
// order: each thread sums a strided subset sequentially, then a fixed tree.
__global__ void k_objective(const double* __restrict__ tobj, int64_t per_inst, double* __restrict__ out,
                            int out_stride) {
  __shared__ double red[256];
  const int b = blockIdx.x;
  const double* p = tobj + static_cast<int64_t>(b) * per_inst;
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < per_inst; i += 256) s += p[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) out[static_cast<int64_t>(b) * out_stride] = red[0];
}

cudaError_t launch_objective(const double* tobj, int B, int64_t groups_per_inst, double* out, int out_stride,
                             cudaStream_t s) {
  chain_break();  // plain launch: the next kernel must not chain to it
  if (fault_hit(kFaultLaunch)) return cudaErrorLaunchFailure;
  count_launch();
  k_objective<<<B, 256, 0, s>>>(tobj, groups_per_inst * 4, out, out_stride);
  return cudaGetLastError();
}

}  // namespace km
