// km_rows.cuh -- per-row helpers shared by the preparation and update kernels:
// loading a point/centroid row, the TF32 hi/lo split and the centroid
// operand emission (bf16 copy or TF32 split, plus the squared norm of exactly
// the values the tensor cores will multiply).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "km_internal.h"

namespace km {

__device__ __forceinline__ float tf32_round(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

__device__ __forceinline__ float load_elem(const void* base, int dtype, int64_t i) {
  if (dtype == kDtypeBF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return reinterpret_cast<const float*>(base)[i];
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One warp writes the assignment operand for centroid row k of an instance
// from float values supplied by `get(j)` (j < D), and returns ||c||^2 of the
// values the MMA uses (bf16-rounded in bf16 mode, the float32 values in f32
// mode).  c_op rows: bf16 [D] or float [3*Dp] = [hi | lo | hi].
template <class Get>
__device__ __forceinline__ float emit_operand_row(Get get, int D, int Dp, int dtype, void* c_op_row, int lane) {
  float s = 0.f;
  if (dtype == kDtypeBF16) {
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(c_op_row);
    for (int j = lane; j < D; j += 32) {
      __nv_bfloat16 h = __float2bfloat16_rn(get(j));
      if (o) o[j] = h;
      float f = __bfloat162float(h);
      s = fmaf(f, f, s);
    }
  } else {
    float* o = reinterpret_cast<float*>(c_op_row);
    for (int j = lane; j < Dp; j += 32) {
      float v = j < D ? get(j) : 0.f;
      if (o) {
        float hi = tf32_round(v);
        float lo = tf32_round(v - hi);
        o[j] = hi;
        o[Dp + j] = lo;
        o[2 * Dp + j] = hi;
      }
      s = fmaf(v, v, s);
    }
  }
  return warp_sum_f(s);
}

}  // namespace km
