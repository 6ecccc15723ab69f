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

// One warp writes the assignment operand for centroid row k of an instance
// from float values supplied by `get(j)` (j < D), and returns ||c||^2 of the
// values the MMA uses (bf16-rounded in bf16 mode, the float32 values in f32
// mode).  The operand holds -2c (exact: a power-of-two scale): bf16 [D], or
// float [3*Dp] = -2 * [hi | lo | hi] for the TF32 split.
template <class Get>
__device__ __forceinline__ float emit_operand_row(Get get, int D, int Dp, int dtype, void* c_op_row, int lane) {
  float s = 0.f;
  if (dtype == kDtypeBF16) {
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(c_op_row);
    for (int j = lane; j < D; j += 32) {
      const __nv_bfloat16 h = __float2bfloat16_rn(get(j));
      const float f = __bfloat162float(h);
      if (o) o[j] = __float2bfloat16_rn(-2.f * f);
      s = fmaf(f, f, s);
    }
  } else {
    float* o = reinterpret_cast<float*>(c_op_row);
    for (int j = lane; j < Dp; j += 32) {
      const float v = j < D ? get(j) : 0.f;
      if (o) {
        const float hi = tf32_round(v);
        const float lo = tf32_round(v - hi);
        o[j] = -2.f * hi;
        o[Dp + j] = -2.f * lo;
        o[2 * Dp + j] = -2.f * hi;
      }
      s = fmaf(v, v, s);
    }
  }
  return warp_sum_f(s);
}

// --------------------------------------------------------------------------
// Norm augmentation.  One extra 32-byte K-slice on each operand makes the
// tensor-core product equal the full squared distance:
//   point row    a_i = [n_hi, n_mid, n_lo, 1, 1, 1, 0, ...]   (n = ||x_i||^2)
//   centroid row b_k = [1, 1, 1, m_hi, m_mid, m_lo, 0, ...]   (m = ||c_k||^2)
//   a_i . b_k = ||x_i||^2 + ||c_k||^2, added to (-2c) . x by the same MMA.
// hi/mid/lo are successive round-to-nearest bf16 (or TF32) pieces of the
// float norm, so their sum carries ~24 significant bits.  A padding centroid
// row (k >= K) is [0, 0, 0, +inf, 0, ...]: its score is +inf, so it never
// wins (the zero entries meet the point row's finite values only).
// bf16 rows hold 16 elements, TF32 rows 8 floats; both are 32 bytes.
constexpr int kAugBytes = 32;

__device__ __forceinline__ void split3_bf16(float v, __nv_bfloat16 (&o)[3]) {
  o[0] = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(o[0]);
  o[1] = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(o[1]);
  o[2] = __float2bfloat16_rn(r2);
}

__device__ __forceinline__ void split3_tf32(float v, float (&o)[3]) {
  o[0] = tf32_round(v);
  const float r1 = v - o[0];
  o[1] = tf32_round(r1);
  o[2] = tf32_round(r1 - o[1]);
}

// role 0: point row, 1: centroid row, 2: padding centroid row.
__device__ __forceinline__ void write_aug_row(void* row, int dtype, float norm, int role) {
  if (dtype == kDtypeBF16) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = 0.f;
    uint32_t bits[16];
    if (role == 2) {
      v[3] = __int_as_float(0x7f800000);
#pragma unroll
      for (int i = 0; i < 16; ++i) bits[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v[i]));
    } else {
      __nv_bfloat16 s[3];
      split3_bf16(norm, s);
      const int at = role == 0 ? 0 : 3, ones = role == 0 ? 3 : 0;
#pragma unroll
      for (int i = 0; i < 3; ++i) v[ones + i] = 1.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) bits[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v[i]));
#pragma unroll
      for (int i = 0; i < 3; ++i) bits[at + i] = __bfloat16_as_ushort(s[i]);
    }
    uint4* d = reinterpret_cast<uint4*>(row);
    d[0] = make_uint4(bits[0] | (bits[1] << 16), bits[2] | (bits[3] << 16), bits[4] | (bits[5] << 16),
                      bits[6] | (bits[7] << 16));
    d[1] = make_uint4(bits[8] | (bits[9] << 16), bits[10] | (bits[11] << 16), bits[12] | (bits[13] << 16),
                      bits[14] | (bits[15] << 16));
  } else {
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (role == 2) {
      v[3] = __int_as_float(0x7f800000);
    } else {
      float s[3];
      split3_tf32(norm, s);
      const int at = role == 0 ? 0 : 3, ones = role == 0 ? 3 : 0;
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        v[at + i] = s[i];
        v[ones + i] = 1.f;
      }
    }
    float4* d = reinterpret_cast<float4*>(row);
    d[0] = make_float4(v[0], v[1], v[2], v[3]);
    d[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

}  // namespace km
