// Device helpers shared by the library's kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sata {

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

// T_P(s) = sum_{p<P} s^p/p!, evaluated by Horner's rule:
// 1 + s(1 + s/2 (1 + s/3 (...))).
__device__ __forceinline__ float taylor_trunc(float s, int P) {
  float t = 1.0f;
  for (int p = P - 1; p >= 1; --p) t = fmaf(t, s * (1.0f / (float)p), 1.0f);
  return t;
}

// Packed basis row (i1 | i2 << 7 | i3 << 14 | i4 << 21 | degree << 28).
__device__ __forceinline__ int packed_index(uint32_t packed, int s) {
  return (packed >> (7 * s)) & 0x7f;
}
__device__ __forceinline__ int packed_degree(uint32_t packed) { return packed >> 28; }
// The packed row of a padding slot: every index at x[dK] (its weight is 0).
__host__ __device__ constexpr uint32_t padding_row(int dK) {
  return (uint32_t)dK | (uint32_t)dK << 7 | (uint32_t)dK << 14 | (uint32_t)dK << 21;
}

// phi_r(x) for one basis row from the packed table entry (unused index slots
// point at x[dK] == 1.0f).
__device__ __forceinline__ float feature_from_packed(const float *x, uint32_t packed, float w) {
  return w * x[packed_index(packed, 0)] * x[packed_index(packed, 1)] *
         x[packed_index(packed, 2)] * x[packed_index(packed, 3)];
}

}  // namespace sata
