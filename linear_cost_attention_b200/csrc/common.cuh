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

// phi_r(x) for one basis row from the packed table entry (unused index slots
// point at x[dK] == 1.0f).
__device__ __forceinline__ float feature_from_packed(const float *x, uint32_t packed, float w) {
  const int i1 = packed & 0xff, i2 = (packed >> 8) & 0xff, i3 = (packed >> 16) & 0xff;
  return w * x[i1] * x[i2] * x[i3];
}

}  // namespace sata
