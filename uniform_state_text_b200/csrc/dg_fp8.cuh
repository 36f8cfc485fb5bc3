// e4m3 helpers shared by the narrow-E kernels: decoding a code, rounding two
// floats to two codes (nearest even, saturated), and the power-of-two exponent
// that brings a row's or block's largest magnitude within the format's 448.
#pragma once
#include <cuda_fp8.h>
#include <stdint.h>

namespace dg {

__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  __nv_fp8_e4m3 v;
  v.__x = c;
  return static_cast<float>(v);
}

// Two floats to two e4m3 codes (x in the lower byte), nearest even, saturated.
__device__ __forceinline__ uint16_t f32x2_to_e4m3(float x, float y) {
  return (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(x, y), __NV_SATFINITE, __NV_E4M3);
}

// Smallest e with amax 2^-e <= 448 = 0.875 2^9: amax = m 2^x, m in [0.5, 1),
// e = x - 9, plus one when m > 0.875 (0 for amax = 0).
__device__ __forceinline__ int e4m3_row_exponent(float amax) {
  if (!(amax > 0.f)) return 0;
  int x;
  const float m = frexpf(amax, &x);
  return x - 9 + (m > 0.875f ? 1 : 0);
}

}  // namespace dg
