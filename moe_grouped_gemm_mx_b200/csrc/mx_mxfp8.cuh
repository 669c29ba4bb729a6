// mx_mxfp8.cuh -- device-side MXFP8 block quantisation of FP32 values (the
// rule of the BF16 quantiser in mx_quant.cu applied to FP32 input), shared by
// the fused SwiGLU epilogue and the transposing quantiser.
#pragma once
#include <cuda_fp8.h>
#include <cstdint>

namespace mxk {

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// MXFP8 quantisation of 32 FP32 values (the BF16 quantiser's rule applied to
// FP32 input): X = floor(log2 amax) - 8 clamped to [-127, 127] (amax 0 gives
// -127), elements x * 2^-X with saturating round-to-nearest-even; a block
// holding NaN or Inf gets scale 0xFF and elements 0x7F.  amax is taken on the
// integer magnitude bits (order-preserving for IEEE patterns, and >= 0x7f800000
// exactly for Inf/NaN).  Returns the scale byte; q receives 32 bytes.
__device__ __forceinline__ uint32_t quant_block32_f32(const float (&h)[32], uint32_t (&q)[8]) {
  uint32_t amax = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) amax = max(amax, __float_as_uint(h[j]) & 0x7FFFFFFFu);
  if (amax >= 0x7F800000u) {
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = 0x7F7F7F7Fu;
    return 0xFFu;
  }
  int x = -127;
  if (amax != 0) {
    const int e = static_cast<int>(amax >> 23);
    const int fl = e > 0 ? e - 127 : (31 - __clz(amax & 0x7FFFFFu)) - 149;  // subnormal: m * 2^-149
    x = fl - 8;
    x = x < -127 ? -127 : (x > 127 ? 127 : x);
  }
  // 2^-X as an FP32 bit pattern: finite FP32 input keeps X <= 119, so the
  // exponent field 127 - X lies in [8, 254]
  const float s = __uint_as_float(static_cast<uint32_t>(127 - x) << 23);
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = e4m3x4(h[4 * i] * s, h[4 * i + 1] * s, h[4 * i + 2] * s, h[4 * i + 3] * s);
  return static_cast<uint32_t>(x + 127);
}

}  // namespace mxk
