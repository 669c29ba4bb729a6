// mx_mxfp8.cuh -- device-side MXFP8 block quantisation of one 32-element
// block, from BF16 (the quantiser and the MoE dispatch) or from FP32 (the
// fused SwiGLU epilogue and the transposing quantiser), with one rule.
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

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Scale exponent X for a block whose largest magnitude has BF16 bits `amax_bits`
// (finite).  X = floor(log2 amax) - 8, clamped to [-127, 127]; amax == 0 -> -127.
__device__ __forceinline__ int bf16_block_exponent(uint32_t amax_bits) {
  if (amax_bits == 0) return -127;
  const int e = static_cast<int>(amax_bits >> 7);
  int fl;
  if (e > 0) {
    fl = e - 127;
  } else {
    const uint32_t m = amax_bits & 0x7Fu;  // subnormal: value = m * 2^-133
    fl = (31 - __clz(m)) - 133;
  }
  const int X = fl - 8;
  return X < -127 ? -127 : (X > 127 ? 127 : X);
}

// MXFP8 quantisation of one 32-element BF16 block held as four 16-byte
// vectors (64 contiguous bytes): the same rule as quant_block32_f32.  amax is
// reduced on the 15 magnitude bits, two values per SIMD max; a pattern >=
// 0x7f80 is Inf or NaN (scale 0xFF, elements 0x7F).  The 32 E4M3 bytes go to
// out0 (elements 0..15) and out1 (16..31); returns the scale byte.
__device__ __forceinline__ uint32_t quant_block32_bf16(const uint4 (&v)[4], uint4& out0, uint4& out1) {
  uint32_t m2 = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    m2 = __vmaxu2(m2, v[j].x & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v[j].y & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v[j].z & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v[j].w & 0x7FFF7FFFu);
  }
  const uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
  if (m >= 0x7F80u) {
    out0 = out1 = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    return 0xFFu;
  }
  const int X = bf16_block_exponent(m);
  const float mult = __uint_as_float(static_cast<uint32_t>(127 - X) << 23);  // 2^-X
  uint32_t o[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    o[2 * j] = e4m3x4(bf16_lo(v[j].x) * mult, bf16_hi(v[j].x) * mult, bf16_lo(v[j].y) * mult,
                      bf16_hi(v[j].y) * mult);
    o[2 * j + 1] = e4m3x4(bf16_lo(v[j].z) * mult, bf16_hi(v[j].z) * mult, bf16_lo(v[j].w) * mult,
                          bf16_hi(v[j].w) * mult);
  }
  out0 = make_uint4(o[0], o[1], o[2], o[3]);
  out1 = make_uint4(o[4], o[5], o[6], o[7]);
  return static_cast<uint32_t>(X + 127);
}

// Byte offset of scale (row r, K-block c) in the tiled scale layout: 128-row x
// 4-block tiles of 512 bytes, ordered (r/128, c/4), byte (r%32)*16 +
// ((r%128)/32)*4 + c%4 inside a tile; sf_ktiles = ceil(kb/4).
__device__ __forceinline__ uint32_t sf_tiled_offset(uint32_t r, uint32_t c, uint32_t sf_ktiles) {
  return ((r >> 7) * sf_ktiles + (c >> 2)) * 512u + (r & 31u) * 16u + ((r & 127u) >> 5) * 4u + (c & 3u);
}

}  // namespace mxk
