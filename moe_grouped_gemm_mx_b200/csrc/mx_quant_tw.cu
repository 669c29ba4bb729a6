// mx_quant_tw.cu -- BF16 -> tile-wise FP32-scaled FP8 (the FP8 format with
// fine-grained FP32 scales that DeepGEMM's GEMMs take: the pages speak of
// "tile-wise" scaling in the FP8 mixed-precision recipe and of DeepGEMM's FP32
// two-level accumulation; the tiles are DeepSeek-V3's 1 x 128 for activations
// and 128 x 128 for weights).
//
// One FP32 scale per tile: s = amax / 448 (IEEE FP32 division; 448 = largest
// E4M3 value), each element x / s (IEEE FP32 division) encoded as E4M3 with
// saturating round-to-nearest-even.  An all-zero tile gets s = 1; a tile
// holding NaN or +-Inf gets s = NaN and every element 0x7F.  Both divisions
// are correctly rounded (__fdiv_rn), so the results are exactly those of the
// definition.
//
//  * rows kernel (activations, [rows, k], scales [k/128, rows]): one warp per
//    (row, 128-element K tile), 8 bytes (4 BF16) per lane, a warp max
//    reduction for amax; HBM-bound.
//  * blocks kernel (weights, [rows, k], scales [ceil(rows/128), k/128]): one
//    256-thread CTA per 128 x 128 block, 64 elements per thread held in
//    registers across the block-wide amax reduction.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mx_launch.h"
#include "mx_mxfp8.cuh"

namespace mxk {

constexpr uint32_t kTwNaN = 0x7FC00000u;  // the quiet NaN written as the scale of a non-finite tile

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

__global__ void __launch_bounds__(256) tw_quant_rows_kernel(const uint2* __restrict__ x, uint32_t* __restrict__ q,
                                                             float* __restrict__ s, int rows, int ktiles) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);  // (tile, row), row fastest
  if (w >= static_cast<int64_t>(rows) * ktiles) return;
  const int row = static_cast<int>(w % rows);
  const int kt = static_cast<int>(w / rows);
  const int64_t k4 = static_cast<int64_t>(ktiles) * 32;  // row length in 4-element units
  const uint2 v = x[row * k4 + kt * 32 + lane];
  float f[4] = {bf16_bits_to_f32(v.x & 0xFFFFu), bf16_bits_to_f32(v.x >> 16), bf16_bits_to_f32(v.y & 0xFFFFu),
                bf16_bits_to_f32(v.y >> 16)};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = max(m, __float_as_uint(f[i]) & 0x7FFFFFFFu);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  uint32_t out;
  float sc;
  if (m >= 0x7F800000u) {
    sc = __uint_as_float(kTwNaN);
    out = 0x7F7F7F7Fu;
  } else {
    sc = m == 0 ? 1.0f : __fdiv_rn(__uint_as_float(m), 448.0f);
    out = e4m3x4(__fdiv_rn(f[0], sc), __fdiv_rn(f[1], sc), __fdiv_rn(f[2], sc), __fdiv_rn(f[3], sc));
  }
  q[row * k4 + kt * 32 + lane] = out;
  if (lane == 0) s[static_cast<int64_t>(kt) * rows + row] = sc;
}

__global__ void __launch_bounds__(256) tw_quant_blocks_kernel(const uint4* __restrict__ x, uint4* __restrict__ q,
                                                               float* __restrict__ s, int rows, int ktiles) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ uint32_t warp_max[8];
  const int kt = blockIdx.x % ktiles;
  const int rb = blockIdx.x / ktiles;
  const int t = threadIdx.x;
  const int r = rb * 128 + (t >> 1);   // this thread's row
  const int half = t & 1;              // which 64 columns of the tile's 128
  const bool valid = r < rows;
  const int64_t k16 = static_cast<int64_t>(ktiles) * 16;  // row length in 16-byte (8-element) units
  const int64_t base = static_cast<int64_t>(r) * k16 + kt * 16 + half * 8;
  uint4 v[8];
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = valid ? x[base + i] : make_uint4(0, 0, 0, 0);
    const uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      m = max(m, (w4[j] << 16) & 0x7FFFFFFFu);
      m = max(m, (w4[j] & 0xFFFF0000u) & 0x7FFFFFFFu);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((t & 31) == 0) warp_max[t >> 5] = m;
  __syncthreads();
  m = warp_max[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = max(m, warp_max[i]);
  const bool nonfinite = m >= 0x7F800000u;
  const float sc = nonfinite ? __uint_as_float(kTwNaN) : (m == 0 ? 1.0f : __fdiv_rn(__uint_as_float(m), 448.0f));
  if (t == 0) s[static_cast<int64_t>(rb) * ktiles + kt] = sc;
  if (!valid) return;
  // input unit i (8 BF16, 16 bytes) becomes 8 output bytes at the same unit
  // index of the byte tensor viewed as 8-byte units
  uint2* q8 = reinterpret_cast<uint2*>(q);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint2 o = make_uint2(0x7F7F7F7Fu, 0x7F7F7F7Fu);
    if (!nonfinite) {
      const uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      float f[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        f[2 * j] = __fdiv_rn(bf16_bits_to_f32(w4[j] & 0xFFFFu), sc);
        f[2 * j + 1] = __fdiv_rn(bf16_bits_to_f32(w4[j] >> 16), sc);
      }
      o.x = e4m3x4(f[0], f[1], f[2], f[3]);
      o.y = e4m3x4(f[4], f[5], f[6], f[7]);
    }
    q8[base + i] = o;
  }
}

static cudaError_t launch_pdl(const void* func, dim3 grid, dim3 block, void** args, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, func, args);
}

cudaError_t launch_tw_quant(const void* x, int64_t rows, int64_t k, void* q, float* s, bool blocks,
                            cudaStream_t stream) {
  int r = static_cast<int>(rows), kt = static_cast<int>(k / 128);
  if (rows == 0 || kt == 0) return cudaSuccess;
  cudaError_t e;
  if (!blocks) {
    const int64_t warps = rows * static_cast<int64_t>(kt);
    const int64_t grid = (warps + 7) / 8;
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const uint2* xp = static_cast<const uint2*>(x);
    uint32_t* qp = static_cast<uint32_t*>(q);
    void* args[] = {&xp, &qp, &s, &r, &kt};
    e = launch_pdl(reinterpret_cast<const void*>(tw_quant_rows_kernel), dim3(static_cast<unsigned>(grid)), dim3(256),
                   args, stream);
  } else {
    const int64_t grid = ((rows + 127) / 128) * kt;
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const uint4* xp = static_cast<const uint4*>(x);
    uint4* qp = static_cast<uint4*>(q);
    void* args[] = {&xp, &qp, &s, &r, &kt};
    e = launch_pdl(reinterpret_cast<const void*>(tw_quant_blocks_kernel), dim3(static_cast<unsigned>(grid)), dim3(256),
                   args, stream);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mxk
