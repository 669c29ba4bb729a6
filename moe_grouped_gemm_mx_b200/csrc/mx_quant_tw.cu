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
//  * rows kernel (activations, [rows, k], scales [k/128, rows]): a half-warp
//    per 1 x 128 tile (16 bytes per lane), 8 tiles per warp with every load in
//    flight before the arithmetic; HBM-bound.
//  * blocks kernel (weights, [rows, k], scales [ceil(rows/128), k/128]): one
//    256-thread CTA per 128 x 128 block, a half-warp per row segment, 64
//    elements per thread held in registers across the block-wide amax
//    reduction.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mx_launch.h"
#include "mx_mxfp8.cuh"

namespace mxk {

constexpr uint32_t kTwNaN = 0x7FC00000u;  // the quiet NaN written as the scale of a non-finite tile

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

// Activations: a half-warp (16 lanes x 16 bytes) holds one 1 x 128 tile; a
// warp takes 8 tiles, all loads issued before any arithmetic (2 KiB in flight
// per warp).  Tiles are numbered with the row fastest, so a warp's scale
// stores are consecutive.
__global__ void __launch_bounds__(256) tw_quant_rows_kernel(const uint4* __restrict__ x, uint2* __restrict__ q,
                                                             float* __restrict__ s, int rows, int ktiles) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;
  const int hl = lane & 15;
  const int64_t units = static_cast<int64_t>(rows) * ktiles;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int64_t k8 = static_cast<int64_t>(ktiles) * 16;  // row length in 8-element units
  uint4 v[4];
  int64_t idx[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t u = w * 8 + j * 2 + half;
    idx[j] = -1;
    v[j] = make_uint4(0, 0, 0, 0);
    if (u < units) {
      const int64_t row = u % rows, kt = u / rows;
      idx[j] = row * k8 + kt * 16 + hl;
      v[j] = x[idx[j]];
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t w4[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m = max(m, (w4[i] << 16) & 0x7FFFFFFFu);
      m = max(m, w4[i] & 0x7FFF0000u);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));  // within the half-warp
    const int64_t u = w * 8 + j * 2 + half;
    if (idx[j] < 0) continue;
    const bool nonfinite = m >= 0x7F800000u;
    const float sc = nonfinite ? __uint_as_float(kTwNaN) : (m == 0 ? 1.0f : __fdiv_rn(__uint_as_float(m), 448.0f));
    uint2 o = make_uint2(0x7F7F7F7Fu, 0x7F7F7F7Fu);
    if (!nonfinite) {
      float f[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[2 * i] = __fdiv_rn(bf16_bits_to_f32(w4[i] & 0xFFFFu), sc);
        f[2 * i + 1] = __fdiv_rn(bf16_bits_to_f32(w4[i] >> 16), sc);
      }
      o.x = e4m3x4(f[0], f[1], f[2], f[3]);
      o.y = e4m3x4(f[4], f[5], f[6], f[7]);
    }
    q[idx[j]] = o;
    if (hl == 0) s[u] = sc;  // scales are [k/128, rows]: index kt * rows + row == u
  }
}

// Weights: one 256-thread CTA per 128 x 128 block; a half-warp reads one row's
// 256 contiguous bytes per load, a warp 16 rows (8 loads per thread, all in
// flight); block-wide amax through shared memory.
__global__ void __launch_bounds__(256) tw_quant_blocks_kernel(const uint4* __restrict__ x, uint2* __restrict__ q,
                                                               float* __restrict__ s, int rows, int ktiles) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ uint32_t warp_max[8];
  const int kt = blockIdx.x % ktiles;
  const int rb = blockIdx.x / ktiles;
  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  const int hl = lane & 15;
  const int64_t k8 = static_cast<int64_t>(ktiles) * 16;  // row length in 8-element units
  uint4 v[8];
  int64_t idx[8];
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = rb * 128 + warp * 16 + i * 2 + (lane >> 4);
    idx[i] = -1;
    v[i] = make_uint4(0, 0, 0, 0);
    if (r < rows) {
      idx[i] = static_cast<int64_t>(r) * k8 + kt * 16 + hl;
      v[i] = x[idx[i]];
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      m = max(m, (w4[j] << 16) & 0x7FFFFFFFu);
      m = max(m, w4[j] & 0x7FFF0000u);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (lane == 0) warp_max[warp] = m;
  __syncthreads();
  m = warp_max[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = max(m, warp_max[i]);
  const bool nonfinite = m >= 0x7F800000u;
  const float sc = nonfinite ? __uint_as_float(kTwNaN) : (m == 0 ? 1.0f : __fdiv_rn(__uint_as_float(m), 448.0f));
  if (t == 0) s[static_cast<int64_t>(rb) * ktiles + kt] = sc;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (idx[i] < 0) continue;
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
    q[idx[i]] = o;  // 8 elements -> 8 bytes at the same unit index
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
    const int64_t warps = (rows * static_cast<int64_t>(kt) + 7) / 8;  // 8 tiles per warp
    const int64_t grid = (warps + 7) / 8;
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const uint4* xp = static_cast<const uint4*>(x);
    uint2* qp = static_cast<uint2*>(q);
    void* args[] = {&xp, &qp, &s, &r, &kt};
    e = launch_pdl(reinterpret_cast<const void*>(tw_quant_rows_kernel), dim3(static_cast<unsigned>(grid)), dim3(256),
                   args, stream);
  } else {
    const int64_t grid = ((rows + 127) / 128) * kt;
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const uint4* xp = static_cast<const uint4*>(x);
    uint2* qp = static_cast<uint2*>(q);
    void* args[] = {&xp, &qp, &s, &r, &kt};
    e = launch_pdl(reinterpret_cast<const void*>(tw_quant_blocks_kernel), dim3(static_cast<unsigned>(grid)), dim3(256),
                   args, stream);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mxk
