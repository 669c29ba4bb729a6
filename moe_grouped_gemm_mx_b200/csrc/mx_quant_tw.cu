// mx_quant_tw.cu -- BF16 -> tile-wise FP32-scaled FP8 (the FP8 format with
// fine-grained FP32 scales that DeepGEMM's GEMMs take: the pages speak of
// "tile-wise" scaling in the FP8 mixed-precision recipe and of DeepGEMM's FP32
// two-level accumulation; the tiles are DeepSeek-V3's 1 x 128 for activations
// and 128 x 128 for weights).
//
// One FP32 scale per tile: s = amax / 448 (IEEE FP32 division; 448 = largest
// E4M3 value), each element x / s (IEEE FP32 division) encoded as E4M3 with
// saturating round-to-nearest-even.  An all-zero tile gets s = 1; a tile
// holding NaN or +-Inf gets s = NaN and every element 0x7F.  The scale is a
// correctly rounded division (__fdiv_rn); each element's quotient is the
// correctly rounded x / s as well, found with one multiply and two FMAs
// (tw_quot below), so the results are exactly those of the definition.
//
//  * rows kernel (activations, [rows, k], scales [k/128, rows]): a warp takes
//    one 128-column tile position of 8 consecutive rows, 4 lanes per 1 x 128
//    tile (32 elements, four 16-byte loads per lane, all in flight before the
//    arithmetic); HBM-bound.
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

// The correctly rounded FP32 quotient x / sc without a division, for x a
// BF16 value and sc = RN(amax / 448) a scale of a tile of BF16 values, with
// r = RN(1 / sc) and sc >= 2^-64.
//
// q0 = RN(x * r) is within a few ulp of x / sc; its residual
// t = RN(q0 * sc - x) is one FMA, and q = RN(q0 - t * r) is one more -- the
// correction step of FMA-based division.  That q equals RN(x / sc) was
// checked exhaustively: a BF16 x has one of 128 significands, and so does
// sc (RN(amax / 448) depends only on amax's significand while it is a
// normal number), and the three roundings scale exactly with the operands'
// exponents while the residual stays a normal number, which sc >= 2^-64
// ensures for every quotient of magnitude 2^-11 or more (smaller ones,
// including BF16 subnormal x, encode as zero however they round).  Signs
// come out right as well, -0 included: t is +0 for x = +-0 and
// RN(-0 * r + q0) keeps q0's zero.
__device__ __forceinline__ float tw_quot(float x, float sc, float r) {
  const float q0 = x * r;
  const float t = fmaf(q0, sc, -x);
  return fmaf(-t, r, q0);
}

// The eight codes of one 16-byte unit (eight BF16 values, lowest address
// first) of a finite tile with scale sc and r = RN(1 / sc).  A tile with a
// scale below 2^-64 (amax below 448 * 2^-64) has each element divided.
__device__ __forceinline__ uint2 tw_codes8(const uint4& v, float sc, float r) {
  const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
  float f[8];
  if (__float_as_uint(sc) >= 0x1F800000u) {  // sc >= 2^-64
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = tw_quot(bf16_bits_to_f32(w4[i] & 0xFFFFu), sc, r);
      f[2 * i + 1] = tw_quot(__uint_as_float(w4[i] & 0xFFFF0000u), sc, r);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __fdiv_rn(bf16_bits_to_f32(w4[i] & 0xFFFFu), sc);
      f[2 * i + 1] = __fdiv_rn(__uint_as_float(w4[i] & 0xFFFF0000u), sc);
    }
  }
  return make_uint2(e4m3x4(f[0], f[1], f[2], f[3]), e4m3x4(f[4], f[5], f[6], f[7]));
}

// Lane-wise maximum of two pairs of 16-bit unsigned integers.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Largest BF16 magnitude pattern among the eight values of a unit, folded
// into m2 (two 16-bit lanes).  For non-negative IEEE patterns integer order
// is value order and every pattern >= 0x7F80 is Inf/NaN, so the same
// maximum detects a non-finite tile.
__device__ __forceinline__ uint32_t fold_amax(uint32_t m2, const uint4& v) {
  m2 = max_u16x2(m2, v.x & 0x7FFF7FFFu);
  m2 = max_u16x2(m2, v.y & 0x7FFF7FFFu);
  m2 = max_u16x2(m2, v.z & 0x7FFF7FFFu);
  return max_u16x2(m2, v.w & 0x7FFF7FFFu);
}

// The tile's scale from its largest magnitude (as FP32 bits).
__device__ __forceinline__ float tw_scale(uint32_t m) {
  return m >= 0x7F800000u ? __uint_as_float(kTwNaN) : (m == 0 ? 1.0f : __fdiv_rn(__uint_as_float(m), 448.0f));
}

// Activations: warp item w covers the 1 x 128 tiles at column block kt of
// rows 8 * rg .. 8 * rg + 7 (items numbered with rg fastest, so a warp's 8
// scales are consecutive in the [k/128, rows] layout).  Lane l owns row
// 8 * rg + l / 4 and the 16-byte chunks l % 4 + 4 i (i < 4) of its tile: each
// load instruction reads 64 contiguous bytes of each of the 8 rows.
__global__ void __launch_bounds__(256) tw_quant_rows_kernel(const uint4* __restrict__ x, uint2* __restrict__ q,
                                                             float* __restrict__ s, int rows, int ktiles) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const uint32_t rgroups = (static_cast<uint32_t>(rows) + 7u) / 8u;
  const uint32_t w = blockIdx.x * 8u + (threadIdx.x >> 5);
  if (w >= rgroups * static_cast<uint32_t>(ktiles)) return;  // the whole warp
  const uint32_t kt = w / rgroups, rg = w - kt * rgroups;
  const int64_t k16 = static_cast<int64_t>(ktiles) * 16;  // row length in 16-byte units
  const int row = static_cast<int>(rg * 8u) + (lane >> 2);
  const bool live = row < rows;
  const int64_t base = static_cast<int64_t>(row) * k16 + kt * 16u + (lane & 3);
  uint4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = live ? x[base + 4 * i] : make_uint4(0, 0, 0, 0);
  uint32_t m2 = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) m2 = fold_amax(m2, v[i]);
  m2 = max_u16x2(m2, __shfl_xor_sync(0xFFFFFFFFu, m2, 1));  // the tile's 4 lanes
  m2 = max_u16x2(m2, __shfl_xor_sync(0xFFFFFFFFu, m2, 2));
  if (!live) return;
  const uint32_t m = max(m2 & 0xFFFFu, m2 >> 16) << 16;
  const float sc = tw_scale(m);
  if ((lane & 3) == 0) s[static_cast<int64_t>(kt) * rows + row] = sc;
  const bool nonfinite = m >= 0x7F800000u;
  const float r = __frcp_rn(sc);
#pragma unroll
  for (int i = 0; i < 4; ++i) q[base + 4 * i] = nonfinite ? make_uint2(0x7F7F7F7Fu, 0x7F7F7F7Fu) : tw_codes8(v[i], sc, r);
}

// Weights: one 256-thread CTA per 128 x 128 block; a half-warp reads one row's
// 256 contiguous bytes per load, a warp 16 rows (8 loads per thread, all in
// flight); block-wide amax through shared memory.  At 62 registers four CTAs
// fit on an SM (three of the 512-thread form did), which shortens the last
// partial wave of the small weight tensors.
__global__ void __launch_bounds__(256, 4) tw_quant_blocks_kernel(const uint4* __restrict__ x, uint2* __restrict__ q,
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
  const int r0 = rb * 128 + warp * 16 + (lane >> 4);  // this thread's rows: r0, r0 + 2, ..., r0 + 14
  const int64_t base = static_cast<int64_t>(r0) * k8 + kt * 16 + hl;
  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = r0 + 2 * i < rows ? x[base + 2 * i * k8] : make_uint4(0, 0, 0, 0);
  uint32_t m2 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) m2 = fold_amax(m2, v[i]);
  uint32_t m = max(m2 & 0xFFFFu, m2 >> 16) << 16;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (lane == 0) warp_max[warp] = m;
  __syncthreads();
  m = warp_max[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = max(m, warp_max[i]);
  const bool nonfinite = m >= 0x7F800000u;
  const float sc = tw_scale(m);
  if (t == 0) s[static_cast<int64_t>(rb) * ktiles + kt] = sc;
  const float r = __frcp_rn(sc);
#pragma unroll
  for (int i = 0; i < 8; ++i)  // 8 elements -> 8 bytes at the same unit index
    if (r0 + 2 * i < rows) q[base + 2 * i * k8] = nonfinite ? make_uint2(0x7F7F7F7Fu, 0x7F7F7F7Fu) : tw_codes8(v[i], sc, r);
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
    const int64_t items = ((rows + 7) / 8) * static_cast<int64_t>(kt);  // one per warp: 8 rows of one column block
    const int64_t grid = (items + 7) / 8;
    if (items > 0xFFFFFFF0LL || grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
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
