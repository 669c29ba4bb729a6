// mx_quant.cu -- BF16 -> MXFP8 (E4M3 elements + UE8M0 block scales) on sm_100a.
//
// The format is the 32-element microscaling FP8 of the B200 MoE-training page
// ("PyTorch and Nebius optimise DeepSeek-V3 MoE training on B200 clusters",
// glossary entry on MXFP8 and the OCP Microscaling specification it cites);
// the quantise step is the first box of that page's MXFP8 pipeline diagram.
//
// Kernel design (HBM-bound: 2 B read, 1 + 1/32 B written per element):
//  * The [rows, K] source is contiguous, so 32-element block b is the 64-byte
//    chunk at byte 64*b regardless of row boundaries.  Four lanes own one
//    block (16 B each); a warp covers 8 consecutive blocks = 512 contiguous
//    bytes, and each thread keeps U such 16-byte loads in flight.
//  * amax is reduced on the integer magnitude bits (bits & 0x7fff) with two
//    xor-shuffles; for non-negative IEEE values integer order is value order,
//    and any pattern >= 0x7f80 is Inf/NaN, so a non-finite block is detected
//    by the same max (an fmaxf reduction would silently drop NaN).
//  * floor(log2 amax) comes from the exponent field (normal) or the position
//    of the top mantissa bit (subnormal); no log2f.
//  * Elements are scaled by the exact power of two 2^-X in fp32 and converted
//    with the hardware's saturating round-to-nearest-even cvt (e4m3x2).
//  * Four consecutive blocks of a row (K-block c..c+3, c % 4 == 0) land in 4
//    consecutive scale bytes, so their scales are gathered into one 32-bit
//    store when K/32 is a multiple of 4.
//  * Extra CTAs beyond the streaming grid write 0x00 into the scale-tile
//    padding (rows up to a multiple of 128, K-blocks up to a multiple of 4).
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mx_launch.h"

namespace mxk {

constexpr int kQuantThreads = 256;
constexpr int kQuantUnroll = 4;  // 16-byte loads in flight per thread

struct QuantArgs {
  const uint4* x;          // BF16 source viewed as 16-byte vectors
  uint2* q;                // E4M3 output viewed as 8-byte vectors
  uint8_t* sf;             // tiled scale output
  int64_t nblk;            // total 32-element blocks = groups*rows*kb
  int64_t kb;              // blocks per row = k/32
  int64_t rows;            // rows per group
  int64_t groups;
  int64_t sf_group_bytes;  // tiled scale bytes per group
  int64_t sf_ktiles;       // ceil(kb/4): 512-byte tiles along K
  int main_blocks;         // CTAs that stream blocks; the rest write padding
  int kb4;                 // kb % 4 == 0
};

__device__ __forceinline__ int64_t sf_tiled_offset(int64_t r, int64_t c, int64_t sf_ktiles) {
  return ((r >> 7) * sf_ktiles + (c >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3);
}

// Scale exponent X for a block whose largest magnitude has BF16 bits `amax_bits`
// (finite).  X = floor(log2 amax) - 8, clamped to [-127, 127]; amax == 0 -> -127.
__device__ __forceinline__ int block_exponent(uint32_t amax_bits) {
  if (amax_bits == 0) return -127;
  const int e = static_cast<int>(amax_bits >> 7);
  int fl;
  if (e > 0) {
    fl = e - 127;
  } else {
    const uint32_t m = amax_bits & 0x7Fu;  // subnormal: value = m * 2^-133
    fl = (31 - __clz(m)) - 133;
  }
  int X = fl - 8;
  return X < -127 ? -127 : (X > 127 ? 127 : X);
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t max_mag(uint32_t w) {
  return max(w & 0x7FFFu, (w >> 16) & 0x7FFFu);
}

__global__ void __launch_bounds__(kQuantThreads) mx_quant_kernel(const QuantArgs a) {
  if (static_cast<int>(blockIdx.x) >= a.main_blocks) {
    // ---- padding of the scale tiles: rows [rows, rpad) x all kb_pad, and
    // rows [0, rows) x blocks [kb, kb_pad), for every group.
    const int64_t kbpad = a.sf_ktiles * 4;
    const int64_t rpad = (a.rows + 127) / 128 * 128;
    const int64_t n1 = (rpad - a.rows) * kbpad;
    const int64_t n2 = a.rows * (kbpad - a.kb);
    const int64_t per_group = n1 + n2;
    const int64_t total = per_group * a.groups;
    const int64_t stride = static_cast<int64_t>(gridDim.x - a.main_blocks) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x - a.main_blocks) * blockDim.x + threadIdx.x;
         i < total; i += stride) {
      const int64_t g = i / per_group;
      const int64_t j = i - g * per_group;
      int64_t r, c;
      if (j < n1) {
        r = a.rows + j / kbpad;
        c = j % kbpad;
      } else {
        const int64_t jj = j - n1;
        const int64_t w = kbpad - a.kb;
        r = jj / w;
        c = a.kb + jj % w;
      }
      a.sf[g * a.sf_group_bytes + sf_tiled_offset(r, c, a.sf_ktiles)] = 0;
    }
    return;
  }

  const int lane = threadIdx.x & 31;
  const int sub = lane & 3;   // which 16-byte quarter of the block
  const int blk = lane >> 2;  // which of the warp's 8 blocks
  const int64_t warp_id = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(a.main_blocks) * blockDim.x) >> 5;
  constexpr int kWarpBlocks = 8 * kQuantUnroll;

  for (int64_t base = warp_id * kWarpBlocks; base < a.nblk; base += nwarps * kWarpBlocks) {
    uint4 v[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int64_t b = base + u * 8 + blk;
      v[u] = b < a.nblk ? __ldcs(a.x + b * 4 + sub) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int64_t b = base + u * 8 + blk;
      uint32_t m = max(max(max_mag(v[u].x), max_mag(v[u].y)), max(max_mag(v[u].z), max_mag(v[u].w)));
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      uint32_t scode;
      uint2 out;
      if (m >= 0x7F80u) {  // Inf or NaN somewhere in the block
        scode = 0xFFu;
        out = make_uint2(0x7F7F7F7Fu, 0x7F7F7F7Fu);
      } else {
        const int X = block_exponent(m);
        scode = static_cast<uint32_t>(X + 127);
        const float mult = __uint_as_float(static_cast<uint32_t>(127 - X) << 23);  // 2^-X
        out.x = pack_e4m3x4(bf16_lo(v[u].x) * mult, bf16_hi(v[u].x) * mult,
                            bf16_lo(v[u].y) * mult, bf16_hi(v[u].y) * mult);
        out.y = pack_e4m3x4(bf16_lo(v[u].z) * mult, bf16_hi(v[u].z) * mult,
                            bf16_lo(v[u].w) * mult, bf16_hi(v[u].w) * mult);
      }
      if (b < a.nblk) __stcs(a.q + b * 4 + sub, out);

      // scale byte(s)
      const int64_t row = b / a.kb;
      const int64_t c = b - row * a.kb;
      const int64_t g = row / a.rows;
      const int64_t rl = row - g * a.rows;
      if (a.kb4) {
        // lanes 0 and 16 each store the 4 scales of blocks blk..blk+3 (one row,
        // K-blocks c..c+3 with c % 4 == 0).
        const int src = lane & 16;
        const uint32_t s0 = __shfl_sync(0xFFFFFFFFu, scode, src + 0);
        const uint32_t s1 = __shfl_sync(0xFFFFFFFFu, scode, src + 4);
        const uint32_t s2 = __shfl_sync(0xFFFFFFFFu, scode, src + 8);
        const uint32_t s3 = __shfl_sync(0xFFFFFFFFu, scode, src + 12);
        if ((lane & 15) == 0 && b < a.nblk) {
          *reinterpret_cast<uint32_t*>(a.sf + g * a.sf_group_bytes + sf_tiled_offset(rl, c, a.sf_ktiles)) =
              s0 | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }
      } else if (sub == 0 && b < a.nblk) {
        a.sf[g * a.sf_group_bytes + sf_tiled_offset(rl, c, a.sf_ktiles)] = static_cast<uint8_t>(scode);
      }
    }
  }
}

// Launch helper used by the C ABI (validation happens there).
cudaError_t launch_quant(const void* x, int64_t groups, int64_t rows, int64_t k, void* q, void* sf,
                         int64_t sf_group_bytes, int num_sms, cudaStream_t stream, int* launches) {
  QuantArgs a;
  a.x = static_cast<const uint4*>(x);
  a.q = static_cast<uint2*>(q);
  a.sf = static_cast<uint8_t*>(sf);
  a.kb = k / 32;
  a.rows = rows;
  a.groups = groups;
  a.nblk = groups * rows * a.kb;
  a.sf_group_bytes = sf_group_bytes;
  a.sf_ktiles = (a.kb + 3) / 4;
  a.kb4 = (a.kb % 4) == 0;
  const int64_t warps_needed = (a.nblk + 8 * kQuantUnroll - 1) / (8 * kQuantUnroll);
  const int64_t ctas_needed = (warps_needed + (kQuantThreads / 32) - 1) / (kQuantThreads / 32);
  const int64_t max_ctas = static_cast<int64_t>(num_sms) * (2048 / kQuantThreads);
  a.main_blocks = static_cast<int>(ctas_needed < max_ctas ? ctas_needed : max_ctas);
  const int64_t kbpad = a.sf_ktiles * 4;
  const int64_t rpad = (rows + 127) / 128 * 128;
  const int64_t pad_entries = ((rpad - rows) * kbpad + rows * (kbpad - a.kb)) * groups;
  int pad_blocks = 0;
  if (pad_entries > 0) {
    const int64_t want = (pad_entries + kQuantThreads - 1) / kQuantThreads;
    pad_blocks = static_cast<int>(want < num_sms ? want : num_sms);
  }
  const int grid = a.main_blocks + pad_blocks;
  if (grid == 0) return cudaSuccess;
  mx_quant_kernel<<<grid, kQuantThreads, 0, stream>>>(a);
  if (launches) *launches += 1;
  return cudaGetLastError();
}

}  // namespace mxk
