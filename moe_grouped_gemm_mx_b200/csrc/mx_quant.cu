// mx_quant.cu -- BF16 -> MXFP8 (E4M3 elements + UE8M0 block scales) on sm_100a.
//
// The format is the 32-element microscaling FP8 of the B200 MoE-training page
// ("PyTorch and Nebius optimise DeepSeek-V3 MoE training on B200 clusters",
// glossary entry on MXFP8 and the OCP Microscaling specification it cites);
// the quantise step is the first box of that page's MXFP8 pipeline diagram.
//
// Kernel design (HBM-bound: 2 B read, 1 + 1/32 B written per element):
//  * The [rows, K] source is contiguous, so 32-element block b is the 64-byte
//    chunk at byte 64*b regardless of row boundaries.  A warp loads 32
//    consecutive blocks (2 KiB) with four coalesced 16-byte loads per lane,
//    staged through swizzled shared memory; then one lane owns one block.  One lane per block keeps
//    the per-element instruction count low: amax, exponent and the scale
//    address are computed once per 32 elements.
//  * amax is reduced on the integer magnitude bits (bits & 0x7fff, two BF16
//    values per 32-bit SIMD max); for non-negative IEEE patterns integer
//    order is value order, and any pattern >= 0x7f80 is Inf/NaN, so a
//    non-finite block is detected by the same max (an fmaxf reduction would
//    silently drop NaN).
//  * floor(log2 amax) comes from the exponent field (normal) or the position
//    of the top mantissa bit (subnormal); no log2f.
//  * Elements are scaled by the exact power of two 2^-X in fp32 and converted
//    with the hardware's saturating round-to-nearest-even cvt (e4m3x2).
//  * Four consecutive blocks of a row (K-block c..c+3, c % 4 == 0) land in 4
//    consecutive scale bytes, so their scales are gathered into one 32-bit
//    store when K/32 is a multiple of 4.  Row / K-block / group indices use
//    32-bit division by launch-time constants (multiply-high and shift).
//  * Extra CTAs beyond the streaming grid write 0x00 into the scale-tile
//    padding (rows up to a multiple of 128, K-blocks up to a multiple of 4).
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mx_fastdiv.h"
#include "mx_launch.h"
#include "mx_mxfp8.cuh"

namespace mxk {

constexpr int kQuantThreads = 256;
// 32-element blocks per lane per loop trip: one (4 x 16 B loads in flight per
// lane, 48 registers, 5 CTAs per SM) streamed 3-5 % faster than two (64
// registers, 4 CTAs per SM) on every workload measured
constexpr int kQuantUnroll = 1;
constexpr uint32_t kSlotBlocks = 32 * kQuantUnroll;  // blocks one warp handles per loop trip

// One tensor to quantise.  Several are processed by one launch: their block
// ranges are laid end to end in "slots" of kSlotBlocks blocks (each job
// starts on a slot boundary, so a warp's slot never spans two jobs).
struct QuantJob {
  const uint4* x;          // BF16 source viewed as 16-byte vectors
  uint4* q;                // E4M3 output viewed as 16-byte vectors
  uint8_t* sf;             // tiled scale output
  uint32_t nblk;           // 32-element blocks = groups*rows*kb (< 2^31)
  uint32_t kb;             // blocks per row = k/32
  uint32_t rows;           // rows per group
  uint32_t groups;
  FastDiv div_kb;          // divide by kb
  FastDiv div_rows;        // divide by rows
  int64_t sf_group_bytes;  // tiled scale bytes per group
  uint32_t sf_ktiles;      // ceil(kb/4): 512-byte tiles along K
  uint32_t kb4;            // kb % 4 == 0
  uint32_t slot0;          // first slot of this job
  int64_t pad0;            // first scale-padding entry of this job
  int64_t pad_n1;          // per group: padding entries in rows [rows, rpad)
  int64_t pad_per_group;   // per group: all padding entries
};

struct QuantBatch {
  QuantJob job[kMaxQuantJobs];
  int count;
  uint32_t total_slots;
  int main_blocks;         // CTAs that stream blocks; the rest write padding
  int64_t pad_total;
};

// Scale-tile padding entry i of one job: rows [rows, rpad) x all kb_pad
// blocks, then rows [0, rows) x blocks [kb, kb_pad), for every group.
__device__ void write_padding(const QuantJob& jb, int64_t i) {
  const int64_t kbpad = static_cast<int64_t>(jb.sf_ktiles) * 4;
  const int64_t g = i / jb.pad_per_group;
  const int64_t j = i - g * jb.pad_per_group;
  int64_t r, c;
  if (j < jb.pad_n1) {
    r = jb.rows + j / kbpad;
    c = j % kbpad;
  } else {
    const int64_t jj = j - jb.pad_n1;
    const int64_t w = kbpad - jb.kb;
    r = jj / w;
    c = jb.kb + jj % w;
  }
  jb.sf[g * jb.sf_group_bytes + sf_tiled_offset(static_cast<uint32_t>(r), static_cast<uint32_t>(c), jb.sf_ktiles)] = 0;
}

// KEEP: the outputs are written with ordinary (write-back) stores, so that
// they stay in L2 for the GEMM that reads them next; otherwise with
// streaming stores (evict-first), which are a little faster for outputs that
// would not fit in L2 anyway.  The BF16 input is always read streaming.
template <bool KEEP>
__device__ __forceinline__ void store_out(uint4* p, const uint4& v) {
  if constexpr (KEEP)
    *p = v;
  else
    __stcs(p, v);
}

// STAGED: the coalesced loads go through a per-warp shared-memory stage (the
// normal form).  Without it (the lean form) each lane loads its own block's
// four pieces straight from global memory: no shared memory at all, so one
// CTA of it fits on an SM beside a GEMM CTA that holds nearly all of the
// shared memory, and the quantisation runs underneath the GEMM.
template <bool KEEP, bool STAGED>
__global__ void __launch_bounds__(kQuantThreads) mx_quant_kernel(const __grid_constant__ QuantBatch B) {
  __shared__ uint4 quant_stage[STAGED ? (kQuantThreads / 32) * kQuantUnroll * 128 : 1];  // 2 KiB per warp and step
  // with programmatic dependent launch the next kernel may start its
  // prologue now; our own reads and writes wait for the previous kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (static_cast<int>(blockIdx.x) >= B.main_blocks) {
    const int64_t stride = static_cast<int64_t>(gridDim.x - B.main_blocks) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x - B.main_blocks) * blockDim.x + threadIdx.x; i < B.pad_total;
         i += stride) {
      int j = 0;
      while (j + 1 < B.count && i >= B.job[j + 1].pad0) ++j;
      write_padding(B.job[j], i - B.job[j].pad0);
    }
    return;
  }

  // ---- streaming part: one lane owns one 32-element block (64 contiguous
  // bytes: four 16-byte loads), so amax, exponent and scale bookkeeping are
  // done once per block with no shuffles; a warp covers 32 consecutive
  // blocks (2 KiB) per unrolled step.
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t warp_id = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (static_cast<uint32_t>(B.main_blocks) * blockDim.x) >> 5;

  for (uint32_t slot = warp_id; slot < B.total_slots; slot += nwarps) {
    int jn = 0;  // warp-uniform job of this slot
    while (jn + 1 < B.count && slot >= B.job[jn + 1].slot0) ++jn;
    const QuantJob& jb = B.job[jn];
    const uint32_t base = (slot - jb.slot0) * kSlotBlocks;

    uint4 v[kQuantUnroll][4];
    if constexpr (!STAGED) {  // lean form: each lane's own 64 bytes, four 16-byte loads
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u) {
        const uint32_t b = base + u * 32 + lane;
        const uint4* src = jb.x + static_cast<size_t>(b) * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) v[u][q] = b < jb.nblk ? __ldcs(src + q) : make_uint4(0, 0, 0, 0);
      }
    } else {
      // Coalesced loads: instruction j of step u brings the 16-byte piece
      // 32j + lane of the step's 2 KiB (512 contiguous bytes per instruction);
      // the pieces go through a per-warp shared-memory stage, swizzled (piece
      // p at slot p ^ ((p >> 3) & 7)) so that both the writes here and each
      // lane's read of its own block's four pieces below are free of bank
      // conflicts.
      uint4* stage = quant_stage + (threadIdx.x >> 5) * (kQuantUnroll * 128);
      {
        uint4 g[kQuantUnroll][4];
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
          const uint32_t b0 = base + u * 32;  // first block of the step
          const uint4* src = jb.x + static_cast<size_t>(b0) * 4;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t p = 32 * j + lane;  // piece p belongs to block b0 + p / 4
            g[u][j] = b0 + (p >> 2) < jb.nblk ? __ldcs(src + p) : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t p = 32 * j + lane;
            stage[u * 128 + (p ^ ((p >> 3) & 7u))] = g[u][j];
          }
      }
      __syncwarp();
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t p = 4 * lane + q;
          v[u][q] = stage[u * 128 + (p ^ ((p >> 3) & 7u))];
        }
      __syncwarp();  // the stage is rewritten by the warp's next slot
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const uint32_t b = base + u * 32 + lane;
      uint4 out0, out1;
      const uint32_t scode = quant_block32_bf16(v[u], out0, out1);
      // the warp's 32 blocks are 1 KB of contiguous output: rearrange it so
      // each store instruction writes 512 contiguous bytes (bytes
      // [16l, 16l + 16) of the first / second half are half l & 1 of block
      // l >> 1 / 16 + (l >> 1))
      {
        const int sa = lane >> 1, sb = 16 + (lane >> 1);
        const bool hi = lane & 1u;
        const uint4 x0 = make_uint4(__shfl_sync(0xFFFFFFFFu, out0.x, sa), __shfl_sync(0xFFFFFFFFu, out0.y, sa),
                                    __shfl_sync(0xFFFFFFFFu, out0.z, sa), __shfl_sync(0xFFFFFFFFu, out0.w, sa));
        const uint4 x1 = make_uint4(__shfl_sync(0xFFFFFFFFu, out1.x, sa), __shfl_sync(0xFFFFFFFFu, out1.y, sa),
                                    __shfl_sync(0xFFFFFFFFu, out1.z, sa), __shfl_sync(0xFFFFFFFFu, out1.w, sa));
        const uint4 y0 = make_uint4(__shfl_sync(0xFFFFFFFFu, out0.x, sb), __shfl_sync(0xFFFFFFFFu, out0.y, sb),
                                    __shfl_sync(0xFFFFFFFFu, out0.z, sb), __shfl_sync(0xFFFFFFFFu, out0.w, sb));
        const uint4 y1 = make_uint4(__shfl_sync(0xFFFFFFFFu, out1.x, sb), __shfl_sync(0xFFFFFFFFu, out1.y, sb),
                                    __shfl_sync(0xFFFFFFFFu, out1.z, sb), __shfl_sync(0xFFFFFFFFu, out1.w, sb));
        const uint32_t b0 = base + u * 32;
        uint4* dst = jb.q + static_cast<size_t>(b0) * 2;
        if (b0 + sa < jb.nblk) store_out<KEEP>(dst + lane, hi ? x1 : x0);
        if (b0 + sb < jb.nblk) store_out<KEEP>(dst + 32 + lane, hi ? y1 : y0);
      }

      // scale byte(s): row / K-block of this block, then its group
      const uint32_t row = fdiv(b, jb.div_kb);
      const uint32_t c = b - row * jb.kb;
      uint32_t g = 0, rl = row;
      if (jb.groups > 1) {
        g = fdiv(row, jb.div_rows);
        rl = row - g * jb.rows;
      }
      uint8_t* sfp = jb.sf + static_cast<int64_t>(g) * jb.sf_group_bytes + sf_tiled_offset(rl, c, jb.sf_ktiles);
      if (jb.kb4) {
        // lanes 4j..4j+3 hold K-blocks c..c+3 (c % 4 == 0) of one row: their
        // four scale bytes are adjacent, so lane 4j stores them as one word.
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, scode, 1);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, scode, 2);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, scode, 3);
        if ((lane & 3u) == 0 && b < jb.nblk)
          *reinterpret_cast<uint32_t*>(sfp) = scode | (s1 << 8) | (s2 << 16) | (s3 << 24);
      } else if (b < jb.nblk) {
        *sfp = static_cast<uint8_t>(scode);
      }
    }
  }
}

// Launch helper used by the C ABI (validation happens there): up to
// kMaxQuantJobs tensors in one launch.  Each job needs groups*rows*(k/32) < 2^31.
cudaError_t launch_quant_batch(const QuantSpec* specs, int count, int num_sms, cudaStream_t stream, int* launches,
                               bool lean) {
  static int resident = 0;  // CTAs of the kernel one SM holds
  static int64_t l2_bytes = 0;
  if (resident == 0) {
    cudaError_t e =
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, mx_quant_kernel<false, true>, kQuantThreads, 0);
    if (e != cudaSuccess || resident <= 0) resident = 2048 / kQuantThreads;
    int dev = 0, l2 = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) == cudaSuccess)
      l2_bytes = l2;
    cudaGetLastError();
  }
  QuantBatch B = {};
  uint32_t slots = 0;
  int64_t pads = 0;
  int64_t out_bytes = 0;
  int n = 0;
  for (int i = 0; i < count; ++i) {
    const QuantSpec& sp = specs[i];
    if (sp.groups == 0 || sp.rows == 0 || sp.k == 0) continue;
    QuantJob& jb = B.job[n++];
    jb.x = static_cast<const uint4*>(sp.x);
    jb.q = static_cast<uint4*>(sp.q);
    jb.sf = static_cast<uint8_t*>(sp.sf);
    jb.kb = static_cast<uint32_t>(sp.k / 32);
    jb.rows = static_cast<uint32_t>(sp.rows);
    jb.groups = static_cast<uint32_t>(sp.groups);
    jb.nblk = static_cast<uint32_t>(sp.groups * sp.rows * (sp.k / 32));
    jb.div_kb = make_fastdiv(jb.kb);
    jb.div_rows = make_fastdiv(jb.rows);
    jb.sf_group_bytes = sp.sf_group_bytes;
    jb.sf_ktiles = (jb.kb + 3) / 4;
    jb.kb4 = (jb.kb % 4) == 0;
    jb.slot0 = slots;
    slots += (jb.nblk + kSlotBlocks - 1) / kSlotBlocks;
    const int64_t kbpad = static_cast<int64_t>(jb.sf_ktiles) * 4;
    const int64_t rpad = (sp.rows + 127) / 128 * 128;
    jb.pad_n1 = (rpad - sp.rows) * kbpad;
    jb.pad_per_group = jb.pad_n1 + sp.rows * (kbpad - jb.kb);
    jb.pad0 = pads;
    pads += jb.pad_per_group * sp.groups;
    out_bytes += static_cast<int64_t>(jb.nblk) * 32 + sp.groups * sp.sf_group_bytes;
  }
  if (n == 0) return cudaSuccess;
  B.count = n;
  B.total_slots = slots;
  B.pad_total = pads;
  const int64_t ctas_needed = (static_cast<int64_t>(slots) + (kQuantThreads / 32) - 1) / (kQuantThreads / 32);
  // the lean form runs one CTA per SM, beside whatever else the SM holds
  const int64_t max_ctas = static_cast<int64_t>(num_sms) * (lean ? 1 : resident);
  B.main_blocks = static_cast<int>(ctas_needed < max_ctas ? ctas_needed : max_ctas);
  int pad_blocks = 0;
  if (pads > 0) {
    const int64_t want = (pads + kQuantThreads - 1) / kQuantThreads;
    pad_blocks = static_cast<int>(want < num_sms ? want : num_sms);
  }
  const int grid = B.main_blocks + pad_blocks;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kQuantThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // outputs that fit in three quarters of L2 are kept there for their consumer
  const bool keep = out_bytes <= l2_bytes / 4 * 3;
  cudaError_t e = lean   ? (keep ? cudaLaunchKernelEx(&cfg, mx_quant_kernel<true, false>, B)
                                : cudaLaunchKernelEx(&cfg, mx_quant_kernel<false, false>, B))
                  : keep ? cudaLaunchKernelEx(&cfg, mx_quant_kernel<true, true>, B)
                         : cudaLaunchKernelEx(&cfg, mx_quant_kernel<false, true>, B);
  if (e != cudaSuccess) return e;
  if (launches) *launches += 1;
  return cudaGetLastError();
}

}  // namespace mxk
