// mx_quant_t.cu -- BF16 -> MXFP8 quantisation along the ROW dimension, written
// in the transposed layout: for x [groups, rows, cols] (row-major) the output
// is q [groups, cols, rows] E4M3 with one UE8M0 scale per 32 consecutive rows
// of a column, tiled as for any [cols, rows] operand.
//
// This is the operand preparation of the training-side MoE GEMMs: the weight
// gradient reduces over tokens, so both of its operands (the output gradient
// and the layer input, [tokens, features]) need their 32-element blocks along
// the token dimension and the token dimension contiguous (K-major for the
// MMA); the input gradient reduces over the layer's output features, so the
// expert weights [E, N, K] need blocks along N and the [E, K, N] layout.  The
// MXFP8 format and the scale rule are those of mx_quant.cu (B200 MoE-training
// page, glossary entry on microscaling FP8; OCP Microscaling specification).
//
// Kernel (HBM-bound: 2 B read, 1 + 1/32 B written per element): persistent
// CTAs of 128 threads walk 128-row x 128-column tiles.  A tile arrives by TMA
// (one 32 KiB box, zero-filled past the edges) into one of two shared-memory
// buffers, and the load of the tile after next is issued as soon as a buffer
// is free, so loads overlap the quantisation and stores of the current tile.
// Thread j walks column j down the staged tile (a warp reads 64 contiguous
// bytes of a row per step, free of bank conflicts) and quantises its four
// 32-row blocks with the FP32 block rule (exact for BF16 input); its four
// scale bytes, adjacent in the tiled layout, leave as one 32-bit store.  The
// E4M3 tile is restaged in (swizzled) shared memory and written out as
// 128-byte row runs by groups of 8 threads.  Scale padding (rows of the
// transposed operand up to a multiple of 128, blocks up to a multiple of 4)
// is written as 0x00 by the CTAs that own it.  Waits on the loads are
// bounded; a timeout sets the status word and the CTA stops.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include <algorithm>

#include "mx_gemm_common.cuh"
#include "mx_launch.h"
#include "mx_mxfp8.cuh"

namespace mxk {

constexpr int kTQTile = 128;  // rows and columns of one tile
constexpr int kTQThreads = 128;
constexpr uint64_t kTQWaitNs = 2000000000ull;  // 2 s: far above any legitimate wait

struct TQArgs {
  uint8_t* q;         // [groups, cols, rows]
  uint8_t* sf;        // groups regions of sf_group_bytes
  int32_t* status;
  int64_t sf_group_bytes;
  int rows, cols;     // rows % 32 == 0, cols % 8 == 0
  int row_tiles, col_tiles, tiles;
  int sf_ktiles;      // ceil(rows / 128): 512-byte tiles along the transposed operand's K
};

struct TQSmem {
  uint16_t tile[2][kTQTile][kTQTile];  // [buffer][row][col] BF16, 2 x 32 KiB
  uint4 stg[kTQTile * 8];               // the E4M3 tile, [column][16-byte chunk], 16 KiB
  uint64_t full[2];
};

__global__ void __launch_bounds__(kTQThreads) mx_quant_t_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                                                const TQArgs a) {
  extern __shared__ uint8_t tq_raw[];
  TQSmem& sm = *reinterpret_cast<TQSmem*>(tq_raw + ((1024u - (smem_u32(tq_raw) & 1023u)) & 1023u));
  const int t = threadIdx.x;
  const uint32_t full0 = smem_u32(&sm.full[0]), full1 = smem_u32(&sm.full[1]);
  if (t == 0) {
    mbar_init(full0, 1);
    mbar_init(full1, 1);
    fence_mbar_init();
    prefetch_tmap(&tmap_x);
  }
  __syncthreads();
  // programmatic dependent launch: let the next kernel start its prologue,
  // and wait for the previous one (which may produce x) before reading
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  auto coords = [&](int tile, int& g, int& rt, int& ct) {
    ct = tile % a.col_tiles;
    rt = (tile / a.col_tiles) % a.row_tiles;
    g = tile / (a.col_tiles * a.row_tiles);
  };
  auto issue = [&](int tile, int b) {  // thread 0 only
    int g, rt, ct;
    coords(tile, g, rt, ct);
    const uint32_t bar = b ? full1 : full0;
    mbar_arrive_expect_tx(bar, kTQTile * kTQTile * 2);
    tma_load_3d(smem_u32(&sm.tile[b][0][0]), &tmap_x, bar, ct * kTQTile, rt * kTQTile, g);
  };
  const int first = blockIdx.x, stride = gridDim.x;
  if (t == 0) {
    if (first < a.tiles) issue(first, 0);
    if (first + stride < a.tiles) issue(first + stride, 1);
  }
  const int c_pad = (a.cols + 127) / 128 * 128;
  int it = 0;
  for (int tile = first; tile < a.tiles; tile += stride, ++it) {
    const int b = it & 1;
    int g, rt, ct;
    coords(tile, g, rt, ct);
    const int r0 = rt * kTQTile, c0 = ct * kTQTile;
    const int rows_here = min(kTQTile, a.rows - r0);  // a multiple of 32
    const int cols_here = min(kTQTile, a.cols - c0);  // a multiple of 8
    const bool got = mbar_wait(b ? full1 : full0, (it >> 1) & 1, nullptr, kTQWaitNs);
    if (__syncthreads_or(!got)) {  // a uniform decision: the block's barriers below need every thread
      if (t == 0) atomicOr(a.status, 0x4);
      // let copies still in flight land before the CTA leaves
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 1000000ull) { }
      return;
    }

    // ---- thread t quantises column c0 + t over the tile's rows
    const int c = c0 + t;
    uint8_t* sfg = a.sf + static_cast<int64_t>(g) * a.sf_group_bytes;
    // scale bytes of (transposed row c, blocks 4*rt .. 4*rt+3): one 32-bit word
    const int64_t sf_off =
        (static_cast<int64_t>(c >> 7) * a.sf_ktiles + rt) * 512 + (c & 31) * 16 + ((c & 127) >> 5) * 4;
    uint32_t qv[32];  // this column's 128 output bytes
    uint32_t sfw = 0;
    if (t < cols_here) {
#pragma unroll
      for (int bl = 0; bl < 4; ++bl) {
        if (bl * 32 < rows_here) {  // blocks past the rows stay 0x00 (scale padding)
          float h[32];
#pragma unroll
          for (int j = 0; j < 32; ++j)
            h[j] = __uint_as_float(static_cast<uint32_t>(sm.tile[b][bl * 32 + j][t]) << 16);
          uint32_t q8[8];
          sfw |= quant_block32_f32(h, q8) << (8 * bl);
#pragma unroll
          for (int i = 0; i < 8; ++i) qv[bl * 8 + i] = q8[i];
        }
      }
      *reinterpret_cast<uint32_t*>(sfg + sf_off) = sfw;
    } else if (c < c_pad) {
      *reinterpret_cast<uint32_t*>(sfg + sf_off) = 0u;  // scale padding rows
    }
    // every thread is done with BF16 buffer b (and with the previous tile's
    // staging reads): refill the buffer with the tile after next
    __syncthreads();
    if (t == 0 && tile + 2 * stride < a.tiles) issue(tile + 2 * stride, b);
    // ---- restage the [128 columns x 128 rows] E4M3 tile so every output row
    // leaves as contiguous 128-byte runs.  Row t of the staging area holds
    // column t's bytes; its 16-byte chunk j sits at slot j ^ (t & 7) so that 8
    // consecutive rows spread over all banks.
    if (t < cols_here) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        sm.stg[t * 8 + (j ^ (t & 7))] = make_uint4(qv[4 * j], qv[4 * j + 1], qv[4 * j + 2], qv[4 * j + 3]);
    }
    __syncthreads();
    const int chunks = rows_here / 16;  // valid 16-byte chunks per output row
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = i * 16 + (t >> 3);  // output row = column c0 + row
      const int j = t & 7;
      if (row < cols_here && j < chunks) {
        uint8_t* dst = a.q + (static_cast<int64_t>(g) * a.cols + c0 + row) * a.rows + r0 + j * 16;
        *reinterpret_cast<uint4*>(dst) = sm.stg[row * 8 + (j ^ (row & 7))];
      }
    }
  }
}

// BF16 x [groups, rows, cols] as a 3-D tensor map with 128 x 128 boxes, no
// swizzle (a thread walks a column of the staged tile), zero fill past the edges.
static bool make_tmap_tq(CUtensorMap* m, const void* x, int64_t groups, int64_t rows, int64_t cols) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(groups)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols * 2), static_cast<cuuint64_t>(rows * cols * 2)};
  const cuuint32_t box[3] = {kTQTile, kTQTile, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(x), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_quant_transposed(const void* x, int64_t groups, int64_t rows, int64_t cols, void* q, void* sf,
                                    int64_t sf_group_bytes, int32_t* status, int num_sms, cudaStream_t stream) {
  TQArgs a;
  a.q = static_cast<uint8_t*>(q);
  a.sf = static_cast<uint8_t*>(sf);
  a.status = status;
  a.sf_group_bytes = sf_group_bytes;
  a.rows = static_cast<int>(rows);
  a.cols = static_cast<int>(cols);
  a.row_tiles = static_cast<int>((rows + kTQTile - 1) / kTQTile);
  a.col_tiles = static_cast<int>((cols + kTQTile - 1) / kTQTile);
  a.sf_ktiles = a.row_tiles;
  const int64_t tiles = groups * a.row_tiles * a.col_tiles;
  if (tiles == 0) return cudaSuccess;
  if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
  a.tiles = static_cast<int>(tiles);
  CUtensorMap tm;
  if (!make_tmap_tq(&tm, x, groups, rows, cols)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(TQSmem) + 1024;
  static cudaError_t attr = cudaErrorNotReady;
  static int per_sm = 0;
  if (attr == cudaErrorNotReady) {
    attr = cudaFuncSetAttribute(mx_quant_t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (attr == cudaSuccess &&
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mx_quant_t_kernel, kTQThreads, smem) != cudaSuccess)
      per_sm = 0;
    cudaGetLastError();
    if (per_sm <= 0) per_sm = 1;
  }
  if (attr != cudaSuccess) return attr;
  const int64_t ctas = std::min<int64_t>(tiles, static_cast<int64_t>(num_sms) * per_sm);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
  cfg.blockDim = dim3(kTQThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, mx_quant_t_kernel, tm, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mxk
