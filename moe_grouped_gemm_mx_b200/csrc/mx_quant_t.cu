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
// Kernel (HBM-bound: 2 B read, 1 + 1/32 B written per element): a CTA of 128
// threads owns a tile of 128 rows x 128 columns of one group.  The tile is
// read with 16-byte coalesced loads (16 per thread, all in flight before any
// shared-memory store) into a 32 KiB row-major staging buffer; then thread j
// walks column j down the 128 rows -- a warp reads 64 contiguous bytes of a
// staged row per step, free of bank conflicts -- and quantises its four
// 32-row blocks with the FP32 block rule (exact for BF16 input); its four
// scale bytes, adjacent in the tiled layout, leave as one 32-bit store.  The
// E4M3 tile is restaged in (swizzled) shared memory and written out as
// 128-byte row runs by groups of 8 threads.  Scale
// padding (rows of the transposed operand up to a multiple of 128, blocks up
// to a multiple of 4) is written as 0x00 by the CTAs that own it.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mx_launch.h"
#include "mx_mxfp8.cuh"

namespace mxk {

constexpr int kTQTile = 128;  // rows and columns of one CTA tile
constexpr int kTQThreads = 128;

struct TQArgs {
  const uint16_t* x;  // BF16 bits [groups, rows, cols]
  uint8_t* q;         // [groups, cols, rows]
  uint8_t* sf;        // groups regions of sf_group_bytes
  int64_t sf_group_bytes;
  int rows, cols;     // rows % 32 == 0, cols % 8 == 0
  int row_tiles, col_tiles;
  int sf_ktiles;      // ceil(rows / 128): 512-byte tiles along the transposed operand's K
};

__global__ void __launch_bounds__(kTQThreads) mx_quant_t_kernel(const TQArgs a) {
  __shared__ __align__(16) uint16_t tile[kTQTile][kTQTile];  // [row][col], 32 KiB
  // programmatic dependent launch: let the next kernel start its prologue,
  // and wait for the previous one (which may produce x) before reading
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int t = threadIdx.x;
  const int ct = blockIdx.x % a.col_tiles;
  const int rt = (blockIdx.x / a.col_tiles) % a.row_tiles;
  const int g = blockIdx.x / (a.col_tiles * a.row_tiles);
  const int r0 = rt * kTQTile, c0 = ct * kTQTile;
  const int rows_here = min(kTQTile, a.rows - r0);   // a multiple of 32
  const int cols_here = min(kTQTile, a.cols - c0);   // a multiple of 8
  const uint16_t* xg = a.x + static_cast<int64_t>(g) * a.rows * a.cols;

  // ---- stage the tile: 16 rounds of 8 rows x 16 lanes x 16 bytes
  uint4 v[16];
  const int lc = (t & 15) * 8;  // this thread's 8 columns
  const int lr = t >> 4;        // row within a round of 8
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = i * 8 + lr;
    v[i] = make_uint4(0, 0, 0, 0);
    if (r < rows_here && lc < cols_here)
      v[i] = *reinterpret_cast<const uint4*>(xg + static_cast<int64_t>(r0 + r) * a.cols + c0 + lc);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) *reinterpret_cast<uint4*>(&tile[i * 8 + lr][lc]) = v[i];
  __syncthreads();

  // ---- thread t quantises column c0 + t over the tile's rows
  const int c = c0 + t;
  uint8_t* sfg = a.sf + static_cast<int64_t>(g) * a.sf_group_bytes;
  // scale bytes of (transposed row c, blocks 4*rt .. 4*rt+3): one 32-bit word
  const int64_t sf_off = (static_cast<int64_t>(c >> 7) * a.sf_ktiles + rt) * 512 + (c & 31) * 16 + ((c & 127) >> 5) * 4;
  const int c_pad = (a.cols + 127) / 128 * 128;
  uint32_t qv[32];  // this column's 128 output bytes
  uint32_t sfw = 0;
  if (t < cols_here) {
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      if (b * 32 < rows_here) {  // blocks past the rows stay 0x00 (scale padding)
        float h[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) h[j] = __uint_as_float(static_cast<uint32_t>(tile[b * 32 + j][t]) << 16);
        uint32_t q8[8];
        sfw |= quant_block32_f32(h, q8) << (8 * b);
#pragma unroll
        for (int i = 0; i < 8; ++i) qv[b * 8 + i] = q8[i];
      }
    }
    *reinterpret_cast<uint32_t*>(sfg + sf_off) = sfw;
  } else if (c < c_pad) {
    *reinterpret_cast<uint32_t*>(sfg + sf_off) = 0u;  // scale padding rows
  }
  // ---- restage the [128 columns x 128 rows] E4M3 tile so every output row
  // leaves as contiguous 128-byte runs (a lane-per-row store pattern would
  // send 16-byte pieces to 32 different rows per instruction).  Row t of the
  // staging area holds column t's bytes; its 16-byte chunk j sits at slot
  // j ^ (t & 7) so that 8 consecutive rows spread over all banks.
  __syncthreads();  // every thread is done reading the BF16 tile
  uint4* stg = reinterpret_cast<uint4*>(&tile[0][0]);  // 16 KiB of the 32 KiB buffer
  if (t < cols_here) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      stg[t * 8 + (j ^ (t & 7))] = make_uint4(qv[4 * j], qv[4 * j + 1], qv[4 * j + 2], qv[4 * j + 3]);
  }
  __syncthreads();
  const int chunks = rows_here / 16;  // valid 16-byte chunks per output row
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = i * 16 + (t >> 3);  // output row = column c0 + row
    const int j = t & 7;
    if (row < cols_here && j < chunks) {
      uint8_t* dst = a.q + (static_cast<int64_t>(g) * a.cols + c0 + row) * a.rows + r0 + j * 16;
      *reinterpret_cast<uint4*>(dst) = stg[row * 8 + (j ^ (row & 7))];
    }
  }
}

cudaError_t launch_quant_transposed(const void* x, int64_t groups, int64_t rows, int64_t cols, void* q, void* sf,
                                    int64_t sf_group_bytes, cudaStream_t stream) {
  TQArgs a;
  a.x = static_cast<const uint16_t*>(x);
  a.q = static_cast<uint8_t*>(q);
  a.sf = static_cast<uint8_t*>(sf);
  a.sf_group_bytes = sf_group_bytes;
  a.rows = static_cast<int>(rows);
  a.cols = static_cast<int>(cols);
  a.row_tiles = static_cast<int>((rows + kTQTile - 1) / kTQTile);
  a.col_tiles = static_cast<int>((cols + kTQTile - 1) / kTQTile);
  a.sf_ktiles = a.row_tiles;
  const int64_t blocks = groups * a.row_tiles * a.col_tiles;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(kTQThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, mx_quant_t_kernel, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mxk
