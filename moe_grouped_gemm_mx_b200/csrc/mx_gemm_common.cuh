// mx_gemm_common.cuh -- definitions shared by the MXFP8 GEMM kernels
// (one-CTA kernel in mx_gemm.cu, CTA-pair kernel in mx_gemm2.cu): problem
// arguments, tile bookkeeping, BF16 packing and tensor-map construction.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mx_ptx.cuh"

namespace mxk {

constexpr int BM = 128;              // MMA M (rows of A per tile)
constexpr int BK = 128;              // K elements per pipeline stage (4 scale blocks)
constexpr int kMaxGroups = 1024;
constexpr int kGemmThreads = 224;  // 7 warps: producer, MMA, 4 epilogue, scale copier
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // default wait bound, 2 s: far above any legitimate wait

enum GemmMode : int { kDense = 0, kContiguous = 1, kMasked = 2, kKGrouped = 3 };

struct GemmArgs {
  const uint8_t* sfa;
  const uint8_t* sfb;
  __nv_bfloat16* d;
  const int32_t* group_offsets;  // contiguous: [groups+1]
  const int32_t* masked_m;       // masked: [groups]
  int32_t* status;
  int64_t sfa_group_bytes;  // masked: tiled scale bytes per expert of A
  int64_t sfb_group_bytes;  // grouped: tiled scale bytes per expert of B
  int m;                    // dense: M; contiguous: m_total; masked: max_m
  int n;
  int k_tiles;              // K / 128 (also the 512-byte scale tiles per 128-row block)
  int n_tiles;              // ceil(N / BN)
  int n_sf_tiles;           // ceil(N / 128)
  int groups;
  int mode;
  int a_box_rows;           // rows of A one TMA box brings (128, or 64/32 for a dense M <= 64)
  // fused SwiGLU + MXFP8 epilogue (CTA-pair kernel only): B holds [gate; up]
  // rows per expert, 2 * swiglu_i of them; the output is E4M3 H = silu(gate)
  // * up [rows, swiglu_i] (through the D tensor map) plus its tiled scales
  int swiglu_i;             // 0: plain BF16 epilogue
  uint8_t* sfh;             // tiled UE8M0 scales of H
  int64_t sfh_group_bytes;  // masked form: tiled scale bytes of H per expert
  uint64_t wait_ns;         // bound of every pipeline wait (mx_set_wait_limit_ns)
};

struct Tile {
  int group;
  int m_blk;  // 128-row block inside the group (masked) or inside A (dense/contiguous)
  int n_blk;
};

// Index of the last entry <= v in the non-decreasing table t[0..n] (n+1 entries).
__device__ __forceinline__ int last_le(const int32_t* t, int n, int32_t v) {
  int lo = 0, hi = n;  // invariant: t[lo] <= v
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (t[mid] <= v) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ Tile decode_tile(const GemmArgs& a, const int32_t* tab0, int t) {
  Tile r;
  if (a.mode == kMasked) {
    const int e = last_le(tab0, a.groups, t);  // tab0 = prefix of tiles per expert
    const int local = t - tab0[e];
    r.group = e;
    r.m_blk = local / a.n_tiles;
    r.n_blk = local - r.m_blk * a.n_tiles;
  } else {
    const int mb = t / a.n_tiles;
    r.n_blk = t - mb * a.n_tiles;
    if (a.mode == kContiguous) {
      r.m_blk = tab0[0] / BM + mb;                               // tab0 = group offsets
      r.group = last_le(tab0, a.groups, r.m_blk * BM);
      if (r.group >= a.groups) r.group = a.groups - 1;
    } else {
      r.m_blk = mb;
      r.group = 0;
    }
  }
  return r;
}

__device__ __forceinline__ void report(int32_t* status, int bits) {
  atomicOr(status, bits);
}

// Teardown of a CTA that gave up: every role has stopped issuing, the MMAs
// and scale copies it issued are drained, but TMA loads issued before the
// give-up may still be landing in its shared memory.  The CTA stays resident
// for 1 ms more (one thread spins; the CTA ends when its last thread does),
// so that they land here and not in the shared memory of a later CTA.
__device__ __forceinline__ void linger_after_abort() {
  const uint64_t t0 = global_timer_ns();
  while (global_timer_ns() - t0 < 1000000ull) { }
}

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo_f32, uint32_t hi_f32) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo_f32), __uint_as_float(hi_f32));
  return *reinterpret_cast<const uint32_t*>(&v);
}

// ======================================================================= host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D BF16 tensor [depth, rows, n] written in boxes of 128 rows x 32 columns
// (64-byte rows, 64-byte swizzle, matching the epilogue's staging layout).
inline bool make_tmap_d(CUtensorMap* m, void* base, int64_t n, int64_t rows, int64_t depth) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(n), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(depth)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(n * 2), static_cast<cuuint64_t>(n * 2 * rows)};
  const cuuint32_t box[3] = {32, static_cast<cuuint32_t>(BM), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 3-D byte tensor [depth, rows, cols] written in boxes of 128 rows x 64 bytes
// (64-byte swizzle, the epilogue's staging layout): the E4M3 output of the
// fused SwiGLU epilogue.
inline bool make_tmap_h(CUtensorMap* m, void* base, int64_t cols, int64_t rows, int64_t depth) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(depth)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(cols * rows)};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(BM), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 3-D byte tensor [depth, rows, k] (k contiguous) read in boxes of box_rows x 128 bytes.
inline bool make_tmap(CUtensorMap* m, const void* base, int64_t k, int64_t rows, int64_t depth, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(depth)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(k * rows)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Epilogue, step 1: read this thread's row of an NCOLS-wide FP32
// accumulator out of TMEM (two 32-column loads in flight at a time) and pack
// it to BF16 pairs: packed[i] holds columns 2i and 2i+1 (RNE).  After this the
// accumulator may be handed back to the MMA warp.
template <int NCOLS>
__device__ __forceinline__ void tmem_row_to_bf16(uint32_t t_row, uint32_t (&packed)[NCOLS / 2]) {
#pragma unroll
  for (int b = 0; b < NCOLS / 64; ++b) {
    uint32_t v0[32], v1[32];
    tc_ld_32x32b_x32(t_row + b * 64, v0);
    tc_ld_32x32b_x32(t_row + b * 64 + 32, v1);
    tc_wait_ld();
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      packed[b * 32 + j] = pack_bf16x2(v0[2 * j], v0[2 * j + 1]);
      packed[b * 32 + 16 + j] = pack_bf16x2(v1[2 * j], v1[2 * j + 1]);
    }
  }
}

// Epilogue, step 2 (the 128 epilogue threads, thread 64 issuing): write the
// WORDS 32-bit words of each row of a 128-row tile through two
// 64-byte-swizzled 8 KiB staging chunks (128 rows x 64 bytes) with TMA stores
// at (x0 + c * CHUNK_ELEMS, y0, z), CHUNK_ELEMS = elements of the tensor map
// per 64 bytes (32 for BF16 D, 64 for E4M3 H); the tensor map clips what lies
// outside the tensor.  `stg_count` alternates the chunks.
template <int WORDS, int CHUNK_ELEMS = 32>
__device__ __forceinline__ void store_words_tma(const uint32_t (&packed)[WORDS], int r_local, uint32_t stg_base,
                                                uint32_t& stg_count, const CUtensorMap* tmap_d, int x0, int y0,
                                                int z) {
#pragma unroll
  for (int c = 0; c < WORDS / 16; ++c) {
    const uint32_t stg = stg_base + (stg_count & 1u) * 8192u;
    // the store issued from this chunk two rounds ago must have read it
    if (threadIdx.x == 64) bulk_wait_group_read<1>();
    named_barrier_sync(1, 128);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t off = r_local * 64 + ((j ^ ((r_local >> 1) & 3)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(stg + off), "r"(packed[c * 16 + j * 4 + 0]),
                   "r"(packed[c * 16 + j * 4 + 1]), "r"(packed[c * 16 + j * 4 + 2]), "r"(packed[c * 16 + j * 4 + 3])
                   : "memory");
    }
    fence_proxy_async_smem();
    named_barrier_sync(1, 128);
    if (threadIdx.x == 64) {
      tma_store_3d(tmap_d, stg, x0 + c * CHUNK_ELEMS, y0, z);
      bulk_commit_group();
    }
    ++stg_count;
  }
}

// BF16 rows of NCOLS columns (NCOLS / 2 packed words).
template <int NCOLS>
__device__ __forceinline__ void store_rows_tma(const uint32_t (&packed)[NCOLS / 2], int r_local, uint32_t stg_base,
                                               uint32_t& stg_count, const CUtensorMap* tmap_d, int x0, int y0,
                                               int z) {
  store_words_tma<NCOLS / 2, 32>(packed, r_local, stg_base, stg_count, tmap_d, x0, y0, z);
}

}  // namespace mxk
