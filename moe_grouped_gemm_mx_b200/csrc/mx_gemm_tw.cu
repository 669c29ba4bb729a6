// mx_gemm_tw.cu -- GEMM on tile-wise FP32-scaled FP8 operands (the format of
// mx_quant_tw.cu: A with one FP32 scale per row and 128-element K tile, B with
// one per 128 x 128 block), dense and contiguous-grouped:
//
//   D[i, j] = sum_kt sa[kt, i] * sb[j/128, kt] * sum_{k in kt} e4m3(a[i,k]) e4m3(b[j,k])
//
// FP32 scales cannot ride inside the tensor core's block-scaled MMA (its
// scales are powers of two), so this is DeepGEMM's two-level accumulation
// ("DeepSeek drops DeepGEMM" page, section 1: FP8 products accumulated by the
// tensor core, promoted into FP32 with the scales applied on CUDA cores),
// rebuilt for B200: the first level is a TMEM accumulator, the promotion reads
// it with tcgen05.ld.
//
// CTA layout (192 threads, one CTA per SM, persistent over 128 x 128 tiles):
//   warp 0      TMA producer: A and B tiles of one 128-element K tile per
//               stage, STAGES-deep ring.
//   warp 1      TMEM owner and MMA issuer: each K tile's four K = 32 FP8
//               MMAs (kind::f8f6f4, no block scales) go into a FRESH partial
//               accumulator, cycling through four 128-column TMEM buffers,
//               so the tensor core runs up to three K tiles ahead of the
//               promotion (a 128 x 128 x 128 tile is only ~256 MMA cycles,
//               less than one promotion round trip).
//   warps 2..5  promotion and epilogue: each thread owns one row of the
//               tile; per K tile it reads the row's 128 partial sums from
//               TMEM, releases the buffer, and adds them times
//               sa[kt, row] * sb[n-block, kt] into FP32 registers; after the
//               last K tile it rounds to BF16 and leaves through swizzled
//               staging and TMA stores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstdlib>

#include "mx_gemm_common.cuh"
#include "mx_launch.h"

namespace mxk {

constexpr int kTwStages = 6;
constexpr int kTwThreads = 192;
constexpr int kTwBufs = 4;  // TMEM partial buffers of 128 columns (all 512 columns)

struct TwLayout {
  static constexpr int A_BYTES = 128 * BK;  // 16 KB
  static constexpr int B_BYTES = 128 * BK;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + kTwStages * A_BYTES;
  static constexpr int OFF_STG = (OFF_B + kTwStages * B_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_BAR = OFF_STG + 2 * 8192;
  // full/empty per stage, accf/acce per partial buffer, drain
  static constexpr int NUM_BARS = 2 * kTwStages + 2 * kTwBufs + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_TAB0 = OFF_MISC + 16;
  static constexpr int BYTES = OFF_TAB0 + (kMaxGroups + 1) * 4;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 128 * kTwBufs;
  static_assert(OFF_B % 1024 == 0 && OFF_STG % 1024 == 0, "swizzled tiles need 1024-B alignment");
  static_assert(ALLOC <= 232448, "shared memory budget");
};

struct TwArgs {
  __nv_bfloat16* d;              // [m, n] (written directly by the split-K form)
  const float* sa;               // [k_tiles, m]
  const float* sb;               // [groups, nb, k_tiles]
  const int32_t* group_offsets;  // contiguous form: [groups + 1]
  int32_t* status;
  int m, n, k_tiles, n_tiles, groups, mode;  // mode 0 dense, 1 contiguous
  uint64_t wait_ns;                          // bound of every pipeline wait
};

// Split-K reduction buffer (reuses the operand ring after the mainloop):
// SPLIT partial slices of 128 rows x 128/SPLIT FP32 columns, in quads of 4
// columns; CTA o owns quads [ceil(o*32/SPLIT), ceil((o+1)*32/SPLIT)).
// [source rank][quad of the slice][row] float4, rows fastest: the 32 lanes of
// a warp (32 consecutive rows) write 512 contiguous bytes per remote store.
template <int SPLIT>
struct TwSplit {
  static constexpr int QUADS = 32;
  static constexpr int MAX_SLICE_QUADS = (QUADS + SPLIT - 1) / SPLIT;
  static constexpr int RED_BYTES = SPLIT * MAX_SLICE_QUADS * BM * 16;
  __host__ __device__ static constexpr int slice_start(int o) { return (o * QUADS + SPLIT - 1) / SPLIT; }
  __host__ __device__ static constexpr int quad_owner(int q) { return (q * SPLIT) / QUADS; }
  static_assert(RED_BYTES <= TwLayout::OFF_STG, "reduction buffer must fit in the operand ring");
};

// SPLIT > 1 (dense form only): a cluster of SPLIT CTAs shares one output
// tile, each CTA promoting a contiguous share of the K tiles into its
// registers; the FP32 sums are then exchanged through distributed shared
// memory (each CTA sums one column slice over the cluster in rank order --
// deterministic -- and stores it as BF16).
template <int SPLIT>
__global__ void __launch_bounds__(kTwThreads, 1)
    mx_gemm_tw_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_d, const TwArgs args) {
  using L = TwLayout;
  using RS = TwSplit<SPLIT>;
  const int split_rank = SPLIT > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int t_first = SPLIT > 1 ? static_cast<int>(blockIdx.x) / SPLIT : static_cast<int>(blockIdx.x);
  const int kt_begin = SPLIT > 1 ? split_rank * args.k_tiles / SPLIT : 0;
  const int kt_end = SPLIT > 1 ? (split_rank + 1) * args.k_tiles / SPLIT : args.k_tiles;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile uint32_t* tmem_slot = misc + 0;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* total_slot = reinterpret_cast<volatile int*>(misc + 2);
  int32_t* tab0 = reinterpret_cast<int32_t*>(smem + L::OFF_TAB0);

  auto full_bar = [&](int s) { return sbase + L::OFF_BAR + 8u * s; };
  auto empty_bar = [&](int s) { return sbase + L::OFF_BAR + 8u * (kTwStages + s); };
  auto accf_bar = [&](int b) { return sbase + L::OFF_BAR + 8u * (2 * kTwStages + b); };
  auto acce_bar = [&](int b) { return sbase + L::OFF_BAR + 8u * (2 * kTwStages + kTwBufs + b); };
  const uint32_t drain_bar = sbase + L::OFF_BAR + 8u * (2 * kTwStages + 2 * kTwBufs);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTwStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < kTwBufs; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 128);
    }
    mbar_init(drain_bar, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_d);
  }
  pdl_launch_dependents();
  pdl_wait_prior();

  int bad = 0;
  if (args.mode == kContiguous) {
    for (int i = threadIdx.x; i <= args.groups; i += blockDim.x) tab0[i] = __ldg(args.group_offsets + i);
    __syncthreads();
    for (int i = threadIdx.x; i <= args.groups; i += blockDim.x) {
      const int32_t v = tab0[i];
      if (v < 0 || (v % BM) != 0 || v > args.m) bad = 1;
      if (i > 0 && v < tab0[i - 1]) bad = 1;
    }
  }
  const int any_bad = __syncthreads_or(bad);
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), L::TMEM_COLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    int total;
    if (args.mode == kContiguous) {
      total = any_bad ? 0 : (tab0[args.groups] - tab0[0]) / BM * args.n_tiles;
      if (any_bad) report(args.status, 0x1);
    } else {
      total = ((args.m + BM - 1) / BM) * args.n_tiles;
    }
    *total_slot = total;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = *total_slot;

  // tile t -> (expert, 128-row block, 128-column block)
  auto decode = [&](int t, int& group, int& m_blk, int& n_blk) {
    const int mb = t / args.n_tiles;
    n_blk = t - mb * args.n_tiles;
    if (args.mode == kContiguous) {
      m_blk = tab0[0] / BM + mb;
      group = last_le(tab0, args.groups, m_blk * BM);
      if (group >= args.groups) group = args.groups - 1;
    } else {
      m_blk = mb;
      group = 0;
    }
  };

  // the promotion warps' FP32 accumulators (one 128-column tile row per
  // thread); at function scope so the split-K exchange below can send them
  float acc[128];
  const int quarter = warp & 3;
  const int r_local = quarter * 32 + lane;

  if (warp == 0) {
    if (lane == 0) {
      // ===== TMA producer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = t_first; t < total && ok; t = SPLIT > 1 ? total : t + static_cast<int>(gridDim.x)) {
        int group, m_blk, n_blk;
        decode(t, group, m_blk, n_blk);
        for (int kt = kt_begin; kt < kt_end; ++kt) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, args.wait_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(stage), L::A_BYTES + L::B_BYTES);
          tma_load_3d(sbase + L::OFF_A + stage * L::A_BYTES, &tmap_a, full_bar(stage), kt * BK, m_blk * BM, 0);
          tma_load_3d(sbase + L::OFF_B + stage * L::B_BYTES, &tmap_b, full_bar(stage), kt * BK, n_blk * 128,
                      args.mode == kContiguous ? group : 0);
          if (++stage == kTwStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {  // loads already in flight land during the teardown's linger
        report(args.status, 0x4);
        *abort_flag = 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ===== MMA issuer
      const uint32_t idesc = idesc_f8_e4m3_f32(BM, 128);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t ib = 0;  // K tiles issued so far (partial buffer = ib % kTwBufs)
      bool ok = true;
      for (int t = t_first; t < total && ok; t = SPLIT > 1 ? total : t + static_cast<int>(gridDim.x)) {
        for (int kt = kt_begin; kt < kt_end; ++kt, ++ib) {
          const uint32_t b = ib % kTwBufs;
          if (!mbar_wait(acce_bar(b), ((ib / kTwBufs) & 1u) ^ 1u, abort_flag, args.wait_ns)) { ok = false; break; }
          if (!mbar_wait(full_bar(stage), phase, abort_flag, args.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = sbase + L::OFF_A + stage * L::A_BYTES;
          const uint32_t b_addr = sbase + L::OFF_B + stage * L::B_BYTES;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb)
            tc_mma_f8(tmem_base + b * 128, desc_kmajor_sw128(a_addr + 32 * kb), desc_kmajor_sw128(b_addr + 32 * kb),
                      idesc, kb != 0 ? 1u : 0u);
          tc_commit(empty_bar(stage));
          tc_commit(accf_bar(b));
          if (++stage == kTwStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        report(args.status, 0x4);
        *abort_flag = 1;
      }
      // every MMA issued must finish before TMEM is freed
      tc_commit(drain_bar);
      mbar_wait(drain_bar, 0, nullptr, 100000000ull);
    }
  } else {
    // ===== promotion and epilogue (warps 2..5 -> TMEM lane quarters 2,3,0,1)
    uint32_t ib = 0;
    uint32_t stg_count = 0;
    bool ok = true;
    for (int t = t_first; t < total && ok; t = SPLIT > 1 ? total : t + static_cast<int>(gridDim.x)) {
      int group, m_blk, n_blk;
      decode(t, group, m_blk, n_blk);
      const int row = m_blk * BM + r_local;
      const bool row_ok = row < args.m;
      const float* sb_t = args.sb + (static_cast<int64_t>(group) * args.n_tiles + n_blk) * args.k_tiles;
      const float* sa_r = args.sa + row;
      auto sa_at = [&](int kt) { return row_ok ? __ldg(sa_r + static_cast<int64_t>(kt) * args.m) : 0.0f; };
      // the scales of K tile kt are loaded two K tiles ahead of their use
      float sa0 = kt_begin < kt_end ? sa_at(kt_begin) : 0.0f, sb0 = kt_begin < kt_end ? __ldg(sb_t + kt_begin) : 0.0f;
      float sa1 = kt_begin + 1 < kt_end ? sa_at(kt_begin + 1) : 0.0f;
      float sb1 = kt_begin + 1 < kt_end ? __ldg(sb_t + kt_begin + 1) : 0.0f;
#pragma unroll
      for (int j = 0; j < 128; ++j) acc[j] = 0.0f;
      for (int kt = kt_begin; kt < kt_end; ++kt, ++ib) {
        const uint32_t b = ib % kTwBufs;
        const float s = sa0 * sb0;
        sa0 = sa1;
        sb0 = sb1;
        if (kt + 2 < kt_end) {
          sa1 = sa_at(kt + 2);
          sb1 = __ldg(sb_t + kt + 2);
        }
        // each warp reads only its own TMEM lane quarter: a warp-uniform
        // decision is enough (the aligned TMEM loads need one)
        const bool got = mbar_wait(accf_bar(b), (ib / kTwBufs) & 1u, abort_flag, args.wait_ns);
        if (!__all_sync(0xFFFFFFFFu, got)) {
          if (lane == 0) report(args.status, 0x4);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + b * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v0[32], v1[32];
          tc_ld_32x32b_x32(t_row + h * 64, v0);
          tc_ld_32x32b_x32(t_row + h * 64 + 32, v1);
          tc_wait_ld();
          if (h == 1) {  // every column of the buffer is in registers: hand it back
            tc_fence_before();
            mbar_arrive(acce_bar(b));
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            acc[h * 64 + j] = fmaf(s, __uint_as_float(v0[j]), acc[h * 64 + j]);
            acc[h * 64 + 32 + j] = fmaf(s, __uint_as_float(v1[j]), acc[h * 64 + 32 + j]);
          }
        }
      }
      if constexpr (SPLIT > 1) break;  // the split-K exchange below finishes the tile
      // one uniform decision per tile before the epilogue's 128-thread
      // barriers: a warp that gave up set abort_flag, which ends the other
      // warps' waits too, so every warp gets here
      if (!named_barrier_and(2, 128, ok)) break;
      uint32_t packed[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) packed[j] = pack_bf16x2(__float_as_uint(acc[2 * j]), __float_as_uint(acc[2 * j + 1]));
      store_rows_tma<128>(packed, r_local, sbase + L::OFF_STG, stg_count, &tmap_d, n_blk * 128, m_blk * BM, 0);
    }
    if (threadIdx.x == 64) bulk_wait_group_all();
  }

  if constexpr (SPLIT > 1) {
    // ---------------------------------------------------------- split-K exchange
    // 1) every CTA of the cluster is past its mainloop, so every operand
    //    ring is free to receive; 2) each promotion thread sends column slice
    //    o of its row to CTA o; 3) each CTA sums the SPLIT partials of its
    //    slice in rank order and stores BF16.  Every thread of every CTA
    //    takes both cluster barriers, whatever happened before.
    tc_fence_before();
    cluster_sync();
    const bool epi = warp >= 2 && t_first < total;
    int m_blk = 0, n_blk = 0;
    if (epi) {
      int group;
      decode(t_first, group, m_blk, n_blk);
    }
    const int row = m_blk * BM + r_local;
    const bool valid = epi && row < args.m;
    if (valid) {
#pragma unroll
      for (int q = 0; q < RS::QUADS; ++q) {
        const int owner = RS::quad_owner(q);
        const uint32_t local =
            sbase + ((split_rank * RS::MAX_SLICE_QUADS + (q - RS::slice_start(owner))) * BM + r_local) * 16;
        st_cluster_v4(map_to_rank(local, owner), __float_as_uint(acc[4 * q]), __float_as_uint(acc[4 * q + 1]),
                      __float_as_uint(acc[4 * q + 2]), __float_as_uint(acc[4 * q + 3]));
      }
    }
    cluster_sync();
    if (valid && !*abort_flag) {
      const float* red = reinterpret_cast<const float*>(smem);
      __nv_bfloat16* drow = args.d + static_cast<int64_t>(row) * args.n;
      const int q_begin = RS::slice_start(split_rank), q_end = RS::slice_start(split_rank + 1);
#pragma unroll 1
      for (int q = q_begin; q < q_end; ++q) {
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int src = 0; src < SPLIT; ++src) {
          const float4 x =
              *reinterpret_cast<const float4*>(red + ((src * RS::MAX_SLICE_QUADS + (q - q_begin)) * BM + r_local) * 4);
          sum.x += x.x; sum.y += x.y; sum.z += x.z; sum.w += x.w;
        }
        const int col = n_blk * 128 + q * 4;
        if (col < args.n) {
          uint2 w;
          w.x = pack_bf16x2(__float_as_uint(sum.x), __float_as_uint(sum.y));
          w.y = pack_bf16x2(__float_as_uint(sum.z), __float_as_uint(sum.w));
          *reinterpret_cast<uint2*>(drow + col) = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) linger_after_abort();
}

template <int SPLIT>
static cudaError_t prepare_tw_kernel() {
  static cudaError_t state = cudaErrorNotReady;
  if (state == cudaErrorNotReady)
    state = cudaFuncSetAttribute(mx_gemm_tw_kernel<SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 TwLayout::ALLOC);
  return state;
}

// How many clusters of SPLIT CTAs the GPU holds at once (0 if unknown).
template <int SPLIT>
static int tw_max_clusters() {
  static int v = -1;
  if (v < 0) {
    v = 0;
    if (prepare_tw_kernel<SPLIT>() == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      cfg.gridDim = dim3(SPLIT, 1, 1);
      cfg.blockDim = dim3(kTwThreads, 1, 1);
      cfg.dynamicSmemBytes = TwLayout::ALLOC;
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = SPLIT;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, mx_gemm_tw_kernel<SPLIT>, &cfg) == cudaSuccess) v = n;
      cudaGetLastError();
    }
  }
  return v;
}

template <int SPLIT>
static cudaError_t launch_tw(const TwProblem& p, int num_sms, cudaStream_t stream) {
  cudaError_t e = prepare_tw_kernel<SPLIT>();
  if (e != cudaSuccess) return e;
  const int64_t b_depth = p.mode == kContiguous ? p.groups : 1;
  CUtensorMap ta, tb, td;
  if (!make_tmap(&ta, p.qa, p.k, p.m, 1, 128)) return cudaErrorInvalidValue;
  if (!make_tmap(&tb, p.qb, p.k, p.n, b_depth, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_d(&td, p.d, p.n, p.m, 1)) return cudaErrorInvalidValue;
  TwArgs a = {};
  a.d = static_cast<__nv_bfloat16*>(p.d);
  a.sa = p.sa;
  a.sb = p.sb;
  a.group_offsets = p.group_offsets;
  a.status = p.status;
  a.wait_ns = wait_limit_ns();
  a.m = static_cast<int>(p.m);
  a.n = static_cast<int>(p.n);
  a.k_tiles = static_cast<int>(p.k / BK);
  a.n_tiles = static_cast<int>((p.n + 127) / 128);
  a.groups = static_cast<int>(p.groups);
  a.mode = p.mode;
  const int64_t tiles_bound = ((p.m + BM - 1) / BM) * a.n_tiles;
  if (tiles_bound == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.blockDim = dim3(kTwThreads, 1, 1);
  cfg.dynamicSmemBytes = TwLayout::ALLOC;
  cfg.stream = stream;
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  if (SPLIT > 1) {  // one cluster of SPLIT CTAs per output tile
    cfg.gridDim = dim3(static_cast<unsigned>(tiles_bound * SPLIT), 1, 1);
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = SPLIT;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl;
    cfg.numAttrs = 2;
  } else {
    cfg.gridDim = dim3(static_cast<unsigned>(tiles_bound < num_sms ? tiles_bound : num_sms), 1, 1);
    attr[0] = pdl;
    cfg.numAttrs = 1;
  }
  cfg.attrs = attr;
  e = cudaLaunchKernelEx(&cfg, mx_gemm_tw_kernel<SPLIT>, ta, tb, td, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

static int tw_max_clusters_of(int split) {
  switch (split) {
    case 2: return tw_max_clusters<2>();
    case 4: return tw_max_clusters<4>();
    case 8: return tw_max_clusters<8>();
    default: return 0;
  }
}

// Dense problems whose 128 x 128 tiles leave most SMs idle split K over a
// cluster of 2, 4 or 8 CTAs: the largest split whose clusters all fit at once
// with at least two K tiles per CTA.  MX_TW_SPLIT=1|2|4|8 forces one (tests).
cudaError_t launch_gemm_tw(const TwProblem& p, int num_sms, cudaStream_t stream) {
  static int forced = -2;
  if (forced == -2) {
    const char* env = getenv("MX_TW_SPLIT");
    forced = env ? atoi(env) : -1;
  }
  const int64_t k_tiles = p.k / BK;
  const int64_t tiles = ((p.m + BM - 1) / BM) * ((p.n + 127) / 128);
  int split = 1;
  if (p.mode != kContiguous) {
    if (forced == 1 || forced == 2 || forced == 4 || forced == 8) {
      if (k_tiles >= forced) split = forced;
    } else if (tiles * 2 <= num_sms) {
      const int order[3] = {8, 4, 2};
      for (int i = 0; i < 3; ++i) {
        const int sp = order[i];
        if (tiles * sp <= num_sms && k_tiles >= 2 * sp && tiles <= tw_max_clusters_of(sp)) {
          split = sp;
          break;
        }
      }
    }
  }
  switch (split) {
    case 2: return launch_tw<2>(p, num_sms, stream);
    case 4: return launch_tw<4>(p, num_sms, stream);
    case 8: return launch_tw<8>(p, num_sms, stream);
    default: return launch_tw<1>(p, num_sms, stream);
  }
}

}  // namespace mxk
