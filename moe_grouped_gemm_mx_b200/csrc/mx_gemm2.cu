// mx_gemm2.cu -- CTA-pair MXFP8 GEMM (tcgen05 cta_group::2) for large problems.
//
// Same computation and C ABI as the one-CTA kernel in mx_gemm.cu (dense,
// contiguous-grouped and masked-grouped forms, FP32 accumulation, BF16 out),
// but two CTAs of a cluster share one 256 x 256 output tile: CTA r holds A
// rows [128r, 128r+128) and B rows [128r, 128r+128) of the tile in its own
// shared memory, and one 2-SM MMA, issued by the leader CTA (rank 0), reads
// both.  Per K step each CTA therefore stages half the B bytes a one-CTA
// 128 x 256 tile needs for the same math, which lowers the operand feed each
// SM must sustain -- the limit of the one-CTA kernel on large problems.
//
//   warp 0 (both CTAs)   TMA producer: the 512-byte scale chunk of its own
//                        128 A rows and the two chunks of all 256 B rows
//                        (every CTA's MMA half needs all N scales), then its
//                        own A half and B half.  Every load completes on a
//                        barrier of the LEADER (scales and operands on two
//                        barriers per stage); the leader announces both
//                        CTAs' bytes.
//   warp 6 (leader)      scale chunks of each stage -> that stage's TMEM
//                        scale buffer (tcgen05.cp, both CTAs) as soon as
//                        they land, while the operands are still in flight;
//                        commit to the stage's "scales ready" barrier.
//   warp 1 (leader)      4 pair MMAs per K tile once its operands have landed
//                        and its scales are ready,
//                        commits multicast to both CTAs' "empty" /
//                        "accumulator full" barriers.
//   warps 2-5 (both)     epilogue of the CTA's own 128 accumulator rows
//                        (TMEM -> BF16 -> swizzled staging -> TMA store);
//                        once a warp's TMEM loads are done, one lane arrives
//                        on the leader's "accumulator empty" (8 arrivals: a
//                        barrier counting all 256 threads, half of them
//                        remote, kept the MMA waiting ~0.7 us per tile).
//
// Grouped forms: a pair tile covers 256 rows of ONE expert; with groups
// aligned to 128 rows, the second CTA's half of an expert's last tile may be
// past the expert's rows, in which case it is computed but not stored.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mx_gemm_common.cuh"
#include "mx_mxfp8.cuh"
#include "mx_launch.h"

namespace mxk {

constexpr int kPairN = 256;  // N of the pair tile (128 B rows per CTA)
constexpr int kPairM = 256;  // M of the pair tile (128 A rows per CTA)
constexpr int kPairKC = 2;   // 128-byte K chunks per pipeline stage (K = 256 per stage)
constexpr int kPairStages = 3;

// One pipeline stage holds two K chunks of 128 bytes for A and B (each chunk
// a 128-row x 128-byte swizzled tile, as the MMA descriptor expects) and the
// matching scale chunks.  Fetching two chunks per TMA operation and issuing 8
// MMAs per barrier wait and commit halves the per-stage fixed costs (TMA
// operations, mbarrier round trips) that bounded 128-K stages.
template <int STAGES>
struct PairLayout {
  static constexpr int CHUNK = 128 * BK;              // 16 KB
  static constexpr int A_BYTES = kPairKC * CHUNK;
  static constexpr int B_BYTES = kPairKC * CHUNK;
  static constexpr int SFA_BYTES = kPairKC * 512;     // [K chunk] of 512-byte scale chunks
  static constexpr int SFB_BYTES = 2 * kPairKC * 512; // [B 128-row half][K chunk]
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
  static constexpr int STG_BYTES = 128 * 32 * 2;
  static constexpr int OFF_STG = (OFF_SFB + STAGES * SFB_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_BAR = OFF_STG + 2 * STG_BYTES;
  // full (operands) / empty / scales-ready / scales-landed per stage, accf,
  // acce, and the drain barriers of the MMA issuer and the scale copier
  static constexpr int NUM_BARS = 4 * STAGES + 4;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_TAB0 = OFF_MISC + 16;
  // (the groups' offsets / masks are read from global memory where needed:
  // a second table here would leave no room on the SM for another kernel's
  // CTA without shared memory, e.g. a quantisation running underneath)
  static constexpr int BYTES = OFF_TAB0 + (kMaxGroups + 1) * 4;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM scale buffer of one stage: per K chunk [SFA 4 cols | SFB 8 cols]
  static constexpr uint32_t SF_CHUNK_COLS = 4 + 8;
  static constexpr uint32_t SF_COLS = kPairKC * SF_CHUNK_COLS;
  static constexpr uint32_t SF_COL0 = kPairN;
  static_assert(SF_COL0 + STAGES * SF_COLS <= TMEM_COLS, "TMEM budget");  // one scale buffer per stage
  static_assert(OFF_B % 1024 == 0 && OFF_SFA % 1024 == 0, "swizzled tiles need 1024-B alignment");
  static_assert(ALLOC <= 232448, "shared memory budget");
};

struct PairTile {
  int group;
  int row0;      // first of the tile's 256 A/D rows (absolute for dense/contiguous, within the expert if masked)
  int rows_end;  // rows at or beyond this are not stored
  int n_blk;     // 256-wide column block
};

// Group i's row offset (contiguous), token offset (K-grouped; i in [0,
// groups]) or valid rows clamped to [0, m] (masked; i < groups), from global
// memory (read once per tile, cached).
__device__ __forceinline__ int32_t group_val(const GemmArgs& a, int i) {
  if (a.mode == kMasked) {
    const int32_t mm = __ldg(a.masked_m + i);
    return mm < 0 ? 0 : (mm > a.m ? a.m : mm);
  }
  return __ldg(a.group_offsets + i);
}

__device__ __forceinline__ PairTile decode_pair_tile(const GemmArgs& a, const int32_t* tab0, int t) {
  PairTile r;
  if (a.mode == kDense) {
    const int mb = t / a.n_tiles;
    r.group = 0;
    r.n_blk = t - mb * a.n_tiles;
    r.row0 = mb * kPairM;
    r.rows_end = a.m;
  } else {
    const int e = last_le(tab0, a.groups, t);  // tab0: prefix of pair tiles per expert
    const int local = t - tab0[e];
    const int mb = local / a.n_tiles;
    r.group = e;
    r.n_blk = local - mb * a.n_tiles;
    if (a.mode == kContiguous) {
      r.row0 = group_val(a, e) + mb * kPairM;
      r.rows_end = group_val(a, e + 1);
    } else if (a.mode == kKGrouped) {  // every expert has the full [m, n] output
      r.row0 = mb * kPairM;
      r.rows_end = a.m;
    } else {  // masked
      r.row0 = mb * kPairM;
      r.rows_end = group_val(a, e);
    }
  }
  return r;
}

// ---------------------------------------------------------------- fused SwiGLU + MXFP8 epilogue

// h = silu(g) * u in FP32, with the logistic function evaluated on -|g| so
// that neither the exponential nor the division can overflow.
__device__ __forceinline__ float swiglu_f32(float g, float u) {
  const float t = __expf(-fabsf(g));       // (0, 1]
  const float r = __fdividef(1.0f, 1.0f + t);  // sigmoid(|g|)
  const float sig = g >= 0.0f ? r : t * r;     // sigmoid(g)
  return g * sig * u;
}

template <int STAGES, bool SWIGLU>
__global__ void __launch_bounds__(kGemmThreads, 1)
    mx_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                        const __grid_constant__ CUtensorMap tmap_d, const __grid_constant__ CUtensorMap tmap_sfa,
                        const __grid_constant__ CUtensorMap tmap_sfb, const GemmArgs args) {
  using L = PairLayout<STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader of the pair
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int npairs = static_cast<int>(gridDim.x) >> 1;

  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile uint32_t* tmem_slot = misc + 0;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* total_slot = reinterpret_cast<volatile int*>(misc + 2);
  int32_t* tab0 = reinterpret_cast<int32_t*>(smem + L::OFF_TAB0);

  auto full_bar = [&](int s) { return sbase + L::OFF_BAR + 8u * s; };
  auto empty_bar = [&](int s) { return sbase + L::OFF_BAR + 8u * (STAGES + s); };
  const uint32_t accf_bar = sbase + L::OFF_BAR + 8u * (2 * STAGES);
  const uint32_t acce_bar = sbase + L::OFF_BAR + 8u * (2 * STAGES + 1);
  const uint32_t drain_bar = sbase + L::OFF_BAR + 8u * (2 * STAGES + 2);
  const uint32_t sf_drain_bar = sbase + L::OFF_BAR + 8u * (2 * STAGES + 3);
  auto sfready_bar = [&](int s) { return sbase + L::OFF_BAR + 8u * (2 * STAGES + 4 + s); };
  auto sffull_bar = [&](int s) { return sbase + L::OFF_BAR + 8u * (3 * STAGES + 4 + s); };

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);   // the leader's producer announces both CTAs' bytes
      mbar_init(empty_bar(s), 1);  // the leader's commit, multicast to both CTAs
      mbar_init(sfready_bar(s), 1);  // the leader's scale-copy commit (leader only)
      mbar_init(sffull_bar(s), 1);   // the leader's producer announces both CTAs' scale bytes
    }
    mbar_init(accf_bar, 1);
    mbar_init(acce_bar, 8);        // one lane of each epilogue warp of both CTAs, after the warp's loads
    mbar_init(drain_bar, 1);
    mbar_init(sf_drain_bar, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_d);
    prefetch_tmap(&tmap_sfa);
    prefetch_tmap(&tmap_sfb);
  }
  pdl_launch_dependents();
  pdl_wait_prior();

  // scheduling table: tab0 = exclusive prefix of pair tiles per expert,
  // after checking the offsets (contiguous, K-grouped) or masks (masked)
  int bad = 0;
  if (args.mode != kDense) {
    if (args.mode == kContiguous || args.mode == kKGrouped) {
      // offsets along M (contiguous) or along K (K-grouped: the token ranges)
      const int limit = args.mode == kContiguous ? args.m : args.k_tiles * BK;
      for (int i = threadIdx.x; i <= args.groups; i += blockDim.x) {
        const int32_t v = __ldg(args.group_offsets + i);
        if (v < 0 || (v % BM) != 0 || v > limit) bad = 1;
        if (i > 0 && v < __ldg(args.group_offsets + i - 1)) bad = 1;
      }
    } else {
      for (int i = threadIdx.x; i < args.groups; i += blockDim.x) {
        const int32_t mm = __ldg(args.masked_m + i);
        if (mm < 0 || mm > args.m) bad = 1;  // clamped where it is read (group_val)
      }
    }
    bad = __syncthreads_or(bad);
    if (warp == 0) {
      const int per = (args.groups + 31) / 32;
      const int lo = lane * per;
      auto tiles_of = [&](int e) -> int {
        if (args.mode == kKGrouped) return bad ? 0 : (args.m + kPairM - 1) / kPairM * args.n_tiles;
        const int rows = args.mode == kContiguous ? (bad ? 0 : group_val(args, e + 1) - group_val(args, e))
                                                  : group_val(args, e);
        return (rows + kPairM - 1) / kPairM * args.n_tiles;
      };
      int sum = 0;
      for (int i = lo; i < lo + per && i < args.groups; ++i) sum += tiles_of(i);
      int incl = sum;
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += y;
      }
      int run = incl - sum;
      for (int i = lo; i < lo + per && i < args.groups; ++i) {
        tab0[i] = run;
        run += tiles_of(i);
      }
      if (lane == 31) tab0[args.groups] = incl;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(tmem_slot)), L::TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (threadIdx.x == 0) {
    int total;
    if (args.mode == kDense) {
      total = ((args.m + kPairM - 1) / kPairM) * args.n_tiles;
    } else {
      total = tab0[args.groups];
      if (bad && rank == 0) report(args.status, args.mode == kMasked ? 0x2 : 0x1);
    }
    *total_slot = total;
  }
  // barriers initialised and TMEM allocated in BOTH CTAs before any cross-CTA traffic
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = *total_slot;
  // K range of a tile in 128-byte chunks: all of K, or (K-grouped) the
  // expert's own token range [off[e], off[e+1])
  auto tile_kc0 = [&](const PairTile& tl) -> int {
    return args.mode == kKGrouped ? group_val(args, tl.group) / BK : 0;
  };
  auto tile_chunks = [&](const PairTile& tl) -> int {
    return args.mode == kKGrouped ? (group_val(args, tl.group + 1) - group_val(args, tl.group)) / BK : args.k_tiles;
  };

  // ---------------------------------------------------------------- roles
  if (warp == 0) {
    if (lane == 0) {
      // ===== TMA producer (both CTAs); every load completes on a barrier of
      // the leader: the scale tiles on the stage's "scales landed" barrier,
      // issued first, so that the copier moves them into TMEM while the
      // operands are still in flight and the MMAs wait for the operands only
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      // the leader announces the bytes of both CTAs' loads for a stage (boxes
      // reaching past the tensor are zero-filled and still count in full)
      const uint32_t bytes_ab = 2u * (L::A_BYTES + L::B_BYTES);
      const uint32_t bytes_sf = 2u * (L::SFA_BYTES + L::SFB_BYTES);
      for (int t = pair; t < total && ok; t += npairs) {
        const PairTile tl = decode_pair_tile(args, tab0, t);
        const int a_row = tl.row0 + 128 * static_cast<int>(rank);
        const int a_z = args.mode == kMasked ? tl.group : 0;
        const int b_z = (args.mode == kDense || args.mode == kKGrouped) ? 0 : tl.group;
        // SwiGLU: CTA 0 takes the 128 gate rows and CTA 1 the matching 128 up
        // rows of the column block, so each CTA's accumulator row holds
        // [gate | up] of the same 128 output columns
        const int b_row = SWIGLU ? (rank != 0 ? args.swiglu_i : 0) + tl.n_blk * 128
                                 : tl.n_blk * kPairN + 128 * static_cast<int>(rank);
        // scale regions as [128-row block][K chunk] of 512-byte chunks
        const int sfa_blk =
            (args.mode == kMasked ? tl.group * static_cast<int>(args.sfa_group_bytes / 512 / args.k_tiles) : 0) +
            a_row / 128;
        const int sfb_grp = (args.mode == kDense || args.mode == kKGrouped) ? 0 : tl.group * args.n_sf_tiles;
        const int sfb_blk = sfb_grp + (SWIGLU ? tl.n_blk : tl.n_blk * 2);
        const int kc0 = tile_kc0(tl);
        const int k_stages = (tile_chunks(tl) + kPairKC - 1) / kPairKC;
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, args.wait_ns)) { ok = false; break; }
          const uint32_t fb = map_to_rank(full_bar(stage), 0);
          const uint32_t sb = map_to_rank(sffull_bar(stage), 0);
          if (rank == 0) {
            mbar_arrive_expect_tx(sffull_bar(stage), bytes_sf);
            mbar_arrive_expect_tx(full_bar(stage), bytes_ab);
          }
          const int kc = kc0 + ks * kPairKC;
          tma_load_3d_pair(sbase + L::OFF_SFA + stage * L::SFA_BYTES, &tmap_sfa, sb, 0, kc, sfa_blk);
          if (SWIGLU) {  // gate and up scale blocks are i/128 blocks apart: two boxes of one block
            tma_load_3d_pair(sbase + L::OFF_SFB + stage * L::SFB_BYTES, &tmap_sfb, sb, 0, kc, sfb_blk);
            tma_load_3d_pair(sbase + L::OFF_SFB + stage * L::SFB_BYTES + kPairKC * 512, &tmap_sfb, sb, 0, kc,
                             sfb_blk + args.swiglu_i / 128);
          } else {
            tma_load_3d_pair(sbase + L::OFF_SFB + stage * L::SFB_BYTES, &tmap_sfb, sb, 0, kc, sfb_blk);
          }
          tma_load_4d_pair(sbase + L::OFF_A + stage * L::A_BYTES, &tmap_a, fb, 0, a_row, kc, a_z);
          tma_load_4d_pair(sbase + L::OFF_B + stage * L::B_BYTES, &tmap_b, fb, 0, b_row, kc, b_z);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {  // loads already in flight land during the teardown's linger
        report(args.status, 0x4);
        *abort_flag = 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ===== MMA issuer (leader only): wait for a stage's scales, 4 pair MMAs, commit
      const uint32_t idesc0 = idesc_mxf8_e4m3(kPairM, kPairN);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs) {
        if (!mbar_wait(acce_bar, acc_phase ^ 1u, abort_flag, args.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const int chunks = tile_chunks(decode_pair_tile(args, tab0, t));
        const int k_stages = (chunks + kPairKC - 1) / kPairKC;
        for (int ks = 0; ks < k_stages; ++ks) {
          // both CTAs' operands of the stage have landed, and its scales are in TMEM
          if (!mbar_wait(full_bar(stage), phase, abort_flag, args.wait_ns)) { ok = false; break; }
          if (!mbar_wait(sfready_bar(stage), phase, abort_flag, args.wait_ns)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < kPairKC; ++c) {
            // a chunk past K holds zeros with zero-code scales and adds nothing;
            // in the K-grouped form a chunk past the expert's tokens belongs to
            // the next expert and is skipped
            if (args.mode == kKGrouped && ks * kPairKC + c >= chunks) break;
            const uint32_t sfa_t = tmem_base + L::SF_COL0 + stage * L::SF_COLS + c * L::SF_CHUNK_COLS;
            const uint32_t sfb_t = sfa_t + 4;
            const uint32_t a_addr = sbase + L::OFF_A + stage * L::A_BYTES + c * L::CHUNK;
            const uint32_t b_addr = sbase + L::OFF_B + stage * L::B_BYTES + c * L::CHUNK;
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
              const uint32_t idesc = idesc_with_sf_ids(idesc0, kb, kb);
              tc_mma_pair_mxf8(tmem_base, desc_kmajor_sw128(a_addr + 32 * kb),
                               desc_kmajor_sw128(b_addr + 32 * kb), idesc,
                               sfa_t | (static_cast<uint32_t>(kb) << 30), sfb_t | (static_cast<uint32_t>(kb) << 30),
                               (ks != 0 || c != 0 || kb != 0) ? 1u : 0u);
            }
          }
          tc_commit_pair_multicast(empty_bar(stage), 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_multicast(accf_bar, 0x3);
        acc_phase ^= 1u;
      }
      if (!ok) {
        report(args.status, 0x4);
        *abort_flag = 1;
      }
      // every pair MMA issued must finish before either CTA frees its TMEM
      // (also when another role gave up while they ran)
      tc_commit_pair_multicast(drain_bar, 0x1);
      mbar_wait(drain_bar, 0, nullptr, 100000000ull);
    }
  } else if (warp == 6) {
    if (lane == 0 && rank == 0) {
      // ===== scale copier (leader only): once both CTAs' scale tiles of
      // stage s have landed, copy each CTA's scale chunks into its TMEM scale
      // buffer s.  Buffer s is free again once the stage's MMAs completed,
      // which both producers have seen (empty) before refilling the stage.
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs) {
        const int k_stages = (tile_chunks(decode_pair_tile(args, tab0, t)) + kPairKC - 1) / kPairKC;
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait(sffull_bar(stage), phase, abort_flag, args.wait_ns)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < kPairKC; ++c) {
            const uint32_t sfa_t = tmem_base + L::SF_COL0 + stage * L::SF_COLS + c * L::SF_CHUNK_COLS;
            const uint32_t sfb_s = sbase + L::OFF_SFB + stage * L::SFB_BYTES + c * 512;
            tc_cp_pair_32x128b_warpx4(sfa_t, desc_sf_32x16(sbase + L::OFF_SFA + stage * L::SFA_BYTES + c * 512));
            tc_cp_pair_32x128b_warpx4(sfa_t + 4, desc_sf_32x16(sfb_s));
            tc_cp_pair_32x128b_warpx4(sfa_t + 8, desc_sf_32x16(sfb_s + kPairKC * 512));
          }
          tc_commit_pair_multicast(sfready_bar(stage), 0x1);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        report(args.status, 0x4);
        *abort_flag = 1;
      }
      // copies still in flight must land before TMEM is freed
      tc_commit_pair_multicast(sf_drain_bar, 0x1);
      mbar_wait(sf_drain_bar, 0, nullptr, 100000000ull);
    }
  } else {
    // ===== epilogue (both CTAs): this CTA's 128 accumulator rows
    const int quarter = warp & 3;
    const int r_local = quarter * 32 + lane;
    const uint32_t acce_leader = map_to_rank(acce_bar, 0);
    uint32_t acc_phase = 0;
    uint32_t stg_count = 0;
    for (int t = pair; t < total; t += npairs) {
      const bool got = mbar_wait(accf_bar, acc_phase, abort_flag, args.wait_ns);
      if (!named_barrier_and(2, 128, got)) {
        if (threadIdx.x == 64) report(args.status, 0x4);
        *abort_flag = 1;
        break;
      }
      acc_phase ^= 1u;
      tc_fence_after();
      const PairTile tl = decode_pair_tile(args, tab0, t);
      const int my_row0 = tl.row0 + 128 * static_cast<int>(rank);
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
      // dense rows past M are clipped by the tensor map; grouped rows past the
      // expert are not ours to write
      const bool dense_rows = args.mode == kDense || args.mode == kKGrouped;
      const bool full = dense_rows ? my_row0 < tl.rows_end : my_row0 + 128 <= tl.rows_end;
      const bool none = my_row0 >= tl.rows_end;
      if constexpr (SWIGLU) {
        // ---- H = silu(gate) * up, requantised to MXFP8 along its columns:
        // each thread owns one row, so a 32-column block is thread-local
        if (none) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acce_leader);
          continue;
        }
        // H for the row's 128 columns first; the accumulator goes back to the
        // MMA warp before the requantisation
        float h[4][32];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          uint32_t g[32], u[32];
          tc_ld_32x32b_x32(t_row + b * 32, g);
          tc_ld_32x32b_x32(t_row + 128 + b * 32, u);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) h[b][j] = swiglu_f32(__uint_as_float(g[j]), __uint_as_float(u[j]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acce_leader);  // TMEM back to the leader's MMA warp before any store
        uint32_t qw[32];  // the row's 128 E4M3 bytes
        uint32_t sfw = 0; // its 4 scale bytes (column blocks 4*n_blk .. 4*n_blk+3)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          uint32_t q8[8];
          sfw |= quant_block32_f32(h[b], q8) << (8 * b);
#pragma unroll
          for (int i = 0; i < 8; ++i) qw[b * 8 + i] = q8[i];
        }
        const int r = my_row0 + r_local;   // absolute row (dense, contiguous) or row within the expert (masked)
        const bool valid = r < tl.rows_end;
        // scales: the 4 bytes of this row for column blocks 4*n_blk..+3 are
        // adjacent in the tiled layout (rows padded to 128, i/128 tiles per row block)
        uint8_t* sfh = args.sfh + (args.mode == kMasked ? tl.group * args.sfh_group_bytes : 0);
        const int64_t sf_off = (static_cast<int64_t>(r >> 7) * (args.swiglu_i / 128) + tl.n_blk) * 512 +
                               (r & 31) * 16 + ((r & 127) >> 5) * 4;
        if (valid)
          *reinterpret_cast<uint32_t*>(sfh + sf_off) = sfw;
        else if (args.mode == kDense)
          *reinterpret_cast<uint32_t*>(sfh + sf_off) = 0u;  // scale padding rows of the last row block
        if (full) {
          store_words_tma<32, 64>(qw, r_local, sbase + L::OFF_STG, stg_count, &tmap_d, tl.n_blk * 128, my_row0,
                                  args.mode == kMasked ? tl.group : 0);
        } else if (valid) {
          // masked expert ending inside this CTA's rows: row-predicated stores
          uint4* hrow = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(args.d) +
                                                 (static_cast<int64_t>(tl.group) * args.m + r) * args.swiglu_i +
                                                 tl.n_blk * 128);
#pragma unroll
          for (int i = 0; i < 8; ++i) hrow[i] = make_uint4(qw[4 * i], qw[4 * i + 1], qw[4 * i + 2], qw[4 * i + 3]);
        }
        continue;
      }
      if (none) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acce_leader);
      } else if (full) {
        uint32_t packed[kPairN / 2];
        if (args.mode == kKGrouped && tile_chunks(tl) == 0) {
#pragma unroll
          for (int j = 0; j < kPairN / 2; ++j) packed[j] = 0u;  // an expert with no tokens has a zero gradient
        } else {
          tmem_row_to_bf16<kPairN>(t_row, packed);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acce_leader);  // TMEM back to the leader's MMA warp before any store
        store_rows_tma<kPairN>(packed, r_local, sbase + L::OFF_STG, stg_count, &tmap_d, tl.n_blk * kPairN, my_row0,
                               (args.mode == kMasked || args.mode == kKGrouped) ? tl.group : 0);
      } else {
        // masked expert ending inside this CTA's rows: row-predicated stores
        const int r = my_row0 + r_local;
        const bool valid = r < tl.rows_end;
        __nv_bfloat16* drow_ptr = args.d + (static_cast<int64_t>(tl.group) * args.m + r) * args.n;
#pragma unroll 1
        for (int c = 0; c < kPairN / 32; ++c) {
          uint32_t v[32];
          tc_ld_32x32b_x32(t_row + c * 32, v);
          tc_wait_ld();
          const int col0 = tl.n_blk * kPairN + c * 32;
          if (valid) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int col = col0 + g * 8;
              if (col < args.n) {
                uint4 w;
                w.x = pack_bf16x2(v[g * 8 + 0], v[g * 8 + 1]);
                w.y = pack_bf16x2(v[g * 8 + 2], v[g * 8 + 3]);
                w.z = pack_bf16x2(v[g * 8 + 4], v[g * 8 + 5]);
                w.w = pack_bf16x2(v[g * 8 + 6], v[g * 8 + 7]);
                *reinterpret_cast<uint4*>(drow_ptr + col) = w;
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acce_leader);
      }
    }
    if (threadIdx.x == 64) bulk_wait_group_all();
  }

  // ---------------------------------------------------------------- teardown
  // neither CTA may leave while its peer can still signal its barriers,
  // read its shared memory or write its TMEM; a CTA that gave up lingers
  // before the second barrier, which keeps its peer resident too (the
  // peer's loads complete on the leader's barriers)
  tc_fence_before();
  cluster_sync();
  if (threadIdx.x == 0 && *abort_flag) linger_after_abort();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
  }
}

// ======================================================================= host

// Operand [depth, rows, k] bytes viewed as 4-D {128, rows, k/128, depth}: one
// box of {128, 128, kPairKC, 1} brings kPairKC consecutive K chunks of 128
// rows, each landing as its own 16 KB 128-byte-swizzled tile.
static bool make_tmap_kc(CUtensorMap* m, const void* base, int64_t k, int64_t rows, int64_t depth) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(k / 128),
                              static_cast<cuuint64_t>(depth)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(k), 128, static_cast<cuuint64_t>(k * rows)};
  const cuuint32_t box[4] = {128, 128, kPairKC, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tiled scale region viewed as 3-D {128 words, K chunks, 128-row blocks}: one
// 512-byte chunk is one box row of 32-bit words (a single TMA request), and a
// box of {128, kPairKC, blocks} brings the chunks of kPairKC consecutive K
// chunks for `blocks` consecutive 128-row blocks.  Chunks past K are
// zero-filled (scale code 0x00), so they scale zeros to zero.
static bool make_tmap_sf(CUtensorMap* m, const void* base, int64_t bytes, int64_t k_chunks, int blocks) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t nblk = static_cast<cuuint64_t>(bytes / 512 / k_chunks);
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(k_chunks), nblk};
  const cuuint64_t strides[2] = {512, static_cast<cuuint64_t>(512 * k_chunks)};
  const cuuint32_t box[3] = {128, kPairKC, static_cast<cuuint32_t>(blocks)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int STAGES, bool SWIGLU>
static cudaError_t prepare_pair_kernel() {
  static cudaError_t state = cudaErrorNotReady;
  if (state == cudaErrorNotReady)
    state = cudaFuncSetAttribute(mx_gemm_pair_kernel<STAGES, SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 PairLayout<STAGES>::ALLOC);
  return state;
}

// Pairs the GPU holds at once (one per two SMs when nothing else runs).
int pair_kernel_max_pairs(int num_sms) {
  static int v = -1;
  if (v < 0) {
    v = num_sms / 2;
    if (prepare_pair_kernel<kPairStages, false>() == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      cfg.gridDim = dim3(2, 1, 1);
      cfg.blockDim = dim3(kGemmThreads, 1, 1);
      cfg.dynamicSmemBytes = PairLayout<kPairStages>::ALLOC;
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, mx_gemm_pair_kernel<kPairStages, false>, &cfg) == cudaSuccess && n > 0) v = n;
      cudaGetLastError();
    }
  }
  return v;
}

template <bool SWIGLU>
static cudaError_t launch_pair(const GemmProblem& p, int num_sms, cudaStream_t stream, int* launches) {
  constexpr int STAGES = kPairStages;
  using L = PairLayout<STAGES>;
  {
    cudaError_t e = prepare_pair_kernel<STAGES, SWIGLU>();
    if (e != cudaSuccess) return e;
  }
  if (SWIGLU && (p.i_dim <= 0 || p.i_dim % 128 != 0 || p.n != 2 * p.i_dim || !p.sf_out))
    return cudaErrorInvalidValue;
  CUtensorMap ta, tb, td, tsa, tsb;
  const int64_t a_depth = p.mode == kMasked ? p.groups : 1;
  const int64_t b_depth = (p.mode == kDense || p.mode == kKGrouped) ? 1 : p.groups;
  const int64_t d_depth = (p.mode == kMasked || p.mode == kKGrouped) ? p.groups : 1;  // K-grouped: D [groups, m, n]
  const int64_t sfa_bytes = a_depth * (((p.m + 127) / 128) * 128 * (p.k / 32));
  const int64_t sfb_bytes = b_depth * (((p.n + 127) / 128) * 128 * (p.k / 32));
  if (!make_tmap_kc(&ta, p.qa, p.k, p.m, a_depth)) return cudaErrorInvalidValue;
  if (!make_tmap_kc(&tb, p.qb, p.k, p.n, b_depth)) return cudaErrorInvalidValue;
  if (SWIGLU) {
    if (!make_tmap_h(&td, p.d, p.i_dim, p.m, d_depth)) return cudaErrorInvalidValue;
  } else {
    if (!make_tmap_d(&td, p.d, p.n, p.m, d_depth)) return cudaErrorInvalidValue;
  }
  if (!make_tmap_sf(&tsa, p.sfa, sfa_bytes, p.k / BK, 1)) return cudaErrorInvalidValue;
  if (!make_tmap_sf(&tsb, p.sfb, sfb_bytes, p.k / BK, SWIGLU ? 1 : 2)) return cudaErrorInvalidValue;

  GemmArgs a = {};
  a.sfa = static_cast<const uint8_t*>(p.sfa);
  a.sfb = static_cast<const uint8_t*>(p.sfb);
  a.d = static_cast<__nv_bfloat16*>(p.d);
  a.group_offsets = p.group_offsets;
  a.masked_m = p.masked_m;
  a.status = p.status;
  a.wait_ns = wait_limit_ns();
  a.k_tiles = static_cast<int>(p.k / BK);
  a.sfa_group_bytes = ((p.m + 127) / 128) * 128 * (p.k / 32);
  a.sfb_group_bytes = ((p.n + 127) / 128) * 128 * (p.k / 32);
  a.m = static_cast<int>(p.m);
  a.n = static_cast<int>(p.n);
  // a SwiGLU tile yields 128 output columns from 128 gate + 128 up rows
  a.n_tiles = SWIGLU ? static_cast<int>(p.i_dim / 128) : static_cast<int>((p.n + kPairN - 1) / kPairN);
  a.n_sf_tiles = static_cast<int>((p.n + 127) / 128);
  a.groups = static_cast<int>(p.groups);
  a.mode = p.mode;
  a.a_box_rows = 128;
  if (SWIGLU) {
    a.swiglu_i = static_cast<int>(p.i_dim);
    a.sfh = static_cast<uint8_t*>(p.sf_out);
    a.sfh_group_bytes = ((p.m + 127) / 128) * 128 * (p.i_dim / 32);
  }

  // upper bound of pair tiles (grouped forms: every expert full)
  int64_t m_blocks;
  if (p.mode == kDense)
    m_blocks = (p.m + kPairM - 1) / kPairM;
  else if (p.mode == kMasked || p.mode == kKGrouped)
    m_blocks = p.groups * ((p.m + kPairM - 1) / kPairM);
  else
    m_blocks = p.m / 128 / 2 + p.groups;  // each expert adds at most one half-used pair tile
  const int64_t tiles_bound = m_blocks * a.n_tiles;
  if (tiles_bound == 0) return cudaSuccess;
  const int64_t max_pairs = pair_kernel_max_pairs(num_sms);
  const int64_t pairs = tiles_bound < max_pairs ? tiles_bound : max_pairs;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3(static_cast<unsigned>(pairs * 2), 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = L::ALLOC;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, mx_gemm_pair_kernel<STAGES, SWIGLU>, ta, tb, td, tsa, tsb, a);
  if (e != cudaSuccess) return e;
  if (launches) *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_gemm_pair(const GemmProblem& p, int num_sms, cudaStream_t stream, int* launches) {
  return p.i_dim > 0 ? launch_pair<true>(p, num_sms, stream, launches) : launch_pair<false>(p, num_sms, stream, launches);
}

}  // namespace mxk
