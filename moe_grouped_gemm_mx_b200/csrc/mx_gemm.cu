// mx_gemm.cu -- MXFP8 block-scaled GEMM kernels for sm_100a (B200).
//
// One persistent, warp-specialised kernel serves the three GEMM forms the
// DeepGEMM pages list ("DeepGEMM" summary page: a plain FP8 GEMM plus MoE
// grouped GEMMs in contiguous and masked layouts; DeepGEMM release page,
// section 4), in the MXFP8 number format of the B200 MoE-training page
// (32-element UE8M0 block scales, FP32 accumulation, BF16 output).
//
//   D[m, n] = sum_b 2^(sa[m,b] + sb[n,b]) * sum_{k in b} e4m3(qa[m,k]) * e4m3(qb[n,k])
//
// CTA layout (224 threads, one CTA per SM):
//   warp 0      TMA producer: A/B tiles (128-byte swizzled, 3-D tensor maps so
//               experts never bleed into each other) and the 512-byte scale
//               tiles (plain bulk copies) into a STAGES-deep shared-memory ring.
//   warp 6      scale copier: as each stage lands, tcgen05.cp its scale tiles
//               into that stage's own TMEM scale buffer and commit to the
//               stage's "scales ready" barrier.
//   warp 1      TMEM owner + MMA issuer: per K-tile, wait for "scales ready",
//               then 4 x tcgen05.mma kind::mxf8f6f4.block_scale (K = 32 each,
//               scale byte k selected by the scale-factor ids), accumulating a
//               128 x BN FP32 tile in TMEM.  tcgen05.commit frees ring slots
//               and publishes finished accumulators.  One 128 x 256 x 32 MMA
//               keeps the tensor pipe busy for about as long as a thread needs
//               to issue two tcgen05 instructions, so the issuer does nothing
//               but wait, issue the MMAs and commit.
//   warps 2..5  epilogue: tcgen05.ld the accumulator (each warp owns the TMEM
//               lane quarter its warp id selects), round to BF16 and store the
//               valid rows/columns.
// The tile scheduler is a static stride over a linear tile index; grouped
// forms map the index to (expert, m-block, n-block) with a table built in
// shared memory from the device-resident offsets / masks, so no host
// synchronisation is needed.  The Hopper-era two-level CUDA-core accumulation
// of the pages is unnecessary here: the tensor core accumulates in FP32 in TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstdlib>

#include "mx_gemm_common.cuh"
#include "mx_launch.h"

namespace mxk {

// BMA: rows of A one stage holds (128, or 64 for a dense M <= 64, which frees
// shared memory for deeper pipelining; the M=128 MMA then also reads the next
// 64 rows of shared memory, which only feed accumulator rows never stored).
template <int BN, int STAGES, int ACC, int SPLIT = 1, int BMA = BM>
struct Layout {
  static constexpr int A_BYTES = BMA * BK;
  static constexpr int B_BYTES = BN * BK;
  static constexpr int SFA_BYTES = 512;
  static constexpr int SFB_TILES = BN / 128;
  static constexpr int SFB_BYTES = SFB_TILES * 512;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
  // epilogue staging: two 128-row x 32-column BF16 chunks (64-byte rows,
  // 64-byte swizzle) that TMA stores read while the next chunk is written
  static constexpr int STG_BYTES = BM * 32 * 2;
  static constexpr int OFF_STG = (OFF_SFB + STAGES * SFB_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_BAR = OFF_STG + 2 * STG_BYTES;
  // full / empty / scales-ready per stage, full / empty per accumulator, and
  // the two drain barriers (MMA issuer, scale copier) used when giving up
  static constexpr int NUM_BARS = 3 * STAGES + 2 * ACC + 2;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_TAB0 = OFF_MISC + 16;
  static constexpr int OFF_TAB1 = OFF_TAB0 + (kMaxGroups + 1) * 4;
  static constexpr int BYTES = OFF_TAB1 + (kMaxGroups + 1) * 4;
  static constexpr int ALLOC = BYTES + 1024;  // room to align the base to 1024 B
  static constexpr uint32_t TMEM_COLS = 512;
  // scale factors in TMEM: one buffer per pipeline stage of
  // [SFA 4 cols | SFB 4 cols per 128 rows of B]
  static constexpr uint32_t SF_COLS = 4 + 4 * SFB_TILES;
  static constexpr uint32_t SF_COL0 = ACC * BN;
  static_assert(BN % 128 == 0 && BN <= 256, "BN must be 128 or 256");
  static_assert(SF_COL0 + STAGES * SF_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(OFF_B % 1024 == 0 && OFF_SFA % 1024 == 0, "swizzled tiles need 1024-B alignment");
  static_assert(BYTES + 1024 <= 232448, "shared memory budget");
  // split-K reduction buffer (reuses the operand ring once the mainloop is
  // done): SPLIT partial slices of 128 rows x BN/SPLIT FP32 columns, rows
  // padded by 4 floats to spread shared-memory banks.
  // Columns are dealt out in quads of 4: CTA o of the cluster owns quads
  // [ceil(o*QUADS/SPLIT), ceil((o+1)*QUADS/SPLIT)).
  static constexpr int QUADS = BN / 4;
  // Receive buffer: [source rank][quad of the slice][row] of float4, rows
  // fastest, so the 32 lanes of a warp (32 consecutive rows) write 512
  // contiguous bytes per remote store and read them back conflict-free.
  static constexpr int MAX_SLICE_QUADS = (QUADS + SPLIT - 1) / SPLIT;
  static constexpr int RED_BYTES = SPLIT * MAX_SLICE_QUADS * BM * 16;
  static_assert(SPLIT == 1 || RED_BYTES <= OFF_BAR, "reduction buffer must fit in the operand ring");
  __host__ __device__ static constexpr int slice_start(int o) { return (o * QUADS + SPLIT - 1) / SPLIT; }
  __host__ __device__ static constexpr int quad_owner(int q) { return (q * SPLIT) / QUADS; }
};

// How the tiles of a problem are shared out.  Tiles [0, bulk) are whole-K
// tiles dealt round robin: a CTA takes first, first + stride, ...  After
// them, cluster `cluster` (of cs CTAs) shares at most one more tile, bulk +
// cluster, each CTA accumulating the K tiles of its rank's share; the cluster
// reduces those partials through distributed shared memory.  `bulk` is all
// tiles (persistent CTAs) or none (one split tile per cluster).
enum BulkMode : int { kBulkAll = 0, kBulkNone = 1 };

struct CtaSchedule {
  int first, stride, cluster, cs, rank, bulk, total, k_tiles;
  __device__ __forceinline__ int split_tile() const {
    return (cs > 1 && bulk + cluster < total) ? bulk + cluster : total;
  }
  __device__ __forceinline__ int begin() const { return first < bulk ? first : split_tile(); }
  __device__ __forceinline__ int next(int t) const {
    if (t >= bulk) return total;
    return t + stride < bulk ? t + stride : split_tile();
  }
  __device__ __forceinline__ bool split(int t) const { return t >= bulk; }
  __device__ __forceinline__ int kt_begin(int t) const { return t >= bulk ? rank * k_tiles / cs : 0; }
  __device__ __forceinline__ int kt_end(int t) const { return t >= bulk ? (rank + 1) * k_tiles / cs : k_tiles; }
};

// One CTA of the GEMM on the problem in `args` (operands through the three
// tensor maps): the tiles of its schedule (CtaSchedule; `bulk` from
// bulk_mode once the tile count is known on the device).  Split tiles need
// cs == SPLIT_MAX; every CTA of a cluster has the same schedule parameters.
template <int BN, int STAGES, int ACC, int SPLIT_MAX, int BMA>
__device__ __forceinline__ void gemm_cta(const CUtensorMap* tmap_a, const CUtensorMap* tmap_b,
                                         const CUtensorMap* tmap_d, const GemmArgs& args, const int bulk_mode,
                                         const int first, const int stride, const int cluster, const int cs,
                                         const int rank) {
  using L = Layout<BN, STAGES, ACC, SPLIT_MAX, BMA>;
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
  int32_t* tab1 = reinterpret_cast<int32_t*>(smem + L::OFF_TAB1);

  auto full_bar = [&](int s) { return sbase + L::OFF_BAR + 8u * s; };
  auto empty_bar = [&](int s) { return sbase + L::OFF_BAR + 8u * (STAGES + s); };
  auto accf_bar = [&](int a) { return sbase + L::OFF_BAR + 8u * (2 * STAGES + a); };
  auto acce_bar = [&](int a) { return sbase + L::OFF_BAR + 8u * (2 * STAGES + ACC + a); };
  auto sfready_bar = [&](int s) { return sbase + L::OFF_BAR + 8u * (2 * STAGES + 2 * ACC + s); };
  const uint32_t drain_bar = sbase + L::OFF_BAR + 8u * (3 * STAGES + 2 * ACC);
  const uint32_t sf_drain_bar = drain_bar + 8u;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
      mbar_init(sfready_bar(s), 1);
    }
    for (int a = 0; a < ACC; ++a) {
      mbar_init(accf_bar(a), 1);
      mbar_init(acce_bar(a), 128);
    }
    mbar_init(drain_bar, 1);
    mbar_init(sf_drain_bar, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(tmap_a);
    prefetch_tmap(tmap_b);
    prefetch_tmap(tmap_d);
  }
  // Everything above touches only this CTA's shared memory and the kernel
  // parameters.  With programmatic dependent launch the next kernel may begin
  // its own prologue now, and from here on we need the previous kernel's
  // results (operands, offsets) and may overwrite what it reads.
  pdl_launch_dependents();
  pdl_wait_prior();

  // scheduling tables
  int bad = 0;
  if (args.mode == kContiguous) {
    for (int i = threadIdx.x; i <= args.groups; i += blockDim.x) tab0[i] = __ldg(args.group_offsets + i);
    __syncthreads();
    for (int i = threadIdx.x; i <= args.groups; i += blockDim.x) {
      const int32_t v = tab0[i];
      if (v < 0 || (v % BM) != 0 || v > args.m) bad = 1;
      if (i > 0 && v < tab0[i - 1]) bad = 1;
    }
  } else if (args.mode == kMasked) {
    for (int i = threadIdx.x; i < args.groups; i += blockDim.x) {
      int32_t mm = __ldg(args.masked_m + i);
      if (mm < 0 || mm > args.m) {
        bad = 1;
        mm = mm < 0 ? 0 : args.m;
      }
      tab1[i] = mm;
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefix of tiles per expert, one warp
      const int per = (args.groups + 31) / 32;
      const int lo = lane * per;
      int sum = 0;
      for (int i = lo; i < lo + per && i < args.groups; ++i) sum += (tab1[i] + BM - 1) / BM * args.n_tiles;
      int incl = sum;
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += y;
      }
      int run = incl - sum;
      for (int i = lo; i < lo + per && i < args.groups; ++i) {
        tab0[i] = run;
        run += (tab1[i] + BM - 1) / BM * args.n_tiles;
      }
      if (lane == 31) tab0[args.groups] = incl;
    }
  }
  const int any_bad = __syncthreads_or(bad);

  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), L::TMEM_COLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    int total;
    if (args.mode == kDense) {
      total = ((args.m + BM - 1) / BM) * args.n_tiles;
    } else if (args.mode == kContiguous) {
      total = any_bad ? 0 : (tab0[args.groups] - tab0[0]) / BM * args.n_tiles;
      if (any_bad) report(args.status, 0x1);
    } else {
      total = tab0[args.groups];
      if (any_bad) report(args.status, 0x2);
    }
    *total_slot = total;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = *total_slot;
  CtaSchedule sch;
  sch.first = first;
  sch.stride = stride;
  sch.cluster = cluster;
  sch.cs = cs;
  sch.rank = rank;
  sch.total = total;
  sch.k_tiles = args.k_tiles;
  sch.bulk = bulk_mode == kBulkNone ? 0 : total;

  int red_acc = 0;  // epilogue threads: the accumulator holding this CTA's split tile

  // ---------------------------------------------------------------- roles
  if (warp == 0) {
    if (lane == 0) {
      // ===== TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = sch.begin(); t < total && ok; t = sch.next(t)) {
        const Tile tl = decode_tile(args, tab0, t);
        const int a_row = tl.m_blk * BM;
        const int a_z = (args.mode == kMasked) ? tl.group : 0;
        const int b_z = (args.mode == kDense) ? 0 : tl.group;
        const uint8_t* sfa_base = args.sfa + (args.mode == kMasked ? tl.group * args.sfa_group_bytes : 0) +
                                  static_cast<int64_t>(tl.m_blk) * args.k_tiles * 512;
        const uint8_t* sfb_grp = args.sfb + (args.mode == kDense ? 0 : tl.group * args.sfb_group_bytes);
        const int sfb_tile0 = tl.n_blk * L::SFB_TILES;
        int nsfb = args.n_sf_tiles - sfb_tile0;
        nsfb = nsfb > L::SFB_TILES ? L::SFB_TILES : nsfb;
        const int kt_begin = sch.kt_begin(t), kt_end = sch.kt_end(t);
        for (int kt = kt_begin; kt < kt_end; ++kt) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, args.wait_ns)) { ok = false; break; }
          // only the A rows that exist are loaded when M is small; the MMA's
          // remaining A rows read stale shared memory and only feed
          // accumulator rows that are never stored
          const uint32_t bytes = args.a_box_rows * BK + L::B_BYTES + L::SFA_BYTES + 512u * nsfb;
          mbar_arrive_expect_tx(full_bar(stage), bytes);
          tma_load_3d(sbase + L::OFF_A + stage * L::A_BYTES, tmap_a, full_bar(stage), kt * BK, a_row, a_z);
          tma_load_3d(sbase + L::OFF_B + stage * L::B_BYTES, tmap_b, full_bar(stage), kt * BK,
                      tl.n_blk * BN, b_z);
          bulk_load(sbase + L::OFF_SFA + stage * L::SFA_BYTES, sfa_base + kt * 512, 512, full_bar(stage));
          for (int j = 0; j < nsfb; ++j)
            bulk_load(sbase + L::OFF_SFB + stage * L::SFB_BYTES + j * 512,
                      sfb_grp + (static_cast<int64_t>(sfb_tile0 + j) * args.k_tiles + kt) * 512, 512,
                      full_bar(stage));
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
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
      const uint32_t idesc0 = idesc_mxf8_e4m3(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = sch.begin(); t < total && ok; t = sch.next(t)) {
        if (!mbar_wait(acce_bar(acc), acc_phase ^ 1u, abort_flag, args.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_t = tmem_base + acc * BN;
        const int kt_begin = sch.kt_begin(t), kt_end = sch.kt_end(t);
        for (int kt = kt_begin; kt < kt_end; ++kt) {
          // the copier's commit implies the stage's operands have landed too
          if (!mbar_wait(sfready_bar(stage), phase, abort_flag, args.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sfa_t = tmem_base + L::SF_COL0 + stage * L::SF_COLS;
          const uint32_t sfb_t = sfa_t + 4;
          const uint32_t a_addr = sbase + L::OFF_A + stage * L::A_BYTES;
          const uint32_t b_addr = sbase + L::OFF_B + stage * L::B_BYTES;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint32_t idesc = idesc_with_sf_ids(idesc0, kb, kb);
            tc_mma_mxf8(d_t, desc_kmajor_sw128(a_addr + 32 * kb), desc_kmajor_sw128(b_addr + 32 * kb), idesc,
                        sfa_t | (static_cast<uint32_t>(kb) << 30), sfb_t | (static_cast<uint32_t>(kb) << 30),
                        (kt != kt_begin || kb != 0) ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(accf_bar(acc));
        if (++acc == ACC) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) {
        report(args.status, 0x4);
        *abort_flag = 1;
      }
      // every MMA this thread issued must finish before TMEM is freed (also
      // when another role gave up while they ran)
      tc_commit(drain_bar);
      mbar_wait(drain_bar, 0, nullptr, 100000000ull);
    }
  } else if (warp == 6) {
    if (lane == 0) {
      // ===== scale copier: stage s's scale tiles -> TMEM scale buffer s.
      // The buffer is free again once the stage's MMAs completed, which the
      // producer has seen (empty) before it refilled the stage (full).
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = sch.begin(); t < total && ok; t = sch.next(t)) {
        for (int kt = sch.kt_begin(t); kt < sch.kt_end(t); ++kt) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, args.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sfa_t = tmem_base + L::SF_COL0 + stage * L::SF_COLS;
          tc_cp_32x128b_warpx4(sfa_t, desc_sf_32x16(sbase + L::OFF_SFA + stage * L::SFA_BYTES));
#pragma unroll
          for (int j = 0; j < L::SFB_TILES; ++j)
            tc_cp_32x128b_warpx4(sfa_t + 4 + 4 * j,
                                 desc_sf_32x16(sbase + L::OFF_SFB + stage * L::SFB_BYTES + j * 512));
          tc_commit(sfready_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        report(args.status, 0x4);
        *abort_flag = 1;
      }
      // copies still in flight must land before TMEM is freed
      tc_commit(sf_drain_bar);
      mbar_wait(sf_drain_bar, 0, nullptr, 100000000ull);
    }
  } else {
    // ===== epilogue (warps 2..5 -> TMEM lane quarters 2,3,0,1)
    const int quarter = warp & 3;
    const int r_local = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t stg_count = 0;  // staging chunks used so far (buffer = count & 1)
    for (int t = sch.begin(); t < total; t = sch.next(t)) {
      // every lane polls; the vote over all four epilogue warps re-converges
      // them before the warp-collective (.sync.aligned) TMEM loads and makes
      // the give-up decision uniform (the warps share named barriers below)
      const bool got = mbar_wait(accf_bar(acc), acc_phase, abort_flag, args.wait_ns);
      if (!named_barrier_and(2, 128, got)) {
        if (threadIdx.x == 64) report(args.status, 0x4);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      if (sch.split(t)) {  // the split-K reduction below finishes this tile
        red_acc = acc;
        break;
      }
      const Tile tl = decode_tile(args, tab0, t);
      int64_t drow;
      bool valid;
      if (args.mode == kMasked) {
        const int r = tl.m_blk * BM + r_local;
        valid = r < tab1[tl.group];
        drow = static_cast<int64_t>(tl.group) * args.m + r;
      } else {
        const int r = tl.m_blk * BM + r_local;
        valid = r < args.m;
        drow = r;
      }
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN;
      // full tiles leave through TMA stores (the tensor map clips rows and
      // columns outside D); a masked-layout tile that ends inside the
      // expert's valid rows is stored row by row from registers
      const bool use_tma = args.mode != kMasked || (tl.m_blk + 1) * BM <= tab1[tl.group];
      if (use_tma) {
        // drain the whole accumulator row into registers first so TMEM goes
        // back to the MMA warp before any store is made
        uint32_t packed[BN / 2];
        tmem_row_to_bf16<BN>(t_row, packed);
        tc_fence_before();
        mbar_arrive(acce_bar(acc));
        store_rows_tma<BN>(packed, r_local, sbase + L::OFF_STG, stg_count, tmap_d, tl.n_blk * BN, tl.m_blk * BM,
                           args.mode == kMasked ? tl.group : 0);
      } else {
        __nv_bfloat16* drow_ptr = args.d + drow * args.n;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tc_ld_32x32b_x32(t_row + c * 32, v);
          tc_wait_ld();
          const int col0 = tl.n_blk * BN + c * 32;
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
        mbar_arrive(acce_bar(acc));
      }
      if (++acc == ACC) { acc = 0; acc_phase ^= 1u; }
    }
    // every TMA store of this CTA must be complete before the CTA exits
    if (threadIdx.x == 64) bulk_wait_group_all();
  }

  const int split_t = sch.split_tile();
  if (SPLIT_MAX > 1 && split_t < total) {
    // ---------------------------------------------------------- split-K reduction
    // (the cluster's split tile; uniform over the cluster, cs == SPLIT_MAX)
    // 1) every CTA of the cluster is past its mainloop, so every operand ring
    //    is free to receive partials; 2) each CTA sends column slice j of its
    //    FP32 partial to CTA j; 3) each CTA sums the SPLIT_MAX partials of its
    //    slice in rank order (deterministic) and stores BF16.
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const int quarter = warp & 3;
    const int r_local = quarter * 32 + lane;
    const Tile tl = decode_tile(args, tab0, split_t);
    const int row = tl.m_blk * BM + r_local;
    // D row of this accumulator row, and whether it is stored (masked form:
    // rows at or beyond the expert's masked_m are not)
    const bool is_masked = args.mode == kMasked;
    const int64_t drow = is_masked ? static_cast<int64_t>(tl.group) * args.m + row : row;
    const bool valid = (is_masked ? row < tab1[tl.group] : row < args.m) && !*abort_flag;
    if (warp >= 2 && warp <= 5) {
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + red_acc * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tc_ld_32x32b_x32(t_row + c * 32, v);
        tc_wait_ld();
        if (valid) {
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const int q = c * 8 + q4;
            const int owner = L::quad_owner(q);
            const int cin = (q - L::slice_start(owner)) * 4;
            const uint32_t local = sbase + ((rank * L::MAX_SLICE_QUADS + cin / 4) * BM + r_local) * 16;
            st_cluster_v4(map_to_rank(local, owner), v[q4 * 4 + 0], v[q4 * 4 + 1], v[q4 * 4 + 2], v[q4 * 4 + 3]);
          }
        }
      }
    }
    cluster_sync();
    if (warp >= 2 && warp <= 5 && valid) {
      const float* red = reinterpret_cast<const float*>(smem);
      __nv_bfloat16* drow_ptr = args.d + drow * args.n;
      const int q_begin = L::slice_start(rank);
      const int q_end = L::slice_start(rank + 1);
#pragma unroll 1
      for (int q = q_begin; q < q_end; ++q) {
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int src = 0; src < SPLIT_MAX; ++src) {
          const float4 x = *reinterpret_cast<const float4*>(
              red + ((src * L::MAX_SLICE_QUADS + (q - q_begin)) * BM + r_local) * 4);
          sum.x += x.x; sum.y += x.y; sum.z += x.z; sum.w += x.w;
        }
        const int col = tl.n_blk * BN + q * 4;
        if (col < args.n) {
          uint2 w;
          w.x = pack_bf16x2(__float_as_uint(sum.x), __float_as_uint(sum.y));
          w.y = pack_bf16x2(__float_as_uint(sum.z), __float_as_uint(sum.w));
          *reinterpret_cast<uint2*>(drow_ptr + col) = w;
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) linger_after_abort();
}

template <int BN, int STAGES, int ACC, int SPLIT, int BMA>
__global__ void __launch_bounds__(kGemmThreads, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                   const __grid_constant__ CUtensorMap tmap_d, const GemmArgs args) {
  // persistent over the problem's tiles, or (SPLIT > 1) one cluster of SPLIT
  // CTAs per tile
  const int cta = static_cast<int>(blockIdx.x);
  const int rank = SPLIT > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  gemm_cta<BN, STAGES, ACC, SPLIT, BMA>(&tmap_a, &tmap_b, &tmap_d, args, SPLIT > 1 ? kBulkNone : kBulkAll, cta,
                                        static_cast<int>(gridDim.x), cta / SPLIT, SPLIT, rank);
}

// ======================================================================= host

// Raise the kernel's dynamic shared-memory limit (once per process).
template <int BN, int STAGES, int ACC, int SPLIT, int BMA>
static cudaError_t prepare_kernel() {
  static cudaError_t state = cudaErrorNotReady;
  if (state == cudaErrorNotReady)
    state = cudaFuncSetAttribute(mx_gemm_kernel<BN, STAGES, ACC, SPLIT, BMA>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Layout<BN, STAGES, ACC, SPLIT, BMA>::ALLOC);
  return state;
}

// How many clusters of the split-K kernel the GPU can hold at once (so a
// launch is sized to a single wave); 0 if the query fails.
template <int SPLIT>
static int max_active_clusters() {
  static int v = -1;
  if (v < 0) {
    v = 0;
    if (prepare_kernel<128, 6, 1, SPLIT, BM>() == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      cfg.gridDim = dim3(SPLIT, 1, 1);
      cfg.blockDim = dim3(kGemmThreads, 1, 1);
      cfg.dynamicSmemBytes = Layout<128, 6, 1, SPLIT, BM>::ALLOC;
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = SPLIT;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, mx_gemm_kernel<128, 6, 1, SPLIT, BM>, &cfg) == cudaSuccess) v = n;
      cudaGetLastError();
    }
  }
  return v;
}

template <int BN, int STAGES, int ACC, int SPLIT, int BMA = BM>
static cudaError_t launch_gemm_cfg(const GemmProblem& p, int num_sms, cudaStream_t stream, int* launches) {
  using L = Layout<BN, STAGES, ACC, SPLIT, BMA>;
  auto kern = mx_gemm_kernel<BN, STAGES, ACC, SPLIT, BMA>;
  {
    cudaError_t e = prepare_kernel<BN, STAGES, ACC, SPLIT, BMA>();
    if (e != cudaSuccess) return e;
  }
  CUtensorMap ta, tb;  // operands
  const int64_t a_depth = p.mode == kMasked ? p.groups : 1;
  const int64_t b_depth = p.mode == kDense ? 1 : p.groups;
  const int a_box_rows = (p.mode == kDense && p.m <= 32) ? 32 : (p.mode == kDense && p.m <= 64) ? 64 : BM;
  if (a_box_rows > BMA) return cudaErrorInvalidValue;
  if (!make_tmap(&ta, p.qa, p.k, p.m, a_depth, a_box_rows)) return cudaErrorInvalidValue;
  if (!make_tmap(&tb, p.qb, p.k, p.n, b_depth, BN)) return cudaErrorInvalidValue;
  CUtensorMap td;
  if (!make_tmap_d(&td, p.d, p.n, p.m, a_depth)) return cudaErrorInvalidValue;

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
  a.n_tiles = static_cast<int>((p.n + BN - 1) / BN);
  a.n_sf_tiles = static_cast<int>((p.n + 127) / 128);
  a.groups = static_cast<int>(p.groups);
  a.mode = p.mode;
  a.a_box_rows = a_box_rows;

  int64_t m_tiles_bound;
  if (p.mode == kMasked)
    m_tiles_bound = p.groups * ((p.m + BM - 1) / BM);
  else
    m_tiles_bound = (p.m + BM - 1) / BM;
  const int64_t tiles_bound = m_tiles_bound * a.n_tiles;
  if (tiles_bound == 0) return cudaSuccess;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = L::ALLOC;
  cfg.stream = stream;
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  if (SPLIT > 1) {
    // one cluster of SPLIT CTAs per output tile
    cfg.gridDim = dim3(static_cast<unsigned>(tiles_bound * SPLIT), 1, 1);
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = SPLIT;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
  } else {
    cfg.gridDim = dim3(static_cast<unsigned>(tiles_bound < num_sms ? tiles_bound : num_sms), 1, 1);
    attr[0] = pdl;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, td, a);
  if (e != cudaSuccess) return e;
  if (launches) *launches += 1;
  return cudaGetLastError();
}

// Tile configuration for one problem.  Large dense and contiguous-grouped
// problems (at least a wave of 256-row tiles) use the CTA-pair 256x256
// kernel; masked-grouped problems use the one-CTA persistent 128x256 kernel;
// dense problems that fit one wave of 128x256 tiles but not of 128x128 ones
// take the 128x256 tiles; smaller ones first try 128x128 tiles with a
// double-buffered accumulator, and dense problems that still leave most SMs
// idle split K across a cluster of 2, 3, 4, 6 or 8 CTAs.
enum GemmConfig : int {
  kCfg256 = 0, kCfg128 = 1, kCfgSplit2 = 2, kCfgSplit4 = 3, kCfgSplit8 = 4, kCfgSplit3 = 5, kCfgSplit6 = 6,
  kCfgPair = 7
};

static int split_of(int c) {
  switch (c) {
    case kCfgSplit2: return 2;
    case kCfgSplit3: return 3;
    case kCfgSplit4: return 4;
    case kCfgSplit6: return 6;
    case kCfgSplit8: return 8;
    default: return 1;
  }
}

static int max_clusters_of(int split) {
  switch (split) {
    case 2: return max_active_clusters<2>();
    case 3: return max_active_clusters<3>();
    case 4: return max_active_clusters<4>();
    case 6: return max_active_clusters<6>();
    case 8: return max_active_clusters<8>();
    default: return 0;
  }
}

static int choose_config(const GemmProblem& p, int num_sms) {
  static int forced = -2;
  if (forced == -2) {
    const char* env = getenv("MX_GEMM_CONFIG");  // tuning override: 0..7
    forced = env ? atoi(env) : -1;
  }
  const int64_t k_tiles = p.k / BK;
  const int64_t m_blocks = (p.mode == kMasked ? p.groups : 1) * ((p.m + BM - 1) / BM);
  const int64_t t256 = m_blocks * ((p.n + 255) / 256);
  const int64_t t128 = m_blocks * ((p.n + 127) / 128);
  int c;
  if (p.mode == kMasked) {
    // decode-style problems stream every expert's weights once: the one-CTA
    // 128x256 tiles keep the most weight bytes in flight per SM
    c = t256 >= num_sms ? kCfg256 : kCfg128;
  } else if (t256 >= num_sms || p.mode != kDense) {
    c = t256 >= num_sms ? kCfgPair : (t128 >= num_sms / 2 ? kCfg128 : kCfgPair);
  } else if (t128 > num_sms && t256 <= num_sms) {
    // one wave of 128x256 tiles instead of more than one of 128x128: the same
    // columns per CTA, one tile's fixed cost instead of two, half the A reads
    c = kCfg256;
  } else if (t128 >= (num_sms * 3) / 4) {
    c = kCfg128;
  } else {
    // Split K over a cluster only where the shorter per-CTA stream pays for
    // the exchange of partial sums through distributed shared memory.  Time
    // model fitted to measured kernels: a CTA streams its operands at about
    // 90 GB/s, the GPU at about 6 TB/s, and the exchange costs about 3 us.
    // Candidates are the splits whose clusters all fit at once and leave no
    // SM doubled up.
    const double a_rows = p.m <= 32 ? 32.0 : p.m <= 64 ? 64.0 : static_cast<double>(BM);
    const double per_cta = (a_rows + 128.0) * static_cast<double>(p.k);
    const double total = static_cast<double>(p.n + p.m) * static_cast<double>(p.k);
    auto est = [&](int sp) {
      const double stream = per_cta / sp / 9.0e10;
      return (stream > total / 6.0e12 ? stream : total / 6.0e12) + (sp > 1 ? 3.0e-6 : 0.0);
    };
    c = kCfg128;
    double best = est(1);
    const int order[5] = {kCfgSplit8, kCfgSplit6, kCfgSplit4, kCfgSplit3, kCfgSplit2};
    for (int i = 0; i < 5; ++i) {
      const int sp = split_of(order[i]);
      if (t128 * sp <= num_sms && k_tiles >= sp && t128 <= max_clusters_of(sp) && est(sp) < best) {
        best = est(sp);
        c = order[i];
      }
    }
  }
  if (forced >= 0 && forced <= 7) {
    const int need = split_of(forced);
    if (need == 1 || (p.mode == kDense && k_tiles >= need)) c = forced;
  }
  return c;
}

cudaError_t launch_gemm(const GemmProblem& p, int num_sms, cudaStream_t stream, int* launches) {
  // fused SwiGLU and K-grouped (weight-gradient) forms: CTA-pair kernel only
  if (p.i_dim > 0 || p.mode == kKGrouped) return launch_gemm_pair(p, num_sms, stream, launches);
  const int c = choose_config(p, num_sms);
  if (c == kCfgPair) return launch_gemm_pair(p, num_sms, stream, launches);
  if (p.mode == kDense && p.m <= 64) {
    // A stages of 64 rows: 8 stages in flight instead of 6
    switch (c) {
      case kCfg128: return launch_gemm_cfg<128, 8, 2, 1, 64>(p, num_sms, stream, launches);
      case kCfgSplit2: return launch_gemm_cfg<128, 8, 1, 2, 64>(p, num_sms, stream, launches);
      case kCfgSplit3: return launch_gemm_cfg<128, 8, 1, 3, 64>(p, num_sms, stream, launches);
      case kCfgSplit4: return launch_gemm_cfg<128, 8, 1, 4, 64>(p, num_sms, stream, launches);
      case kCfgSplit6: return launch_gemm_cfg<128, 8, 1, 6, 64>(p, num_sms, stream, launches);
      case kCfgSplit8: return launch_gemm_cfg<128, 8, 1, 8, 64>(p, num_sms, stream, launches);
      default: return launch_gemm_cfg<256, 4, 1, 1>(p, num_sms, stream, launches);
    }
  }
  switch (c) {
    case kCfg128: return launch_gemm_cfg<128, 6, 2, 1>(p, num_sms, stream, launches);
    case kCfgSplit2: return launch_gemm_cfg<128, 6, 1, 2>(p, num_sms, stream, launches);
    case kCfgSplit3: return launch_gemm_cfg<128, 6, 1, 3>(p, num_sms, stream, launches);
    case kCfgSplit4: return launch_gemm_cfg<128, 6, 1, 4>(p, num_sms, stream, launches);
    case kCfgSplit6: return launch_gemm_cfg<128, 6, 1, 6>(p, num_sms, stream, launches);
    case kCfgSplit8: return launch_gemm_cfg<128, 6, 1, 8>(p, num_sms, stream, launches);
    default: return launch_gemm_cfg<256, 4, 1, 1>(p, num_sms, stream, launches);
  }
}

// ======================================================================= batch

// Independent dense problems in ONE launch.  Each CTA belongs to one problem
// (problem p owns CTAs [cta0[p], cta0[p+1]), a whole number of clusters) and
// runs the one-CTA kernel's body on it with 128 x BN tiles (BN = 128: six
// stages and two accumulators; BN = 256: four stages, one accumulator, half
// the re-reads of A): persistently over the problem's tiles, or with K split
// over the CS CTAs of each of its clusters (one tile per cluster, partials
// reduced through distributed shared memory).  The host sizes every
// problem's share of the GPU so that all of them finish at about the same
// time: small problems stream their operands on all SMs at once instead of
// one after another.
template <int BN>
struct BatchCfg {
  static constexpr int STAGES = BN == 128 ? 6 : 4;
  static constexpr int ACC = BN == 128 ? 2 : 1;
};

struct BatchMaps {
  CUtensorMap a[kMaxBatch];
  CUtensorMap b[kMaxBatch];
  CUtensorMap d[kMaxBatch];
};

struct BatchArgs {
  GemmArgs args[kMaxBatch];
  int cta0[kMaxBatch + 1];
  int split[kMaxBatch];  // 1, or CS: the CTAs of a cluster share one tile
  int count;
};

template <int BN, int CS>
__global__ void __launch_bounds__(kGemmThreads, 1)
    mx_gemm_batch_kernel(const __grid_constant__ BatchMaps maps, const __grid_constant__ BatchArgs bat) {
  const int cta = static_cast<int>(blockIdx.x);
  int p = 0;
  while (p + 1 < bat.count && cta >= bat.cta0[p + 1]) ++p;
  const GemmArgs& args = bat.args[p];
  const int local = cta - bat.cta0[p];
  const int ctas = bat.cta0[p + 1] - bat.cta0[p];
  const int split = bat.split[p];
  const int rank = split > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  gemm_cta<BN, BatchCfg<BN>::STAGES, BatchCfg<BN>::ACC, CS, BM>(&maps.a[p], &maps.b[p], &maps.d[p], args,
                                                                 split > 1 ? kBulkNone : kBulkAll, local, ctas,
                                                                 local / split, split, rank);
}

template <int BN, int CS>
using BatchLayout = Layout<BN, BatchCfg<BN>::STAGES, BatchCfg<BN>::ACC, CS, BM>;

template <int BN, int CS>
static cudaError_t prepare_batch_kernel() {
  static cudaError_t state = cudaErrorNotReady;
  if (state == cudaErrorNotReady)
    state = cudaFuncSetAttribute(mx_gemm_batch_kernel<BN, CS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 BatchLayout<BN, CS>::ALLOC);
  return state;
}

// Clusters of CS CTAs the GPU holds at once (0 if unknown).
template <int BN, int CS>
static int batch_max_clusters() {
  static int v = -1;
  if (v < 0) {
    v = 0;
    if (prepare_batch_kernel<BN, CS>() == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      cfg.gridDim = dim3(CS, 1, 1);
      cfg.blockDim = dim3(kGemmThreads, 1, 1);
      cfg.dynamicSmemBytes = BatchLayout<BN, CS>::ALLOC;
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = CS;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, mx_gemm_batch_kernel<BN, CS>, &cfg) == cudaSuccess) v = n;
      cudaGetLastError();
    }
  }
  return v;
}

// Share of the GPU for each problem: a time model (a CTA of this kernel
// streams its operands at ~62 GB/s with 128-wide tiles and ~52 GB/s with
// 256-wide ones, fitted to the page shapes' batch; a tile costs ~0.5 us
// more, a split-K exchange ~3 us).  Every problem gets a cluster, then each further
// cluster goes to the problem that would finish last, with the better of
// "no split" and "split K over the cluster" for its share.
struct BatchPlan {
  int ctas[kMaxBatch];
  int split[kMaxBatch];
  double time;
};

static double batch_time(int64_t tiles, double tile_bytes, int64_t k_tiles, int ctas, int bn, int cs, int* split) {
  const double rate = bn == 128 ? 6.2e10 : 5.2e10, per_tile = 0.5e-6, exchange = 3.0e-6;
  const int64_t groups1 = ctas;
  double best = static_cast<double>((tiles + groups1 - 1) / groups1) * (tile_bytes / rate + per_tile);
  *split = 1;
  const int64_t groups_s = ctas / cs;
  if (cs > 1 && k_tiles >= cs && groups_s >= tiles) {  // one tile per cluster
    const double t = tile_bytes / cs / rate + per_tile + exchange;
    if (t < best) {
      best = t;
      *split = cs;
    }
  }
  return best;
}

static BatchPlan plan_batch(const GemmProblem* ps, int count, int bn, int cs, int clusters) {
  BatchPlan pl = {};
  int64_t tiles[kMaxBatch];
  double tile_bytes[kMaxBatch];
  double t[kMaxBatch];
  int left = clusters;
  for (int i = 0; i < count; ++i) {
    tiles[i] = ((ps[i].m + BM - 1) / BM) * ((ps[i].n + bn - 1) / bn);
    const int64_t a_rows = ps[i].m < BM ? (ps[i].m <= 32 ? 32 : ps[i].m <= 64 ? 64 : BM) : BM;
    tile_bytes[i] = static_cast<double>((a_rows + bn) * ps[i].k) * (1.0 + 1.0 / 32.0);
    pl.ctas[i] = cs;
    --left;
    t[i] = batch_time(tiles[i], tile_bytes[i], ps[i].k / BK, pl.ctas[i], bn, cs, &pl.split[i]);
  }
  while (left > 0) {
    int worst = -1;
    for (int i = 0; i < count; ++i) {
      const bool useful = pl.ctas[i] < tiles[i] * cs;  // more CTAs than tiles x cluster size cannot help
      if (useful && (worst < 0 || t[i] > t[worst])) worst = i;
    }
    if (worst < 0) break;
    pl.ctas[worst] += cs;
    --left;
    t[worst] =
        batch_time(tiles[worst], tile_bytes[worst], ps[worst].k / BK, pl.ctas[worst], bn, cs, &pl.split[worst]);
  }
  pl.time = 0.0;
  for (int i = 0; i < count; ++i) pl.time = t[i] > pl.time ? t[i] : pl.time;
  return pl;
}

template <int BN, int CS>
static cudaError_t launch_batch_cs(const GemmProblem* ps, int count, const BatchPlan& pl, cudaStream_t stream,
                                   int* launches) {
  using L = BatchLayout<BN, CS>;
  {
    cudaError_t e = prepare_batch_kernel<BN, CS>();
    if (e != cudaSuccess) return e;
  }
  BatchMaps maps;
  BatchArgs bat = {};
  bat.count = count;
  int cta = 0;
  for (int i = 0; i < count; ++i) {
    const GemmProblem& p = ps[i];
    const int a_box_rows = p.m <= 32 ? 32 : p.m <= 64 ? 64 : BM;
    if (!make_tmap(&maps.a[i], p.qa, p.k, p.m, 1, a_box_rows)) return cudaErrorInvalidValue;
    if (!make_tmap(&maps.b[i], p.qb, p.k, p.n, 1, BN)) return cudaErrorInvalidValue;
    if (!make_tmap_d(&maps.d[i], p.d, p.n, p.m, 1)) return cudaErrorInvalidValue;
    GemmArgs& a = bat.args[i];
    a.sfa = static_cast<const uint8_t*>(p.sfa);
    a.sfb = static_cast<const uint8_t*>(p.sfb);
    a.d = static_cast<__nv_bfloat16*>(p.d);
    a.status = p.status;
    a.wait_ns = wait_limit_ns();
    a.k_tiles = static_cast<int>(p.k / BK);
    a.sfa_group_bytes = ((p.m + 127) / 128) * 128 * (p.k / 32);
    a.sfb_group_bytes = ((p.n + 127) / 128) * 128 * (p.k / 32);
    a.m = static_cast<int>(p.m);
    a.n = static_cast<int>(p.n);
    a.n_tiles = static_cast<int>((p.n + BN - 1) / BN);
    a.n_sf_tiles = static_cast<int>((p.n + 127) / 128);
    a.groups = 1;
    a.mode = kDense;
    a.a_box_rows = a_box_rows;
    bat.cta0[i] = cta;
    bat.split[i] = pl.split[i];
    cta += pl.ctas[i];
  }
  bat.cta0[count] = cta;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3(static_cast<unsigned>(cta), 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = L::ALLOC;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, mx_gemm_batch_kernel<BN, CS>, maps, bat);
  if (e != cudaSuccess) return e;
  if (launches) *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_gemm_batch(const GemmProblem* ps_in, int count, int num_sms, cudaStream_t stream, int* launches) {
  (void)num_sms;
  if (count < 0 || count > kMaxBatch) return cudaErrorInvalidValue;
  GemmProblem ps[kMaxBatch];
  int n = 0;
  for (int i = 0; i < count; ++i)  // empty problems take no CTAs
    if (ps_in[i].m > 0 && ps_in[i].n > 0 && ps_in[i].k > 0) ps[n++] = ps_in[i];
  if (n == 0) return cudaSuccess;
  static int forced_cs = -2, forced_bn = -2;  // tuning overrides: cluster size 2 or 4, tile width 128 or 256
  if (forced_cs == -2) {
    const char* env = getenv("MX_BATCH_CLUSTER");
    forced_cs = env ? atoi(env) : -1;
    env = getenv("MX_BATCH_BN");
    forced_bn = env ? atoi(env) : -1;
  }
  // candidate (tile width, cluster size) forms; the one the model finishes first
  const int cl[4] = {batch_max_clusters<128, 2>(), batch_max_clusters<128, 4>(), batch_max_clusters<256, 2>(),
                     batch_max_clusters<256, 4>()};
  const int bns[4] = {128, 128, 256, 256}, css[4] = {2, 4, 2, 4};
  int best = -1;
  BatchPlan plans[4];
  for (int c = 0; c < 4; ++c) {
    if (cl[c] < n) continue;
    if ((forced_cs == 2 || forced_cs == 4) && css[c] != forced_cs) continue;
    if ((forced_bn == 128 || forced_bn == 256) && bns[c] != forced_bn) continue;
    plans[c] = plan_batch(ps, n, bns[c], css[c], cl[c]);
    if (best < 0 || plans[c].time < plans[best].time) best = c;
  }
  switch (best) {
    case 0: return launch_batch_cs<128, 2>(ps, n, plans[0], stream, launches);
    case 1: return launch_batch_cs<128, 4>(ps, n, plans[1], stream, launches);
    case 2: return launch_batch_cs<256, 2>(ps, n, plans[2], stream, launches);
    case 3: return launch_batch_cs<256, 4>(ps, n, plans[3], stream, launches);
    default: return cudaErrorInvalidConfiguration;
  }
}

}  // namespace mxk
