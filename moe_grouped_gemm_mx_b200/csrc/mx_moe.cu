// mx_moe.cu -- the data movement around the grouped GEMM of a mixture-of-
// experts expert layer, on sm_100a: the routing plan, the dispatch (each
// token quantised to MXFP8 once and its row placed at every expert row it is
// routed to, in the contiguous grouped layout), the row scatter / gather of
// the all-to-all buffers of expert parallelism, the gate-weighted combine, and
// the peer-memory forms of dispatch and combine for expert parallelism over
// NVLink (rows written straight into, and read straight from, the buffers of
// the rank that owns the expert, through a device table of every rank's
// pointers) with the plan that places each entry there.
//
// Sources: the B200 MoE-training page (the diagram of the MXFP8 expert layer:
// router output -> BF16 -> MXFP8 -> grouped GEMM -> BF16 -> all-to-all
// combine; the glossary entry on all-to-all: tokens go to the experts that
// process them and the results are gathered back; the DeepEP section) and the
// DeepGEMM release page, section 4 (the contiguous layout: each expert's
// tokens grouped, one group after another, each group padded to the GEMM's
// 128-row tile).
//
// Everything here is HBM-bound data movement; each kernel reads and writes
// every byte once.  Indices that come from device memory (rows, ids) are
// checked before any access: a bad one skips the access and sets a bit of the
// caller's status word.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mx_launch.h"
#include "mx_mxfp8.cuh"
#include "mx_ptx.cuh"

namespace mxk {

constexpr int kRouteThreads = 1024;
constexpr int kRowWarps = 8;  // warps per CTA of the row kernels (one row per warp)
constexpr int kDevBadIndex = 0x8;
constexpr int kCombineBatch = 8;  // routed rows of a token whose loads the combine has in flight at once

__device__ __forceinline__ void moe_report(int32_t* status, int bits) { atomicOr(status, bits); }

// ------------------------------------------------------------------ routing plan
// A cluster of kRouteCluster CTAs of 32 warps; CTA c owns the contiguous
// segment c of the entries and warp w of it a contiguous sub-segment, so entry
// order is (CTA, warp, position).
//  1. each warp streams its sub-segment 32 entries per step (four steps'
//     loads in flight): a lane's rank among the step's entries of its expert
//     comes from __match_any_sync, the warp's running count of that expert
//     from its own row of a [32][E] shared-memory table; the rank within the
//     sub-segment is parked in row[i];
//  2. one thread per expert turns its column into exclusive per-warp
//     prefixes and the CTA's total; after a cluster barrier each CTA reads
//     the other CTAs' totals through distributed shared memory (the earlier
//     CTAs' sum is its base, all of them the expert's count), and a block
//     scan over the padded counts gives the group offsets (the same in every
//     CTA; CTA 0 writes them out);
//  3. each warp adds offset + CTA base + warp prefix to its parked ranks.
// A second cluster barrier keeps every CTA resident until its peers have
// read its totals.
constexpr int kRouteUnroll = 4;
constexpr int kRouteCluster = 8;

__device__ __forceinline__ int32_t ld_cluster_s32(uint32_t addr) {
  int32_t v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__global__ void __launch_bounds__(kRouteThreads) moe_route_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                                  int pad, int32_t* __restrict__ counts,
                                                                  int32_t* __restrict__ offsets,
                                                                  int32_t* __restrict__ row,
                                                                  int32_t* __restrict__ dropped) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ int32_t route_smem[];
  int32_t* wc = route_smem;          // [32][E] per-warp counts, then per-warp exclusive prefixes
  int32_t* tot = wc + 32 * E;        // [E] this CTA's count per expert (read by the other CTAs)
  int32_t* base = tot + E;           // [E] group offset + earlier CTAs' counts
  int32_t* wsum = base + E;          // [32] warp totals of the scan
  int32_t* nbad = wsum + 32;         // [1] dropped entries of this CTA (read by CTA 0)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int crank = static_cast<int>(cluster_ctarank());
  for (int i = tid; i < 32 * E; i += blockDim.x) wc[i] = 0;
  if (tid == 0) *nbad = 0;
  __syncthreads();

  const int cseg = (n + kRouteCluster - 1) / kRouteCluster;
  const int cbeg = min(n, crank * cseg);
  const int cend = min(n, cbeg + cseg);
  const int seg = (cend - cbeg + 31) / 32;
  const int begin = min(cend, cbeg + warp * seg);
  const int end = min(cend, begin + seg);
  const uint32_t lower = (1u << lane) - 1u;
  int32_t* my = wc + warp * E;
  int bad = 0;
  for (int s0 = begin; s0 < end; s0 += 32 * kRouteUnroll) {
    int ev[kRouteUnroll];
#pragma unroll
    for (int u = 0; u < kRouteUnroll; ++u) {
      const int i = s0 + u * 32 + lane;
      ev[u] = i < end ? __ldg(ids + i) : -1;
    }
#pragma unroll
    for (int u = 0; u < kRouteUnroll; ++u) {
      const int i = s0 + u * 32 + lane;
      const bool in = i < end;
      const bool valid = in && ev[u] >= 0 && ev[u] < E;
      if (in && !valid) ++bad;
      const int key = valid ? ev[u] : -1;
      const uint32_t peers = __match_any_sync(0xFFFFFFFFu, key);
      int b = 0;
      if (valid) {
        b = my[key];
        row[i] = b + __popc(peers & lower);
      } else if (in) {
        row[i] = -1;
      }
      __syncwarp();
      if (valid && (peers & lower) == 0) my[key] = b + __popc(peers);
      __syncwarp();
    }
  }
  if (bad) atomicAdd(nbad, bad);
  __syncthreads();

  if (tid < E) {
    int t = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = wc[w * E + tid];
      wc[w * E + tid] = t;
      t += c;
    }
    tot[tid] = t;
  }
  cluster_arrive_release();  // every CTA's totals are written ...
  cluster_wait_acquire();    // ... and visible cluster-wide
  int pre = 0, all = 0;
  if (tid < E) {
    const uint32_t a = smem_u32(tot + tid);
    for (int c = 0; c < kRouteCluster; ++c) {
      const int v = c == crank ? tot[tid] : ld_cluster_s32(map_to_rank(a, c));
      if (c < crank) pre += v;
      all += v;
    }
  }
  int nbad_all = 0;
  if (crank == 0 && tid == 0) {
    const uint32_t a = smem_u32(nbad);
    for (int c = 0; c < kRouteCluster; ++c) nbad_all += c == 0 ? *nbad : ld_cluster_s32(map_to_rank(a, c));
  }
  cluster_arrive_release();  // done reading the other CTAs' shared memory

  const int v = tid < E ? (all + pad - 1) / pad * pad : 0;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = wsum[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, wi, o);
      if (lane >= o) wi += y;
    }
    wsum[lane] = wi - w;
  }
  __syncthreads();
  const int excl = incl - v + wsum[warp];
  if (tid < E) {
    base[tid] = excl + pre;
    if (crank == 0) {
      counts[tid] = all;
      offsets[tid] = excl;
      if (tid == E - 1) offsets[E] = excl + v;
    }
  }
  if (crank == 0 && tid == 0 && dropped != nullptr) *dropped = nbad_all;
  __syncthreads();

  for (int i = begin + lane; i < end; i += 32) {
    const int r = row[i];  // written by this thread in step 1
    if (r < 0) continue;
    const int e = __ldg(ids + i);
    row[i] = base[e] + my[e] + r;
  }
  cluster_wait_acquire();  // peers may still read this CTA's totals until here
}

// ------------------------------------------------------------------ dispatch / scatter
struct PlaceArgs {
  const void* src;          // QUANT: BF16 tokens [n_src, k]; else E4M3 rows [n_src, k]
  const uint8_t* src_sf;    // !QUANT: row-major scales [n_src, k/32]
  const int32_t* row;       // destination rows [n_src * fan]
  const int32_t* counts;    // [E] real rows per group (padding clearing)
  const int32_t* offsets;   // [E+1] padded group starts
  uint8_t* q;               // E4M3 rows [m_rows, k] (PEER: this rank's receive rows, padding only)
  uint8_t* sf;              // scales of q: tiled, or row-major [m_rows, k/32]
  uint8_t* const* q_peers;  // PEER: [ranks] every rank's receive rows [m_rows, k]
  uint8_t* const* sf_peers; // PEER: [ranks] their tiled scales
  const int32_t* row_rank;  // PEER: destination rank of each destination row [n_src * fan]
  int ranks;
  int32_t* status;
  int64_t n_src;
  int64_t m_rows;
  int k;
  int fan;                  // destination rows per source row (top-k for the dispatch, 1 for a scatter)
  int E;                    // groups whose padding rows are cleared (0: none)
  int pad_slots;            // padding rows per group at most (pad - 1)
  int sf_row_major;
};

// Scale word of blocks c..c+3 (c % 4 == 0) of row r of the scales at sf.
__device__ __forceinline__ uint32_t* scale_word(const PlaceArgs& a, uint8_t* sf, int64_t r, uint32_t c, uint32_t kb) {
  const int64_t off = a.sf_row_major ? r * kb + c : static_cast<int64_t>(sf_tiled_offset(static_cast<uint32_t>(r), c, kb / 4));
  return reinterpret_cast<uint32_t*>(sf + off);
}

// One warp per (source row, chunk of 32 blocks = 1024 elements): QUANT
// quantises the BF16 token's blocks, one per lane, with the quantiser's rule;
// else it copies the E4M3 bytes and scales.  The chunk is then written to each
// of the row's `fan` destinations.  The warps after the last source chunk
// clear the group padding rows (E4M3 0, scale 0: the quantisation of a zero
// row), one (padding slot, chunk) each.  Splitting rows into chunks keeps
// enough warps in flight when there are few tokens.  PEER: destination j of a
// row is row `row` of rank `row_rank`'s receive buffer, reached through the
// pointer tables (another GPU's memory over NVLink, by plain stores); the
// padding rows cleared are those of this rank's own receive buffer.
template <bool QUANT, bool PEER>
__global__ void __launch_bounds__(kRowWarps * 32) moe_place_kernel(const PlaceArgs a) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  const uint32_t kb = static_cast<uint32_t>(a.k / 32);
  const int64_t chunks = (kb + 31) / 32;
  const int64_t src_units = a.n_src * chunks;
  if (w < src_units) {
    const int64_t src = w / chunks;
    const uint32_t b = static_cast<uint32_t>(w - src * chunks) * 32 + lane;
    const bool on = b < kb;  // kb % 4 == 0: each group of 4 lanes is all on or all off
    uint4 out0 = make_uint4(0, 0, 0, 0), out1 = out0;
    uint32_t scode = 0;
    if (QUANT) {
      uint4 v[4];
      const uint4* sp = static_cast<const uint4*>(a.src) + (src * kb + b) * 4;
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = on ? __ldcs(sp + j) : make_uint4(0, 0, 0, 0);
      scode = quant_block32_bf16(v, out0, out1);
    } else if (on) {
      const uint4* sp = static_cast<const uint4*>(a.src) + (src * kb + b) * 2;
      out0 = __ldcs(sp);
      out1 = __ldcs(sp + 1);
      scode = a.src_sf[src * kb + b];
    }
    const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, scode, 1);
    const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, scode, 2);
    const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, scode, 3);
    const uint32_t word = scode | (s1 << 8) | (s2 << 16) | (s3 << 24);
    // rearrange so each store instruction writes 512 contiguous bytes: bytes
    // [16l, 16l + 16) of the chunk's first (second) 512 are half l & 1 of
    // block l >> 1 (16 + (l >> 1))
    const int sa = lane >> 1, sb = 16 + (lane >> 1);
    const bool hi = lane & 1;
    uint4 st0, st1;
    {
      const uint4 x0 = make_uint4(__shfl_sync(0xFFFFFFFFu, out0.x, sa), __shfl_sync(0xFFFFFFFFu, out0.y, sa),
                                  __shfl_sync(0xFFFFFFFFu, out0.z, sa), __shfl_sync(0xFFFFFFFFu, out0.w, sa));
      const uint4 x1 = make_uint4(__shfl_sync(0xFFFFFFFFu, out1.x, sa), __shfl_sync(0xFFFFFFFFu, out1.y, sa),
                                  __shfl_sync(0xFFFFFFFFu, out1.z, sa), __shfl_sync(0xFFFFFFFFu, out1.w, sa));
      const uint4 y0 = make_uint4(__shfl_sync(0xFFFFFFFFu, out0.x, sb), __shfl_sync(0xFFFFFFFFu, out0.y, sb),
                                  __shfl_sync(0xFFFFFFFFu, out0.z, sb), __shfl_sync(0xFFFFFFFFu, out0.w, sb));
      const uint4 y1 = make_uint4(__shfl_sync(0xFFFFFFFFu, out1.x, sb), __shfl_sync(0xFFFFFFFFu, out1.y, sb),
                                  __shfl_sync(0xFFFFFFFFu, out1.z, sb), __shfl_sync(0xFFFFFFFFu, out1.w, sb));
      st0 = hi ? x1 : x0;
      st1 = hi ? y1 : y0;
    }
    const uint32_t b0 = b - lane;  // first block of the chunk
    const bool on0 = b0 + sa < kb, on1 = b0 + sb < kb;
    for (int j = 0; j < a.fan; ++j) {
      const int32_t r = a.row[src * a.fan + j];
      if (r < 0) continue;  // a dropped entry
      uint8_t* qb = a.q;
      uint8_t* sfb = a.sf;
      if constexpr (PEER) {
        const int32_t rk = a.row_rank[src * a.fan + j];
        if (rk < 0 || rk >= a.ranks) {
          if (lane == 0) moe_report(a.status, kDevBadIndex);
          continue;
        }
        qb = a.q_peers[rk];
        sfb = a.sf_peers[rk];
      }
      if (r >= a.m_rows) {
        if (lane == 0) moe_report(a.status, kDevBadIndex);
        continue;
      }
      uint4* dst = reinterpret_cast<uint4*>(qb) + (static_cast<int64_t>(r) * kb + b0) * 2;
      if (on0) dst[lane] = st0;
      if (on1) dst[32 + lane] = st1;
      if (on && (lane & 3) == 0) *scale_word(a, sfb, r, b, kb) = word;
    }
    return;
  }
  // padding rows, one (slot, chunk) per warp
  if (a.E == 0 || a.pad_slots == 0) return;
  const int64_t p = (w - src_units) / chunks;
  const uint32_t c = static_cast<uint32_t>((w - src_units) - p * chunks);
  const int e = static_cast<int>(p / a.pad_slots);
  if (e >= a.E) return;
  const int s = static_cast<int>(p - static_cast<int64_t>(e) * a.pad_slots);
  const int64_t r = static_cast<int64_t>(a.offsets[e]) + a.counts[e] + s;
  if (r >= a.offsets[e + 1]) return;
  if (r < 0 || r >= a.m_rows) {
    if (lane == 0) moe_report(a.status, kDevBadIndex);
    return;
  }
  const uint32_t b = c * 32 + lane;
  if (b < kb) {
    uint4* dst = reinterpret_cast<uint4*>(a.q) + (r * kb + b) * 2;
    dst[0] = make_uint4(0, 0, 0, 0);
    dst[1] = make_uint4(0, 0, 0, 0);
    if ((lane & 3) == 0) *scale_word(a, a.sf, r, b, kb) = 0;
  }
}

// ------------------------------------------------------------------ row gather
// dst[i] = src[idx[i]] for rows of `row_vecs` 16-byte vectors; an index
// outside [0, src_rows) gives a zero row and the status bit.  One warp per row.
__global__ void __launch_bounds__(kRowWarps * 32) moe_gather_kernel(const uint4* __restrict__ src, int64_t src_rows,
                                                                    int64_t row_vecs, const int32_t* __restrict__ idx,
                                                                    int64_t n, uint4* __restrict__ dst,
                                                                    int32_t* status) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  if (i >= n) return;
  const int32_t r = idx[i];
  uint4* d = dst + i * row_vecs;
  if (r < 0 || r >= src_rows) {
    if (lane == 0) moe_report(status, kDevBadIndex);
    for (int64_t c = lane; c < row_vecs; c += 32) d[c] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4* s = src + static_cast<int64_t>(r) * row_vecs;
  for (int64_t c = lane; c < row_vecs; c += 32) d[c] = __ldcs(s + c);
}

// ------------------------------------------------------------------ combine
// out[t, :] = sum_j w[t, j] * y[row[t*topk + j], :], FP32 fused multiply-adds
// in j order, rounded once to BF16 (RNE).  One warp per (token, chunk of 256
// columns): 8 columns (one 16-byte vector) per lane, eight routed rows' loads
// in flight.  PEER: routed row j of a token is row `row` of rank `row_rank`'s
// expert output, read through the pointer table (another GPU's memory over
// NVLink, by plain loads).
template <bool PEER>
__global__ void __launch_bounds__(kRowWarps * 32) moe_combine_kernel(const uint4* __restrict__ y,
                                                                     const uint4* const* __restrict__ y_peers,
                                                                     const int32_t* __restrict__ row_rank, int ranks,
                                                                     int64_t y_rows, int64_t n_vecs,
                                                                     const int32_t* __restrict__ row,
                                                                     const float* __restrict__ wt, int64_t tokens,
                                                                     int topk, uint4* __restrict__ out,
                                                                     int32_t* status) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  const int64_t chunks = (n_vecs + 31) / 32;
  const int64_t t = w / chunks;
  if (t >= tokens) return;
  const int64_t c = (w - t * chunks) * 32 + lane;
  const int32_t* rt = row + t * topk;
  const float* wt_t = wt + t * topk;
  bool bad = false;
  if (c < n_vecs) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int j0 = 0; j0 < topk; j0 += kCombineBatch) {
      // three branch-free phases, each with the batch's loads in flight
      // together: the rows (and ranks), the ranks' addresses, the data
      int32_t r[kCombineBatch], rk[kCombineBatch];
#pragma unroll
      for (int u = 0; u < kCombineBatch; ++u) {
        const int j = j0 + u;
        r[u] = j < topk ? rt[j] : -1;
        rk[u] = PEER && j < topk ? row_rank[t * topk + j] : 0;
      }
      const uint4* yb[kCombineBatch];
#pragma unroll
      for (int u = 0; u < kCombineBatch; ++u) {
        const bool rank_ok = !PEER || (rk[u] >= 0 && rk[u] < ranks);
        if (r[u] >= 0 && (!rank_ok || r[u] >= y_rows)) {
          bad = true;
          r[u] = -1;
        }
        yb[u] = PEER ? y_peers[r[u] >= 0 ? rk[u] : 0] : y;  // entry 0 exists: ranks >= 1
      }
      uint4 v[kCombineBatch];
      float wj[kCombineBatch];
#pragma unroll
      for (int u = 0; u < kCombineBatch; ++u) {
        wj[u] = r[u] >= 0 ? wt_t[j0 + u] : 0.0f;
        v[u] = r[u] >= 0 ? __ldcs(yb[u] + static_cast<int64_t>(r[u]) * n_vecs + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kCombineBatch; ++u) {
        if (j0 + u >= topk) break;
        const uint32_t x4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = fmaf(wj[u], bf16_lo(x4[i]), acc[2 * i]);
          acc[2 * i + 1] = fmaf(wj[u], bf16_hi(x4[i]), acc[2 * i + 1]);
        }
      }
    }
    uint4 o;
    uint32_t* op = &o.x;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      op[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    out[t * n_vecs + c] = o;
  }
  if (bad && lane == 0) moe_report(status, kDevBadIndex);
}

// ------------------------------------------------------------------ expert-parallel placement plan
// Rank `rank` of `ranks` owns the experts [rank * el, (rank + 1) * el),
// el = E / ranks.  count[src][e] is the number of entries rank src routes to
// (global) expert e; this rank's entries were routed with pad 1, so
// row_send[i] = (its entries for experts before e) + (the rank of entry i
// among its entries for e).  On the owner o = e / el, expert e's rows come
// source rank by source rank, each source's in its own order, and every
// local expert's group is padded to `pad` rows:
//   dst_rank[i] = o
//   dst_row[i]  = gstart(e) + sum_{src < rank} count[src][e] + (row_send[i] - own_start(e))
// with gstart(e) the padded start of e among its owner's experts.  Block 0
// also writes this rank's own receive plan: counts_local[l] = total entries
// of expert rank * el + l over all sources, offsets_local = their padded
// starts (el + 1 values).  An id outside [0, E) is a dropped entry (-1, -1).
constexpr int kPlanThreads = 256;

__global__ void __launch_bounds__(kPlanThreads) moe_peer_plan_kernel(
    const int32_t* __restrict__ ids, const int32_t* __restrict__ row_send, int64_t n,
    const int32_t* __restrict__ count, int ranks, int rank, int E, int pad, int32_t* __restrict__ dst_rank,
    int32_t* __restrict__ dst_row, int32_t* __restrict__ counts_local, int32_t* __restrict__ offsets_local,
    int32_t* status) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ int32_t plan_sh[];
  int32_t* tot = plan_sh;     // [E] entries of expert e over all source ranks
  int32_t* pre = tot + E;     // [E] ... over the source ranks before this one
  int32_t* own = pre + E;     // [E] this rank's entries of e
  int32_t* start = own + E;   // [E] this rank's entries of the experts before e
  int32_t* gsc = start + E;   // [E] exclusive scan of the padded totals over all experts
  const int el = E / ranks;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t t = 0, p = 0;
    for (int src = 0; src < ranks; ++src) {
      const int32_t c = __ldg(count + static_cast<int64_t>(src) * E + e);
      t += c;
      if (src < rank) p += c;
    }
    tot[e] = t;
    pre[e] = p;
    own[e] = __ldg(count + static_cast<int64_t>(rank) * E + e);
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // two exclusive scans, 32 experts per step
    const int lane = threadIdx.x;
    int32_t carry_s = 0, carry_g = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int32_t vs = e < E ? own[e] : 0;
      const int32_t vg = e < E ? (tot[e] + pad - 1) / pad * pad : 0;
      int32_t xs = vs, xg = vg;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t ys = __shfl_up_sync(0xFFFFFFFFu, xs, o);
        const int32_t yg = __shfl_up_sync(0xFFFFFFFFu, xg, o);
        if (lane >= o) {
          xs += ys;
          xg += yg;
        }
      }
      if (e < E) {
        start[e] = carry_s + xs - vs;
        gsc[e] = carry_g + xg - vg;
      }
      carry_s += __shfl_sync(0xFFFFFFFFu, xs, 31);
      carry_g += __shfl_sync(0xFFFFFFFFu, xg, 31);
    }
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    const int e0 = rank * el;
    for (int l = threadIdx.x; l <= el; l += blockDim.x) {
      if (l < el) {
        counts_local[l] = tot[e0 + l];
        offsets_local[l] = gsc[e0 + l] - gsc[e0];
      } else {
        offsets_local[el] = gsc[e0 + el - 1] - gsc[e0] + (tot[e0 + el - 1] + pad - 1) / pad * pad;
      }
    }
  }
  bool bad = false;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int32_t e = ids[i];
    int32_t dr = -1, drow = -1;
    if (e >= 0 && e < E) {
      const int32_t within = row_send[i] - start[e];
      if (within < 0 || within >= own[e]) {
        bad = true;
      } else {
        const int o = e / el;
        dr = o;
        drow = gsc[e] - gsc[o * el] + pre[e] + within;
      }
    }
    dst_rank[i] = dr;
    dst_row[i] = drow;
  }
  if (bad) moe_report(status, kDevBadIndex);
}

// ======================================================================= host

static cudaError_t launch_pdl_cfg(const void* func, dim3 grid, dim3 block, size_t smem, void** args,
                                  cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelExC(&cfg, func, args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_moe_route(const int32_t* ids, int64_t n, int E, int pad, int32_t* counts, int32_t* offsets,
                             int32_t* row, int32_t* dropped, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(34 * E + 33) * 4;  // at most 139 KB (E = 1024)
  static cudaError_t attr = cudaErrorNotReady;
  if (attr == cudaErrorNotReady)
    attr = cudaFuncSetAttribute(moe_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 34 * 1024 * 4 + 33 * 4);
  if (attr != cudaSuccess) return attr;
  int ni = static_cast<int>(n);
  void* args[] = {&ids, &ni, &E, &pad, &counts, &offsets, &row, &dropped};
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[2];
  cfg.gridDim = dim3(kRouteCluster);
  cfg.blockDim = dim3(kRouteThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kRouteCluster;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(moe_route_kernel), args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_moe_place(const MoePlace& p, cudaStream_t stream) {
  PlaceArgs a = {};
  a.src = p.src;
  a.src_sf = static_cast<const uint8_t*>(p.src_sf);
  a.row = p.row;
  a.counts = p.counts;
  a.offsets = p.offsets;
  a.q = static_cast<uint8_t*>(p.q);
  a.sf = static_cast<uint8_t*>(p.sf);
  a.status = p.status;
  a.n_src = p.n_src;
  a.m_rows = p.m_rows;
  a.k = static_cast<int>(p.k);
  a.fan = p.fan;
  a.E = p.pad > 1 ? p.experts : 0;
  a.pad_slots = p.pad > 1 ? p.pad - 1 : 0;
  a.sf_row_major = p.sf_row_major;
  a.q_peers = reinterpret_cast<uint8_t* const*>(p.q_peers);
  a.sf_peers = reinterpret_cast<uint8_t* const*>(p.sf_peers);
  a.row_rank = p.row_rank;
  a.ranks = p.ranks;
  const bool peer = p.q_peers != nullptr;
  const int64_t chunks = (p.k / 32 + 31) / 32;
  const int64_t warps = (p.n_src + static_cast<int64_t>(a.E) * a.pad_slots) * chunks;
  if (warps == 0) return cudaSuccess;
  const int64_t grid = (warps + kRowWarps - 1) / kRowWarps;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
  void* args[] = {&a};
  const void* f = peer ? (p.quantize ? reinterpret_cast<const void*>(moe_place_kernel<true, true>)
                                     : reinterpret_cast<const void*>(moe_place_kernel<false, true>))
                       : (p.quantize ? reinterpret_cast<const void*>(moe_place_kernel<true, false>)
                                     : reinterpret_cast<const void*>(moe_place_kernel<false, false>));
  return launch_pdl_cfg(f, dim3(static_cast<unsigned>(grid)), dim3(kRowWarps * 32), 0, args, stream);
}

cudaError_t launch_moe_gather(const void* src, int64_t src_rows, int64_t row_bytes, const int32_t* idx, int64_t n,
                              void* dst, int32_t* status, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int64_t grid = (n + kRowWarps - 1) / kRowWarps;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const uint4* s = static_cast<const uint4*>(src);
  uint4* d = static_cast<uint4*>(dst);
  int64_t vecs = row_bytes / 16;
  void* args[] = {&s, &src_rows, &vecs, &idx, &n, &d, &status};
  return launch_pdl_cfg(reinterpret_cast<const void*>(moe_gather_kernel), dim3(static_cast<unsigned>(grid)),
                        dim3(kRowWarps * 32), 0, args, stream);
}

cudaError_t launch_moe_combine(const void* y, const void* const* y_peers, const int32_t* row_rank, int ranks,
                               int64_t y_rows, int64_t n_cols, const int32_t* row, const float* w, int64_t tokens,
                               int topk, void* out, int32_t* status, cudaStream_t stream) {
  if (tokens == 0) return cudaSuccess;
  const int64_t warps = tokens * ((n_cols / 8 + 31) / 32);
  const int64_t grid = (warps + kRowWarps - 1) / kRowWarps;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const uint4* yp = static_cast<const uint4*>(y);
  const uint4* const* ypp = reinterpret_cast<const uint4* const*>(y_peers);
  uint4* op = static_cast<uint4*>(out);
  int64_t vecs = n_cols / 8;
  void* args[] = {&yp, &ypp, &row_rank, &ranks, &y_rows, &vecs, &row, &w, &tokens, &topk, &op, &status};
  const void* f = y_peers ? reinterpret_cast<const void*>(moe_combine_kernel<true>)
                          : reinterpret_cast<const void*>(moe_combine_kernel<false>);
  return launch_pdl_cfg(f, dim3(static_cast<unsigned>(grid)), dim3(kRowWarps * 32), 0, args, stream);
}

cudaError_t launch_moe_peer_plan(const int32_t* ids, const int32_t* row_send, int64_t n, const int32_t* count,
                                 int ranks, int rank, int E, int pad, int32_t* dst_rank, int32_t* dst_row,
                                 int32_t* counts_local, int32_t* offsets_local, int32_t* status, int num_sms,
                                 cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(5) * E * 4;  // at most 20 KB (E = 1024)
  int64_t grid = (n + kPlanThreads - 1) / kPlanThreads;
  if (grid < 1) grid = 1;  // block 0 writes the receive plan even with no entries
  if (grid > 2 * static_cast<int64_t>(num_sms)) grid = 2 * static_cast<int64_t>(num_sms);
  void* args[] = {&ids, &row_send, &n, &count, &ranks, &rank, &E, &pad, &dst_rank, &dst_row,
                  &counts_local, &offsets_local, &status};
  return launch_pdl_cfg(reinterpret_cast<const void*>(moe_peer_plan_kernel), dim3(static_cast<unsigned>(grid)),
                        dim3(kPlanThreads), smem, args, stream);
}

}  // namespace mxk
