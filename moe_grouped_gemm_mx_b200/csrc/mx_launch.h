// mx_launch.h -- host-side launch entry points shared by the C ABI (mx_api.cu)
// and the kernel translation units.  Internal to the library.
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

namespace mxk {

constexpr int kMaxQuantJobs = 8;  // tensors one quantiser launch handles

// Bound, in ns, of every pipeline wait of the GEMM kernels launched from now
// on (mx_set_wait_limit_ns; 2 s unless changed).
uint64_t wait_limit_ns();

struct QuantSpec {
  const void* x;            // BF16 [groups, rows, k]
  void* q;                  // E4M3 out, same shape
  void* sf;                 // tiled scales out, groups regions of sf_group_bytes
  int64_t groups, rows, k;
  int64_t sf_group_bytes;
};

// lean: the shared-memory-free form, one CTA per SM (to run beside a GEMM)
cudaError_t launch_quant_batch(const QuantSpec* specs, int count, int num_sms, cudaStream_t stream, int* launches,
                               bool lean = false);

// Quantisation along the rows of x [groups, rows, cols] into q [groups, cols,
// rows] with per-group tiled scales of the [cols, rows] operand.
cudaError_t launch_quant_transposed(const void* x, int64_t groups, int64_t rows, int64_t cols, void* q, void* sf,
                                    int64_t sf_group_bytes, int32_t* status, int num_sms, cudaStream_t stream);

struct GemmProblem {
  const void* qa;
  const void* sfa;
  const void* qb;
  const void* sfb;
  void* d;
  const int32_t* group_offsets;  // contiguous form only (device, groups + 1)
  const int32_t* masked_m;       // masked form only (device, groups)
  int32_t* status;               // device status word, never null
  int64_t m, n, k;               // m: dense M / contiguous m_total / masked max_m
  int64_t groups;                // experts (1 for the dense form)
  int mode;                      // 0 dense, 1 contiguous, 2 masked
  // fused SwiGLU + MXFP8 requantisation epilogue (i_dim > 0): qb holds
  // [gate; up] = 2 * i_dim rows per expert, d receives E4M3 H [.., i_dim]
  // and sf_out its tiled scales
  int64_t i_dim = 0;
  void* sf_out = nullptr;
};

cudaError_t launch_gemm(const GemmProblem& p, int num_sms, cudaStream_t stream, int* launches);

// Up to kMaxBatch independent dense problems (mode 0) in one launch, the
// GPU shared among them (mx_gemm.cu).  Empty problems are skipped.
constexpr int kMaxBatch = 4;
cudaError_t launch_gemm_batch(const GemmProblem* ps, int count, int num_sms, cudaStream_t stream, int* launches);

// CTA-pair (2-SM MMA) kernel for large problems, any of the three forms.
cudaError_t launch_gemm_pair(const GemmProblem& p, int num_sms, cudaStream_t stream, int* launches);

// Tile-wise FP32-scaled FP8 (mx_quant_tw.cu): blocks == false -> one scale per
// row and 128-element K tile, s [k/128, rows]; true -> one per 128 x 128 block,
// s [ceil(rows/128), k/128].
cudaError_t launch_tw_quant(const void* x, int64_t rows, int64_t k, void* q, float* s, bool blocks,
                            cudaStream_t stream);

struct TwProblem {
  const void* qa;                // [m, k] E4M3
  const float* sa;               // [k/128, m]
  const void* qb;                // [groups, n, k] E4M3
  const float* sb;               // [groups, ceil(n/128), k/128]
  void* d;                       // [m, n] BF16
  const int32_t* group_offsets;  // contiguous form only
  int32_t* status;
  int64_t m, n, k, groups;
  int mode;                      // 0 dense, 1 contiguous
};

cudaError_t launch_gemm_tw(const TwProblem& p, int num_sms, cudaStream_t stream);

// MoE expert-layer data movement (mx_moe.cu).
cudaError_t launch_moe_route(const int32_t* ids, int64_t n, int E, int pad, int32_t* counts, int32_t* offsets,
                             int32_t* row, int32_t* dropped, cudaStream_t stream);

struct MoePlace {
  const void* src;          // quantize: BF16 [n_src, k]; else E4M3 [n_src, k]
  const void* src_sf;       // !quantize: row-major scales [n_src, k/32]
  const int32_t* row;       // [n_src * fan] destination rows (-1: none)
  const int32_t* counts;    // [experts]
  const int32_t* offsets;   // [experts + 1]
  void* q;                  // [m_rows, k]
  void* sf;                 // tiled over m_rows, or row-major [m_rows, k/32]
  int32_t* status;
  int64_t n_src, m_rows, k;
  int fan, experts, pad, sf_row_major;
  bool quantize;
  // peer form (expert parallelism over peer memory): destination j of source
  // row i is row row[i*fan+j] of rank row_rank[i*fan+j]'s buffers, device
  // tables q_peers / sf_peers [ranks]; q / sf are this rank's own (padding)
  void* const* q_peers = nullptr;
  void* const* sf_peers = nullptr;
  const int32_t* row_rank = nullptr;
  int ranks = 0;
};
cudaError_t launch_moe_place(const MoePlace& p, cudaStream_t stream);
cudaError_t launch_moe_gather(const void* src, int64_t src_rows, int64_t row_bytes, const int32_t* idx, int64_t n,
                              void* dst, int32_t* status, cudaStream_t stream);
// y_peers != nullptr: the peer form, routed row j of token t is row
// row[t*topk+j] of rank row_rank[t*topk+j]'s output (device table [ranks]).
cudaError_t launch_moe_combine(const void* y, const void* const* y_peers, const int32_t* row_rank, int ranks,
                               int64_t y_rows, int64_t n_cols, const int32_t* row, const float* w, int64_t tokens,
                               int topk, void* out, int32_t* status, cudaStream_t stream);
cudaError_t launch_moe_peer_plan(const int32_t* ids, const int32_t* row_send, int64_t n, const int32_t* count,
                                 int ranks, int rank, int E, int pad, int32_t* dst_rank, int32_t* dst_row,
                                 int32_t* counts_local, int32_t* offsets_local, int32_t* status, int num_sms,
                                 cudaStream_t stream);

}  // namespace mxk
