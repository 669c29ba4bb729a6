// mx_api.cu -- the extern "C" boundary declared in include/mx.h: argument
// validation, then one kernel launch per call on the caller's stream.  No
// memory is allocated per call; the only device memory the library owns is the
// 4-byte internal status word below.
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>

#include "../../include/mx.h"

#include "mx_launch.h"

namespace {

constexpr int64_t kMaxGroups = 1024;
constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

__device__ int32_t g_internal_status = 0;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  static int cached_dev = -1, cached = 0;
  if (dev != cached_dev) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached = v;
    cached_dev = dev;
  }
  return cached;
}

int32_t* internal_status_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_internal_status) != cudaSuccess) return nullptr;
  return static_cast<int32_t*>(p);
}

mx_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MX_OK : MX_ERR_CUDA; }

constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // 2 s
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};

}  // namespace

uint64_t mxk::wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

extern "C" {

const char* mx_status_string(int status) {
  switch (status) {
    case MX_OK: return "MX_OK";
    case MX_ERR_INVALID_ARGUMENT: return "MX_ERR_INVALID_ARGUMENT";
    case MX_ERR_UNSUPPORTED_SHAPE: return "MX_ERR_UNSUPPORTED_SHAPE";
    case MX_ERR_MISALIGNED: return "MX_ERR_MISALIGNED";
    case MX_ERR_CUDA: return "MX_ERR_CUDA";
    default: return "MX_ERR_UNKNOWN";
  }
}

size_t mx_scale_bytes(int64_t rows, int64_t k) {
  if (rows <= 0 || k <= 0) return 0;
  const int64_t kb = (k + 31) / 32;
  return static_cast<size_t>(((rows + 127) / 128) * 128 * ((kb + 3) / 4) * 4);
}

// Host-side checks of one quantisation job; MX_OK with *empty set for a no-op.
static mx_status check_quant_job(const void* x, int64_t groups, int64_t rows, int64_t k, const void* q,
                                 const void* sf, bool* empty) {
  *empty = false;
  if (groups < 0 || rows < 0 || k < 0) return MX_ERR_INVALID_ARGUMENT;
  if (k % 32 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (groups == 0 || rows == 0 || k == 0) {
    *empty = true;
    return MX_OK;
  }
  if (!x || !q || !sf) return MX_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(q) || !aligned16(sf)) return MX_ERR_MISALIGNED;
  if (rows > kMaxDim || groups * rows > kMaxDim || groups * rows * (k / 32) >= (int64_t(1) << 31))
    return MX_ERR_UNSUPPORTED_SHAPE;
  return MX_OK;
}

static mx_status quantize_impl(const void* x, int64_t groups, int64_t rows, int64_t k, void* q, void* sf,
                               mx_stream_t stream) {
  bool empty = false;
  mx_status st = check_quant_job(x, groups, rows, k, q, sf, &empty);
  if (st != MX_OK || empty) return st;
  const int sms = num_sms();
  if (sms <= 0) return MX_ERR_CUDA;
  mxk::QuantSpec spec{x, q, sf, groups, rows, k, static_cast<int64_t>(mx_scale_bytes(rows, k))};
  return from_cuda(mxk::launch_quant_batch(&spec, 1, sms, reinterpret_cast<cudaStream_t>(stream), nullptr));
}

mx_status mx_quantize_bf16_to_e4m3(const void* x_bf16, int64_t rows, int64_t k, void* q_e4m3, void* sf_ue8m0,
                                   mx_stream_t stream) {
  return quantize_impl(x_bf16, 1, rows, k, q_e4m3, sf_ue8m0, stream);
}

mx_status mx_quantize_bf16_to_e4m3_grouped(const void* x_bf16, int64_t groups, int64_t rows, int64_t k,
                                           void* q_e4m3, void* sf_ue8m0, mx_stream_t stream) {
  return quantize_impl(x_bf16, groups, rows, k, q_e4m3, sf_ue8m0, stream);
}

static mx_status quantize_multi(const mx_quant_job* jobs, int32_t count, mx_stream_t stream, bool lean) {
  if (count < 0 || (count > 0 && !jobs)) return MX_ERR_INVALID_ARGUMENT;
  // validate everything before launching anything
  int nonempty = 0;
  for (int32_t i = 0; i < count; ++i) {
    bool empty = false;
    mx_status st = check_quant_job(jobs[i].x_bf16, jobs[i].groups, jobs[i].rows, jobs[i].k, jobs[i].q_e4m3,
                                   jobs[i].sf_ue8m0, &empty);
    if (st != MX_OK) return st;
    nonempty += empty ? 0 : 1;
  }
  if (nonempty == 0) return MX_OK;
  const int sms = num_sms();
  if (sms <= 0) return MX_ERR_CUDA;
  mxk::QuantSpec specs[mxk::kMaxQuantJobs];
  int n = 0;
  for (int32_t i = 0; i < count; ++i) {
    const mx_quant_job& j = jobs[i];
    if (j.groups == 0 || j.rows == 0 || j.k == 0) continue;
    specs[n++] = mxk::QuantSpec{j.x_bf16, j.q_e4m3, j.sf_ue8m0, j.groups, j.rows, j.k,
                                static_cast<int64_t>(mx_scale_bytes(j.rows, j.k))};
    if (n == mxk::kMaxQuantJobs) {
      cudaError_t e = mxk::launch_quant_batch(specs, n, sms, reinterpret_cast<cudaStream_t>(stream), nullptr, lean);
      if (e != cudaSuccess) return MX_ERR_CUDA;
      n = 0;
    }
  }
  if (n > 0) {
    cudaError_t e = mxk::launch_quant_batch(specs, n, sms, reinterpret_cast<cudaStream_t>(stream), nullptr, lean);
    if (e != cudaSuccess) return MX_ERR_CUDA;
  }
  return MX_OK;
}

mx_status mx_quantize_bf16_to_e4m3_multi(const mx_quant_job* jobs, int32_t count, mx_stream_t stream) {
  return quantize_multi(jobs, count, stream, false);
}

mx_status mx_quantize_bf16_to_e4m3_multi_lean(const mx_quant_job* jobs, int32_t count, mx_stream_t stream) {
  return quantize_multi(jobs, count, stream, true);
}

mx_status mx_quantize_bf16_to_e4m3_transposed(const void* x_bf16, int64_t groups, int64_t rows, int64_t cols,
                                              void* q_e4m3, void* sf_ue8m0, mx_stream_t stream) {
  if (groups < 0 || rows < 0 || cols < 0) return MX_ERR_INVALID_ARGUMENT;
  if (rows % 32 != 0 || cols % 8 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (groups == 0 || rows == 0 || cols == 0) return MX_OK;
  if (!x_bf16 || !q_e4m3 || !sf_ue8m0) return MX_ERR_INVALID_ARGUMENT;
  if (!aligned16(x_bf16) || !aligned16(q_e4m3) || !aligned16(sf_ue8m0)) return MX_ERR_MISALIGNED;
  if (rows > kMaxDim || cols > kMaxDim || groups * rows * cols / 32 >= (int64_t(1) << 40))
    return MX_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(mxk::launch_quant_transposed(x_bf16, groups, rows, cols, q_e4m3, sf_ue8m0,
                                                static_cast<int64_t>(mx_scale_bytes(cols, rows)),
                                                internal_status_ptr(), num_sms(),
                                                reinterpret_cast<cudaStream_t>(stream)));
}

static mx_status check_gemm_common(const void* qa, const void* sfa, const void* qb, const void* sfb, void* d,
                                   int64_t m, int64_t n, int64_t k, int64_t groups) {
  if (m < 0 || n < 0 || k < 0 || groups < 0) return MX_ERR_INVALID_ARGUMENT;
  if (k == 0 || k % 128 != 0 || n % 16 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (m > kMaxDim || n > kMaxDim || k > kMaxDim || groups > kMaxGroups) return MX_ERR_UNSUPPORTED_SHAPE;
  if (!qa || !sfa || !qb || !sfb || !d) return MX_ERR_INVALID_ARGUMENT;
  if (!aligned16(qa) || !aligned16(sfa) || !aligned16(qb) || !aligned16(sfb) || !aligned16(d))
    return MX_ERR_MISALIGNED;
  return MX_OK;
}

mx_status mx_gemm(const void* qa, const void* sfa, const void* qb, const void* sfb, void* d_bf16, int64_t m,
                  int64_t n, int64_t k, int32_t* dev_status, mx_stream_t stream) {
  if (m < 0 || n < 0 || k < 0) return MX_ERR_INVALID_ARGUMENT;
  if (m == 0 || n == 0) {
    if (k % 128 != 0 || k == 0 || n % 16 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
    return MX_OK;
  }
  mx_status st = check_gemm_common(qa, sfa, qb, sfb, d_bf16, m, n, k, 1);
  if (st != MX_OK) return st;
  const int sms = num_sms();
  if (sms <= 0) return MX_ERR_CUDA;
  int32_t* status = dev_status ? dev_status : internal_status_ptr();
  if (!status) return MX_ERR_CUDA;
  mxk::GemmProblem p{qa, sfa, qb, sfb, d_bf16, nullptr, nullptr, status, m, n, k, 1, 0};
  return from_cuda(mxk::launch_gemm(p, sms, reinterpret_cast<cudaStream_t>(stream), nullptr));
}

mx_status mx_gemm_batch(const mx_gemm_problem* problems, int32_t count, int32_t* dev_status, mx_stream_t stream) {
  static_assert(MX_GEMM_BATCH_MAX == mxk::kMaxBatch, "batch limit");
  if (!problems || count < 1 || count > MX_GEMM_BATCH_MAX) return MX_ERR_INVALID_ARGUMENT;
  mxk::GemmProblem ps[MX_GEMM_BATCH_MAX];
  int32_t* status = nullptr;
  int n_live = 0;
  for (int32_t i = 0; i < count; ++i) {  // every problem checked before anything is launched
    const mx_gemm_problem& q = problems[i];
    if (q.m < 0 || q.n < 0 || q.k < 0) return MX_ERR_INVALID_ARGUMENT;
    if (q.m == 0 || q.n == 0) {
      if (q.k % 128 != 0 || q.k == 0 || q.n % 16 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
      continue;
    }
    mx_status st = check_gemm_common(q.qa, q.sfa, q.qb, q.sfb, q.d_bf16, q.m, q.n, q.k, 1);
    if (st != MX_OK) return st;
    ++n_live;
  }
  if (n_live == 0) return MX_OK;
  const int sms = num_sms();
  if (sms <= 0) return MX_ERR_CUDA;
  status = dev_status ? dev_status : internal_status_ptr();
  if (!status) return MX_ERR_CUDA;
  int n = 0;
  for (int32_t i = 0; i < count; ++i) {
    const mx_gemm_problem& q = problems[i];
    if (q.m == 0 || q.n == 0) continue;
    ps[n++] = mxk::GemmProblem{q.qa, q.sfa, q.qb, q.sfb, q.d_bf16, nullptr, nullptr, status, q.m, q.n, q.k, 1, 0};
  }
  return from_cuda(mxk::launch_gemm_batch(ps, n, sms, reinterpret_cast<cudaStream_t>(stream), nullptr));
}

mx_status mx_grouped_gemm_contiguous(const void* qa, const void* sfa, const void* qb, const void* sfb,
                                     const int32_t* group_offsets, int32_t groups, int64_t m_total, int64_t n,
                                     int64_t k, void* d_bf16, int32_t* dev_status, mx_stream_t stream) {
  if (groups < 0 || m_total < 0 || n < 0 || k < 0) return MX_ERR_INVALID_ARGUMENT;
  if (k == 0 || k % 128 != 0 || n % 16 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (groups == 0 || m_total == 0 || n == 0) return MX_OK;
  if (!group_offsets) return MX_ERR_INVALID_ARGUMENT;
  mx_status st = check_gemm_common(qa, sfa, qb, sfb, d_bf16, m_total, n, k, groups);
  if (st != MX_OK) return st;
  if (reinterpret_cast<uintptr_t>(group_offsets) & 3u) return MX_ERR_MISALIGNED;
  const int sms = num_sms();
  if (sms <= 0) return MX_ERR_CUDA;
  int32_t* status = dev_status ? dev_status : internal_status_ptr();
  if (!status) return MX_ERR_CUDA;
  mxk::GemmProblem p{qa, sfa, qb, sfb, d_bf16, group_offsets, nullptr, status, m_total, n, k, groups, 1};
  return from_cuda(mxk::launch_gemm(p, sms, reinterpret_cast<cudaStream_t>(stream), nullptr));
}

mx_status mx_grouped_gemm_masked(const void* qa, const void* sfa, const void* qb, const void* sfb,
                                 const int32_t* masked_m, int32_t groups, int64_t max_m, int64_t n, int64_t k,
                                 void* d_bf16, int32_t* dev_status, mx_stream_t stream) {
  if (groups < 0 || max_m < 0 || n < 0 || k < 0) return MX_ERR_INVALID_ARGUMENT;
  if (k == 0 || k % 128 != 0 || n % 16 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (groups == 0 || max_m == 0 || n == 0) return MX_OK;
  if (!masked_m) return MX_ERR_INVALID_ARGUMENT;
  if (groups * max_m > kMaxDim) return MX_ERR_UNSUPPORTED_SHAPE;
  mx_status st = check_gemm_common(qa, sfa, qb, sfb, d_bf16, max_m, n, k, groups);
  if (st != MX_OK) return st;
  if (reinterpret_cast<uintptr_t>(masked_m) & 3u) return MX_ERR_MISALIGNED;
  const int sms = num_sms();
  if (sms <= 0) return MX_ERR_CUDA;
  int32_t* status = dev_status ? dev_status : internal_status_ptr();
  if (!status) return MX_ERR_CUDA;
  mxk::GemmProblem p{qa, sfa, qb, sfb, d_bf16, nullptr, masked_m, status, max_m, n, k, groups, 2};
  return from_cuda(mxk::launch_gemm(p, sms, reinterpret_cast<cudaStream_t>(stream), nullptr));
}

mx_status mx_grouped_gemm_kgrouped(const void* qa, const void* sfa, const void* qb, const void* sfb,
                                   const int32_t* group_offsets, int32_t groups, int64_t m, int64_t n,
                                   int64_t k_total, void* d_bf16, int32_t* dev_status, mx_stream_t stream) {
  if (groups < 0 || m < 0 || n < 0 || k_total < 0) return MX_ERR_INVALID_ARGUMENT;
  if (k_total == 0 || k_total % 128 != 0 || n % 16 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (groups == 0 || m == 0 || n == 0) return MX_OK;
  if (!group_offsets) return MX_ERR_INVALID_ARGUMENT;
  if (groups * m > kMaxDim) return MX_ERR_UNSUPPORTED_SHAPE;
  mx_status st = check_gemm_common(qa, sfa, qb, sfb, d_bf16, m, n, k_total, groups);
  if (st != MX_OK) return st;
  if (reinterpret_cast<uintptr_t>(group_offsets) & 3u) return MX_ERR_MISALIGNED;
  const int sms = num_sms();
  if (sms <= 0) return MX_ERR_CUDA;
  int32_t* status = dev_status ? dev_status : internal_status_ptr();
  if (!status) return MX_ERR_CUDA;
  mxk::GemmProblem p{qa, sfa, qb, sfb, d_bf16, group_offsets, nullptr, status, m, n, k_total, groups, 3};
  return from_cuda(mxk::launch_gemm(p, sms, reinterpret_cast<cudaStream_t>(stream), nullptr));
}

// ---------------------------------------------------------------- tile-wise FP32-scaled FP8

static mx_status tw_quantize(const void* x, int64_t rows, int64_t k, void* q, float* s, bool blocks,
                             mx_stream_t stream) {
  if (rows < 0 || k < 0) return MX_ERR_INVALID_ARGUMENT;
  if (k % 128 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0 || k == 0) return MX_OK;
  if (!x || !q || !s) return MX_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(s) & 3u)) return MX_ERR_MISALIGNED;
  if (rows > kMaxDim || k > kMaxDim) return MX_ERR_UNSUPPORTED_SHAPE;
  // the 1 x 128 kernel numbers its (8 rows x 128 columns) items in 32 bits
  if ((rows + 7) / 8 * (k / 128) > 0xFFFFFFF0LL) return MX_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(mxk::launch_tw_quant(x, rows, k, q, s, blocks, reinterpret_cast<cudaStream_t>(stream)));
}

mx_status mx_quantize_bf16_to_e4m3_tile1x128(const void* x_bf16, int64_t rows, int64_t k, void* q_e4m3,
                                             float* scales, mx_stream_t stream) {
  return tw_quantize(x_bf16, rows, k, q_e4m3, scales, false, stream);
}

mx_status mx_quantize_bf16_to_e4m3_block128x128(const void* x_bf16, int64_t rows, int64_t k, void* q_e4m3,
                                                float* scales, mx_stream_t stream) {
  return tw_quantize(x_bf16, rows, k, q_e4m3, scales, true, stream);
}

static mx_status tw_gemm(const void* qa, const float* sa, const void* qb, const float* sb,
                         const int32_t* group_offsets, int32_t groups, int64_t m, int64_t n, int64_t k, void* d,
                         int32_t* dev_status, int mode, mx_stream_t stream) {
  if (groups < 0 || m < 0 || n < 0 || k < 0) return MX_ERR_INVALID_ARGUMENT;
  if (k == 0 || k % 128 != 0 || n % 16 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (groups == 0 || m == 0 || n == 0) return MX_OK;
  if (!qa || !sa || !qb || !sb || !d || (mode == 1 && !group_offsets)) return MX_ERR_INVALID_ARGUMENT;
  if (!aligned16(qa) || !aligned16(qb) || !aligned16(d) || (reinterpret_cast<uintptr_t>(sa) & 3u) ||
      (reinterpret_cast<uintptr_t>(sb) & 3u) || (reinterpret_cast<uintptr_t>(group_offsets) & 3u))
    return MX_ERR_MISALIGNED;
  if (m > kMaxDim || n > kMaxDim || k > kMaxDim || groups > kMaxGroups) return MX_ERR_UNSUPPORTED_SHAPE;
  const int sms = num_sms();
  if (sms <= 0) return MX_ERR_CUDA;
  int32_t* status = dev_status ? dev_status : internal_status_ptr();
  if (!status) return MX_ERR_CUDA;
  mxk::TwProblem p{qa, sa, qb, sb, d, group_offsets, status, m, n, k, groups, mode};
  return from_cuda(mxk::launch_gemm_tw(p, sms, reinterpret_cast<cudaStream_t>(stream)));
}

mx_status mx_gemm_tilewise(const void* qa, const float* sa, const void* qb, const float* sb, void* d_bf16,
                           int64_t m, int64_t n, int64_t k, int32_t* dev_status, mx_stream_t stream) {
  return tw_gemm(qa, sa, qb, sb, nullptr, 1, m, n, k, d_bf16, dev_status, 0, stream);
}

mx_status mx_grouped_gemm_contiguous_tilewise(const void* qa, const float* sa, const void* qb, const float* sb,
                                              const int32_t* group_offsets, int32_t groups, int64_t m_total,
                                              int64_t n, int64_t k, void* d_bf16, int32_t* dev_status,
                                              mx_stream_t stream) {
  return tw_gemm(qa, sa, qb, sb, group_offsets, groups, m_total, n, k, d_bf16, dev_status, 1, stream);
}

// ---------------------------------------------------------------- fused SwiGLU + MXFP8 (expert MLP, first half)

static mx_status check_swiglu(const void* qh, const void* sfh, int64_t i_dim) {
  if (i_dim <= 0) return MX_ERR_INVALID_ARGUMENT;
  if (i_dim % 128 != 0 || 2 * i_dim > kMaxDim) return MX_ERR_UNSUPPORTED_SHAPE;
  if (!qh || !sfh) return MX_ERR_INVALID_ARGUMENT;
  if (!aligned16(qh) || !aligned16(sfh)) return MX_ERR_MISALIGNED;
  return MX_OK;
}

mx_status mx_gemm_swiglu_quant(const void* qa, const void* sfa, const void* qb, const void* sfb, void* qh,
                               void* sfh, int64_t m, int64_t i_dim, int64_t k, int32_t* dev_status,
                               mx_stream_t stream) {
  if (m < 0 || i_dim < 0 || k < 0) return MX_ERR_INVALID_ARGUMENT;
  if (k == 0 || k % 128 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (m == 0) return i_dim % 128 == 0 ? MX_OK : MX_ERR_UNSUPPORTED_SHAPE;
  mx_status st = check_swiglu(qh, sfh, i_dim);
  if (st != MX_OK) return st;
  st = check_gemm_common(qa, sfa, qb, sfb, qh, m, 2 * i_dim, k, 1);
  if (st != MX_OK) return st;
  const int sms = num_sms();
  if (sms <= 0) return MX_ERR_CUDA;
  int32_t* status = dev_status ? dev_status : internal_status_ptr();
  if (!status) return MX_ERR_CUDA;
  mxk::GemmProblem p{qa, sfa, qb, sfb, qh, nullptr, nullptr, status, m, 2 * i_dim, k, 1, 0};
  p.i_dim = i_dim;
  p.sf_out = sfh;
  return from_cuda(mxk::launch_gemm(p, sms, reinterpret_cast<cudaStream_t>(stream), nullptr));
}

mx_status mx_grouped_gemm_contiguous_swiglu_quant(const void* qa, const void* sfa, const void* qb, const void* sfb,
                                                  const int32_t* group_offsets, int32_t groups, int64_t m_total,
                                                  int64_t i_dim, int64_t k, void* qh, void* sfh,
                                                  int32_t* dev_status, mx_stream_t stream) {
  if (groups < 0 || m_total < 0 || i_dim < 0 || k < 0) return MX_ERR_INVALID_ARGUMENT;
  if (k == 0 || k % 128 != 0 || i_dim % 128 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (groups == 0 || m_total == 0 || i_dim == 0) return MX_OK;
  if (!group_offsets) return MX_ERR_INVALID_ARGUMENT;
  mx_status st = check_swiglu(qh, sfh, i_dim);
  if (st != MX_OK) return st;
  st = check_gemm_common(qa, sfa, qb, sfb, qh, m_total, 2 * i_dim, k, groups);
  if (st != MX_OK) return st;
  if (reinterpret_cast<uintptr_t>(group_offsets) & 3u) return MX_ERR_MISALIGNED;
  const int sms = num_sms();
  if (sms <= 0) return MX_ERR_CUDA;
  int32_t* status = dev_status ? dev_status : internal_status_ptr();
  if (!status) return MX_ERR_CUDA;
  mxk::GemmProblem p{qa, sfa, qb, sfb, qh, group_offsets, nullptr, status, m_total, 2 * i_dim, k, groups, 1};
  p.i_dim = i_dim;
  p.sf_out = sfh;
  return from_cuda(mxk::launch_gemm(p, sms, reinterpret_cast<cudaStream_t>(stream), nullptr));
}

mx_status mx_grouped_gemm_masked_swiglu_quant(const void* qa, const void* sfa, const void* qb, const void* sfb,
                                              const int32_t* masked_m, int32_t groups, int64_t max_m, int64_t i_dim,
                                              int64_t k, void* qh, void* sfh, int32_t* dev_status,
                                              mx_stream_t stream) {
  if (groups < 0 || max_m < 0 || i_dim < 0 || k < 0) return MX_ERR_INVALID_ARGUMENT;
  if (k == 0 || k % 128 != 0 || i_dim % 128 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (groups == 0 || max_m == 0 || i_dim == 0) return MX_OK;
  if (!masked_m) return MX_ERR_INVALID_ARGUMENT;
  if (groups * max_m > kMaxDim) return MX_ERR_UNSUPPORTED_SHAPE;
  mx_status st = check_swiglu(qh, sfh, i_dim);
  if (st != MX_OK) return st;
  st = check_gemm_common(qa, sfa, qb, sfb, qh, max_m, 2 * i_dim, k, groups);
  if (st != MX_OK) return st;
  if (reinterpret_cast<uintptr_t>(masked_m) & 3u) return MX_ERR_MISALIGNED;
  const int sms = num_sms();
  if (sms <= 0) return MX_ERR_CUDA;
  int32_t* status = dev_status ? dev_status : internal_status_ptr();
  if (!status) return MX_ERR_CUDA;
  mxk::GemmProblem p{qa, sfa, qb, sfb, qh, nullptr, masked_m, status, max_m, 2 * i_dim, k, groups, 2};
  p.i_dim = i_dim;
  p.sf_out = sfh;
  return from_cuda(mxk::launch_gemm(p, sms, reinterpret_cast<cudaStream_t>(stream), nullptr));
}

int64_t mx_moe_max_rows(int64_t n, int32_t experts, int32_t pad) {
  if (n < 0 || experts <= 0 || pad <= 0) return 0;
  const int64_t rows = n + static_cast<int64_t>(experts) * (pad - 1);
  return (rows + 127) / 128 * 128;
}

mx_status mx_moe_route(const int32_t* ids, int64_t n, int32_t experts, int32_t pad, int32_t* counts,
                       int32_t* offsets, int32_t* row, int32_t* dropped, mx_stream_t stream) {
  if (n < 0 || experts < 1 || experts > kMaxGroups || pad < 1 || pad > 128) return MX_ERR_INVALID_ARGUMENT;
  if (n > kMaxDim - 1024) return MX_ERR_UNSUPPORTED_SHAPE;
  if (!counts || !offsets || (n > 0 && (!ids || !row))) return MX_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(ids) | reinterpret_cast<uintptr_t>(counts) | reinterpret_cast<uintptr_t>(offsets) |
       reinterpret_cast<uintptr_t>(row) | reinterpret_cast<uintptr_t>(dropped)) & 3u)
    return MX_ERR_MISALIGNED;
  return from_cuda(mxk::launch_moe_route(ids, n, experts, pad, counts, offsets, row, dropped,
                                         static_cast<cudaStream_t>(stream)));
}

static mx_status check_place(const void* src, int64_t n_src, int64_t k, const int32_t* row, int32_t fan,
                             const int32_t* counts, const int32_t* offsets, int32_t experts, int32_t pad,
                             int64_t m_rows, const void* q, const void* sf, bool tiled) {
  if (n_src < 0 || k < 0 || m_rows < 0 || fan < 1 || fan > 64 || pad < 1 || pad > 128 || experts < 0 ||
      experts > kMaxGroups)
    return MX_ERR_INVALID_ARGUMENT;
  if (k % 128 != 0 || (tiled && m_rows % 128 != 0)) return MX_ERR_UNSUPPORTED_SHAPE;
  if (k > kMaxDim || m_rows > kMaxDim || n_src > kMaxDim || n_src * static_cast<int64_t>(fan) > kMaxDim)
    return MX_ERR_UNSUPPORTED_SHAPE;
  if (pad > 1 && experts > 0 && (!counts || !offsets)) return MX_ERR_INVALID_ARGUMENT;
  if (k == 0 || (n_src == 0 && (pad == 1 || experts == 0))) return MX_OK;
  if (!q || !sf || (n_src > 0 && (!src || !row))) return MX_ERR_INVALID_ARGUMENT;
  if (!aligned16(src) || !aligned16(q) || !aligned16(sf)) return MX_ERR_MISALIGNED;
  return MX_OK;
}

mx_status mx_moe_dispatch_quant(const void* x_bf16, int64_t tokens, int64_t k, const int32_t* row, int32_t topk,
                                const int32_t* counts, const int32_t* offsets, int32_t experts, int32_t pad,
                                int64_t m_rows, void* q_e4m3, void* sf, int32_t sf_row_major,
                                int32_t* dev_status, mx_stream_t stream) {
  mx_status st = check_place(x_bf16, tokens, k, row, topk, counts, offsets, experts, pad, m_rows, q_e4m3, sf,
                             sf_row_major == 0);
  if (st != MX_OK) return st;
  if (k == 0 || (tokens == 0 && (pad == 1 || experts == 0))) return MX_OK;
  mxk::MoePlace p = {};
  p.src = x_bf16;
  p.row = row;
  p.counts = counts;
  p.offsets = offsets;
  p.q = q_e4m3;
  p.sf = sf;
  p.status = dev_status ? dev_status : internal_status_ptr();
  p.n_src = tokens;
  p.m_rows = m_rows;
  p.k = k;
  p.fan = topk;
  p.experts = experts;
  p.pad = pad;
  p.sf_row_major = sf_row_major != 0;
  p.quantize = true;
  return from_cuda(mxk::launch_moe_place(p, static_cast<cudaStream_t>(stream)));
}

mx_status mx_moe_scatter_rows(const void* q_src, const void* sf_src, int64_t n_src, int64_t k,
                              const int32_t* dst_row, const int32_t* counts, const int32_t* offsets,
                              int32_t experts, int32_t pad, int64_t m_rows, void* q_dst, void* sf_dst,
                              int32_t* dev_status, mx_stream_t stream) {
  mx_status st = check_place(q_src, n_src, k, dst_row, 1, counts, offsets, experts, pad, m_rows, q_dst, sf_dst, true);
  if (st != MX_OK) return st;
  if (k == 0 || (n_src == 0 && (pad == 1 || experts == 0))) return MX_OK;
  if (n_src > 0 && !sf_src) return MX_ERR_INVALID_ARGUMENT;
  mxk::MoePlace p = {};
  p.src = q_src;
  p.src_sf = sf_src;
  p.row = dst_row;
  p.counts = counts;
  p.offsets = offsets;
  p.q = q_dst;
  p.sf = sf_dst;
  p.status = dev_status ? dev_status : internal_status_ptr();
  p.n_src = n_src;
  p.m_rows = m_rows;
  p.k = k;
  p.fan = 1;
  p.experts = experts;
  p.pad = pad;
  p.sf_row_major = 0;
  p.quantize = false;
  return from_cuda(mxk::launch_moe_place(p, static_cast<cudaStream_t>(stream)));
}

mx_status mx_gather_rows(const void* src, int64_t src_rows, int64_t row_bytes, const int32_t* idx, int64_t n,
                         void* dst, int32_t* dev_status, mx_stream_t stream) {
  if (src_rows < 0 || row_bytes < 0 || n < 0) return MX_ERR_INVALID_ARGUMENT;
  if (row_bytes % 16 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (n > kMaxDim || src_rows > kMaxDim) return MX_ERR_UNSUPPORTED_SHAPE;
  if (n == 0 || row_bytes == 0) return MX_OK;
  if (!idx || !dst || (src_rows > 0 && !src)) return MX_ERR_INVALID_ARGUMENT;
  if (!aligned16(src) || !aligned16(dst)) return MX_ERR_MISALIGNED;
  int32_t* status = dev_status ? dev_status : internal_status_ptr();
  return from_cuda(mxk::launch_moe_gather(src, src_rows, row_bytes, idx, n, dst, status,
                                          static_cast<cudaStream_t>(stream)));
}

mx_status mx_moe_combine(const void* y_bf16, int64_t y_rows, int64_t n_cols, const int32_t* row, const float* w,
                         int64_t tokens, int32_t topk, void* out_bf16, int32_t* dev_status, mx_stream_t stream) {
  if (y_rows < 0 || n_cols < 0 || tokens < 0 || topk < 1 || topk > 64) return MX_ERR_INVALID_ARGUMENT;
  if (n_cols % 8 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (tokens > kMaxDim || y_rows > kMaxDim || tokens * static_cast<int64_t>(topk) > kMaxDim)
    return MX_ERR_UNSUPPORTED_SHAPE;
  if (tokens == 0 || n_cols == 0) return MX_OK;
  if (!row || !w || !out_bf16 || (y_rows > 0 && !y_bf16)) return MX_ERR_INVALID_ARGUMENT;
  if (!aligned16(y_bf16) || !aligned16(out_bf16) || (reinterpret_cast<uintptr_t>(w) & 3u) ||
      (reinterpret_cast<uintptr_t>(row) & 3u))
    return MX_ERR_MISALIGNED;
  int32_t* status = dev_status ? dev_status : internal_status_ptr();
  return from_cuda(mxk::launch_moe_combine(y_bf16, nullptr, nullptr, 0, y_rows, n_cols, row, w, tokens, topk,
                                           out_bf16, status, static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------ expert parallelism over peer memory

mx_status mx_moe_peer_plan(const int32_t* ids, const int32_t* row_send, int64_t n, const int32_t* count_table,
                           int32_t ranks, int32_t rank, int32_t experts, int32_t pad, int32_t* dst_rank,
                           int32_t* dst_row, int32_t* counts_local, int32_t* offsets_local, int32_t* dev_status,
                           mx_stream_t stream) {
  if (n < 0 || ranks < 1 || ranks > kMaxGroups || rank < 0 || rank >= ranks || experts < 1 ||
      experts > kMaxGroups || pad < 1 || pad > 128 || experts % ranks != 0)
    return MX_ERR_INVALID_ARGUMENT;
  // every entry of every rank plus each expert's padding: the largest row
  // index and padded offset the plan can produce must fit in int32
  if (n * static_cast<int64_t>(ranks) + static_cast<int64_t>(experts) * (pad - 1) > kMaxDim)
    return MX_ERR_UNSUPPORTED_SHAPE;
  if (!count_table || !counts_local || !offsets_local || (n > 0 && (!ids || !row_send || !dst_rank || !dst_row)))
    return MX_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(ids) | reinterpret_cast<uintptr_t>(row_send) |
       reinterpret_cast<uintptr_t>(count_table) | reinterpret_cast<uintptr_t>(dst_rank) |
       reinterpret_cast<uintptr_t>(dst_row) | reinterpret_cast<uintptr_t>(counts_local) |
       reinterpret_cast<uintptr_t>(offsets_local)) & 3u)
    return MX_ERR_MISALIGNED;
  const int sms = num_sms();
  if (sms <= 0) return MX_ERR_CUDA;
  int32_t* status = dev_status ? dev_status : internal_status_ptr();
  if (!status) return MX_ERR_CUDA;
  return from_cuda(mxk::launch_moe_peer_plan(ids, row_send, n, count_table, ranks, rank, experts, pad, dst_rank,
                                             dst_row, counts_local, offsets_local, status, sms,
                                             static_cast<cudaStream_t>(stream)));
}

mx_status mx_moe_dispatch_quant_peer(const void* x_bf16, int64_t tokens, int64_t k, const int32_t* dst_rank,
                                     const int32_t* dst_row, int32_t topk, void* const* q_peers,
                                     void* const* sf_peers, int32_t ranks, int64_t m_rows, void* q_local,
                                     void* sf_local, const int32_t* counts_local, const int32_t* offsets_local,
                                     int32_t experts_local, int32_t pad, int32_t* dev_status, mx_stream_t stream) {
  if (ranks < 1 || ranks > kMaxGroups) return MX_ERR_INVALID_ARGUMENT;
  mx_status st = check_place(x_bf16, tokens, k, dst_row, topk, counts_local, offsets_local, experts_local, pad,
                             m_rows, q_local, sf_local, true);
  if (st != MX_OK) return st;
  if (k == 0 || (tokens == 0 && (pad == 1 || experts_local == 0))) return MX_OK;
  if (tokens > 0 && (!dst_rank || !q_peers || !sf_peers)) return MX_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(q_peers) | reinterpret_cast<uintptr_t>(sf_peers)) & 7u ||
      (reinterpret_cast<uintptr_t>(dst_rank) & 3u))
    return MX_ERR_MISALIGNED;
  mxk::MoePlace p = {};
  p.src = x_bf16;
  p.row = dst_row;
  p.counts = counts_local;
  p.offsets = offsets_local;
  p.q = q_local;
  p.sf = sf_local;
  p.status = dev_status ? dev_status : internal_status_ptr();
  p.n_src = tokens;
  p.m_rows = m_rows;
  p.k = k;
  p.fan = topk;
  p.experts = experts_local;
  p.pad = pad;
  p.sf_row_major = 0;
  p.quantize = true;
  p.q_peers = q_peers;
  p.sf_peers = sf_peers;
  p.row_rank = dst_rank;
  p.ranks = ranks;
  return from_cuda(mxk::launch_moe_place(p, static_cast<cudaStream_t>(stream)));
}

mx_status mx_moe_combine_peer(const void* const* y_peers, int32_t ranks, int64_t y_rows, int64_t n_cols,
                              const int32_t* src_rank, const int32_t* src_row, const float* w, int64_t tokens,
                              int32_t topk, void* out_bf16, int32_t* dev_status, mx_stream_t stream) {
  if (ranks < 1 || ranks > kMaxGroups || y_rows < 0 || n_cols < 0 || tokens < 0 || topk < 1 || topk > 64)
    return MX_ERR_INVALID_ARGUMENT;
  if (n_cols % 8 != 0) return MX_ERR_UNSUPPORTED_SHAPE;
  if (tokens > kMaxDim || y_rows > kMaxDim || tokens * static_cast<int64_t>(topk) > kMaxDim)
    return MX_ERR_UNSUPPORTED_SHAPE;
  if (tokens == 0 || n_cols == 0) return MX_OK;
  if (!y_peers || !src_rank || !src_row || !w || !out_bf16) return MX_ERR_INVALID_ARGUMENT;
  if (!aligned16(out_bf16) || (reinterpret_cast<uintptr_t>(y_peers) & 7u) ||
      ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(src_rank) |
        reinterpret_cast<uintptr_t>(src_row)) & 3u))
    return MX_ERR_MISALIGNED;
  int32_t* status = dev_status ? dev_status : internal_status_ptr();
  return from_cuda(mxk::launch_moe_combine(nullptr, y_peers, src_rank, ranks, y_rows, n_cols, src_row, w, tokens,
                                           topk, out_bf16, status, static_cast<cudaStream_t>(stream)));
}

mx_status mx_set_wait_limit_ns(uint64_t ns) {
  g_wait_ns.store(ns == 0 ? kDefaultWaitNs : ns, std::memory_order_relaxed);
  return MX_OK;
}

uint64_t mx_wait_limit_ns(void) { return g_wait_ns.load(std::memory_order_relaxed); }

mx_status mx_read_internal_status(int32_t* host_out, int clear) {
  if (!host_out) return MX_ERR_INVALID_ARGUMENT;
  if (cudaDeviceSynchronize() != cudaSuccess) return MX_ERR_CUDA;
  if (cudaMemcpyFromSymbol(host_out, g_internal_status, sizeof(int32_t)) != cudaSuccess) return MX_ERR_CUDA;
  if (clear) {
    const int32_t zero = 0;
    if (cudaMemcpyToSymbol(g_internal_status, &zero, sizeof(int32_t)) != cudaSuccess) return MX_ERR_CUDA;
  }
  return MX_OK;
}

}  // extern "C"
