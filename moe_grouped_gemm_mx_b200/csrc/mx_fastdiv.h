// mx_fastdiv.h -- division of 32-bit unsigned integers by a divisor fixed at
// launch time, by multiply-high and shift (the "round-up" method of Granlund
// & Montgomery, "Division by invariant integers using multiplication", PLDI
// 1994): with s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1,
//     n / d = (umulhi(n, m) + n) >> s        for every 0 <= n < 2^32.
// Host and device code; the host side also serves the CPU unit test.
#pragma once
#include <cstdint>

#if defined(__CUDACC__)
#define MX_HD __host__ __device__ __forceinline__
#else
#define MX_HD inline
#endif

namespace mxk {

struct FastDiv {
  uint32_t d, m, s;
};

inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t s = 0;
  while ((uint64_t(1) << s) < d) ++s;
  const uint64_t m = ((uint64_t(1) << 32) * ((uint64_t(1) << s) - d)) / d + 1;
  return FastDiv{d, static_cast<uint32_t>(m), s};
}

MX_HD uint32_t mulhi32(uint32_t a, uint32_t b) {
#if defined(__CUDA_ARCH__)
  return __umulhi(a, b);
#else
  return static_cast<uint32_t>((static_cast<uint64_t>(a) * b) >> 32);
#endif
}

MX_HD uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return static_cast<uint32_t>((static_cast<uint64_t>(mulhi32(n, f.m)) + n) >> f.s);
}

}  // namespace mxk
