"""The quantiser's launch-time integer division (multiply-high and shift)
against exact integer division, compiled for the host from the same header
the kernel uses."""
import os
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "moe_grouped_gemm_mx_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <cstdint>
#include "mx_fastdiv.h"
int main() {
  using namespace mxk;
  uint64_t bad = 0, checked = 0;
  uint32_t ds[] = {1u, 2u, 3u, 4u, 5u, 7u, 16u, 48u, 56u, 64u, 127u, 128u, 200u, 224u, 256u, 4096u,
                   7168u, 65536u, 69632u, 1000003u, 2147483647u, 2147483648u, 2147483649u, 4294967295u};
  uint64_t x = 88172645463325252ull;
  for (uint32_t d : ds) {
    FastDiv f = make_fastdiv(d);
    for (uint64_t n = 0; n < 70000; ++n) { checked++; if (fdiv((uint32_t)n, f) != (uint32_t)n / d) bad++; }
    for (uint64_t n = 0xFFFFFFFFull - 70000; n <= 0xFFFFFFFFull; ++n) { checked++; if (fdiv((uint32_t)n, f) != (uint32_t)n / d) bad++; }
    for (int i = 0; i < 200000; ++i) {
      x ^= x << 13; x ^= x >> 7; x ^= x << 17;
      uint32_t n = (uint32_t)x; checked++;
      if (fdiv(n, f) != n / d) bad++;
    }
    for (uint64_t q = 1; q * d < 0xFFFFFFFFull && q < 5000; ++q) {   // around multiples of d
      for (int64_t e = -1; e <= 1; ++e) { uint64_t n = q * d + e; if (n > 0xFFFFFFFFull) continue;
        checked++; if (fdiv((uint32_t)n, f) != (uint32_t)n / d) bad++; }
    }
  }
  printf("%llu %llu\n", (unsigned long long)checked, (unsigned long long)bad);
  return bad != 0;
}
"""


def test_fastdiv_matches_integer_division():
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "t.cpp")
        exe = os.path.join(td, "t")
        open(src, "w").write(PROGRAM)
        subprocess.run(["g++", "-O2", "-std=c++17", "-I", HDR, "-o", exe, src], check=True)
        out = subprocess.run([exe], capture_output=True, text=True)
        checked, bad = map(int, out.stdout.split())
        assert checked > 1_000_000
        assert bad == 0, out.stdout
