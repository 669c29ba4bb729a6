"""The tile-wise quantisers divide each element by its tile's FP32 scale
without a division instruction: q0 = RN(x * r) with r = RN(1 / s), then one
FMA correction, q = RN(q0 - RN(q0 * s - x) * r).  The kernels rely on q
being the correctly rounded quotient RN(x / s) for every BF16 x and every
scale s = RN(amax / 448) of a BF16 amax.  Both have only 128 significands,
and the roundings scale exactly with the exponents while no value leaves the
normal range, so the claim reduces to 128 x 128 significand pairs; this test
checks them (over several exponent offsets) on the host with IEEE single
precision and the C library's correctly rounded fmaf, and that the
uncorrected product alone is not enough."""
import os
import subprocess
import tempfile

import pytest

SRC = r"""
#include <math.h>
#include <stdio.h>
int main(void) {
    long bad_q0 = 0, bad_q = 0, total = 0;
    const int ea_list[3] = {-40, 0, 40};
    for (int e = 0; e < 3; ++e)
    for (int k = 0; k < 128; ++k) {
        volatile float amax = ldexpf(1.0f + k / 128.0f, ea_list[e]);
        volatile float s = amax / 448.0f;
        volatile float r = 1.0f / s;
        for (int d = -14; d <= 0; ++d)
        for (int j = 0; j < 128; ++j) {
            volatile float x = ldexpf(1.0f + j / 128.0f, ea_list[e] + d);
            if (x > amax) continue;
            for (int sg = 0; sg < 2; ++sg) {
                volatile float xs = sg ? -x : x;
                volatile float ref = xs / s;
                volatile float q0 = xs * r;
                volatile float t = fmaf(q0, s, -xs);
                volatile float q = fmaf(-t, r, q0);
                ++total;
                bad_q0 += q0 != ref;
                bad_q += q != ref;
            }
        }
    }
    printf("%ld %ld %ld\n", total, bad_q0, bad_q);
    return 0;
}
"""


def test_fma_corrected_quotient_is_correctly_rounded():
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "q.c")
        exe = os.path.join(td, "q")
        with open(src, "w") as f:
            f.write(SRC)
        try:
            subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", exe, src, "-lm"], check=True,
                           capture_output=True, timeout=120)
        except (FileNotFoundError, subprocess.CalledProcessError) as e:
            pytest.skip(f"no C compiler: {e}")
        out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=300).stdout.split()
    total, bad_q0, bad_q = (int(v) for v in out)
    assert total > 1_000_000
    assert bad_q0 > 0          # the product alone is often off by an ulp
    assert bad_q == 0, f"{bad_q} of {total} corrected quotients differ from RN(x / s)"
