"""Every GEMM tile configuration (persistent 128x256, persistent 128x128 with
a double-buffered accumulator, split-K over clusters of 2/4/8 CTAs) on the
same shapes against the oracle.  The configuration is forced through the
library's tuning override MX_GEMM_CONFIG, read once per process, so each
configuration runs in a child process."""
import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch

import mx_inputs
from mxtest_util import assert_gemm_close, oracle_quantize

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = [(200, 272, 1152), (64, 528, 1024), (129, 256, 1280)]

CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import moe_grouped_gemm_mx_b200 as mx, mx_inputs
out = sys.argv[2]
res = {}
for (m, n, k) in %r:
    a, b = mx_inputs.dense_problem(m, n, k, seed=m + n, kind="outlier")
    qa, sfa = mx.mx_quantize_bf16_to_e4m3(a.cuda())
    qb, sfb = mx.mx_quantize_bf16_to_e4m3(b.cuda())
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    d = mx.mx_gemm(qa, sfa, qb, sfb, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, hex(int(st.item()))
    res[f"{m}x{n}x{k}"] = d.float().cpu().numpy()
np.savez(out, **res)
""" % (SHAPES,)


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4], ids=["128x256", "128x128x2acc", "split2", "split4", "split8"])
def test_forced_config(oracle, cfg):
    with tempfile.TemporaryDirectory() as td:
        out = os.path.join(td, "d.npz")
        env = dict(os.environ, MX_GEMM_CONFIG=str(cfg))
        r = subprocess.run([sys.executable, "-c", CHILD, ROOT, out], env=env, capture_output=True, text=True,
                           timeout=300)
        assert r.returncode == 0, r.stderr[-2000:]
        got = np.load(out)
        for (m, n, k) in SHAPES:
            a, b = mx_inputs.dense_problem(m, n, k, seed=m + n, kind="outlier")
            qa, sfa = oracle_quantize(oracle, a)
            qb, sfb = oracle_quantize(oracle, b)
            d_ref, absd = oracle.gemm(qa, sfa, qb, sfb)
            assert_gemm_close(got[f"{m}x{n}x{k}"].astype(np.float64), d_ref, absd, f"cfg {cfg} {m}x{n}x{k}")
