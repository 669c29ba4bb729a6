"""Failure detection in the GEMM kernels: every wait inside a kernel is
bounded, and a wait that runs out makes the kernel give up cleanly.

The wait bound is lowered (mx_set_wait_limit_ns) to 1 us, far below the
legitimate wait of the epilogue for an accumulator that needs a K loop of
512K elements (about a millisecond), so that wait runs out on every CTA.
Each call must then report MX_DEV_TIMEOUT in its status word, leave every
byte outside D untouched, and leave the context usable: with the default
bound restored, the same GEMM reports nothing and matches the oracle on
sampled rows, and so does the PR1 GEMM.  The give-up path is taken with
TMA loads, block-scaled MMAs and scale copies in flight, so it exercises
the drains (MMAs and copies waited on, loads allowed to land before the CTA
ends, TMEM freed last).

Each tile configuration runs in a child process (MX_GEMM_CONFIG forces the
one-CTA persistent kernel, split-K over a cluster of 2, or the CTA-pair
kernel), so that a failure there cannot affect the other tests."""
import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest

import mx_inputs
from mxtest_util import assert_gemm_close, oracle_quantize

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
M, N, K = 256, 512, 512 * 1024
ROWS = [0, 1, 127, 128, 200, 255]
GUARD = 4096        # BF16 elements of sentinel before and after D

CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import moe_grouped_gemm_mx_b200 as mx, mx_inputs
M, N, K, GUARD = %d, %d, %d, %d
ROWS = %r
out = sys.argv[2]
dev = torch.device("cuda")
a, b = mx_inputs.dense_problem(M, N, K, seed=21, device=dev)
qa, sfa = mx.mx_quantize_bf16_to_e4m3(a)
qb, sfb = mx.mx_quantize_bf16_to_e4m3(b)
sentinel = torch.tensor([0x7FBF], dtype=torch.int16).view(torch.bfloat16)   # a NaN pattern no result has
buf = sentinel.to(dev).repeat(M * N + 2 * GUARD)
d = buf[GUARD:GUARD + M * N].view(M, N)
st = torch.zeros(1, dtype=torch.int32, device=dev)
res = {}
for rep in range(2):                                # two failing calls in a row
    mx.mx_set_wait_limit_ns(1000)
    mx.mx_gemm(qa, sfa, qb, sfb, d=d, dev_status=st)
    torch.cuda.synchronize()
    res[f"timeout_status_{rep}"] = np.array(int(st.item()))
    st.zero_()
    g = buf.view(torch.int16)
    res[f"guards_intact_{rep}"] = np.array(bool((g[:GUARD] == 0x7FBF).all()) and bool((g[-GUARD:] == 0x7FBF).all()))
mx.mx_set_wait_limit_ns(0)
res["limit_restored"] = np.array(mx.mx_wait_limit_ns())
mx.mx_gemm(qa, sfa, qb, sfb, d=d, dev_status=st)
torch.cuda.synchronize()
res["status_after"] = np.array(int(st.item()))
res["d_rows"] = d[ROWS].float().cpu().numpy()
res["a_rows"] = a[ROWS].cpu().view(torch.int16).numpy()
res["b"] = b.cpu().view(torch.int16).numpy()
a1, b1 = mx_inputs.dense_problem(128, 256, 512, seed=0)      # generated on the CPU, as the parent does
q1, s1 = mx.mx_quantize_bf16_to_e4m3(a1.to(dev))
q2, s2 = mx.mx_quantize_bf16_to_e4m3(b1.to(dev))
st.zero_()
res["pr1"] = mx.mx_gemm(q1, s1, q2, s2, dev_status=st).float().cpu().numpy()
torch.cuda.synchronize()
res["pr1_status"] = np.array(int(st.item()))
np.savez(out, **res)
""" % (M, N, K, GUARD, ROWS)


@pytest.mark.parametrize("cfg", [0, 2, 7], ids=["one-cta-128x256", "split2", "pair256"])
def test_wait_timeout_reported_and_recovered(oracle, cfg):
    import torch
    with tempfile.TemporaryDirectory() as td:
        out = os.path.join(td, "r.npz")
        env = dict(os.environ, MX_GEMM_CONFIG=str(cfg))
        r = subprocess.run([sys.executable, "-c", CHILD, ROOT, out], env=env, capture_output=True, text=True,
                           timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        got = np.load(out)
        import moe_grouped_gemm_mx_b200 as mx
        for rep in range(2):
            assert int(got[f"timeout_status_{rep}"]) & mx.MX_DEV_TIMEOUT, \
                f"call {rep}: status {int(got[f'timeout_status_{rep}']):#x}, no timeout reported"
            assert bool(got[f"guards_intact_{rep}"]), f"call {rep}: bytes outside D were written"
        assert int(got["limit_restored"]) == 2_000_000_000
        assert int(got["status_after"]) == 0, f"status {int(got['status_after']):#x} after restoring the bound"
        # the GEMM after the failures: sampled rows against the oracle
        a_rows = torch.from_numpy(got["a_rows"]).view(torch.bfloat16)
        b = torch.from_numpy(got["b"]).view(torch.bfloat16)
        qa, sfa = oracle_quantize(oracle, a_rows)
        qb, sfb = oracle_quantize(oracle, b)
        d_ref, absd = oracle.gemm(qa, sfa, qb, sfb)
        assert_gemm_close(got["d_rows"].astype(np.float64), d_ref, absd, f"cfg {cfg}: GEMM after the timeouts")
        # and the PR1 GEMM
        assert int(got["pr1_status"]) == 0
        a1, b1 = mx_inputs.dense_problem(128, 256, 512, seed=0)
        qa, sfa = oracle_quantize(oracle, a1)
        qb, sfb = oracle_quantize(oracle, b1)
        d_ref, absd = oracle.gemm(qa, sfa, qb, sfb)
        assert_gemm_close(got["pr1"].astype(np.float64), d_ref, absd, f"cfg {cfg}: PR1 after the timeouts")
