"""Every GEMM tile configuration (persistent 128x256, persistent 128x128 with
a double-buffered accumulator, split-K over clusters of 2/3/4/6/8 CTAs, and
the CTA-pair 256x256 kernel with 2-SM MMAs) on the
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
SHAPES = [(200, 272, 1152), (64, 528, 1024), (129, 256, 1280), (17, 400, 1152)]

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


@pytest.mark.parametrize("cfg", [0, 1, 2, 5, 3, 6, 4, 7],
                         ids=["128x256", "128x128x2acc", "split2", "split3", "split4", "split6", "split8",
                              "pair256"])
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


GROUPED_CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import moe_grouped_gemm_mx_b200 as mx, mx_inputs
out = sys.argv[2]
counts = torch.tensor([0, 5, 128, 300, 1, 0, 77, 256], dtype=torch.int64)
c = mx_inputs.contiguous_problem(n=528, k=384, seed=11, counts=counts)
qa, sfa = mx.mx_quantize_bf16_to_e4m3(c.a.cuda())
qb, sfb = mx.mx_quantize_bf16_to_e4m3(c.b.cuda())
st = torch.zeros(1, dtype=torch.int32, device="cuda")
d = torch.full((c.a.shape[0] + 128, 528), 7.0, dtype=torch.bfloat16, device="cuda")
mx.mx_grouped_gemm_contiguous(qa, sfa, qb, sfb, c.offsets.cuda(), d=d[:c.a.shape[0]], dev_status=st)
mm = torch.tensor([0, 256, 1, 129, 128, 200, 255], dtype=torch.int32)
p = mx_inputs.masked_problem(n=272, k=256, experts=7, max_m=256, seed=12, masked_m=mm)
qa2, sfa2 = mx.mx_quantize_bf16_to_e4m3(p.a.cuda())
qb2, sfb2 = mx.mx_quantize_bf16_to_e4m3(p.b.cuda())
d2 = torch.full((7, 256, 272), 7.0, dtype=torch.bfloat16, device="cuda")
mx.mx_grouped_gemm_masked(qa2, sfa2, qb2, sfb2, mm.cuda(), d=d2, dev_status=st)
torch.cuda.synchronize()
assert int(st.item()) == 0, hex(int(st.item()))
np.savez(out, contiguous=d.float().cpu().numpy(), masked=d2.float().cpu().numpy())
"""


@pytest.mark.parametrize("cfg", [0, 7], ids=["128x256", "pair256"])
def test_forced_config_grouped(oracle, cfg):
    """Both persistent kernels on ragged contiguous groups (odd numbers of
    128-row blocks, empty experts) and on masked experts ending at every
    kind of boundary; rows outside the groups / masks keep their sentinel."""
    with tempfile.TemporaryDirectory() as td:
        out = os.path.join(td, "d.npz")
        env = dict(os.environ, MX_GEMM_CONFIG=str(cfg))
        r = subprocess.run([sys.executable, "-c", GROUPED_CHILD, ROOT, out], env=env, capture_output=True,
                           text=True, timeout=300)
        assert r.returncode == 0, r.stderr[-2000:]
        got = np.load(out)
        counts = torch.tensor([0, 5, 128, 300, 1, 0, 77, 256], dtype=torch.int64)
        c = mx_inputs.contiguous_problem(n=528, k=384, seed=11, counts=counts)
        qa, sfa = oracle_quantize(oracle, c.a)
        qb, sfb = oracle_quantize(oracle, c.b)
        m_end = int(c.offsets[-1])
        d_ref, absd = oracle.grouped_contiguous(qa, sfa, qb.reshape(8, 528, 384), sfb, c.offsets.numpy())
        assert_gemm_close(got["contiguous"][:m_end].astype(np.float64), d_ref, absd, f"cfg {cfg} contiguous")
        assert np.all(got["contiguous"][m_end:] == 7.0)
        mm = np.array([0, 256, 1, 129, 128, 200, 255], dtype=np.int32)
        p = mx_inputs.masked_problem(n=272, k=256, experts=7, max_m=256, seed=12,
                                     masked_m=torch.from_numpy(mm))
        qa2, sfa2 = oracle_quantize(oracle, p.a)
        qb2, sfb2 = oracle_quantize(oracle, p.b)
        d2_ref, abs2 = oracle.grouped_masked(qa2.reshape(7, 256, 256), sfa2, qb2.reshape(7, 272, 256), sfb2, mm)
        for e in range(7):
            assert np.all(got["masked"][e, mm[e]:] == 7.0), f"cfg {cfg} expert {e} rows >= masked_m written"
            if mm[e]:
                assert_gemm_close(got["masked"][e, :mm[e]].astype(np.float64), d2_ref[e, :mm[e]],
                                  abs2[e, :mm[e]], f"cfg {cfg} masked e={e}")


CHILD_BATCH = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import moe_grouped_gemm_mx_b200 as mx, mx_inputs
out = sys.argv[2]
qs = []
for (m, n, k) in %r:
    a, b = mx_inputs.dense_problem(m, n, k, seed=m + n, kind="outlier")
    qa, sfa = mx.mx_quantize_bf16_to_e4m3(a.cuda())
    qb, sfb = mx.mx_quantize_bf16_to_e4m3(b.cuda())
    qs.append((qa, sfa, qb, sfb))
st = torch.zeros(1, dtype=torch.int32, device="cuda")
ds = mx.mx_gemm_batch(qs, dev_status=st)
torch.cuda.synchronize()
assert int(st.item()) == 0, hex(int(st.item()))
np.savez(out, **{f"{m}x{n}x{k}": d.float().cpu().numpy() for (m, n, k), d in zip(%r, ds)})
""" % (SHAPES, SHAPES)


@pytest.mark.parametrize("bn", [128, 256])
@pytest.mark.parametrize("cluster", [2, 4])
def test_batch_forced_cluster(oracle, cluster, bn):
    """mx_gemm_batch over the four shapes above with its cluster size and tile
    width forced (MX_BATCH_CLUSTER, MX_BATCH_BN, read once per process): the
    planner's split-K over clusters of 2 or 4 and its persistent shares, with
    128- and 256-wide tiles, against the oracle."""
    with tempfile.TemporaryDirectory() as td:
        out = os.path.join(td, "d.npz")
        env = dict(os.environ, MX_BATCH_CLUSTER=str(cluster), MX_BATCH_BN=str(bn))
        r = subprocess.run([sys.executable, "-c", CHILD_BATCH, ROOT, out], env=env, capture_output=True, text=True,
                           timeout=300)
        assert r.returncode == 0, r.stderr[-2000:]
        got = np.load(out)
        for (m, n, k) in SHAPES:
            a, b = mx_inputs.dense_problem(m, n, k, seed=m + n, kind="outlier")
            qa, sfa = oracle_quantize(oracle, a)
            qb, sfb = oracle_quantize(oracle, b)
            d_ref, absd = oracle.gemm(qa, sfa, qb, sfb)
            assert_gemm_close(got[f"{m}x{n}x{k}"].astype(np.float64), d_ref, absd,
                              f"batch cluster {cluster} bn {bn} {m}x{n}x{k}")
