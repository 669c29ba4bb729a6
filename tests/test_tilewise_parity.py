"""Tile-wise FP32-scaled FP8 (DeepGEMM's format: 1 x 128 activation tiles,
128 x 128 weight blocks, s = amax / 448) on the GPU vs the CPU oracle: both
quantisers bit-exact (scales compared as FP32 bit patterns, NaN included),
and the two-level-accumulation GEMM (TMEM partial per 128-element K tile,
promoted with its scales in FP32) in dense and contiguous-grouped form within
the GEMM tolerance."""
import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch

import mx_inputs
from mxtest_util import assert_gemm_close, to_np_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    import moe_grouped_gemm_mx_b200 as m
    return m


def bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def check_quant(mx, oracle, x, blocks: bool):
    dev = torch.device("cuda")
    if blocks:
        q, s = mx.mx_quantize_bf16_to_e4m3_block128x128(x.to(dev))
        rq, rs = oracle.tw_quantize_blocks(x)
    else:
        q, s = mx.mx_quantize_bf16_to_e4m3_tile1x128(x.to(dev))
        rq, rs = oracle.tw_quantize_rows(x)
    torch.cuda.synchronize()
    q = q.cpu().numpy()
    s = s.cpu().numpy()
    assert np.array_equal(bits(s), bits(rs)), f"{(bits(s) != bits(rs)).sum()} scales differ"
    assert np.array_equal(q, rq), f"{(q != rq).sum()} element bytes differ"


@pytest.mark.parametrize("blocks", [False, True])
def test_tilewise_quant_every_bf16_pattern(mx, oracle, blocks):
    bits16 = np.random.default_rng(1).permutation(np.arange(65536, dtype=np.int64)).astype(np.uint16)
    x = torch.from_numpy(bits16.view(np.int16).reshape(256, 256).copy()).view(torch.bfloat16)
    check_quant(mx, oracle, x, blocks)


@pytest.mark.parametrize("shape", [(300, 512), (64, 7168), (129, 256), (1, 128)])
@pytest.mark.parametrize("blocks", [False, True])
def test_tilewise_quant_shapes(mx, oracle, shape, blocks):
    x = mx_inputs.outlier_bf16(shape, seed=21)
    if shape[0] >= 130:
        x[129, 128:256] = 0.0           # a zero 1x128 tile (its block stays non-zero)
        x[0, 300] = float("nan")        # a non-finite tile / block
    check_quant(mx, oracle, x, blocks)


def tw_dense(mx, oracle, m, n, k, seed, rows=None):
    dev = torch.device("cuda")
    a = mx_inputs.outlier_bf16((m, k), seed=seed)
    b = mx_inputs.normal_bf16((n, k), 0.02, seed + 1)
    qa, sa = mx.mx_quantize_bf16_to_e4m3_tile1x128(a.to(dev))
    qb, sb = mx.mx_quantize_bf16_to_e4m3_block128x128(b.to(dev))
    d = mx.mx_gemm_tilewise(qa, sa, qb, sb)
    torch.cuda.synchronize()
    d_ref, absd = oracle.tw_gemm(qa.cpu().numpy(), sa.cpu().numpy(), qb.cpu().numpy(), sb.cpu().numpy(), rows=rows)
    dg = to_np_f64(d if rows is None else d[torch.as_tensor(rows, device=d.device)])
    assert_gemm_close(dg, d_ref, absd, f"tile-wise {m}x{n}x{k}")


@pytest.mark.parametrize("m,n,k", [(128, 256, 512), (200, 272, 1152), (17, 400, 128), (300, 128, 2048)])
def test_tilewise_gemm_dense(mx, oracle, m, n, k):
    tw_dense(mx, oracle, m, n, k, seed=30)


def test_tilewise_gemm_page_shape(mx, oracle):
    """The first dense shape of the DeepGEMM comparison table, 64 x 2112 x 7168."""
    tw_dense(mx, oracle, 64, 2112, 7168, seed=31)


def test_tilewise_gemm_contiguous(mx, oracle):
    counts = torch.tensor([0, 5, 128, 200, 1, 0, 77], dtype=torch.int64)
    n, k = 272, 384
    prob = mx_inputs.contiguous_problem(n=n, k=k, seed=32, counts=counts)
    e = len(counts)
    dev = torch.device("cuda")
    qa, sa = mx.mx_quantize_bf16_to_e4m3_tile1x128(prob.a.to(dev))
    # expert weights [E, N, K] quantised as one [E*N, K] matrix: with N not a
    # multiple of 128 the blocks would straddle experts, so quantise per expert
    qb = torch.empty((e, n, k), dtype=torch.uint8, device=dev)
    nb = (n + 127) // 128
    sb = torch.empty((e, nb, k // 128), dtype=torch.float32, device=dev)
    for x in range(e):
        mx.mx_quantize_bf16_to_e4m3_block128x128(prob.b[x].to(dev), q=qb[x], s=sb[x])
    off = prob.offsets.to(dev)
    d = mx.mx_grouped_gemm_contiguous_tilewise(qa, sa, qb, sb, off)
    torch.cuda.synchronize()
    qa_h, sa_h, qb_h, sb_h = qa.cpu().numpy(), sa.cpu().numpy(), qb.cpu().numpy(), sb.cpu().numpy()
    offs = prob.offsets.numpy()
    for x in range(e):
        r0, r1 = int(offs[x]), int(offs[x + 1])
        if r1 == r0:
            continue
        d_ref, absd = oracle.tw_gemm(qa_h[r0:r1], np.ascontiguousarray(sa_h[:, r0:r1]), qb_h[x], sb_h[x])
        assert_gemm_close(to_np_f64(d[r0:r1]), d_ref, absd, f"tile-wise contiguous expert {x}")


# ---------------------------------------------------------------- ragged shapes and experts

TW_SHAPES = [(256, 512, 512), (300, 272, 1152), (17, 400, 128), (600, 2112, 384)]
TW_COUNTS = [0, 5, 128, 300, 1, 0, 77, 256]   # ragged experts, empty ones, a row block ending mid-tile


@pytest.mark.parametrize("m,n,k", TW_SHAPES)
def test_tilewise_gemm_ragged(mx, oracle, m, n, k):
    """Ragged M, N tails and a single K tile (K = 128)."""
    dev = torch.device("cuda")
    a = mx_inputs.outlier_bf16((m, k), seed=m + k)
    b = mx_inputs.normal_bf16((n, k), 0.02, m + n)
    qa, sa = mx.mx_quantize_bf16_to_e4m3_tile1x128(a.to(dev))
    qb, sb = mx.mx_quantize_bf16_to_e4m3_block128x128(b.to(dev))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    d = mx.mx_gemm_tilewise(qa, sa, qb, sb, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    d_ref, absd = oracle.tw_gemm(qa.cpu().numpy(), sa.cpu().numpy(), qb.cpu().numpy(), sb.cpu().numpy())
    assert_gemm_close(to_np_f64(d), d_ref, absd, f"tile-wise {m}x{n}x{k}")


def test_tilewise_gemm_contiguous_ragged(mx, oracle):
    counts = torch.tensor(TW_COUNTS, dtype=torch.int64)
    n, k = 256, 640
    prob = mx_inputs.contiguous_problem(n=n, k=k, seed=40, counts=counts)
    e = len(counts)
    dev = torch.device("cuda")
    qa, sa = mx.mx_quantize_bf16_to_e4m3_tile1x128(prob.a.to(dev))
    qb = torch.empty((e, n, k), dtype=torch.uint8, device=dev)
    sb = torch.empty((e, n // 128, k // 128), dtype=torch.float32, device=dev)
    for x in range(e):
        mx.mx_quantize_bf16_to_e4m3_block128x128(prob.b[x].to(dev), q=qb[x], s=sb[x])
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    d = mx.mx_grouped_gemm_contiguous_tilewise(qa, sa, qb, sb, prob.offsets.to(dev), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    qa_h, sa_h, qb_h, sb_h = qa.cpu().numpy(), sa.cpu().numpy(), qb.cpu().numpy(), sb.cpu().numpy()
    offs = prob.offsets.numpy()
    for x in range(e):
        r0, r1 = int(offs[x]), int(offs[x + 1])
        if r1 == r0:
            continue
        d_ref, absd = oracle.tw_gemm(qa_h[r0:r1], np.ascontiguousarray(sa_h[:, r0:r1]), qb_h[x], sb_h[x])
        assert_gemm_close(to_np_f64(d[r0:r1]), d_ref, absd, f"tile-wise contiguous expert {x}")


@pytest.mark.parametrize("blocks", [False, True])
def test_tilewise_quant_midpoints_and_tiny_scales(mx, oracle, blocks):
    """Rounding corner cases of x / s: tiles scaled so that s = 1 exactly
    with elements on E4M3 rounding midpoints (ties to even), tiles of BF16
    subnormals (a subnormal FP32 scale), and rows spread over many binades,
    plus a large random matrix."""
    g = torch.Generator().manual_seed(77)
    rows, k = 256, 512
    x = torch.randn(rows, k, generator=g)
    mids = torch.tensor([1.0625, 1.1875, 1.3125, 1.4375, 1.5625, 1.6875, 1.8125, 1.9375,
                         0.0029296875, 0.0048828125, 0.0009765625, 0.001953125 * 1.5])
    for r in range(0, 128):                       # amax 448 in every 128x128 block and 1x128 tile
        x[r] = mids[torch.randint(0, len(mids), (k,), generator=g)] * (2.0 ** torch.randint(-6, 8, (k,), generator=g))
        x[r, ::128] = 448.0
    x[128:160] = torch.randn(32, k, generator=g) * 1e-39  # BF16 subnormals: a tiny scale
    x[160] = torch.randn(k, generator=g) * (2.0 ** torch.randint(-30, 30, (k,), generator=g).float())
    x = x.to(torch.bfloat16)
    check_quant(mx, oracle, x, blocks)
    big = torch.randn(2048, 1024, generator=g).to(torch.bfloat16)
    check_quant(mx, oracle, big, blocks)


def _near_boundary_counts(x: torch.Tensor, s: np.ndarray, blocks: bool):
    """Elements of x whose approximate quotient RN(|x| * RN(1 / s)) lies within
    8 FP32 grid steps of an E4M3 rounding boundary -- the ones whose code a
    quotient a few ulp off would change: returns (how many, how many of those
    are not exact quotients).  Counts coverage only; the codes themselves are
    compared with the oracle."""
    a = np.abs(x.float().numpy())
    rows, k = a.shape
    if blocks:
        st = np.repeat(np.repeat(s, 128, axis=0)[:rows], 128, axis=1)
    else:
        st = np.repeat(s.T, 128, axis=1)
    st = st.astype(np.float32)
    ok = np.isfinite(st) & (st >= np.float32(2.0 ** -64))
    r = np.float32(1.0) / st
    q0 = (a.astype(np.float32) * r).astype(np.float32)
    b = q0.view(np.uint32).astype(np.int64)
    lo = np.maximum(b - 8, 0).astype(np.uint32).view(np.float32)
    hi = (b + 8).astype(np.uint32).view(np.float32)

    def code(v):
        return torch.from_numpy(np.minimum(v, np.float32(448.0))).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    near = (code(lo) != code(hi)) & ok
    inexact = near & (a.astype(np.float64) != q0.astype(np.float64) * st.astype(np.float64))
    return int(near.sum()), int(inexact.sum())


@pytest.mark.parametrize("blocks", [False, True])
def test_tilewise_quant_near_rounding_boundaries(mx, oracle, blocks):
    """Random tiles over many binades, large enough that thousands of
    quotients x / s sit on or within a few ulp of an E4M3 rounding boundary
    (exact ties against scales with short significands, and thousands of
    inexact near-ties), bit-exact against the oracle."""
    g = torch.Generator().manual_seed(91)
    x = torch.randn(4096, 2048, generator=g) * torch.exp(torch.randn(4096, 1, generator=g) * 3.0)
    x = x.to(torch.bfloat16)
    _, rs = (oracle.tw_quantize_blocks if blocks else oracle.tw_quantize_rows)(x)
    near, inexact = _near_boundary_counts(x, rs, blocks)
    assert near >= 1000 and inexact >= 20, (near, inexact)
    check_quant(mx, oracle, x, blocks)


def _every_significand_pair() -> torch.Tensor:
    """128 blocks of 128 x 128 BF16 values.  Block b's largest magnitude has
    significand 1 + b/128 (element [0, 0], one binade above the rest); row i
    of a block peaks at significand 1 + ((b + i) % 128)/128; every other
    element takes each of the 128 BF16 significands at 0 to 12 binades below
    its row's peak, with random signs.  So both kernels see every scale
    significand (a scale RN(amax / 448) has one per amax significand), each
    paired with every element significand across the E4M3 normal and
    subnormal ranges of the quotient.  Every value is exact in BF16."""
    g = np.random.default_rng(123)
    blocks = []
    sig = 1.0 + np.arange(128) / 128.0
    for b in range(128):
        blk = np.empty((128, 128), dtype=np.float64)
        for i in range(128):
            peak = sig[(b + i) % 128]
            j = g.permutation(128)[:127]
            d = g.integers(0, 13, 127)
            blk[i, 1:] = sig[j] * np.exp2(-d - 1.0) * np.where(g.random(127) < 0.5, -1.0, 1.0)
            blk[i, 0] = peak
        blk[0, 0] = sig[b] * 2.0
        blocks.append(blk * 2.0 ** (b % 7 - 3))
    return torch.from_numpy(np.concatenate(blocks)).to(torch.bfloat16)


@pytest.mark.parametrize("blocks", [False, True])
def test_tilewise_quant_every_significand_pair(mx, oracle, blocks):
    check_quant(mx, oracle, _every_significand_pair(), blocks)


# ---------------------------------------------------------------- split-K over a cluster

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
# ragged M and N, K tiles not a multiple of the split (9 over 2/4/8), exactly
# one K tile per CTA (8 over 8), a single row and a single 16-column block,
# fewer K tiles than the split asks for (5: the split is not taken), and the
# page's first dense shape
SPLIT_SHAPES = [(200, 272, 1152), (17, 400, 1152), (129, 256, 1024), (1, 16, 1024), (256, 128, 640),
                (64, 2112, 7168)]

SPLIT_CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import moe_grouped_gemm_mx_b200 as mx, mx_inputs
out = sys.argv[2]
res = {}
for (m, n, k) in %r:
    a = mx_inputs.outlier_bf16((m, k), seed=m + k)
    b = mx_inputs.normal_bf16((n, k), 0.02, n + k)
    qa, sa = mx.mx_quantize_bf16_to_e4m3_tile1x128(a.cuda())
    qb, sb = mx.mx_quantize_bf16_to_e4m3_block128x128(b.cuda())
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    buf = torch.full((m + 128, n), 7.0, dtype=torch.bfloat16, device="cuda")
    mx.mx_gemm_tilewise(qa, sa, qb, sb, d=buf[:m], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, hex(int(st.item()))
    res[f"{m}x{n}x{k}"] = buf.float().cpu().numpy()
    res[f"{m}x{n}x{k}_q"] = np.concatenate([qa.cpu().numpy().ravel(), qb.cpu().numpy().ravel()])
    res[f"{m}x{n}x{k}_sa"] = sa.cpu().numpy()
    res[f"{m}x{n}x{k}_sb"] = sb.cpu().numpy()
np.savez(out, **res)
""" % (SPLIT_SHAPES,)


@pytest.mark.parametrize("split", [1, 2, 4, 8, 0], ids=["split1", "split2", "split4", "split8", "auto"])
def test_tilewise_gemm_split_k(oracle, split):
    """The dense tile-wise GEMM with K split over a cluster of 1/2/4/8 CTAs
    (forced through the library's MX_TW_SPLIT override, read once per
    process, so each split runs in a child process) and with the library's
    own choice; rows past M keep their sentinel."""
    with tempfile.TemporaryDirectory() as td:
        out = os.path.join(td, "d.npz")
        env = dict(os.environ)
        env.pop("MX_TW_SPLIT", None)
        if split:
            env["MX_TW_SPLIT"] = str(split)
        r = subprocess.run([sys.executable, "-c", SPLIT_CHILD, ROOT, out], env=env, capture_output=True, text=True,
                           timeout=300)
        assert r.returncode == 0, r.stderr[-2000:]
        got = np.load(out)
        for (m, n, k) in SPLIT_SHAPES:
            key = f"{m}x{n}x{k}"
            q = got[key + "_q"]
            qa, qb = q[:m * k].reshape(m, k), q[m * k:].reshape(n, k)
            d_ref, absd = oracle.tw_gemm(qa, got[key + "_sa"], qb, got[key + "_sb"])
            assert_gemm_close(got[key][:m].astype(np.float64), d_ref, absd, f"split {split} {key}")
            assert np.all(got[key][m:] == 7.0), f"split {split} {key}: rows past M written"
