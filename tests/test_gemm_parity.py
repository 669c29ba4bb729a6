"""Dense MXFP8 GEMM on the GPU vs the CPU oracle.

The GPU side runs the whole path (its own quantiser, then mx_gemm); the oracle
quantises the same BF16 inputs itself and sums the dequantised products in
fp64.  Outputs must satisfy |D_gpu - D_ref| <= 1e-2*sum|a*b| + 1e-3 element-
wise, be finite, and leave every byte outside D untouched."""
import numpy as np
import pytest
import torch

import mx_inputs
from mxtest_util import sampled_rows, assert_gemm_close, is_sentinel, oracle_quantize, sentinel_fill, to_np_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    import moe_grouped_gemm_mx_b200 as m
    return m


def gpu_dense(mx, a_cpu, b_cpu, guard_rows=3):
    dev = torch.device("cuda")
    a, b = a_cpu.to(dev), b_cpu.to(dev)
    qa, sfa = mx.mx_quantize_bf16_to_e4m3(a)
    qb, sfb = mx.mx_quantize_bf16_to_e4m3(b)
    m, n = a.shape[0], b.shape[0]
    buf = sentinel_fill((m + guard_rows, n))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    d = mx.mx_gemm(qa, sfa, qb, sfb, d=buf[:m], dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item()):#x}"
    assert bool(is_sentinel(buf[m:]).all()), "mx_gemm wrote past the end of D"
    return d


def check_dense(mx, oracle, a, b, rows=None, what=""):
    d = gpu_dense(mx, a, b)
    qa, sfa = oracle_quantize(oracle, a)
    qb, sfb = oracle_quantize(oracle, b)
    d_ref, absd = oracle.gemm(qa, sfa, qb, sfb, rows=rows)
    d_gpu = to_np_f64(d if rows is None else d[torch.as_tensor(rows, device=d.device)])
    assert_gemm_close(d_gpu, d_ref, absd, what)
    return d


def test_pr1(mx, oracle):
    a, b = mx_inputs.dense_problem(128, 256, 512, seed=0)
    check_dense(mx, oracle, a, b, what="PR1 128x256x512")


@pytest.mark.parametrize("seed", [1, 2])
def test_pr1_other_seeds(mx, oracle, seed):
    a, b = mx_inputs.dense_problem(128, 256, 512, seed=seed)
    check_dense(mx, oracle, a, b, what=f"PR1 seed {seed}")


@pytest.mark.parametrize("m,n,k", [
    (1, 16, 128), (63, 144, 128), (64, 256, 256), (65, 272, 128), (127, 16, 384),
    (128, 528, 256), (129, 256, 640), (300, 400, 256), (257, 512, 1024),
])
def test_edge_shapes(mx, oracle, m, n, k):
    a, b = mx_inputs.dense_problem(m, n, k, seed=m + n + k, kind="outlier")
    check_dense(mx, oracle, a, b, what=f"{m}x{n}x{k}")


def test_small_integers_exact(mx, oracle):
    """Integer operands in [-4, 4] with a +-4 in every block: every product
    and every partial sum is an exact integer far below 2^24, so the FP32
    accumulator is exact and D must equal the BF16 rounding (RNE) of the
    integer product."""
    g = torch.Generator().manual_seed(3)
    m, n, k = 130, 272, 256

    def mat(rows):
        x = torch.randint(-4, 5, (rows, k), generator=g).float()
        col = torch.randint(0, 32, (rows, k // 32), generator=g) + torch.arange(0, k, 32)
        sign = torch.randint(0, 2, (rows, k // 32), generator=g).float() * 2 - 1
        x.scatter_(1, col, 4.0 * sign)
        return x
    a, b = mat(m), mat(n)
    want = (a.double() @ b.double().T)
    assert float(want.abs().max()) < 2 ** 24
    d = gpu_dense(mx, a.to(torch.bfloat16), b.to(torch.bfloat16))
    assert torch.equal(d.cpu().view(torch.int16), want.float().to(torch.bfloat16).view(torch.int16))


def test_zero_blocks_and_extremes(mx, oracle):
    """All-zero blocks, a huge and a tiny block scale side by side."""
    a, b = mx_inputs.dense_problem(128, 256, 512, seed=4)
    a = a.clone()
    a[:, 0:32] = 0
    a[5, 32:64] = a[5, 32:64].float().mul(2.0 ** 100).to(torch.bfloat16)
    a[6, 64:96] = a[6, 64:96].float().mul(2.0 ** -100).to(torch.bfloat16)
    check_dense(mx, oracle, a, b, what="zero/extreme blocks")


@pytest.mark.parametrize("shape", mx_inputs.PAGE_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_page_shapes_all_rows(mx, oracle, shape):
    m, n, k = shape
    a, b = mx_inputs.dense_problem(m, n, k, seed=0, kind="outlier")
    check_dense(mx, oracle, a, b, what=f"page shape {shape}")


def gpu_batch(mx, problems):
    """D_i of mx_gemm_batch over BF16 (A_i, B_i) pairs, with the status word."""
    dev = torch.device("cuda")
    qs = []
    for a, b in problems:
        qa, sfa = mx.mx_quantize_bf16_to_e4m3(a.to(dev))
        qb, sfb = mx.mx_quantize_bf16_to_e4m3(b.to(dev))
        qs.append((qa, sfa, qb, sfb))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    ds = mx.mx_gemm_batch(qs, dev_status=st)
    torch.cuda.synchronize()
    return ds, int(st.item())


def test_page_shapes_batch_all_rows(mx, oracle):
    """The three page shapes as one mx_gemm_batch launch (the GPU shared
    among them, K split over clusters where the model says so): every row of
    every problem against the oracle."""
    probs = [mx_inputs.dense_problem(m, n, k, seed=0, kind="outlier") for (m, n, k) in mx_inputs.PAGE_SHAPES]
    ds, st = gpu_batch(mx, probs)
    assert st == 0
    for (a, b), d, shape in zip(probs, ds, mx_inputs.PAGE_SHAPES):
        qa, sfa = oracle_quantize(oracle, a)
        qb, sfb = oracle_quantize(oracle, b)
        d_ref, absd = oracle.gemm(qa, sfa, qb, sfb)
        assert_gemm_close(to_np_f64(d), d_ref, absd, f"batch page shape {shape}")


@pytest.mark.parametrize("shapes", [
    [(1, 16, 128), (63, 144, 384), (200, 272, 1152), (129, 400, 256)],
    [(17, 528, 2048), (64, 256, 128)],
    [(300, 400, 256)],
], ids=["four-ragged", "two", "one"])
def test_batch_ragged(mx, oracle, shapes):
    """Ragged batches: M of 1, 63, 129, 200, 300 rows, N not a multiple of
    128, K of one 128-element tile (no split possible) to 2048; one problem
    alone is mx_gemm's problem."""
    probs = [mx_inputs.dense_problem(m, n, k, seed=m + n + k, kind="outlier") for (m, n, k) in shapes]
    ds, st = gpu_batch(mx, probs)
    assert st == 0
    for (a, b), d, shape in zip(probs, ds, shapes):
        qa, sfa = oracle_quantize(oracle, a)
        qb, sfb = oracle_quantize(oracle, b)
        d_ref, absd = oracle.gemm(qa, sfa, qb, sfb)
        assert_gemm_close(to_np_f64(d), d_ref, absd, f"batch {shape}")


def test_batch_with_empty_problem_and_sentinels(mx, oracle):
    """An empty problem in the batch takes no work; the others' outputs are
    written exactly in their [M, N] (sentinel rows around each untouched)."""
    dev = torch.device("cuda")
    shapes = [(64, 2112, 1024), (0, 256, 512), (128, 512, 768)]
    qs, refs, bufs = [], [], []
    for (m, n, k) in shapes:
        a, b = mx_inputs.dense_problem(max(m, 1), n, k, seed=7 + n, kind="outlier")
        a = a[:m]
        qa, sfa = mx.mx_quantize_bf16_to_e4m3(a.to(dev)) if m else (torch.empty((0, k), dtype=torch.uint8, device=dev),
                                                                  torch.zeros(16, dtype=torch.uint8, device=dev))
        qb, sfb = mx.mx_quantize_bf16_to_e4m3(b.to(dev))
        qs.append((qa, sfa, qb, sfb))
        buf = sentinel_fill((m + 2, n))
        bufs.append(buf)
        refs.append((a, b))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    mx.mx_gemm_batch(qs, outs=[bf[1:1 + m] for bf, (m, _, _) in zip(bufs, shapes)], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for (a, b), bf, (m, n, k) in zip(refs, bufs, shapes):
        assert bool(is_sentinel(bf[0]).all()) and bool(is_sentinel(bf[m + 1]).all()), f"{(m, n, k)}: guard rows"
        if m == 0:
            continue
        qa, sfa = oracle_quantize(oracle, a)
        qb, sfb = oracle_quantize(oracle, b)
        d_ref, absd = oracle.gemm(qa, sfa, qb, sfb)
        assert_gemm_close(to_np_f64(bf[1:1 + m]), d_ref, absd, f"batch {(m, n, k)}")


@pytest.mark.parametrize("nk", mx_inputs.LARGE_NK, ids=lambda s: "x".join(map(str, s)))
def test_large_dense_sampled_rows(mx, oracle, nk):
    n, k = nk
    m = mx_inputs.LARGE_M
    a, b = mx_inputs.dense_problem(m, n, k, seed=0, kind="loguniform")
    # 256 random rows plus the first and last row of every 128-row M tile
    rows = sampled_rows(m, 256, seed=0)
    assert len(rows) >= 256 + 2 * (m // 128) - 8
    check_dense(mx, oracle, a, b, rows=rows, what=f"large {m}x{n}x{k}")


def test_empty_m_is_noop(mx):
    dev = torch.device("cuda")
    qa = torch.empty((0, 128), dtype=torch.uint8, device=dev)
    qb = torch.zeros((16, 128), dtype=torch.uint8, device=dev)
    sf = torch.zeros(mx.scale_bytes(16, 128), dtype=torch.uint8, device=dev)
    d = mx.mx_gemm(qa, sf, qb, sf)
    assert d.shape == (0, 16)
