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
