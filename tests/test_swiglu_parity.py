"""Fused MoE expert MLP, first half, on the GPU vs the CPU oracle:
gate/up GEMM -> SwiGLU -> MXFP8 requantisation in one kernel (dense,
contiguous-grouped and masked-grouped forms), and the down GEMM run directly
on its output.

The requantised H cannot be bit-exact against an fp64 oracle (the FP32 GEMM
accumulation decides E4M3 rounding near code midpoints), so each element is
held to one E4M3 step at its block scale plus the GEMM tolerance carried
through silu(g) * u, scales to the rule, and almost all codes to the
oracle's own quantisation (``mxtest_util.check_swiglu_quant``).  The down
GEMM on the GPU's H is held to the plain GEMM tolerance."""
import numpy as np
import pytest
import torch

import mx_inputs
from mxtest_util import (assert_gemm_close, check_swiglu_quant, gpu_sf_rowmajor, oracle_quantize, to_np_f64)

pytestmark = pytest.mark.gpu

H_SENTINEL = 0x5A  # a byte pattern the kernel must leave alone in untouched rows


@pytest.fixture(scope="module")
def mx():
    import moe_grouped_gemm_mx_b200 as m
    return m


def split_gate_up(oracle, qb, sfb_rm, groups, i_dim, k):
    """The oracle's [gate; up] operands per expert: bytes [E, i, k] and their
    row-major scales, from the quantised [E, 2i, k] projection."""
    qb3 = qb.reshape(groups, 2 * i_dim, k)
    sf3 = sfb_rm.reshape(groups, 2 * i_dim, k // 32)
    return (np.ascontiguousarray(qb3[:, :i_dim]), np.ascontiguousarray(sf3[:, :i_dim].reshape(-1, k // 32)),
            np.ascontiguousarray(qb3[:, i_dim:]), np.ascontiguousarray(sf3[:, i_dim:].reshape(-1, k // 32)))


# ---------------------------------------------------------------- dense

@pytest.mark.parametrize("m,i_dim,k,wstd", [(200, 384, 512, 0.02), (64, 128, 384, 0.1), (300, 256, 1152, 0.05)])
def test_dense_swiglu_quant(mx, oracle, m, i_dim, k, wstd):
    dev = torch.device("cuda")
    a = mx_inputs.normal_bf16((m, k), 1.0, 31, dev)
    w = mx_inputs.normal_bf16((2 * i_dim, k), wstd, 32, dev)
    qa, sfa = mx.mx_quantize_bf16_to_e4m3(a)
    qb, sfb = mx.mx_quantize_bf16_to_e4m3(w)
    sfh = torch.full((mx.scale_bytes(m, i_dim),), H_SENTINEL, dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    qh, sfh = mx.mx_gemm_swiglu_quant(qa, sfa, qb, sfb, sfh=sfh, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rqa, rsa = oracle_quantize(oracle, a.cpu())
    rqb, rsb = oracle_quantize(oracle, w.cpu())
    g, gabs = oracle.gemm(rqa, rsa, rqb[:i_dim], rsb[:i_dim])
    u, uabs = oracle.gemm(rqa, rsa, rqb[i_dim:], rsb[i_dim:])
    sf_rm = gpu_sf_rowmajor(oracle, sfh, 1, m, i_dim)
    check_swiglu_quant(oracle, qh.cpu().numpy(), sf_rm[:m], g, u, gabs, uabs, f"dense {m}x{i_dim}x{k}")
    # scale padding rows of the last 128-row block are written as 0x00
    pad_rows = (-m) % 128
    if pad_rows:
        full = gpu_sf_rowmajor(oracle, sfh, 1, m + pad_rows, i_dim)
        assert not full[m:].any()


# ---------------------------------------------------------------- contiguous

def run_contiguous(mx, prob, i_dim):
    dev = torch.device("cuda")
    a = prob.a.to(dev)
    w = prob.b.to(dev)
    qa, sfa = mx.mx_quantize_bf16_to_e4m3(a)
    qb, sfb = mx.mx_quantize_bf16_to_e4m3(w)
    m_total = a.shape[0]
    qh = torch.full((m_total, i_dim), H_SENTINEL, dtype=torch.uint8, device=dev)
    sfh = torch.full((mx.scale_bytes(m_total, i_dim),), H_SENTINEL, dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    off = prob.offsets.to(dev)
    mx.mx_grouped_gemm_contiguous_swiglu_quant(qa, sfa, qb, sfb, off, qh=qh, sfh=sfh, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return qh, sfh


def test_contiguous_swiglu_quant_ragged_then_down(mx, oracle):
    counts = torch.tensor([0, 5, 128, 200, 1, 0, 77], dtype=torch.int64)
    i_dim, k, n_down = 256, 384, 272
    prob = mx_inputs.contiguous_problem(n=2 * i_dim, k=k, seed=4, counts=counts)
    extra = 128  # rows past the last group: must stay untouched
    m_end = int(prob.offsets[-1])
    prob.a = torch.cat([prob.a, torch.ones(extra, k, dtype=prob.a.dtype)])
    qh, sfh = run_contiguous(mx, prob, i_dim)
    groups = len(counts)
    rqa, rsa = oracle_quantize(oracle, prob.a)
    rqb, rsb = oracle_quantize(oracle, prob.b)
    qg, sg, qu, su = split_gate_up(oracle, rqb, rsb, groups, i_dim, k)
    off = prob.offsets.numpy()
    g, gabs = oracle.grouped_contiguous(rqa, rsa, qg, sg, off)
    u, uabs = oracle.grouped_contiguous(rqa, rsa, qu, su, off)
    m_total = prob.a.shape[0]
    sf_rm = gpu_sf_rowmajor(oracle, sfh, 1, m_total, i_dim)
    qh_np = qh.cpu().numpy()
    check_swiglu_quant(oracle, qh_np[:m_end], sf_rm[:m_end], g, u, gabs, uabs, "contiguous ragged")
    assert np.all(qh_np[m_end:] == H_SENTINEL), "H rows past the last group were written"
    assert np.all(sf_rm[m_end:] == H_SENTINEL), "scale rows past the last group were written"
    # the down GEMM consumes (qh, sfh) as they stand
    w2 = mx_inputs.normal_bf16((groups, n_down, i_dim), 0.02, 77)
    dev = torch.device("cuda")
    qw2, sfw2 = mx.mx_quantize_bf16_to_e4m3(w2.to(dev))
    d = mx.mx_grouped_gemm_contiguous(qh, sfh, qw2, sfw2, prob.offsets.to(dev))
    torch.cuda.synchronize()
    rqw2, rsw2 = oracle_quantize(oracle, w2)
    y_ref, yabs = oracle.grouped_contiguous(qh_np, sf_rm, rqw2.reshape(groups, n_down, i_dim), rsw2, off)
    assert_gemm_close(to_np_f64(d[:m_end]), y_ref, yabs, "down GEMM on the fused output")


def test_contiguous_swiglu_quant_moe_config_sampled(mx, oracle):
    """The MoE workload's gate/up shape (32 experts, 8192 tokens x top-8 with
    Zipf(1.1) popularity, 2I = 4096, K = 7168) on sampled rows: the first and
    last row of every group and 256 random rows."""
    i_dim, k = 2048, 7168
    counts = mx_inputs.zipf_routing_counts(seed=0)
    prob = mx_inputs.contiguous_problem(n=2 * i_dim, k=k, seed=0, counts=counts)
    qh, sfh = run_contiguous(mx, prob, i_dim)
    off = prob.offsets.numpy()
    rng = np.random.default_rng(1)
    rows = set(rng.integers(0, int(off[-1]), 256).tolist())
    for e in range(len(counts)):
        if off[e + 1] > off[e]:
            rows.update([int(off[e]), int(off[e + 1]) - 1])
    rows = np.array(sorted(rows), dtype=np.int64)
    rqa, rsa = oracle_quantize(oracle, prob.a)
    rqb, rsb = oracle_quantize(oracle, prob.b)
    qg, sg, qu, su = split_gate_up(oracle, rqb, rsb, len(counts), i_dim, k)
    g, gabs = oracle.grouped_contiguous(rqa, rsa, qg, sg, off, rows=rows)
    u, uabs = oracle.grouped_contiguous(rqa, rsa, qu, su, off, rows=rows)
    sf_rm = gpu_sf_rowmajor(oracle, sfh, 1, prob.a.shape[0], i_dim)
    check_swiglu_quant(oracle, qh.cpu().numpy()[rows], sf_rm[rows], g, u, gabs, uabs, "MoE gate/up sampled")


# ---------------------------------------------------------------- masked

def test_masked_swiglu_quant(mx, oracle):
    dev = torch.device("cuda")
    mm = torch.tensor([0, 1, 100, 256, 129], dtype=torch.int32)
    i_dim, k = 256, 256
    prob = mx_inputs.masked_problem(n=2 * i_dim, k=k, experts=5, max_m=256, seed=6, masked_m=mm)
    e, max_m, _ = prob.a.shape
    qa, sfa = mx.mx_quantize_bf16_to_e4m3(prob.a.to(dev))
    qb, sfb = mx.mx_quantize_bf16_to_e4m3(prob.b.to(dev))
    qh = torch.full((e, max_m, i_dim), H_SENTINEL, dtype=torch.uint8, device=dev)
    sfh = torch.full((e * mx.scale_bytes(max_m, i_dim),), H_SENTINEL, dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    mx.mx_grouped_gemm_masked_swiglu_quant(qa, sfa, qb, sfb, mm.to(dev), qh=qh, sfh=sfh, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rqa, rsa = oracle_quantize(oracle, prob.a)
    rqb, rsb = oracle_quantize(oracle, prob.b)
    qg, sg, qu, su = split_gate_up(oracle, rqb, rsb, e, i_dim, k)
    g, gabs = oracle.grouped_masked(rqa.reshape(e, max_m, k), rsa, qg, sg, mm.numpy())
    u, uabs = oracle.grouped_masked(rqa.reshape(e, max_m, k), rsa, qu, su, mm.numpy())
    sf_rm = gpu_sf_rowmajor(oracle, sfh, e, max_m, i_dim).reshape(e, max_m, i_dim // 32)
    qh_np = qh.cpu().numpy()
    for x in range(e):
        r = int(mm[x])
        if r:
            check_swiglu_quant(oracle, qh_np[x, :r], sf_rm[x, :r], g[x, :r], u[x, :r], gabs[x, :r], uabs[x, :r],
                               f"masked expert {x}")
        assert np.all(qh_np[x, r:] == H_SENTINEL), f"expert {x}: H rows >= masked_m written"
        assert np.all(sf_rm[x, r:] == H_SENTINEL), f"expert {x}: scale rows >= masked_m written"
