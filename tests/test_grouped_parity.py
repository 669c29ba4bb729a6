"""MoE grouped MXFP8 GEMMs (contiguous and masked layouts) on the GPU vs the
CPU oracle, including empty experts, ragged groups, NaN padding rows that must
be ignored, rows that must stay untouched, and bad offsets / masks that must
be reported through the device status word without writing anything."""
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


# ---------------------------------------------------------------- contiguous

def gpu_contiguous(mx, prob, extra_rows=0, offsets=None):
    dev = torch.device("cuda")
    a = prob.a.to(dev)
    if extra_rows:
        a = torch.cat([a, torch.ones(extra_rows, a.shape[1], dtype=a.dtype, device=dev)])
    b = prob.b.to(dev)
    qa, sfa = mx.mx_quantize_bf16_to_e4m3(a)
    qb, sfb = mx.mx_quantize_bf16_to_e4m3(b)
    off = (prob.offsets if offsets is None else offsets).to(dev)
    d = sentinel_fill((a.shape[0], b.shape[1]))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    mx.mx_grouped_gemm_contiguous(qa, sfa, qb, sfb, off, d=d, dev_status=status)
    torch.cuda.synchronize()
    return d, int(status.item())


def check_contiguous(mx, oracle, prob, rows=None, extra_rows=0, what=""):
    d, st = gpu_contiguous(mx, prob, extra_rows)
    assert st == 0, f"device status {st:#x}"
    m_end = int(prob.offsets[-1])
    assert bool(is_sentinel(d[m_end:]).all()), "rows past the last group were written"
    qa, sfa = oracle_quantize(oracle, prob.a)
    e, n, k = prob.b.shape
    qb, sfb = oracle_quantize(oracle, prob.b)
    d_ref, absd = oracle.grouped_contiguous(qa, sfa, qb.reshape(e, n, k), sfb, prob.offsets.numpy(), rows=rows)
    d_gpu = to_np_f64(d[:m_end] if rows is None else d[torch.as_tensor(rows, device=d.device)])
    assert_gemm_close(d_gpu, d_ref, absd, what)


def test_contiguous_small_ragged(mx, oracle):
    counts = torch.tensor([0, 5, 128, 200, 1, 0, 77], dtype=torch.int64)
    prob = mx_inputs.contiguous_problem(n=272, k=256, seed=1, counts=counts)
    check_contiguous(mx, oracle, prob, extra_rows=64, what="contiguous ragged")


def test_contiguous_single_group_equals_dense(mx, oracle):
    """One expert in the contiguous layout and the dense GEMM on the same
    operands both match the oracle (the tile configurations, hence the FP32
    summation order, may differ, so the two are compared within tolerance)."""
    counts = torch.tensor([256], dtype=torch.int64)
    prob = mx_inputs.contiguous_problem(n=256, k=512, seed=2, counts=counts)
    d, st = gpu_contiguous(mx, prob)
    assert st == 0
    dev = torch.device("cuda")
    qa, sfa = mx.mx_quantize_bf16_to_e4m3(prob.a.to(dev))
    qb, sfb = mx.mx_quantize_bf16_to_e4m3(prob.b[0].to(dev))
    dd = mx.mx_gemm(qa, sfa, qb, sfb)
    torch.cuda.synchronize()
    ra, rsa = oracle_quantize(oracle, prob.a)
    rb, rsb = oracle_quantize(oracle, prob.b[0])
    d_ref, absd = oracle.gemm(ra, rsa, rb, rsb)
    assert_gemm_close(to_np_f64(d), d_ref, absd, "contiguous E=1")
    assert_gemm_close(to_np_f64(dd), d_ref, absd, "dense")


def test_contiguous_all_empty(mx):
    counts = torch.zeros(4, dtype=torch.int64)
    prob = mx_inputs.contiguous_problem(n=64, k=128, seed=3, counts=counts)
    prob.a = torch.zeros((128, 128), dtype=torch.bfloat16)
    d, st = gpu_contiguous(mx, prob)
    assert st == 0
    assert bool(is_sentinel(d).all())


@pytest.mark.parametrize("bad", ["not_multiple", "decreasing", "past_end"])
def test_contiguous_bad_offsets_reported(mx, bad):
    counts = torch.tensor([128, 128], dtype=torch.int64)
    prob = mx_inputs.contiguous_problem(n=64, k=128, seed=4, counts=counts)
    off = {"not_multiple": [0, 100, 256], "decreasing": [0, 256, 128], "past_end": [0, 128, 384]}[bad]
    d, st = gpu_contiguous(mx, prob, offsets=torch.tensor(off, dtype=torch.int32))
    assert st & mx.MX_DEV_BAD_OFFSETS
    assert bool(is_sentinel(d).all()), "nothing may be written when offsets are invalid"


@pytest.mark.parametrize("which", ["gate_up", "down"])
def test_contiguous_moe_sampled(mx, oracle, which):
    """Full-size MoE grouped GEMMs (32 experts, 8192 tokens x top-8, Zipf
    routing): gate/up (N=4096, K=7168) and down (N=7168, K=2048) -- 256
    random rows, the first and last row of every 128-row tile (each CTA half
    of a pair tile), and the first and last real row of every non-empty
    expert, against the oracle."""
    n, k = mx_inputs.MOE_GATE_NK if which == "gate_up" else mx_inputs.MOE_DOWN_NK
    prob = mx_inputs.contiguous_problem(n=n, k=k, seed=0 if which == "gate_up" else 100)
    off = prob.offsets.numpy()
    ends = []
    for e in range(len(prob.counts)):
        if prob.counts[e] > 0:
            ends += [int(off[e]), int(off[e]) + int(prob.counts[e]) - 1]
    rows = sampled_rows(int(off[-1]), 256, seed=0, extra=ends)
    check_contiguous(mx, oracle, prob, rows=rows, what=f"MoE {which}")


# ---------------------------------------------------------------- masked

def gpu_masked(mx, prob, masked_m=None):
    dev = torch.device("cuda")
    a, b = prob.a.to(dev), prob.b.to(dev)
    qa, sfa = mx.mx_quantize_bf16_to_e4m3(a)
    qb, sfb = mx.mx_quantize_bf16_to_e4m3(b)
    mm = (prob.masked_m if masked_m is None else masked_m).to(dev)
    e, max_m, _ = a.shape
    d = sentinel_fill((e, max_m, b.shape[1]))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    mx.mx_grouped_gemm_masked(qa, sfa, qb, sfb, mm, d=d, dev_status=status)
    torch.cuda.synchronize()
    return d, int(status.item())


def check_masked(mx, oracle, prob, what="", sample_per_expert=None, whole_experts=()):
    """All rows of every expert (or, with sample_per_expert, the first and
    last valid row plus that many random valid rows, and every valid row of
    the experts in whole_experts) against the oracle; all rows at or beyond
    masked_m must still hold the sentinel."""
    d, st = gpu_masked(mx, prob)
    assert st == 0, f"device status {st:#x}"
    e, max_m, k = prob.a.shape
    n = prob.b.shape[1]
    mm = prob.masked_m.tolist()
    for g in range(e):
        assert bool(is_sentinel(d[g, mm[g]:]).all()), f"expert {g}: rows >= masked_m written"
    rng = np.random.default_rng(0)
    rows = []
    for g in range(e):
        if mm[g] == 0:
            continue
        if sample_per_expert is None or g in whole_experts:
            rows.extend(g * max_m + r for r in range(mm[g]))
        else:
            pick = {0, mm[g] - 1} | set(rng.integers(0, mm[g], sample_per_expert).tolist())
            rows.extend(g * max_m + r for r in sorted(pick))
    if not rows:
        return
    rows = np.array(rows, dtype=np.int64)
    qa, sfa = oracle_quantize(oracle, prob.a)
    qb, sfb = oracle_quantize(oracle, prob.b)
    d_ref, absd = oracle.grouped_masked(qa.reshape(e, max_m, k), sfa, qb.reshape(e, n, k), sfb,
                                        prob.masked_m.numpy(), rows=rows)
    d_gpu = to_np_f64(d.reshape(e * max_m, n)[torch.as_tensor(rows, device=d.device)])
    assert_gemm_close(d_gpu, d_ref, absd, what)


def test_masked_small(mx, oracle):
    mm = torch.tensor([0, 200, 1, 129, 128], dtype=torch.int32)
    prob = mx_inputs.masked_problem(n=272, k=256, experts=5, max_m=200, seed=1, masked_m=mm)
    check_masked(mx, oracle, prob, "masked small")


def test_masked_all_empty(mx):
    mm = torch.zeros(3, dtype=torch.int32)
    prob = mx_inputs.masked_problem(n=64, k=128, experts=3, max_m=64, seed=2, masked_m=mm)
    d, st = gpu_masked(mx, prob)
    assert st == 0 and bool(is_sentinel(d).all())


def test_masked_bad_mask_reported_and_clamped(mx, oracle):
    mm = torch.tensor([300, -5], dtype=torch.int32)
    prob = mx_inputs.masked_problem(n=64, k=128, experts=2, max_m=128, seed=3,
                                    masked_m=torch.tensor([128, 0], dtype=torch.int32))
    d, st = gpu_masked(mx, prob, masked_m=mm)
    assert st & mx.MX_DEV_BAD_MASK
    assert bool(is_sentinel(d[1]).all())
    assert not bool(is_sentinel(d[0]).any())


def test_masked_decode_config(mx, oracle):
    """Full masked decode config: 32 experts x max 256 rows, masked_m ~
    U{0..256}, N=4096, K=7168, NaN padding rows; every valid row of the four
    experts with the most rows (a tile boundary inside each) and of the
    expert with the fewest non-zero rows, the first, last and 8 random valid
    rows of every other expert, against the oracle."""
    n, k = mx_inputs.MASKED_NK
    prob = mx_inputs.masked_problem(n=n, k=k, seed=0)
    mm = prob.masked_m.numpy()
    order = np.argsort(-mm, kind="stable")
    whole = set(order[:4].tolist())
    nz = [g for g in range(len(mm)) if mm[g] > 0]
    whole.add(min(nz, key=lambda g: mm[g]))
    assert sum(int(mm[g]) for g in whole) >= 4 * 128
    check_masked(mx, oracle, prob, "masked decode", sample_per_expert=8, whole_experts=whole)
