"""Training-side MoE GEMMs on the GPU vs the CPU oracle: quantisation along the
token dimension into the transposed layout (bit-exact, every BF16 pattern,
ragged tiles, padding), the K-grouped weight-gradient GEMM (ragged experts,
an empty expert, odd 128-token chunk counts, bad offsets, the MoE gate/up
shape sampled), and the input-gradient GEMM on weights quantised along N."""
import numpy as np
import pytest
import torch

import mx_inputs
from mxtest_util import sampled_rows, assert_gemm_close, is_sentinel, sentinel_fill, to_np_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    import moe_grouped_gemm_mx_b200 as m
    return m


def run_transposed(mx, x):
    dev = torch.device("cuda")
    xd = x.to(dev)
    groups = 1 if x.dim() == 2 else x.shape[0]
    rows, cols = x.shape[-2], x.shape[-1]
    sf = torch.full((groups * mx.scale_bytes(cols, rows),), 0x5A, dtype=torch.uint8, device=dev)
    q, sf = mx.mx_quantize_bf16_to_e4m3_transposed(xd, sf=sf)
    torch.cuda.synchronize()
    return q.cpu().numpy().reshape(groups * cols, rows), sf.cpu().numpy()


def check_transposed(mx, oracle, x):
    groups = 1 if x.dim() == 2 else x.shape[0]
    rows, cols = x.shape[-2], x.shape[-1]
    q, sf = run_transposed(mx, x)
    rq, rsf = oracle.quantize_transposed(x)
    assert np.array_equal(q, rq), f"{(q != rq).sum()} element bytes differ"
    # the whole tiled region, padding included, against the oracle's tiling
    per = oracle.scale_bytes(cols, rows)
    for g in range(groups):
        want = oracle.sf_tile(rsf[g * cols:(g + 1) * cols], cols, rows)
        assert np.array_equal(sf[g * per:(g + 1) * per], want), f"group {g}: tiled scales differ"


def test_transposed_every_bf16_pattern(mx, oracle):
    """All 65536 BF16 bit patterns (NaN and Inf included), shuffled into a
    [2048, 32] matrix so every 32-row block of a column mixes magnitudes."""
    bits = np.random.default_rng(0).permutation(np.arange(65536, dtype=np.int64)).astype(np.uint16)
    x = torch.from_numpy(bits.view(np.int16).reshape(2048, 32).copy()).view(torch.bfloat16)
    check_transposed(mx, oracle, x)


@pytest.mark.parametrize("shape", [(288, 200), (32, 8), (128, 128), (3, 64, 136), (2, 416, 264)])
def test_transposed_ragged_tiles(mx, oracle, shape):
    """Row tiles of 128 with a 32/64/96-row tail, column tiles with a tail of
    8..120, groups; outliers, zero blocks and a NaN block included."""
    x = mx_inputs.outlier_bf16(shape, seed=3)
    if len(shape) == 2 and shape[0] >= 64:
        x[32:64, 0] = 0.0          # an all-zero block
        x[0:32, 1] = float("nan")  # a non-finite block
    check_transposed(mx, oracle, x)


# ---------------------------------------------------------------- K-grouped weight gradient

def kgrouped_problem(m, n, offsets, seed):
    t = int(offsets[-1])
    dy = mx_inputs.normal_bf16((t, m), 1.0, seed)          # output gradient [tokens, m]
    x = mx_inputs.normal_bf16((t, n), 1.0, seed + 1)       # layer input [tokens, n]
    return dy, x


def run_kgrouped(mx, dy, x, offsets, groups, d=None, status=None):
    dev = torch.device("cuda")
    qa, sfa = mx.mx_quantize_bf16_to_e4m3_transposed(dy.to(dev))   # [m, tokens]
    qb, sfb = mx.mx_quantize_bf16_to_e4m3_transposed(x.to(dev))    # [n, tokens]
    off = torch.as_tensor(offsets, dtype=torch.int32, device=dev)
    d = mx.mx_grouped_gemm_kgrouped(qa, sfa, qb, sfb, off, groups=groups, d=d, dev_status=status)
    torch.cuda.synchronize()
    return d


def test_kgrouped_ragged_experts(mx, oracle):
    """Experts with 1, 0, 2, 1 and 3 chunks of 128 tokens (odd counts leave
    half of a 256-token stage to the next expert, which must not leak in);
    M = 200 and N = 272 are not multiples of the 256-wide tiles."""
    offsets = np.array([0, 128, 128, 384, 512, 896], dtype=np.int32)
    m, n = 200, 272
    dy, x = kgrouped_problem(m, n, offsets, seed=40)
    dev = torch.device("cuda")
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    d = run_kgrouped(mx, dy, x, offsets, 5, status=st)
    assert int(st.item()) == 0
    qa, sfa = oracle.quantize_transposed(dy)
    qb, sfb = oracle.quantize_transposed(x)
    d_ref, absd = oracle.grouped_kgrouped(qa, sfa, qb, sfb, offsets)
    dg = to_np_f64(d)
    assert not dg[1].any(), "the expert with no tokens must get a zero gradient"
    for e in range(5):
        assert_gemm_close(dg[e], d_ref[e], absd[e], f"K-grouped expert {e}")


def test_kgrouped_bad_offsets_reported(mx):
    dev = torch.device("cuda")
    dy, x = kgrouped_problem(128, 128, np.array([0, 256]), seed=41)
    d = sentinel_fill((2, 128, 128))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    run_kgrouped(mx, dy, x, np.array([0, 200, 256], dtype=np.int32), 2, d=d, status=st)
    assert int(st.item()) & mx.MX_DEV_BAD_OFFSETS
    assert bool(is_sentinel(d).all()), "nothing may be written when offsets are invalid"


def test_kgrouped_moe_gate_up_wgrad_sampled(mx, oracle):
    """Weight gradient of the MoE gate/up projection: 32 experts, 8192 tokens x
    top-8 (Zipf 1.1), groups padded to 128 tokens; dW[e] = dY_e^T X_e with
    dY [tokens, 4096], X [tokens, 7168]; 256 sampled (expert, row) pairs plus
    the first and last row of every expert."""
    n_out, k_in = mx_inputs.MOE_GATE_NK
    counts = mx_inputs.zipf_routing_counts(seed=0)
    offsets = mx_inputs.padded_offsets(counts).numpy().astype(np.int32)
    t = int(offsets[-1])
    dy = mx_inputs.normal_bf16((t, n_out), 1.0, 50)
    x = mx_inputs.normal_bf16((t, k_in), 1.0, 51)
    groups = len(counts)
    d = run_kgrouped(mx, dy, x, offsets, groups)
    rng = np.random.default_rng(2)
    ids = set(rng.integers(0, groups * n_out, 256).tolist())
    for e in range(groups):
        ids.update([e * n_out, e * n_out + n_out - 1])
    ids = np.array(sorted(ids), dtype=np.int64)
    qa, sfa = oracle.quantize_transposed(dy)
    qb, sfb = oracle.quantize_transposed(x)
    d_ref, absd = oracle.grouped_kgrouped(qa, sfa, qb, sfb, offsets, rows=ids)
    dg = d.reshape(groups * n_out, k_in)[torch.as_tensor(ids, device=d.device)]
    assert_gemm_close(to_np_f64(dg), d_ref, absd, "MoE gate/up wgrad (sampled)")


# ---------------------------------------------------------------- input gradient

def test_dgrad_on_weights_quantised_along_n(mx, oracle):
    """dX = dY W per expert: the contiguous grouped GEMM with the expert
    weights [E, N, K] quantised along N into [E, K, N]."""
    counts = torch.tensor([5, 0, 200, 77], dtype=torch.int64)
    offsets = mx_inputs.padded_offsets(counts)
    e, n, k = len(counts), 256, 384
    t = int(offsets[-1])
    dev = torch.device("cuda")
    dy = mx_inputs.normal_bf16((t, n), 1.0, 60)
    w = mx_inputs.normal_bf16((e, n, k), 0.02, 61)
    q_dy, sf_dy = mx.mx_quantize_bf16_to_e4m3(dy.to(dev))
    q_wt, sf_wt = mx.mx_quantize_bf16_to_e4m3_transposed(w.to(dev))     # [E, K, N]
    dx = mx.mx_grouped_gemm_contiguous(q_dy, sf_dy, q_wt, sf_wt, offsets.to(dev))
    torch.cuda.synchronize()
    r_dy, rs_dy = oracle.quantize(dy.view(torch.int16).numpy().view(np.uint16))
    r_wt, rs_wt = oracle.quantize_transposed(w)
    d_ref, absd = oracle.grouped_contiguous(r_dy, rs_dy, r_wt.reshape(e, k, n), rs_wt, offsets.numpy())
    m_end = int(offsets[-1])
    assert_gemm_close(to_np_f64(dx[:m_end]), d_ref, absd, "dgrad")


def test_dgrad_moe_shape_sampled(mx, oracle):
    """dX = dY W13 at the MoE gate/up shape (32 experts, 8192 tokens x top-8,
    Zipf routing, dY [T, 4096], W13 [32, 4096, 7168] quantised along N into
    [32, 7168, 4096]): 256 random rows, the first and last row of every
    128-row tile and of every non-empty expert, against the oracle."""
    counts = mx_inputs.zipf_routing_counts(seed=0)
    offsets = mx_inputs.padded_offsets(counts)
    n_out, k_in = mx_inputs.MOE_GATE_NK
    e = len(counts)
    t = int(offsets[-1])
    dev = torch.device("cuda")
    dy = mx_inputs.normal_bf16((t, n_out), 1.0, 62)
    pad = torch.repeat_interleave(torch.arange(e), (offsets[1:] - offsets[:-1]).long())
    local = torch.arange(t) - offsets[:-1].long()[pad]
    dy[local >= counts[pad]] = 0                    # padding rows of the grouped layout are zero
    w = mx_inputs.normal_bf16((e, n_out, k_in), 0.02, 63)
    q_dy, sf_dy = mx.mx_quantize_bf16_to_e4m3(dy.to(dev))
    q_wt, sf_wt = mx.mx_quantize_bf16_to_e4m3_transposed(w.to(dev))     # [E, K, N]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    dx = mx.mx_grouped_gemm_contiguous(q_dy, sf_dy, q_wt, sf_wt, offsets.to(dev), dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ends = []
    for g in range(e):
        if counts[g] > 0:
            ends += [int(offsets[g]), int(offsets[g]) + int(counts[g]) - 1]
    rows = sampled_rows(t, 256, seed=3, extra=ends)
    r_dy, rs_dy = oracle.quantize(dy.view(torch.int16).numpy().view(np.uint16))
    r_wt, rs_wt = oracle.quantize_transposed(w)
    d_ref, absd = oracle.grouped_contiguous(r_dy, rs_dy, r_wt.reshape(e, k_in, n_out), rs_wt,
                                            offsets.numpy().astype(np.int32), rows=rows)
    dg = dx[torch.as_tensor(rows, device=dev)]
    assert_gemm_close(to_np_f64(dg), d_ref, absd, "MoE dgrad (sampled)")
