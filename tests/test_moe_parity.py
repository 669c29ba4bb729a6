"""The MoE expert layer's data movement on the GPU vs the CPU oracle (the B200
MoE-training page's MXFP8 expert layer: router output -> MXFP8 -> grouped
GEMM -> BF16 -> combine; DeepGEMM's contiguous layout, release page section 4).

* routing plan: bit-exact (counts, padded offsets, the row of every entry,
  dropped entries);
* dispatch: bit-exact E4M3 rows and scales (tiled and row-major), padding rows
  zero, non-finite tokens;
* scatter / gather of all-to-all buffers: bit-exact;
* combine: FP32 in j order then BF16, against the fp64 sum, within
  2^-8 * sum_j |w y| + 2^-9 |out| (BF16 rounding of the result plus at most
  topk FP32 roundings);
* the whole single-GPU layer (route, dispatch, gate/up + SwiGLU + MXFP8,
  down, combine) against the oracle's down GEMM and combine of the GPU's own
  hidden activations, at a small size and at the full MoE shape (sampled
  tokens)."""
import numpy as np
import pytest
import torch

import mx_inputs
from mxtest_util import assert_gemm_close, bf16_bits_np, gpu_sf_rowmajor, oracle_quantize, to_np_f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.fixture(scope="module")
def mx():
    import moe_grouped_gemm_mx_b200 as m
    return m


def route_both(mx, oracle, ids: np.ndarray, E: int, pad: int):
    counts, offsets, row, dropped = mx.mx_moe_route(torch.from_numpy(ids.reshape(-1).copy()).to(DEV), E, pad)
    rc, ro, rr, rb = oracle.moe_route(ids, E, pad)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(row.cpu().numpy(), rr)
    assert int(dropped.item()) == rb
    return counts, offsets, row


@pytest.mark.parametrize("T,topk,E,pad", [(300, 8, 32, 128), (300, 8, 32, 1), (5, 2, 3, 2), (1, 1, 1, 128),
                                          (2000, 6, 1000, 128), (4100, 4, 7, 16)])
def test_route(mx, oracle, T, topk, E, pad):
    ids = mx_inputs.topk_ids(T, topk, E, seed=T + E)
    route_both(mx, oracle, ids, E, pad)


def test_route_invalid_ids_and_empty(mx, oracle):
    ids = mx_inputs.topk_ids(700, 4, 9, seed=2)
    ids[3, 1] = -1
    ids[100, 0] = 9
    ids[699, 3] = 1 << 30
    route_both(mx, oracle, ids, 9, 128)
    route_both(mx, oracle, np.zeros((0, 4), dtype=np.int32), 9, 128)


def test_route_full_moe_shape(mx, oracle):
    ids = mx_inputs.topk_ids(mx_inputs.MOE_TOKENS, mx_inputs.MOE_TOPK, mx_inputs.MOE_EXPERTS, seed=0)
    route_both(mx, oracle, ids, mx_inputs.MOE_EXPERTS, 128)


def dispatch_check(mx, oracle, x, ids, E, pad, row_major=False):
    T, topk = ids.shape
    k = x.shape[1]
    counts, offsets, row = route_both(mx, oracle, ids, E, pad)
    m_rows = mx.mx_moe_max_rows(T * topk, E, pad)
    q = torch.full((m_rows, k), 0xAB, dtype=torch.uint8, device=DEV)
    sf_bytes = m_rows * (k // 32) if row_major else mx.scale_bytes(m_rows, k)
    sf = torch.full((sf_bytes,), 0xAB, dtype=torch.uint8, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    mx.mx_moe_dispatch_quant(x.to(DEV), row, topk, counts, offsets, pad, m_rows, q=q, sf=sf,
                             sf_row_major=row_major, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    used = int(offsets[-1].item())
    rq, rsf = oracle.moe_dispatch(x, row.cpu().numpy(), topk, m_rows)
    qh = q.cpu().numpy()
    assert np.array_equal(qh[:used], rq[:used]), f"{(qh[:used] != rq[:used]).sum()} element bytes differ"
    assert np.all(qh[used:] == 0xAB), "rows past the plan were written"
    if row_major:
        sfh = sf.cpu().numpy().reshape(m_rows, k // 32)
    else:
        sfh = gpu_sf_rowmajor(oracle, sf, 1, m_rows, k)
    assert np.array_equal(sfh[:used], rsf[:used]), f"{(sfh[:used] != rsf[:used]).sum()} scale bytes differ"
    return q, sf, counts, offsets, row, m_rows


@pytest.mark.parametrize("T,k,topk,E,pad", [(300, 512, 8, 32, 128), (77, 128, 3, 5, 128), (64, 256, 2, 4, 1),
                                            (513, 1024, 6, 16, 32)])
def test_dispatch(mx, oracle, T, k, topk, E, pad):
    x = mx_inputs.outlier_bf16((T, k), seed=T + k)
    ids = mx_inputs.topk_ids(T, topk, E, seed=T)
    dispatch_check(mx, oracle, x, ids, E, pad)


def test_dispatch_row_major_and_nonfinite(mx, oracle):
    x = mx_inputs.normal_bf16((90, 384), 1.0, 4)
    x[3, 40] = float("nan")
    x[7, 300] = float("inf")
    x[8] = 0.0
    x[9, :32] = 1e-40                      # BF16 subnormals
    ids = mx_inputs.topk_ids(90, 4, 8, seed=5)
    dispatch_check(mx, oracle, x, ids, 8, 1, row_major=True)
    dispatch_check(mx, oracle, x, ids, 8, 128, row_major=False)


def test_dispatch_bad_row_reports(mx):
    x = mx_inputs.normal_bf16((4, 128), 1.0, 6).to(DEV)
    row = torch.tensor([0, 1, 2, 999, 3, 4, 5, 6], dtype=torch.int32, device=DEV)   # 999 >= m_rows
    q = torch.zeros((128, 128), dtype=torch.uint8, device=DEV)
    sf = torch.zeros(mx.scale_bytes(128, 128), dtype=torch.uint8, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    mx.mx_moe_dispatch_quant(x, row, 2, None, None, 1, 128, q=q, sf=sf, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & mx.MX_DEV_BAD_INDEX


def test_dispatch_full_moe_shape(mx, oracle):
    T, topk, E = mx_inputs.MOE_TOKENS, mx_inputs.MOE_TOPK, mx_inputs.MOE_EXPERTS
    k = mx_inputs.MOE_GATE_NK[1]
    x = mx_inputs.normal_bf16((T, k), 1.0, 21)
    ids = mx_inputs.topk_ids(T, topk, E, seed=0)
    dispatch_check(mx, oracle, x, ids, E, 128)


def test_scatter_and_gather_rows(mx, oracle):
    """The expert-parallel path: dispatch into an unpadded, expert-ordered send
    buffer (row-major scales), then scatter it into the padded grouped layout;
    the result equals a direct dispatch into that layout.  Gather moves rows
    back."""
    T, k, topk, E = 200, 256, 4, 6
    x = mx_inputs.outlier_bf16((T, k), seed=31)
    ids = mx_inputs.topk_ids(T, topk, E, seed=32)
    qs, sfs, _, _, row_send, n_send = dispatch_check(mx, oracle, x, ids, E, 1, row_major=True)
    n = T * topk
    # send-buffer row i holds entry order[i]; in the padded plan that entry sits at row_pad[order[i]]
    counts, offsets, row_pad = route_both(mx, oracle, ids, E, 128)
    order = np.argsort(row_send.cpu().numpy())
    dst = torch.from_numpy(row_pad.cpu().numpy()[order].astype(np.int32)).to(DEV)
    m_rows = mx.mx_moe_max_rows(n, E, 128)
    q = torch.full((m_rows, k), 0xAB, dtype=torch.uint8, device=DEV)
    sf = torch.full((mx.scale_bytes(m_rows, k),), 0xAB, dtype=torch.uint8, device=DEV)
    mx.mx_moe_scatter_rows(qs[:n].contiguous(), sfs[: n * (k // 32)].contiguous(), dst, counts, offsets, 128, m_rows,
                           q=q, sf=sf)
    torch.cuda.synchronize()
    used = int(offsets[-1].item())
    rq, rsf = oracle.moe_dispatch(x, row_pad.cpu().numpy(), topk, m_rows)
    assert np.array_equal(q.cpu().numpy()[:used], rq[:used])
    assert np.array_equal(gpu_sf_rowmajor(oracle, sf, 1, m_rows, k)[:used], rsf[:used])
    # gather: BF16 rows back into send order, with one out-of-range index
    y = mx_inputs.normal_bf16((used, 64), 1.0, 33).to(DEV)
    idx = dst.clone()
    idx[5] = used + 7
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    g = mx.mx_gather_rows(y, idx, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & mx.MX_DEV_BAD_INDEX
    yb = bf16_bits_np(y)
    gb = bf16_bits_np(g)
    ref = yb[np.clip(idx.cpu().numpy(), 0, used - 1)]
    ref[5] = 0
    assert np.array_equal(gb, ref)


def combine_check(mx, oracle, y, row, w, tokens=None):
    out = mx.mx_moe_combine(y, row, w)
    torch.cuda.synchronize()
    wn = w.cpu().numpy()
    rn = row.cpu().numpy().reshape(wn.shape)
    if tokens is None:
        tokens = np.arange(wn.shape[0])
    yb = bf16_bits_np(y)
    ref, absd = oracle.moe_combine(yb, np.ascontiguousarray(rn[tokens]), np.ascontiguousarray(wn[tokens]))
    got = to_np_f64(out)[tokens]
    err = np.abs(got - ref)
    tol = 2.0 ** -8 * absd + 2.0 ** -9 * np.abs(ref) + 1e-30
    assert np.all(err <= tol), f"{(err > tol).sum()} combine outputs outside tolerance"
    return out


def test_combine(mx, oracle):
    T, topk, N, rows = 333, 8, 200, 3000
    y = mx_inputs.normal_bf16((rows, N), 1.0, 40).to(DEV)
    rng = np.random.default_rng(41)
    row = rng.integers(0, rows, size=T * topk).astype(np.int32)
    row[::17] = -1                                   # dropped entries
    w = torch.from_numpy(mx_inputs.gate_weights(T, topk, seed=42)).to(DEV)
    combine_check(mx, oracle, y, torch.from_numpy(row).to(DEV), w)


def test_combine_bad_row_reports(mx):
    y = torch.zeros((4, 16), dtype=torch.bfloat16, device=DEV)
    row = torch.tensor([0, 4], dtype=torch.int32, device=DEV)
    w = torch.ones((1, 2), dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    mx.mx_moe_combine(y, row, w, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & mx.MX_DEV_BAD_INDEX


def moe_layer(mx, x, ids, w_gate_up, w_down, gate_w, E, pad=128):
    """One MoE expert layer on the GPU, every step a library call."""
    T, topk = ids.shape
    counts, offsets, row, _ = mx.mx_moe_route(torch.from_numpy(ids.reshape(-1).copy()).to(DEV), E, pad)
    m_rows = mx.mx_moe_max_rows(T * topk, E, pad)
    qa, sfa = mx.mx_moe_dispatch_quant(x.to(DEV), row, topk, counts, offsets, pad, m_rows)
    q13, sf13 = mx.mx_quantize_bf16_to_e4m3(w_gate_up.to(DEV))
    q2, sf2 = mx.mx_quantize_bf16_to_e4m3(w_down.to(DEV))
    qh, sfh = mx.mx_grouped_gemm_contiguous_swiglu_quant(qa, sfa, q13, sf13, offsets)
    d = mx.mx_grouped_gemm_contiguous(qh, sfh, q2, sf2, offsets)
    out = mx.mx_moe_combine(d, row, torch.from_numpy(gate_w).to(DEV))
    torch.cuda.synchronize()
    return dict(counts=counts, offsets=offsets, row=row, m_rows=m_rows, qh=qh, sfh=sfh, d=d, out=out)


def layer_check(mx, oracle, x, ids, w_down, gate_w, E, r, sample_tokens=None):
    """The layer's output against the oracle: down GEMM of the GPU's hidden
    MXFP8 activations (fp64), then the combine in fp64, within the GEMM
    tolerance carried through the gate weights plus the combine's rounding."""
    T, topk = ids.shape
    offsets = r["offsets"].cpu().numpy()
    rown = r["row"].cpu().numpy().reshape(T, topk)
    tokens = np.arange(T) if sample_tokens is None else sample_tokens
    rows = np.ascontiguousarray(rown[tokens].reshape(-1).astype(np.int64))
    i_dim = r["qh"].shape[1]
    qh = r["qh"].cpu().numpy()
    sfh = gpu_sf_rowmajor(oracle, r["sfh"], 1, r["m_rows"], i_dim)
    q2, sf2 = oracle_quantize(oracle, w_down)
    n = w_down.shape[1]
    q2 = q2.reshape(E, n, i_dim)
    sf2 = sf2.reshape(E, n, i_dim // 32)
    d_ref, d_abs = oracle.grouped_contiguous(qh, sfh, q2, sf2, offsets, rows=rows)
    # the GPU's D rows themselves meet the GEMM tolerance
    d_rows = to_np_f64(r["d"][torch.from_numpy(rows).to(DEV)])   # rows past the plan are never computed
    assert_gemm_close(d_rows, d_ref, d_abs, "moe layer down GEMM")
    wt = gate_w[tokens].astype(np.float64)
    d_ref = d_ref.reshape(len(tokens), topk, n)
    d_abs = d_abs.reshape(len(tokens), topk, n)
    ref = np.einsum("tj,tjn->tn", wt, d_ref)
    tol = np.einsum("tj,tjn->tn", np.abs(wt), 1e-2 * d_abs + 1e-3 + 2.0 ** -9 * np.abs(d_ref))
    tol += 2.0 ** -8 * np.einsum("tj,tjn->tn", np.abs(wt), np.abs(d_ref)) + 2.0 ** -9 * np.abs(ref)
    got = to_np_f64(r["out"][torch.from_numpy(tokens).to(DEV)])
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{bad.sum()} of {bad.size} layer outputs outside tolerance"


def test_moe_layer_small(mx, oracle):
    T, topk, E, H, I, N = 200, 4, 6, 256, 256, 384
    x = mx_inputs.normal_bf16((T, H), 1.0, 50)
    ids = mx_inputs.topk_ids(T, topk, E, seed=51)
    gate_w = mx_inputs.gate_weights(T, topk, seed=52)
    w13 = mx_inputs.normal_bf16((E, 2 * I, H), 0.05, 53)
    w2 = mx_inputs.normal_bf16((E, N, I), 0.05, 54)
    r = moe_layer(mx, x, ids, w13, w2, gate_w, E)
    layer_check(mx, oracle, x, ids, w2, gate_w, E, r)


def test_moe_layer_full_shape_sampled(mx, oracle):
    """8192 tokens x top-8 of 32 experts, hidden 7168, intermediate 2048 (the
    contiguous workload's gate/up 4096 x 7168 and down 7168 x 2048): 96
    sampled tokens, among them the first and last."""
    T, topk, E = mx_inputs.MOE_TOKENS, mx_inputs.MOE_TOPK, mx_inputs.MOE_EXPERTS
    H = mx_inputs.MOE_GATE_NK[1]
    I = mx_inputs.MOE_GATE_NK[0] // 2
    N = mx_inputs.MOE_DOWN_NK[0]
    x = mx_inputs.normal_bf16((T, H), 1.0, 60, device=DEV)
    ids = mx_inputs.topk_ids(T, topk, E, seed=0)
    gate_w = mx_inputs.gate_weights(T, topk, seed=0)
    w13 = mx_inputs.normal_bf16((E, 2 * I, H), 0.02, 61, device=DEV)
    w2 = mx_inputs.normal_bf16((E, N, I), 0.02, 62, device=DEV)
    r = moe_layer(mx, x, ids, w13, w2, gate_w, E)
    rng = np.random.default_rng(63)
    tokens = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 94, replace=False)]))
    layer_check(mx, oracle, x, ids, w2.cpu(), gate_w, E, r, sample_tokens=tokens)


def test_ep_layer_one_rank_matches_direct_layer(mx):
    """The expert-parallel layer with one rank (send buffer in expert order,
    scatter into the padded layout, gather back) computes exactly what the
    direct single-GPU layer computes."""
    from moe_grouped_gemm_mx_b200.ep import ep_moe_layer
    T, topk, E, H, I, N = 300, 4, 8, 256, 256, 256
    x = mx_inputs.normal_bf16((T, H), 1.0, 70).to(DEV)
    ids = mx_inputs.topk_ids(T, topk, E, seed=71)
    ids[5, 2] = -1                                   # a dropped entry
    gate_w = mx_inputs.gate_weights(T, topk, seed=72)
    w13 = mx_inputs.normal_bf16((E, 2 * I, H), 0.05, 73)
    w2 = mx_inputs.normal_bf16((E, N, I), 0.05, 74)
    r = moe_layer(mx, x, ids, w13, w2, gate_w, E)
    q13, sf13 = mx.mx_quantize_bf16_to_e4m3(w13.to(DEV))
    q2, sf2 = mx.mx_quantize_bf16_to_e4m3(w2.to(DEV))
    y = ep_moe_layer(x, torch.from_numpy(ids).to(DEV), torch.from_numpy(gate_w).to(DEV), E, q13, sf13, q2, sf2)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), r["out"].view(torch.int16))
