"""Expert parallelism with the exchange over peer memory (the DeepEP role on
the B200 MoE-training page: tokens go to the ranks holding their experts and
the results come back), emulated on one GPU: R ranks' receive and output
buffers are R buffer sets on the same device, reached by the kernels through
the same device address tables they would use with one GPU per rank, and the
phases run rank after rank (what the stream barriers between phases give
with one process per GPU; no kernel waits on another).

* placement plan: bit-exact against the oracle's (owner rank and row of
  every entry, each owner's counts and padded offsets);
* dispatch: every owner's receive buffer bit-exact (E4M3 rows and tiled
  scales of the routed tokens, the oracle's quantisation; zero padding rows);
* the whole layer on 2 and 4 emulated ranks: bit-identical to the
  single-GPU layer on the same tokens (both route every row through the same
  kernels; a row's result does not depend on where it sits);
* bad ranks in the address tables' range checks set MX_DEV_BAD_INDEX."""
import numpy as np
import pytest
import torch

import mx_inputs
from mxtest_util import bf16_bits_np, gpu_sf_rowmajor

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.fixture(scope="module")
def mx():
    import moe_grouped_gemm_mx_b200 as m
    return m


def rank_inputs(ranks, tokens, topk, experts, seed):
    ids_list = [mx_inputs.topk_ids(tokens[r], topk, experts, seed=seed + r) for r in range(ranks)]
    if tokens[0] > 3:
        ids_list[0][3, 1] = -1          # a dropped entry
    return ids_list


def gpu_plans(mx, ids_list, experts, pad):
    """Every rank's plan from the library: route (pad 1), the count table,
    the placement."""
    routes = [mx.mx_moe_route(torch.from_numpy(ids.reshape(-1).copy()).to(DEV), experts, 1) for ids in ids_list]
    table = torch.stack([r[0] for r in routes])
    plans = []
    for r, ids in enumerate(ids_list):
        flat = torch.from_numpy(ids.reshape(-1).copy()).to(DEV)
        plans.append(mx.mx_moe_peer_plan(flat, routes[r][2], table, r, experts, pad))
    torch.cuda.synchronize()
    return plans


@pytest.mark.parametrize("ranks,experts,pad", [(1, 8, 128), (2, 8, 128), (3, 6, 1), (4, 32, 128), (4, 64, 32)])
def test_peer_plan(mx, oracle, ranks, experts, pad):
    tokens = [150, 0, 97, 300][:ranks] if ranks > 1 else [150]
    ids_list = rank_inputs(ranks, tokens, 4, experts, seed=100 * ranks + experts)
    plans = gpu_plans(mx, ids_list, experts, pad)
    per, counts, offsets = oracle.moe_peer_plan(ids_list, experts, pad=pad)
    for r in range(ranks):
        dst_rank, dst_row, cl, ol = (t.cpu().numpy() for t in plans[r])
        assert np.array_equal(dst_rank, per[r][0]), f"rank {r}: owners differ"
        assert np.array_equal(dst_row, per[r][1]), f"rank {r}: rows differ"
        assert np.array_equal(cl, counts[r]) and np.array_equal(ol, offsets[r]), f"rank {r}: receive plan differs"


def test_peer_dispatch_receive_buffers(mx, oracle):
    """Three ranks holding 2 of 6 experts each: every owner's receive buffer
    holds the oracle's MXFP8 row of each routed token at the planned row, and
    zero rows in the group padding."""
    from moe_grouped_gemm_mx_b200.ep import LibraryOps, PeerBuffers
    ranks, experts, topk, H, N, pad = 3, 6, 3, 256, 128, 128
    tokens = [120, 45, 200]
    ids_list = rank_inputs(ranks, tokens, topk, experts, seed=7)
    xs = [mx_inputs.normal_bf16((tokens[r], H), 1.0, 20 + r).to(DEV) for r in range(ranks)]
    xs[1][5, 17] = float("nan")                 # a non-finite token: its blocks are NaN-coded
    m_cap = mx.mx_moe_max_rows(sum(tokens) * topk, experts // ranks, pad)
    bufs = PeerBuffers.emulated(ranks, m_cap, H, N, DEV)
    for b in bufs:                               # stale data everywhere
        b.q.fill_(0xAB)
        b.sf.fill_(0xCD)
    plans = gpu_plans(mx, ids_list, experts, pad)
    ops = LibraryOps(mx)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    for r in range(ranks):
        dst_rank, dst_row, cl, ol = plans[r]
        mx.mx_moe_dispatch_quant_peer(xs[r], dst_rank, dst_row, topk, bufs[r].q_ptrs, bufs[r].sf_ptrs, m_cap,
                                      bufs[r].q, bufs[r].sf, cl, ol, pad, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    per, counts, offsets = oracle.moe_peer_plan(ids_list, experts, pad=pad)
    for o in range(ranks):
        q = bufs[o].q.cpu().numpy()
        sf = gpu_sf_rowmajor(oracle, bufs[o].sf, 1, m_cap, H)
        seen = np.zeros(m_cap, dtype=bool)
        for r in range(ranks):
            qx, sx = oracle.quantize(bf16_bits_np(xs[r]))
            dr, drow = per[r]
            for i in np.nonzero(dr == o)[0]:
                t = i // topk
                assert np.array_equal(q[drow[i]], qx[t]), f"owner {o} row {drow[i]} (rank {r} entry {i})"
                assert np.array_equal(sf[drow[i]], sx[t]), f"owner {o} scales of row {drow[i]}"
                seen[drow[i]] = True
        for l in range(experts // ranks):
            lo, hi = offsets[o][l] + counts[o][l], offsets[o][l + 1]
            assert not q[lo:hi].any() and not sf[lo:hi].any(), f"owner {o} expert {l}: padding rows not zero"
            seen[lo:hi] = True
        assert seen[:offsets[o][-1]].all()      # every row of the plan is a routed row or padding


@pytest.mark.parametrize("ranks", [2, 4])
def test_peer_layer_matches_single_gpu_layer(mx, ranks):
    """The whole expert layer over R emulated ranks (plan, dispatch into the
    owners, each owner's fused gate/up + SwiGLU + MXFP8 and down GEMMs in
    place, combine from the owners) gives every rank's tokens exactly what
    the single-GPU layer gives them."""
    from moe_grouped_gemm_mx_b200.ep import PeerBuffers, ep_moe_layer_peer_emulated
    experts, topk, H, I, N, pad = 8, 4, 256, 256, 256, 128
    tokens = [300, 64, 211, 128][:ranks]
    ids_list = rank_inputs(ranks, tokens, topk, experts, seed=40 + ranks)
    xs = [mx_inputs.normal_bf16((tokens[r], H), 1.0, 60 + r).to(DEV) for r in range(ranks)]
    gws = [torch.from_numpy(mx_inputs.gate_weights(tokens[r], topk, seed=70 + r)).to(DEV) for r in range(ranks)]
    w13 = mx_inputs.normal_bf16((experts, 2 * I, H), 0.05, 80).to(DEV)
    w2 = mx_inputs.normal_bf16((experts, N, I), 0.05, 81).to(DEV)
    q13, sf13 = mx.mx_quantize_bf16_to_e4m3(w13)
    q2, sf2 = mx.mx_quantize_bf16_to_e4m3(w2)
    el = experts // ranks
    per13 = mx.scale_bytes(2 * I, H)
    per2 = mx.scale_bytes(N, I)
    weights = [(q13[r * el:(r + 1) * el], sf13[r * el * per13:(r + 1) * el * per13],
                q2[r * el:(r + 1) * el], sf2[r * el * per2:(r + 1) * el * per2]) for r in range(ranks)]
    m_cap = mx.mx_moe_max_rows(sum(tokens) * topk, el, pad)
    bufs = PeerBuffers.emulated(ranks, m_cap, H, N, DEV)
    mx.read_internal_status()   # clear what earlier calls may have left
    outs = ep_moe_layer_peer_emulated(xs, [torch.from_numpy(i).to(DEV) for i in ids_list], gws, experts, weights,
                                      bufs, pad=pad)
    for r in range(ranks):
        counts, offsets, row, _ = mx.mx_moe_route(torch.from_numpy(ids_list[r].reshape(-1).copy()).to(DEV),
                                                  experts, pad)
        m_rows = mx.mx_moe_max_rows(tokens[r] * topk, experts, pad)
        qa, sfa = mx.mx_moe_dispatch_quant(xs[r], row, topk, counts, offsets, pad, m_rows)
        qh, sfh = mx.mx_grouped_gemm_contiguous_swiglu_quant(qa, sfa, q13, sf13, offsets)
        d = mx.mx_grouped_gemm_contiguous(qh, sfh, q2, sf2, offsets)
        ref = mx.mx_moe_combine(d, row, gws[r])
        torch.cuda.synchronize()
        assert torch.equal(outs[r].view(torch.int16), ref.view(torch.int16)), f"rank {r} differs"
    assert mx.read_internal_status() == 0


def test_peer_bad_ranks_report(mx):
    """A destination or source rank outside the tables is skipped and sets
    MX_DEV_BAD_INDEX; nothing is written for it."""
    from moe_grouped_gemm_mx_b200.ep import PeerBuffers
    bufs = PeerBuffers.emulated(2, 128, 128, 128, DEV)
    x = mx_inputs.normal_bf16((2, 128), 1.0, 5).to(DEV)
    dst_rank = torch.tensor([0, 2], dtype=torch.int32, device=DEV)
    dst_row = torch.tensor([0, 1], dtype=torch.int32, device=DEV)
    counts = torch.zeros(1, dtype=torch.int32, device=DEV)
    offsets = torch.zeros(2, dtype=torch.int32, device=DEV)
    bufs[1].q.fill_(0x11)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    mx.mx_moe_dispatch_quant_peer(x, dst_rank, dst_row, 1, bufs[0].q_ptrs, bufs[0].sf_ptrs, 128, bufs[0].q,
                                  bufs[0].sf, counts, offsets, 1, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & mx.MX_DEV_BAD_INDEX
    assert bool((bufs[1].q == 0x11).all())
    st.zero_()
    w = torch.ones((1, 2), dtype=torch.float32, device=DEV)
    mx.mx_moe_combine_peer(bufs[0].y_ptrs, 128, 128, torch.tensor([1, -3], dtype=torch.int32, device=DEV),
                           torch.tensor([0, 0], dtype=torch.int32, device=DEV), w, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & mx.MX_DEV_BAD_INDEX


def test_peer_layer_undersized_buffers_raise(mx):
    """Receive buffers too small for the plan: the dispatch skips the rows
    past the buffer, the grouped GEMMs refuse the offsets and the combine
    skips the rows it cannot load -- each reports it, and the layer raises
    instead of returning the stale contents of the output buffers."""
    from moe_grouped_gemm_mx_b200.ep import PeerBuffers, ep_moe_layer_peer_emulated
    ranks, experts, topk, H, I, N, pad = 2, 4, 2, 128, 128, 128, 128
    tokens = [200, 150]
    ids_list = rank_inputs(ranks, tokens, topk, experts, seed=90)
    xs = [mx_inputs.normal_bf16((tokens[r], H), 1.0, 91 + r).to(DEV) for r in range(ranks)]
    gws = [torch.from_numpy(mx_inputs.gate_weights(tokens[r], topk, seed=93 + r)).to(DEV) for r in range(ranks)]
    q13, sf13 = mx.mx_quantize_bf16_to_e4m3(mx_inputs.normal_bf16((experts, 2 * I, H), 0.05, 95).to(DEV))
    q2, sf2 = mx.mx_quantize_bf16_to_e4m3(mx_inputs.normal_bf16((experts, N, I), 0.05, 96).to(DEV))
    el = experts // ranks
    per13, per2 = mx.scale_bytes(2 * I, H), mx.scale_bytes(N, I)
    weights = [(q13[r * el:(r + 1) * el], sf13[r * el * per13:(r + 1) * el * per13],
                q2[r * el:(r + 1) * el], sf2[r * el * per2:(r + 1) * el * per2]) for r in range(ranks)]
    need = mx.mx_moe_max_rows(sum(tokens) * topk, el, pad)
    assert need > 256
    bufs = PeerBuffers.emulated(ranks, 256, H, N, DEV)      # far below the rows the plans need
    with pytest.raises(RuntimeError, match="device status"):
        ep_moe_layer_peer_emulated(xs, [torch.from_numpy(i).to(DEV) for i in ids_list], gws, experts, weights,
                                   bufs, pad=pad)
    # the same layer with buffers of the right size runs clean
    bufs = PeerBuffers.emulated(ranks, need, H, N, DEV)
    outs = ep_moe_layer_peer_emulated(xs, [torch.from_numpy(i).to(DEV) for i in ids_list], gws, experts, weights,
                                      bufs, pad=pad)
    assert all(bool(torch.isfinite(o.float()).all()) for o in outs)
