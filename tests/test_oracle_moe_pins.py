"""Pins of the oracle's MoE expert-layer data movement (routing plan,
dispatch into the contiguous grouped layout, weighted combine) to facts that
do not come from the oracle itself: hand-worked examples, a library routine
(numpy's stable argsort) for the unpadded plan, the worked MXFP8 example of
32 ones (scale 0x77, elements 0x78), dequantisation error bounds, one-hot
combines and an fp64 einsum.

The layer is the B200 MoE-training page's MXFP8 expert layer (router output
-> MXFP8 -> grouped GEMM -> BF16 -> all-to-all combine; glossary entry on
all-to-all); the grouped layout is DeepGEMM's contiguous one (release page,
section 4)."""
import numpy as np
import pytest
import torch

import mx_inputs


def test_route_hand_example():
    # T = 3 tokens, top-2; entries in token-major order have experts 2,0 | 0,1 | 2,1
    ids = np.array([[2, 0], [0, 1], [2, 1]], dtype=np.int32)
    from oracle import moe_route
    counts, offsets, row, bad = moe_route(ids, 3, pad=2)
    assert bad == 0
    assert counts.tolist() == [2, 2, 2]
    assert offsets.tolist() == [0, 2, 4, 6]
    # expert 0 gets entries 1, 2 -> rows 0, 1; expert 1 entries 3, 5 -> 2, 3; expert 2 entries 0, 4 -> 4, 5
    assert row.tolist() == [4, 0, 1, 2, 5, 3]
    counts, offsets, row, bad = moe_route(ids, 3, pad=4)
    assert offsets.tolist() == [0, 4, 8, 12]
    assert row.tolist() == [8, 0, 1, 4, 9, 5]


def test_route_drops_invalid_ids_and_pads_empty_groups():
    from oracle import moe_route
    ids = np.array([[0, 5], [-1, 0]], dtype=np.int32)
    counts, offsets, row, bad = moe_route(ids, 3, pad=128)
    assert bad == 2
    assert counts.tolist() == [2, 0, 0]
    assert offsets.tolist() == [0, 128, 128, 128]   # empty groups take no rows
    assert row.tolist() == [0, -1, -1, 1]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_route_unpadded_is_inverse_stable_argsort(seed):
    from oracle import moe_route
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, 7, size=(50, 3)).astype(np.int32)
    counts, offsets, row, bad = moe_route(ids, 7, pad=1)
    order = np.argsort(ids.reshape(-1), kind="stable")      # entries sorted by expert, ties in entry order
    inv = np.empty_like(order)
    inv[order] = np.arange(order.size)
    assert np.array_equal(row, inv)
    assert np.array_equal(counts, np.bincount(ids.reshape(-1), minlength=7))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))


def test_route_padded_invariants():
    from oracle import moe_route
    ids = mx_inputs.topk_ids(300, 8, 32, seed=5)
    counts, offsets, row, bad = moe_route(ids, 32, pad=128)
    flat = ids.reshape(-1)
    assert bad == 0
    assert np.all(offsets % 128 == 0)
    gaps = np.diff(offsets) - counts
    assert np.all((gaps >= 0) & (gaps < 128))
    assert len(np.unique(row)) == row.size
    for e in range(32):
        rs = row[flat == e]
        assert np.array_equal(rs, np.arange(offsets[e], offsets[e] + counts[e]))  # entry order, no holes


def test_dispatch_worked_example_and_padding():
    from oracle import moe_dispatch, moe_route
    # token 0: 64 ones (two blocks), token 1: ones times 2^3
    x = torch.ones(2, 64, dtype=torch.bfloat16)
    x[1] *= 8
    ids = np.array([[1, 0], [1, 1]], dtype=np.int32)   # token 1 twice to expert 1 (duplicates are kept)
    counts, offsets, row, _ = moe_route(ids, 2, pad=4)
    assert offsets.tolist() == [0, 4, 8]
    q, sf = moe_dispatch(x, row, 2, int(offsets[-1]))
    # 32 ones -> scale code 0x77 (2^-8), elements 0x78 (256): the worked example
    assert q[row[1]].tolist() == [0x78] * 64 and sf[row[1]].tolist() == [0x77, 0x77]
    # x 8 = 2^3 -> scale code 0x7A, same elements
    for r in (row[2], row[3]):
        assert q[r].tolist() == [0x78] * 64 and sf[r].tolist() == [0x7A, 0x7A]
    used = set(row.tolist())
    for r in range(int(offsets[-1])):
        if r not in used:                       # padding rows are zero rows
            assert not q[r].any() and not sf[r].any()


def test_dispatch_dequantises_to_its_token():
    from oracle import e4m3_table, moe_dispatch, moe_route
    x = mx_inputs.outlier_bf16((40, 256), seed=9)
    ids = mx_inputs.topk_ids(40, 4, 6, seed=10)
    counts, offsets, row, _ = moe_route(ids, 6, pad=128)
    q, sf = moe_dispatch(x, row, 4, int(offsets[-1]))
    tab = e4m3_table()
    xf = x.float().numpy().astype(np.float64)
    for t in range(40):
        for j in range(4):
            r = row[t * 4 + j]
            scale = np.exp2(sf[r].astype(np.float64) - 127.0).repeat(32)
            deq = tab[q[r]] * scale
            # E4M3 keeps 3 mantissa bits: error <= 2^-4 |x| for normal codes,
            # half the subnormal step 2^-10 * scale below them, and the
            # saturation of scaled values in (448, 512) to 448
            ax = np.abs(xf[t])
            err = np.abs(deq - xf[t])
            bound = ax * 2.0 ** -4 + scale * 2.0 ** -10 + np.maximum(ax - 448.0 * scale, 0.0)
            assert np.all(err <= bound), (t, j)


def test_combine_one_hot_and_einsum():
    from oracle import moe_combine
    rng = np.random.default_rng(3)
    y = torch.from_numpy(rng.standard_normal((12, 40)).astype(np.float32)).to(torch.bfloat16)
    row = rng.permutation(12)[:10].astype(np.int32).reshape(5, 2)
    # one-hot weights select one routed row exactly
    w = np.zeros((5, 2), dtype=np.float32)
    w[:, 1] = 1.0
    out, _ = moe_combine(y, row, w)
    yf = y.float().numpy().astype(np.float64)
    assert np.array_equal(out, yf[row[:, 1]])
    # general weights: an fp64 einsum over the gathered rows
    w = rng.random((5, 2)).astype(np.float32)
    out, absd = moe_combine(y, row, w)
    ref = np.einsum("tj,tjn->tn", w.astype(np.float64), yf[row])
    assert np.allclose(out, ref, rtol=1e-15, atol=0)
    assert np.allclose(absd, np.einsum("tj,tjn->tn", np.abs(w.astype(np.float64)), np.abs(yf[row])), rtol=1e-15)
    # dropped entries (row -1) contribute nothing
    row2 = row.copy()
    row2[:, 0] = -1
    out2, _ = moe_combine(y, row2, w)
    assert np.allclose(out2, w[:, 1:2].astype(np.float64) * yf[row[:, 1]], rtol=1e-15, atol=0)


def test_layer_grouped_rows_match_per_token_dense():
    """Through the plan, row r of the contiguous grouped GEMM is token t's
    row times its expert's weights: the grouped oracle and the dense oracle
    agree on every routed (t, j)."""
    from oracle import gemm, grouped_contiguous, moe_dispatch, moe_route, quantize
    T, topk, E, n, k = 20, 3, 5, 48, 128
    x = mx_inputs.normal_bf16((T, k), 1.0, 11)
    w = mx_inputs.normal_bf16((E, n, k), 0.02, 12)
    qb, sfb = quantize(w)
    qb = qb.reshape(E, n, k)
    sfb = sfb.reshape(E, n, k // 32)
    ids = mx_inputs.topk_ids(T, topk, E, seed=13)
    counts, offsets, row, _ = moe_route(ids, E, pad=128)
    q, sf = moe_dispatch(x, row, topk, int(offsets[-1]))
    d, _ = grouped_contiguous(q, sf, qb, sfb, offsets)
    qx, sfx = quantize(x)
    for t in range(T):
        for j in range(topk):
            e = int(ids[t, j])
            dt, _ = gemm(qx[t:t + 1], sfx[t:t + 1], qb[e], sfb[e])
            assert np.array_equal(d[row[t * topk + j]], dt[0])


# ---------------------------------------------------------------- expert-parallel placement

def test_peer_plan_hand_example():
    """Two ranks, four experts (rank 0 owns 0-1, rank 1 owns 2-3), pad 2.
    Rank 0's entries have experts 0,3,1,0 and rank 1's 2,0,3,3.  Totals: e0 3
    (rank 0 entries 0, 3, then rank 1 entry 1), e1 1, e2 1, e3 3 (rank 0
    entry 1, then rank 1 entries 2, 3).  Owner 0: e0 rows 0-2 (padded to 4),
    e1 row 4 (padded to 2): offsets 0, 4, 6.  Owner 1: e2 row 0 (padded to
    2), e3 rows 2-4 (padded to 4): offsets 0, 2, 6."""
    from oracle import moe_peer_plan
    per, counts, offsets = moe_peer_plan([np.array([0, 3, 1, 0]), np.array([2, 0, 3, 3])], 4, pad=2)
    assert per[0][0].tolist() == [0, 1, 0, 0] and per[0][1].tolist() == [0, 2, 4, 1]
    assert per[1][0].tolist() == [1, 0, 1, 1] and per[1][1].tolist() == [0, 2, 3, 4]
    assert counts.tolist() == [[3, 1], [1, 3]]
    assert offsets.tolist() == [[0, 4, 6], [0, 2, 6]]


@pytest.mark.parametrize("pad", [1, 128])
def test_peer_plan_one_rank_is_the_routing_plan(pad):
    """With one rank the placement is the single-GPU routing plan."""
    from oracle import moe_peer_plan, moe_route
    ids = mx_inputs.topk_ids(300, 4, 8, seed=81)
    ids[7, 1] = -1
    ids[9, 0] = 8
    per, counts, offsets = moe_peer_plan([ids], 8, pad=pad)
    rc, ro, rr, _ = moe_route(ids, 8, pad=pad)
    assert np.array_equal(per[0][1], rr)
    assert np.array_equal(per[0][0], np.where(rr >= 0, 0, -1))
    assert np.array_equal(counts[0], rc) and np.array_equal(offsets[0], ro)


@pytest.mark.parametrize("ranks,experts", [(2, 8), (3, 6), (4, 32)])
def test_peer_plan_is_the_owners_routing_plan(ranks, experts):
    """On every owner, the rows are those the single-GPU routing plan gives
    to the owner's experts over all ranks' entries taken rank by rank (the
    entries of other owners' experts dropped), and the plan's counts and
    offsets are that plan's."""
    from oracle import moe_peer_plan, moe_route
    rng = np.random.default_rng(ranks * experts)
    ids_list = [mx_inputs.topk_ids(int(rng.integers(0, 200)), 4, experts, seed=90 + r) for r in range(ranks)]
    ids_list[0][:3, 0] = -1                       # dropped entries
    per, counts, offsets = moe_peer_plan(ids_list, experts, pad=128)
    el = experts // ranks
    allids = np.concatenate([a.reshape(-1) for a in ids_list])
    dr = np.concatenate([p[0] for p in per])
    drow = np.concatenate([p[1] for p in per])
    for o in range(ranks):
        local = np.where((allids >= o * el) & (allids < (o + 1) * el), allids - o * el, -1).astype(np.int32)
        rc, ro, rr, _ = moe_route(local, el, pad=128)
        mine = local >= 0
        assert np.all(dr[mine] == o)
        assert np.array_equal(drow[mine], rr[mine])
        assert np.array_equal(counts[o], rc) and np.array_equal(offsets[o], ro)
    assert np.all((dr == -1) == (allids < 0)) and np.all((drow == -1) == (allids < 0))
