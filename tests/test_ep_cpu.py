"""Expert parallelism on two and four gloo ranks (CPU): the layer's multi-rank
plumbing (per-expert count exchange, the row all-to-alls with uneven and
empty splits, the receive-side plan, the return path and the combine) gives
exactly the output of the same layer computed in one process over all
tokens and all experts; so does the layer with the exchange over peer
memory (count all-gather, placement, stores into the owners' receive
buffers and loads from their outputs, the barriers between the phases),
with every rank's buffers as shared-memory CPU tensors.  The steps that run as CUDA kernels on a GPU are
replaced by oracle-backed CPU stand-ins (tests/ep_ref_ops.py), identical in
both runs, so any difference is the plumbing's."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))

TOPK, H, I, N = 2, 128, 128, 96


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _problem(case: str, world: int):
    """Per-rank tokens, routing and gate weights, and the global experts (two
    per rank)."""
    sys.path[:0] = [ROOT, TESTS]
    import mx_inputs
    import oracle
    E = 2 * world
    ranks = []
    for r in range(world):
        T = 40 + 13 * r
        x = mx_inputs.normal_bf16((T, H), 1.0, 100 + r)
        ids = mx_inputs.topk_ids(T, TOPK, E, seed=200 + r)
        if case == "skewed":
            if r == 1:
                ids = ids % 2 + 2            # rank 1 sends nothing to rank 0's experts (nor rank 2's, ...)
            ids[3, 1] = -1                   # a dropped entry
        gw = mx_inputs.gate_weights(T, TOPK, seed=300 + r)
        ranks.append((x, ids, gw))
    w13 = mx_inputs.normal_bf16((E, 2 * I, H), 0.05, 400)
    w2 = mx_inputs.normal_bf16((E, N, I), 0.05, 401)
    q13, sf13 = oracle.quantize(w13)
    q2, sf2 = oracle.quantize(w2)
    experts = (q13.reshape(E, 2 * I, H), sf13.reshape(E, 2 * I, H // 32),
               q2.reshape(E, N, I), sf2.reshape(E, N, I // 32))
    return ranks, experts, E


def _rank_main(rank, world, port, case, out):
    import torch.distributed as dist
    sys.path[:0] = [ROOT, TESTS]
    from ep_ref_ops import OracleOps
    from moe_grouped_gemm_mx_b200.ep import ep_moe_layer
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        ranks, (q13, sf13, q2, sf2), E = _problem(case, world)
        x, ids, gw = ranks[rank]
        lo, hi = rank * (E // world), (rank + 1) * (E // world)
        y = ep_moe_layer(x, torch.from_numpy(ids), torch.from_numpy(gw), E,
                         torch.from_numpy(q13[lo:hi].copy()), torch.from_numpy(sf13[lo:hi].copy()),
                         torch.from_numpy(q2[lo:hi].copy()), torch.from_numpy(sf2[lo:hi].copy()),
                         ops=OracleOps())
        out[rank] = y.view(torch.int16).numpy().copy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module", autouse=True)
def _library():
    if not os.path.exists(os.path.join(ROOT, "moe_grouped_gemm_mx_b200", "libmx.so")):
        import __graft_entry__
        __graft_entry__.build()


@pytest.mark.parametrize("world,case", [(2, "uniform"), (2, "skewed"), (4, "skewed")])
def test_ep_ranks_match_one_process(world, case):
    from ep_ref_ops import OracleOps
    from moe_grouped_gemm_mx_b200.ep import ep_moe_layer
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, case, out), nprocs=world, join=True)
    ranks, (q13, sf13, q2, sf2), E = _problem(case, world)
    x = torch.cat([r[0] for r in ranks])
    ids = torch.from_numpy(np.concatenate([r[1] for r in ranks]))
    gw = torch.from_numpy(np.concatenate([r[2] for r in ranks]))
    ref = ep_moe_layer(x, ids, gw, E, torch.from_numpy(q13), torch.from_numpy(sf13), torch.from_numpy(q2),
                       torch.from_numpy(sf2), ops=OracleOps())
    ref_bits = ref.view(torch.int16).numpy()
    t0 = 0
    for r in range(world):
        t1 = t0 + ranks[r][0].shape[0]
        assert np.array_equal(out[r], ref_bits[t0:t1]), f"rank {r}"
        t0 = t1
    assert np.abs(ref.float().numpy()).max() > 0      # the layer produced something


def _rank_main_peer(rank, world, port, case, shared, out):
    import torch.distributed as dist
    sys.path[:0] = [ROOT, TESTS]
    from ep_ref_ops import OracleOps
    from moe_grouped_gemm_mx_b200.ep import PeerBuffers, ep_moe_layer_peer
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        ranks, (q13, sf13, q2, sf2), E = _problem(case, world)
        x, ids, gw = ranks[rank]
        lo, hi = rank * (E // world), (rank + 1) * (E // world)
        q_all, sf_all, y_all = shared
        no_table = torch.zeros(world, dtype=torch.int64)     # the CPU stand-ins index the shared tensors instead
        bufs = PeerBuffers(q_all[rank], sf_all[rank], y_all[rank], no_table, no_table, no_table, rank)
        bufs.peer_q, bufs.peer_sf, bufs.peer_y = q_all, sf_all, y_all
        y = ep_moe_layer_peer(x, torch.from_numpy(ids), torch.from_numpy(gw), E,
                              torch.from_numpy(q13[lo:hi].copy()), torch.from_numpy(sf13[lo:hi].copy()),
                              torch.from_numpy(q2[lo:hi].copy()), torch.from_numpy(sf2[lo:hi].copy()),
                              bufs, ops=OracleOps())
        out[rank] = y.view(torch.int16).numpy().copy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [(2, "uniform"), (2, "skewed"), (4, "skewed")])
def test_ep_peer_ranks_match_one_process(world, case):
    from ep_ref_ops import OracleOps
    from moe_grouped_gemm_mx_b200.ep import ep_moe_layer
    ranks, (q13, sf13, q2, sf2), E = _problem(case, world)
    entries = sum(r[1].size for r in ranks)
    el = E // world
    m_cap = (entries + el * 127 + 127) // 128 * 128
    shared = ([torch.full((m_cap, H), 0xAB, dtype=torch.uint8).share_memory_() for _ in range(world)],
              [torch.full((m_cap, H // 32), 0xCD, dtype=torch.uint8).share_memory_() for _ in range(world)],
              [torch.zeros((m_cap, N), dtype=torch.bfloat16).share_memory_() for _ in range(world)])
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_rank_main_peer, args=(world, port, case, shared, out), nprocs=world, join=True)
    x = torch.cat([r[0] for r in ranks])
    ids = torch.from_numpy(np.concatenate([r[1] for r in ranks]))
    gw = torch.from_numpy(np.concatenate([r[2] for r in ranks]))
    ref = ep_moe_layer(x, ids, gw, E, torch.from_numpy(q13), torch.from_numpy(sf13), torch.from_numpy(q2),
                       torch.from_numpy(sf2), ops=OracleOps())
    ref_bits = ref.view(torch.int16).numpy()
    t0 = 0
    for r in range(world):
        t1 = t0 + ranks[r][0].shape[0]
        assert np.array_equal(out[r], ref_bits[t0:t1]), f"rank {r}"
        t0 = t1


@pytest.mark.parametrize("pad", [1, 64, 256])
def test_ep_layers_reject_pad_off_the_gemm_grid(pad):
    """Both layer forms refuse a pad other than 128 before any work: the
    grouped GEMM takes groups that start on 128-row boundaries, and a plan
    padded otherwise would make it skip every tile."""
    from ep_ref_ops import OracleOps
    from moe_grouped_gemm_mx_b200.ep import PeerBuffers, ep_moe_layer, ep_moe_layer_peer
    ranks, (q13, sf13, q2, sf2), E = _problem("uniform", 1)
    x, ids, gw = ranks[0]
    w = [torch.from_numpy(a) for a in (q13, sf13, q2, sf2)]
    with pytest.raises(ValueError, match="pad"):
        ep_moe_layer(x, torch.from_numpy(ids), torch.from_numpy(gw), E, *w, ops=OracleOps(), pad=pad)
    table = torch.zeros(1, dtype=torch.int64)
    bufs = PeerBuffers(torch.zeros((128, H), dtype=torch.uint8), torch.zeros((128, H // 32), dtype=torch.uint8),
                       torch.zeros((128, N), dtype=torch.bfloat16), table, table, table, 0)
    with pytest.raises(ValueError, match="pad"):
        ep_moe_layer_peer(x, torch.from_numpy(ids), torch.from_numpy(gw), E, *w, bufs, ops=OracleOps(), pad=pad)


# ---------------------------------------------------------------- bench plumbing

BT, BE, BH, BI, BN = 48, 16, 128, 128, 96     # tokens per rank, experts, hidden, intermediate, output


def _rank_main_bench(rank, world, port, shared, out):
    """One rank of `bench.py --workload moe_layer_ep` at toy size: the bench's
    own process-group set-up, rank problem and max-over-ranks timing
    reduction around the peer-memory layer (oracle stand-ins for the
    kernels, shared CPU tensors for the mapped buffers)."""
    sys.path[:0] = [ROOT, TESTS]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    import mx_inputs
    import oracle
    import torch.distributed as dist
    from ep_ref_ops import OracleOps
    from moe_grouped_gemm_mx_b200.ep import PeerBuffers, ep_moe_layer_peer
    w, r, local = bench.dist_init(None)
    try:
        assert (w, r, local) == (world, rank, rank)
        bench.EP_CTX.update(world=w, rank=r, mode="peer")
        x, ids, gw, w13, w2 = bench.ep_rank_problem(mx_inputs, r, w, BT, BE, BH, BI, BN, seed=5)
        el = BE // w
        q13, sf13 = oracle.quantize(w13)
        q2, sf2 = oracle.quantize(w2)
        q_all, sf_all, y_all = shared
        no_table = torch.zeros(w, dtype=torch.int64)
        bufs = PeerBuffers(q_all[r], sf_all[r], y_all[r], no_table, no_table, no_table, r)
        bufs.peer_q, bufs.peer_sf, bufs.peer_y = q_all, sf_all, y_all
        y = ep_moe_layer_peer(x, ids, torch.as_tensor(gw), BE,
                              torch.from_numpy(q13.reshape(el, 2 * BI, BH)),
                              torch.from_numpy(sf13.reshape(el, 2 * BI, BH // 32)),
                              torch.from_numpy(q2.reshape(el, BN, BI)), torch.from_numpy(sf2.reshape(el, BN, BI // 32)),
                              bufs, ops=OracleOps())
        t_max = bench.max_over_ranks(w, 1.0 + r, torch.device("cpu"))
        out[r] = (y.view(torch.int16).numpy().copy(), t_max)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_bench_ep_workload_plumbing():
    """Two gloo ranks through bench.py's moe_layer_ep plumbing: every rank's
    output equals the one-process layer over all ranks' tokens and all
    experts (the ranks' expert shares together are one set of experts), the
    step time is the max over ranks, and the interleaved expert placement
    gives each rank every W-th popularity rank."""
    import bench
    import mx_inputs
    import oracle
    from ep_ref_ops import OracleOps
    from moe_grouped_gemm_mx_b200.ep import ep_moe_layer
    world = 2
    el = BE // world
    assert [bench.ep_expert_label(p, BE, world) // el for p in range(BE)] == [p % world for p in range(BE)]
    entries = world * BT * min(8, BE)
    m_cap = (entries + el * 127 + 127) // 128 * 128
    shared = ([torch.full((m_cap, BH), 0xAB, dtype=torch.uint8).share_memory_() for _ in range(world)],
              [torch.full((m_cap, BH // 32), 0xCD, dtype=torch.uint8).share_memory_() for _ in range(world)],
              [torch.zeros((m_cap, BN), dtype=torch.bfloat16).share_memory_() for _ in range(world)])
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_rank_main_bench, args=(world, port, shared, out), nprocs=world, join=True)
    parts = [bench.ep_rank_problem(mx_inputs, r, world, BT, BE, BH, BI, BN, seed=5) for r in range(world)]
    one = bench.ep_rank_problem(mx_inputs, 0, 1, BT, BE, BH, BI, BN, seed=5)
    w13 = torch.cat([p[3] for p in parts])
    w2 = torch.cat([p[4] for p in parts])
    assert torch.equal(w13.view(torch.int16), one[3].view(torch.int16))   # expert e's weights depend on e only
    q13, sf13 = oracle.quantize(w13)
    q2, sf2 = oracle.quantize(w2)
    x = torch.cat([p[0] for p in parts])
    ids = torch.cat([p[1] for p in parts])
    gw = torch.cat([torch.as_tensor(p[2]) for p in parts])
    ref = ep_moe_layer(x, ids, gw, BE, torch.from_numpy(q13.reshape(BE, 2 * BI, BH)),
                       torch.from_numpy(sf13.reshape(BE, 2 * BI, BH // 32)), torch.from_numpy(q2.reshape(BE, BN, BI)),
                       torch.from_numpy(sf2.reshape(BE, BN, BI // 32)), ops=OracleOps())
    ref_bits = ref.view(torch.int16).numpy()
    for r in range(world):
        y_bits, t_max = out[r]
        assert np.array_equal(y_bits, ref_bits[r * BT:(r + 1) * BT]), f"rank {r}"
        assert t_max == float(world)
    assert np.abs(ref.float().numpy()).max() > 0
