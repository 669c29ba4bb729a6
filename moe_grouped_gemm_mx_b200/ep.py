"""Expert parallelism for the MoE expert layer.

Each of W ranks holds E/W experts (rank d owns experts [d*E/W, (d+1)*E/W))
and its own tokens.  One layer:

1. route the rank's (token, expert) entries with pad 1: the send buffer is
   ordered by expert, hence by the rank that owns it;
2. dispatch: quantise every token to MXFP8 once, its row written to each
   send-buffer row it is routed to (row-major scales travel with the row:
   1 + 1/32 bytes per element on the wire instead of BF16's 2);
3. all-to-all of the per-expert row counts, then of the rows and scales;
4. route the received rows by local expert (their order is source rank,
   expert, source order, so a stable plan keeps each source's rows together)
   and scatter them into the padded contiguous grouped layout;
5. fused gate/up GEMM + SwiGLU + MXFP8 requantisation, down GEMM;
6. gather the output rows back into receive order, all-to-all them home,
   and take the gate-weighted sum per token (combine).

This is the role DeepEP plays on the B200 MoE-training page (its DeepEP
section and the glossary entry on all-to-all: tokens are sent to the
experts that process them and the results gathered back), around the
grouped GEMM of that page's MXFP8 expert-layer diagram.  The collectives
are NCCL all-to-alls through torch.distributed; their split sizes need one
device-to-host read of the row counts per exchange.  Every step of the data
path is a library kernel; this module only sequences them (``ops``), and the
few index vectors it builds with torch are bookkeeping over the count table.

``ep_moe_layer_peer`` is the same layer with the exchange fused into the
kernels over peer memory instead of all-to-alls: every rank's receive and
output buffers are mapped on every rank (``PeerBuffers``); after an
all-gather of the per-expert counts, one plan kernel gives each entry its
owner and its row there, the dispatch kernel quantises each token once and
stores its MXFP8 row straight into the owner's receive buffer (NVLink
stores), the owner runs its experts in place, and the combine kernel loads
the expert outputs straight from the owners' buffers (NVLink loads) into the
gate-weighted sum.  Stream-ordered barriers (a one-element all-reduce)
separate the three phases; no kernel waits on another rank.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class LibraryOps:
    """The steps of the layer as calls into the CUDA library.

    Every call ORs its data-dependent errors (bad offsets, rows beyond a
    buffer, indices outside a table) into the int32 device word ``status``;
    ``check()`` reads it back and raises if any step reported one."""

    def __init__(self, mx=None, status: torch.Tensor | None = None):
        if mx is None:
            import moe_grouped_gemm_mx_b200 as mx
        self.mx = mx
        self.status = status

    def max_rows(self, n, experts, pad):
        return self.mx.mx_moe_max_rows(n, experts, pad)

    def route(self, ids, experts, pad):
        counts, offsets, row, _ = self.mx.mx_moe_route(ids.reshape(-1), experts, pad)
        return counts, offsets, row

    def dispatch(self, x, row, topk, counts, offsets, pad, m_rows, row_major):
        return self.mx.mx_moe_dispatch_quant(x, row, topk, counts, offsets, pad, m_rows, sf_row_major=row_major,
                                             dev_status=self.status)

    def scatter(self, q_src, sf_src, dst_row, counts, offsets, pad, m_rows):
        return self.mx.mx_moe_scatter_rows(q_src, sf_src, dst_row, counts, offsets, pad, m_rows,
                                           dev_status=self.status)

    def gate_up_swiglu(self, qa, sfa, q13, sf13, offsets):
        return self.mx.mx_grouped_gemm_contiguous_swiglu_quant(qa, sfa, q13, sf13, offsets, dev_status=self.status)

    def down(self, qh, sfh, q2, sf2, offsets, d=None):
        return self.mx.mx_grouped_gemm_contiguous(qh, sfh, q2, sf2, offsets, d=d, dev_status=self.status)

    def gather(self, src, idx):
        return self.mx.mx_gather_rows(src, idx, dev_status=self.status)

    def combine(self, y, row, w):
        return self.mx.mx_moe_combine(y, row, w, dev_status=self.status)

    def peer_plan(self, ids, row_send, count_table, rank, experts, pad):
        return self.mx.mx_moe_peer_plan(ids, row_send, count_table, rank, experts, pad, dev_status=self.status)

    def dispatch_peer(self, x, dst_rank, dst_row, topk, bufs, counts_l, offsets_l, pad):
        self.mx.mx_moe_dispatch_quant_peer(x, dst_rank, dst_row, topk, bufs.q_ptrs, bufs.sf_ptrs, bufs.m_cap,
                                           bufs.q, bufs.sf, counts_l, offsets_l, pad, dev_status=self.status)

    def combine_peer(self, bufs, n, dst_rank, dst_row, w, out=None):
        return self.mx.mx_moe_combine_peer(bufs.y_ptrs, bufs.m_cap, n, dst_rank, dst_row, w, out=out,
                                           dev_status=self.status)

    def check(self, what: str = "expert layer"):
        """Raise if any call since the last check reported a device error
        (one device-to-host read), then clear the word."""
        if self.status is None:
            return
        v = int(self.status.item())
        if v:
            self.status.zero_()
            raise RuntimeError(f"{what}: device status {v:#x} (bad offsets 0x1, bad mask 0x2, timeout 0x4, "
                               f"index or row outside its buffer 0x8)")


def _default_ops(ops, device):
    """The caller's ops, or library ops with a fresh status word that the
    layer checks before it returns."""
    if ops is not None:
        return ops, False
    return LibraryOps(status=torch.zeros(1, dtype=torch.int32, device=device)), True


def _check_pad(pad: int):
    # the contiguous grouped GEMM takes groups that start on 128-row
    # boundaries, and the routing kernels pad groups to at most 128 rows
    if pad != 128:
        raise ValueError(f"pad must be 128: the grouped GEMM's groups start on 128-row boundaries (got {pad})")


def _all_to_all_rows(src: torch.Tensor, send_rows, recv_rows, group):
    """all_to_all_single of whole rows of a 2-D tensor (split sizes in rows)."""
    out = torch.empty((sum(recv_rows),) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    dist.all_to_all_single(out, src[: sum(send_rows)].contiguous(), list(recv_rows), list(send_rows), group=group)
    return out


def ep_moe_layer(x: torch.Tensor, ids: torch.Tensor, gate_w: torch.Tensor, experts: int,
                 q13, sf13, q2, sf2, group=None, ops=None, pad: int = 128) -> torch.Tensor:
    """One expert-parallel MoE layer on this rank.

    x      BF16 [T, H] this rank's tokens; ids int32 [T, topk] global expert
           ids; gate_w float32 [T, topk].
    q13/sf13, q2/sf2  this rank's E/W experts, quantised: [E/W, 2I, H] and
           [E/W, N, I] E4M3 with per-expert tiled scales.
    pad    rows each local expert's group is padded to: 128 (the grouped
           GEMM's groups start on 128-row boundaries; anything else raises).
    ops    the steps (default: the CUDA library, with a device status word
           that is checked before returning -- a RuntimeError names any
           data-dependent error a kernel reported).
    Returns BF16 [T, N]: sum_j gate_w[t, j] * expert_{ids[t,j]}(x[t])."""
    _check_pad(pad)
    ops, own_status = _default_ops(ops, x.device)
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if experts % world:
        raise ValueError("the experts must divide evenly over the ranks")
    e_loc = experts // world
    T, topk = ids.shape
    H = x.shape[1]
    dev = x.device

    # 1-2: expert-ordered send buffer, one MXFP8 row per (token, expert) entry
    counts, _, row_send = ops.route(ids, experts, 1)
    n_send = T * topk
    q_send, sf_send = ops.dispatch(x, row_send, topk, None, None, 1, ops.max_rows(n_send, experts, 1),
                                   row_major=True)
    sf_send = sf_send.view(-1, H // 32)

    # 3: counts per (destination rank, local expert), then rows and scales
    if world > 1:
        recv_counts = torch.empty_like(counts)
        dist.all_to_all_single(recv_counts, counts, group=group)   # [source rank][local expert]
    else:
        recv_counts = counts
    table = torch.stack([counts.view(world, e_loc), recv_counts.view(world, e_loc)]).cpu()
    send_rows = table[0].sum(1).tolist()
    recv_rows = table[1].sum(1).tolist()
    n_recv = sum(recv_rows)
    if world > 1:
        q_recv = _all_to_all_rows(q_send, send_rows, recv_rows, group)
        sf_recv = _all_to_all_rows(sf_send, send_rows, recv_rows, group)
    else:
        q_recv, sf_recv = q_send[:n_recv], sf_send[:n_recv]

    # 4: local expert of each received row (source-major, then expert), its
    # row in the padded grouped layout, and the scatter
    local_ids = torch.arange(e_loc, dtype=torch.int32).repeat(world)
    ids_recv = torch.repeat_interleave(local_ids, table[1].reshape(-1).long()).to(dev)
    counts_l, offsets_l, dst_row = ops.route(ids_recv, e_loc, pad)
    m_rows = ops.max_rows(n_recv, e_loc, pad)
    qa, sfa = ops.scatter(q_recv.contiguous(), sf_recv.contiguous(), dst_row, counts_l, offsets_l, pad, m_rows)

    # 5: the local experts
    qh, sfh = ops.gate_up_swiglu(qa, sfa, q13, sf13, offsets_l)
    d = ops.down(qh, sfh, q2, sf2, offsets_l)

    # 6: back to the tokens' ranks in receive order, then the weighted sum
    y_back = ops.gather(d, dst_row)
    if world > 1:
        y_home = _all_to_all_rows(y_back, recv_rows, send_rows, group)
    else:
        y_home = y_back
    out = ops.combine(y_home, row_send, gate_w)
    if own_status:
        ops.check("ep_moe_layer")
    return out


# ---------------------------------------------------------------- exchange over peer memory

class PeerBuffers:
    """One rank's buffers for the peer-memory exchange, and device tables of
    every rank's addresses of the same buffers.

    q  uint8 [m_cap, H]: the MXFP8 rows routed to this rank's experts;
    sf uint8: their tiled scales (``scale_bytes(m_cap, H)``);
    y  BF16 [m_cap, N]: this rank's expert outputs, row for row;
    q_ptrs / sf_ptrs / y_ptrs  int64 [ranks] device tensors (rank r's address).
    m_cap must hold the rows of the largest plan any rank receives (at most
    mx_moe_max_rows(ranks * tokens * topk, E / ranks, pad))."""

    def __init__(self, q, sf, y, q_ptrs, sf_ptrs, y_ptrs, rank):
        self.q, self.sf, self.y = q, sf, y
        self.q_ptrs, self.sf_ptrs, self.y_ptrs = q_ptrs, sf_ptrs, y_ptrs
        self.rank = rank
        self.ranks = q_ptrs.numel()
        self.m_cap = q.shape[0]

    @staticmethod
    def _alloc(alloc, m_cap, H, N, device, scale_bytes):
        q = alloc((m_cap, H), torch.uint8, device)
        sf = alloc((scale_bytes(m_cap, H),), torch.uint8, device)
        y = alloc((m_cap, N), torch.bfloat16, device)
        return q, sf, y

    @classmethod
    def emulated(cls, ranks: int, m_cap: int, H: int, N: int, device, mx=None):
        """``ranks`` ranks' buffers on one GPU, one PeerBuffers per emulated
        rank, all sharing the same address tables (the kernels see exactly
        what they would see with each buffer on its own GPU)."""
        if mx is None:
            import moe_grouped_gemm_mx_b200 as mx
        bufs = [cls._alloc(lambda shape, dt, dev: torch.empty(shape, dtype=dt, device=dev), m_cap, H, N, device,
                           mx.scale_bytes) for _ in range(ranks)]
        tables = [torch.tensor([b[i].data_ptr() for b in bufs], dtype=torch.int64, device=device) for i in range(3)]
        return [cls(*bufs[r], *tables, r) for r in range(ranks)]

    @classmethod
    def symmetric(cls, m_cap: int, H: int, N: int, group=None, mx=None):
        """Buffers in torch's symmetric memory, mapped on every rank of
        ``group`` (one process per GPU; peers reached over NVLink)."""
        if mx is None:
            import moe_grouped_gemm_mx_b200 as mx
        import os
        # the kernels use plain peer loads and stores: no NVLink multicast
        # object is needed for these buffers
        os.environ.setdefault("TORCH_SYMM_MEM_DISABLE_MULTICAST", "1")
        import torch.distributed._symmetric_memory as symm
        group = dist.group.WORLD if group is None else group
        device = torch.device("cuda", torch.cuda.current_device())
        bufs = cls._alloc(lambda shape, dt, dev: symm.empty(*shape, dtype=dt, device=dev), m_cap, H, N, device,
                          mx.scale_bytes)
        tables = []
        for b in bufs:
            h = symm.rendezvous(b, group)
            tables.append(torch.tensor(list(h.buffer_ptrs), dtype=torch.int64, device=device))
        return cls(*bufs, *tables, dist.get_rank(group))


def peer_route(ids, experts, ops=None):
    """This rank's entries routed with pad 1: (counts [E], row_send [n]) --
    the row of the count table every rank contributes, and each entry's
    place in expert order (the placement plan's input)."""
    ops = LibraryOps() if ops is None else ops
    counts, _, row_send = ops.route(ids.reshape(-1), experts, 1)
    return counts, row_send


def count_table(counts, group=None):
    """[ranks, experts] table of every rank's per-expert counts (one NCCL
    all-gather; the single row itself with one rank)."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world == 1:
        return counts.view(1, -1)
    if counts.is_cuda:   # NCCL gathers straight into the table
        table = torch.empty((world, counts.numel()), dtype=counts.dtype, device=counts.device)
        dist.all_gather_into_tensor(table, counts, group=group)
        return table
    parts = [torch.empty_like(counts) for _ in range(world)]   # gloo (CPU ranks)
    dist.all_gather(parts, counts, group=group)
    return torch.stack(parts)


def peer_dispatch(x, ids, experts, table, bufs: PeerBuffers, ops=None, pad: int = 128, row_send=None):
    """Phase 1 on one rank: plan this rank's entries against the all-ranks
    count table and store every routed MXFP8 row in its owner's receive
    buffer.  ``row_send``: peer_route's, if already computed.  Returns the
    plan (dst_rank, dst_row, counts_local, offsets_local)."""
    ops = LibraryOps() if ops is None else ops
    T, topk = ids.shape
    flat = ids.reshape(-1)
    if row_send is None:
        _, row_send = peer_route(flat, experts, ops)
    dst_rank, dst_row, counts_l, offsets_l = ops.peer_plan(flat, row_send, table, bufs.rank, experts, pad)
    ops.dispatch_peer(x, dst_rank, dst_row, topk, bufs, counts_l, offsets_l, pad)
    return dst_rank, dst_row, counts_l, offsets_l


def peer_experts(bufs: PeerBuffers, plan, q13, sf13, q2, sf2, ops=None):
    """Phase 2 on one rank: its experts over its receive buffer, the outputs
    left in its output buffer y (row for row)."""
    ops = LibraryOps() if ops is None else ops
    offsets_l = plan[3]
    qh, sfh = ops.gate_up_swiglu(bufs.q, bufs.sf, q13, sf13, offsets_l)
    ops.down(qh, sfh, q2, sf2, offsets_l, d=bufs.y)


def peer_combine(bufs: PeerBuffers, plan, gate_w, n: int, ops=None, out=None):
    """Phase 3 on one rank: the gate-weighted sum of its tokens' expert
    outputs, loaded from their owners' output buffers (into ``out`` if
    given)."""
    ops = LibraryOps() if ops is None else ops
    if out is None:
        return ops.combine_peer(bufs, n, plan[0], plan[1], gate_w)
    return ops.combine_peer(bufs, n, plan[0], plan[1], gate_w, out=out)


def route_counts(ids, experts, ops=None):
    """This rank's entries per global expert (the row of the count table)."""
    return peer_route(ids, experts, ops)[0]


def _stream_barrier(group, device):
    """Every rank's work so far on its current stream is complete before any
    rank's later work on its stream starts (a one-element all-reduce on the
    stream; on CPU ranks, a plain barrier)."""
    t = torch.zeros(1, dtype=torch.int32, device=device)
    dist.all_reduce(t, group=group)


def ep_moe_layer_peer(x: torch.Tensor, ids: torch.Tensor, gate_w: torch.Tensor, experts: int,
                      q13, sf13, q2, sf2, bufs: PeerBuffers, group=None, ops=None, pad: int = 128,
                      check: bool = True, out: torch.Tensor | None = None) -> torch.Tensor:
    """One expert-parallel MoE layer on this rank with the exchange over peer
    memory (arguments as ep_moe_layer; ``bufs`` from PeerBuffers.symmetric).
    With the default ops and ``check`` the layer verifies, before it
    returns, that no kernel reported an error -- in particular that every
    owner's plan fitted its receive buffer (rows beyond bufs.m_cap are
    skipped by the dispatch and reported, and would leave stale expert
    outputs behind): a RuntimeError otherwise.  ``check=False`` skips that
    device-to-host read (the caller reads ``ops.status`` later, e.g. after
    a timed loop).  Returns BF16 [T, N] (``out`` if given)."""
    _check_pad(pad)
    ops, own_status = _default_ops(ops, x.device)
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if experts % world or bufs.ranks != world:
        raise ValueError("the experts must divide evenly over the ranks, one buffer set per rank")
    counts, row_send = peer_route(ids, experts, ops)
    table = count_table(counts, group)
    plan = peer_dispatch(x, ids, experts, table, bufs, ops, pad, row_send=row_send)
    if world > 1:
        _stream_barrier(group, x.device)
    peer_experts(bufs, plan, q13, sf13, q2, sf2, ops)
    if world > 1:
        _stream_barrier(group, x.device)
    out = peer_combine(bufs, plan, gate_w, bufs.y.shape[1], ops, out=out)
    if world > 1:
        _stream_barrier(group, x.device)  # the outputs are read before any rank overwrites its buffers
    if own_status and check:
        ops.check("ep_moe_layer_peer")
    return out


def ep_moe_layer_peer_emulated(xs, ids_list, gate_ws, experts, weights, bufs_list, ops=None, pad: int = 128):
    """The peer-memory layer for R ranks emulated on one GPU: each phase runs
    for every rank before the next phase starts (what the barriers of
    ep_moe_layer_peer guarantee).  weights[r] = (q13, sf13, q2, sf2) of rank
    r's experts.  Returns every rank's output; with the default ops, raises
    if any kernel reported an error."""
    _check_pad(pad)
    ops, own_status = _default_ops(ops, xs[0].device)
    table = torch.stack([route_counts(ids, experts, ops) for ids in ids_list])
    plans = [peer_dispatch(xs[r], ids_list[r], experts, table, bufs_list[r], ops, pad) for r in range(len(xs))]
    for r in range(len(xs)):
        peer_experts(bufs_list[r], plans[r], *weights[r], ops)
    outs = [peer_combine(bufs_list[r], plans[r], gate_ws[r], bufs_list[r].y.shape[1], ops) for r in range(len(xs))]
    if own_status:
        ops.check("ep_moe_layer_peer_emulated")
    return outs
