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
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class LibraryOps:
    """The steps of the layer as calls into the CUDA library."""

    def __init__(self, mx=None):
        if mx is None:
            import moe_grouped_gemm_mx_b200 as mx
        self.mx = mx

    def max_rows(self, n, experts, pad):
        return self.mx.mx_moe_max_rows(n, experts, pad)

    def route(self, ids, experts, pad):
        counts, offsets, row, _ = self.mx.mx_moe_route(ids.reshape(-1), experts, pad)
        return counts, offsets, row

    def dispatch(self, x, row, topk, counts, offsets, pad, m_rows, row_major):
        return self.mx.mx_moe_dispatch_quant(x, row, topk, counts, offsets, pad, m_rows, sf_row_major=row_major)

    def scatter(self, q_src, sf_src, dst_row, counts, offsets, pad, m_rows):
        return self.mx.mx_moe_scatter_rows(q_src, sf_src, dst_row, counts, offsets, pad, m_rows)

    def gate_up_swiglu(self, qa, sfa, q13, sf13, offsets):
        return self.mx.mx_grouped_gemm_contiguous_swiglu_quant(qa, sfa, q13, sf13, offsets)

    def down(self, qh, sfh, q2, sf2, offsets):
        return self.mx.mx_grouped_gemm_contiguous(qh, sfh, q2, sf2, offsets)

    def gather(self, src, idx):
        return self.mx.mx_gather_rows(src, idx)

    def combine(self, y, row, w):
        return self.mx.mx_moe_combine(y, row, w)


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
    Returns BF16 [T, N]: sum_j gate_w[t, j] * expert_{ids[t,j]}(x[t])."""
    ops = LibraryOps() if ops is None else ops
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
    return ops.combine(y_home, row_send, gate_w)
