"""CPU stand-ins for the library steps of the expert-parallel MoE layer,
built on the oracle (fp64 GEMMs, exact quantisation), so the layer's
multi-rank plumbing (count exchange, all-to-all splits, row orders, the
return path) can run on gloo ranks without a GPU.  Scales stay row-major
throughout: these ops both produce and consume them."""
import numpy as np
import torch

import oracle


def _np(t):
    return t.detach().cpu().numpy() if isinstance(t, torch.Tensor) else np.asarray(t)


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


class OracleOps:
    def max_rows(self, n, experts, pad):
        return (n + experts * (pad - 1) + 127) // 128 * 128

    def route(self, ids, experts, pad):
        c, o, r, _ = oracle.moe_route(_np(ids).reshape(-1).astype(np.int32), experts, pad)
        return torch.from_numpy(c), torch.from_numpy(o), torch.from_numpy(r)

    def dispatch(self, x, row, topk, counts, offsets, pad, m_rows, row_major):
        q, sf = oracle.moe_dispatch(x, _np(row), topk, m_rows)
        return torch.from_numpy(q), torch.from_numpy(sf.reshape(-1).copy())

    def scatter(self, q_src, sf_src, dst_row, counts, offsets, pad, m_rows):
        q_src, sf_src, dst = _np(q_src), _np(sf_src), _np(dst_row)
        q = np.zeros((m_rows, q_src.shape[1]), dtype=np.uint8)
        sf = np.zeros((m_rows, sf_src.shape[1]), dtype=np.uint8)
        q[dst] = q_src
        sf[dst] = sf_src
        return torch.from_numpy(q), torch.from_numpy(sf)

    def gate_up_swiglu(self, qa, sfa, q13, sf13, offsets):
        off = _np(offsets).astype(np.int32)
        d, _ = oracle.grouped_contiguous(_np(qa), _np(sfa), _np(q13), _np(sf13), off)
        i_dim = d.shape[1] // 2
        h = oracle.swiglu(d[:, :i_dim], d[:, i_dim:]).astype(np.float32)
        qh = np.zeros((qa.shape[0], i_dim), dtype=np.uint8)
        sfh = np.zeros((qa.shape[0], i_dim // 32), dtype=np.uint8)
        if len(h):
            qh[: len(h)], sfh[: len(h)] = oracle.quantize_f32(h)
        return torch.from_numpy(qh), torch.from_numpy(sfh)

    def down(self, qh, sfh, q2, sf2, offsets, d=None):
        off = _np(offsets).astype(np.int32)
        dd, _ = oracle.grouped_contiguous(_np(qh), _np(sfh), _np(q2), _np(sf2), off)
        out = np.zeros((qh.shape[0], dd.shape[1]), dtype=np.float64)
        out[: len(dd)] = dd
        if d is None:
            return _bf16(out)
        d.copy_(_bf16(out))
        return d

    def gather(self, src, idx):
        return src[torch.as_tensor(_np(idx)).long()]

    def combine(self, y, row, w):
        out, _ = oracle.moe_combine(y.contiguous(), _np(row), _np(w))
        return _bf16(out)

    # -- the exchange over peer memory, with every rank's buffers as shared
    # CPU tensors (bufs.peer_q / peer_sf / peer_y, indexed by rank)

    def peer_plan(self, ids, row_send, count_table, rank, experts, pad):
        """The placement from the count table alone (what each rank can
        compute): owner o = e // (E/R); row = padded start of e among o's
        experts + entries of e on the ranks before this one + the entry's
        rank among this rank's entries of e."""
        ids, table = _np(ids).reshape(-1), _np(count_table)
        ranks = table.shape[0]
        el = experts // ranks
        tot = table.sum(0)
        padded = (tot + pad - 1) // pad * pad
        before = table[:rank].sum(0)
        seen = np.zeros(experts, dtype=np.int64)
        dst_rank = np.full(ids.size, -1, dtype=np.int32)
        dst_row = np.full(ids.size, -1, dtype=np.int32)
        for i, e in enumerate(ids):
            if 0 <= e < experts:
                o = e // el
                dst_rank[i] = o
                dst_row[i] = padded[o * el:e].sum() + before[e] + seen[e]
                seen[e] += 1
        mine = slice(rank * el, (rank + 1) * el)
        offsets = np.concatenate([[0], np.cumsum(padded[mine])]).astype(np.int32)
        return (torch.from_numpy(dst_rank), torch.from_numpy(dst_row), torch.from_numpy(tot[mine].astype(np.int32)),
                torch.from_numpy(offsets))

    def dispatch_peer(self, x, dst_rank, dst_row, topk, bufs, counts_l, offsets_l, pad):
        q, sf = oracle.quantize(x)
        for i, (rk, r) in enumerate(zip(_np(dst_rank).tolist(), _np(dst_row).tolist())):
            if r >= 0:
                bufs.peer_q[rk][r] = torch.from_numpy(q[i // topk])
                bufs.peer_sf[rk][r] = torch.from_numpy(sf[i // topk])
        cl, ol = _np(counts_l), _np(offsets_l)
        for l in range(cl.size):                # this rank's own padding rows
            bufs.q[ol[l] + cl[l]:ol[l + 1]] = 0
            bufs.sf[ol[l] + cl[l]:ol[l + 1]] = 0

    def combine_peer(self, bufs, n, dst_rank, dst_row, w, out=None):
        dr, drow = _np(dst_rank).reshape(-1), _np(dst_row).reshape(-1)
        y = torch.zeros((dr.size, n), dtype=torch.bfloat16)
        for i, (rk, r) in enumerate(zip(dr.tolist(), drow.tolist())):
            if r >= 0:
                y[i] = bufs.peer_y[rk][r]
        rows = np.where(drow >= 0, np.arange(dr.size), -1).astype(np.int32)
        res = self.combine(y, rows, w)
        if out is None:
            return res
        out.copy_(res)
        return out
