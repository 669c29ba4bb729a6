"""CPU oracle for MXFP8 quantisation and GEMM -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference arm of ``bench.py`` may import this package.  The product path
(``moe_grouped_gemm_mx_b200``) never imports it, and it never imports the
product path.  The arithmetic lives in ``mx_oracle.c`` (plain C, fp64); this
module only builds that library and marshals numpy arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mx_oracle.c")
_LIB = os.path.join(_HERE, "libmx_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math, OpenMP across rows)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "mx_oracle.h")))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-D_DEFAULT_SOURCE", "-fopenmp", "-shared", "-fPIC",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I32 = ctypes.c_int32
        L.mxo_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.mxo_e4m3_decode.restype = ctypes.c_double
        L.mxo_e4m3_encode.argtypes = [ctypes.c_double]
        L.mxo_e4m3_encode.restype = ctypes.c_uint8
        L.mxo_ue8m0_decode.argtypes = [ctypes.c_uint8]
        L.mxo_ue8m0_decode.restype = ctypes.c_double
        L.mxo_floor_log2.argtypes = [ctypes.c_double]
        L.mxo_floor_log2.restype = ctypes.c_int
        L.mxo_e4m3_table.argtypes = [P]
        L.mxo_e4m3_table.restype = None
        L.mxo_quantize_block.argtypes = [P, P, P]
        L.mxo_quantize_block.restype = None
        L.mxo_quantize.argtypes = [P, I64, I64, P, P]
        L.mxo_quantize.restype = None
        L.mxo_quantize_block_f32.argtypes = [P, P, P]
        L.mxo_quantize_block_f32.restype = None
        L.mxo_quantize_f32.argtypes = [P, I64, I64, P, P]
        L.mxo_quantize_f32.restype = None
        L.mxo_silu.argtypes = [ctypes.c_double]
        L.mxo_silu.restype = ctypes.c_double
        L.mxo_swiglu.argtypes = [P, P, I64, P]
        L.mxo_swiglu.restype = None
        L.mxo_scale_bytes.argtypes = [I64, I64]
        L.mxo_scale_bytes.restype = I64
        L.mxo_sf_offset.argtypes = [I64, I64, I64]
        L.mxo_sf_offset.restype = I64
        L.mxo_sf_tile.argtypes = [P, I64, I64, P]
        L.mxo_sf_tile.restype = None
        L.mxo_sf_untile.argtypes = [P, I64, I64, P]
        L.mxo_sf_untile.restype = None
        L.mxo_gemm.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P, P]
        L.mxo_gemm.restype = None
        L.mxo_grouped_contiguous.argtypes = [P, P, P, P, P, I32, I64, I64, P, I64, P, P]
        L.mxo_grouped_contiguous.restype = None
        L.mxo_grouped_masked.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, I64, P, P]
        L.mxo_grouped_masked.restype = None
        L.mxo_grouped_kgrouped.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, I64, P, P]
        L.mxo_grouped_kgrouped.restype = None
        L.mxo_tw_quantize_rows.argtypes = [P, I64, I64, P, P]
        L.mxo_tw_quantize_rows.restype = None
        L.mxo_tw_quantize_blocks.argtypes = [P, I64, I64, P, P]
        L.mxo_tw_quantize_blocks.restype = None
        L.mxo_tw_gemm.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P, P]
        L.mxo_tw_gemm.restype = None
        L.mxo_moe_route.argtypes = [P, I64, I32, I32, P, P, P]
        L.mxo_moe_route.restype = I64
        L.mxo_moe_peer_plan.argtypes = [P, P, I32, I32, I32, P, P, P, P]
        L.mxo_moe_peer_plan.restype = None
        L.mxo_moe_dispatch.argtypes = [P, I64, I64, P, I64, I64, P, P]
        L.mxo_moe_dispatch.restype = None
        L.mxo_moe_combine.argtypes = [P, I64, P, P, I64, I64, P, P]
        L.mxo_moe_combine.restype = None
        L.mxo_num_threads.argtypes = []
        L.mxo_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _u16(x) -> np.ndarray:
    """Accept a numpy uint16 array or a torch bfloat16 tensor (its raw bits)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # only for turning a bf16 tensor into its bit pattern
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


# ---------------------------------------------------------------- scalars

def e4m3_decode(code: int) -> float:
    return lib().mxo_e4m3_decode(code)


def e4m3_encode(v: float) -> int:
    return lib().mxo_e4m3_encode(v)


def ue8m0_decode(code: int) -> float:
    return lib().mxo_ue8m0_decode(code)


def floor_log2(a: float) -> int:
    return lib().mxo_floor_log2(a)


def e4m3_table() -> np.ndarray:
    out = np.zeros(256, dtype=np.float64)
    lib().mxo_e4m3_table(_p(out))
    return out


# ---------------------------------------------------------------- quantiser

def quantize_block(x_bits: np.ndarray):
    x = _u16(x_bits).reshape(32)
    q = np.zeros(32, dtype=np.uint8)
    s = np.zeros(1, dtype=np.uint8)
    lib().mxo_quantize_block(_p(x), _p(q), _p(s))
    return q, int(s[0])


def quantize(x):
    """BF16 [..., k] -> (q uint8 [rows, k], sf uint8 row-major [rows, k/32]),
    rows = product of the leading dimensions."""
    xb = _u16(x)
    k = xb.shape[-1]
    rows = xb.size // k if k else 0
    assert k % 32 == 0
    q = np.zeros((rows, k), dtype=np.uint8)
    sf = np.zeros((rows, k // 32), dtype=np.uint8)
    lib().mxo_quantize(_p(xb), rows, k, _p(q), _p(sf))
    return q, sf


def quantize_block_f32(x: np.ndarray):
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(32)
    q = np.zeros(32, dtype=np.uint8)
    s = np.zeros(1, dtype=np.uint8)
    lib().mxo_quantize_block_f32(_p(x), _p(q), _p(s))
    return q, int(s[0])


def quantize_f32(x: np.ndarray):
    """FP32 [..., k] -> (q uint8 [rows, k], sf uint8 row-major [rows, k/32]),
    the same scale and rounding rule as ``quantize``."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    k = x.shape[-1]
    rows = x.size // k if k else 0
    assert k % 32 == 0
    q = np.zeros((rows, k), dtype=np.uint8)
    sf = np.zeros((rows, k // 32), dtype=np.uint8)
    lib().mxo_quantize_f32(_p(x), rows, k, _p(q), _p(sf))
    return q, sf


def silu(x: float) -> float:
    return lib().mxo_silu(x)


def swiglu(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """h = silu(g) * u elementwise, fp64."""
    g = np.ascontiguousarray(g, dtype=np.float64)
    u = np.ascontiguousarray(u, dtype=np.float64)
    assert g.shape == u.shape
    h = np.zeros(g.shape, dtype=np.float64)
    lib().mxo_swiglu(_p(g), _p(u), g.size, _p(h))
    return h


def scale_bytes(rows: int, k: int) -> int:
    return lib().mxo_scale_bytes(rows, k)


def sf_offset(r: int, c: int, k: int) -> int:
    return lib().mxo_sf_offset(r, c, k)


def sf_tile(sf_rm: np.ndarray, rows: int, k: int) -> np.ndarray:
    sf_rm = np.ascontiguousarray(sf_rm, dtype=np.uint8)
    out = np.zeros(scale_bytes(rows, k), dtype=np.uint8)
    lib().mxo_sf_tile(_p(sf_rm), rows, k, _p(out))
    return out


def sf_untile(tiled: np.ndarray, rows: int, k: int) -> np.ndarray:
    tiled = np.ascontiguousarray(tiled, dtype=np.uint8)
    out = np.zeros((rows, k // 32), dtype=np.uint8)
    lib().mxo_sf_untile(_p(tiled), rows, k, _p(out))
    return out


# ---------------------------------------------------------------- GEMMs

def gemm(qa, sfa, qb, sfb, rows=None):
    """D = deq(A) * deq(B)^T in fp64 for the listed rows (all if None).

    Returns (d, abssum), both [nrows, n] float64; abssum = sum_k |a*b|."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sfa = np.ascontiguousarray(sfa, dtype=np.uint8)
    sfb = np.ascontiguousarray(sfb, dtype=np.uint8)
    m, k = qa.shape
    n = qb.shape[0]
    ids = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nrows = m if ids is None else len(ids)
    d = np.zeros((nrows, n), dtype=np.float64)
    a = np.zeros((nrows, n), dtype=np.float64)
    lib().mxo_gemm(_p(qa), _p(sfa), _p(qb), _p(sfb), m, n, k, _p(ids), nrows, _p(d), _p(a))
    return d, a


def grouped_contiguous(qa, sfa, qb, sfb, offsets, rows=None):
    """qa [m_total, k], qb [groups, n, k]; offsets int32 [groups+1]."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sfa = np.ascontiguousarray(sfa, dtype=np.uint8)
    sfb = np.ascontiguousarray(sfb, dtype=np.uint8)
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    groups = len(off) - 1
    _, n, k = qb.shape
    ids = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nrows = int(off[-1]) if ids is None else len(ids)
    d = np.zeros((nrows, n), dtype=np.float64)
    a = np.zeros((nrows, n), dtype=np.float64)
    lib().mxo_grouped_contiguous(_p(qa), _p(sfa), _p(qb), _p(sfb), _p(off), groups, n, k,
                                 _p(ids), nrows, _p(d), _p(a))
    return d, a


def grouped_masked(qa, sfa, qb, sfb, masked_m, rows=None):
    """qa [groups, max_m, k], qb [groups, n, k]; rows >= masked_m[e] are NaN.

    Without ``rows`` returns (d, abssum) of shape [groups, max_m, n]; with
    ``rows`` (flat indices e*max_m + r) returns [len(rows), n]."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sfa = np.ascontiguousarray(sfa, dtype=np.uint8)
    sfb = np.ascontiguousarray(sfb, dtype=np.uint8)
    mm = np.ascontiguousarray(masked_m, dtype=np.int32)
    groups, max_m, k = qa.shape
    n = qb.shape[1]
    ids = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nrows = groups * max_m if ids is None else len(ids)
    d = np.zeros((nrows, n), dtype=np.float64)
    a = np.zeros((nrows, n), dtype=np.float64)
    lib().mxo_grouped_masked(_p(qa), _p(sfa), _p(qb), _p(sfb), _p(mm), groups, max_m, n, k,
                             _p(ids), nrows, _p(d), _p(a))
    if ids is None:
        return d.reshape(groups, max_m, n), a.reshape(groups, max_m, n)
    return d, a


def quantize_transposed(x):
    """Quantisation along the ROW dimension of x [..., rows, cols] (blocks of
    32 consecutive rows of one column), returned in the transposed layout:
    by definition the row-wise quantisation of x^T.  For a 3-D x each group
    is transposed on its own: q [groups*cols, rows], sf [groups*cols, rows/32]."""
    xb = _u16(x)
    if xb.ndim == 2:
        xb = xb[None]
    xt = np.ascontiguousarray(np.swapaxes(xb, -1, -2))
    return quantize(xt)


def grouped_kgrouped(qa, sfa, qb, sfb, offsets, rows=None):
    """d[e] = deq(A[:, off[e]:off[e+1]]) * deq(B[:, off[e]:off[e+1]])^T in fp64.

    qa [m, k_total], qb [n, k_total] (the token dimension is the reduction
    dimension), sfa / sfb row-major [., k_total/32]; offsets int32
    [groups+1].  Returns (d, abssum) of shape [groups, m, n], or
    [len(rows), n] for the listed flat indices e*m + i."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sfa = np.ascontiguousarray(sfa, dtype=np.uint8)
    sfb = np.ascontiguousarray(sfb, dtype=np.uint8)
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    groups = len(off) - 1
    m, k_total = qa.shape
    n = qb.shape[0]
    ids = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nrows = groups * m if ids is None else len(ids)
    d = np.zeros((nrows, n), dtype=np.float64)
    a = np.zeros((nrows, n), dtype=np.float64)
    lib().mxo_grouped_kgrouped(_p(qa), _p(sfa), _p(qb), _p(sfb), _p(off), groups, m, n, k_total,
                               _p(ids), nrows, _p(d), _p(a))
    if ids is None:
        return d.reshape(groups, m, n), a.reshape(groups, m, n)
    return d, a


# ---------------------------------------------------------------- tile-wise FP32-scaled FP8

def tw_quantize_rows(x):
    """BF16 [rows, k] -> (q uint8 [rows, k], s float32 [k/128, rows]): one FP32
    scale per row and 128-element K tile."""
    xb = _u16(x)
    rows, k = xb.shape
    assert k % 128 == 0
    q = np.zeros((rows, k), dtype=np.uint8)
    s = np.zeros((k // 128, rows), dtype=np.float32)
    lib().mxo_tw_quantize_rows(_p(xb), rows, k, _p(q), _p(s))
    return q, s


def tw_quantize_blocks(x):
    """BF16 [rows, k] -> (q uint8 [rows, k], s float32 [ceil(rows/128), k/128]):
    one FP32 scale per 128 x 128 block."""
    xb = _u16(x)
    rows, k = xb.shape
    assert k % 128 == 0
    q = np.zeros((rows, k), dtype=np.uint8)
    s = np.zeros(((rows + 127) // 128, k // 128), dtype=np.float32)
    lib().mxo_tw_quantize_blocks(_p(xb), rows, k, _p(q), _p(s))
    return q, s


def tw_gemm(qa, sa, qb, sb, rows=None):
    """D = deq(A) deq(B)^T in fp64 with tile-wise FP32 scales (sa [k/128, m],
    sb [ceil(n/128), k/128]).  Returns (d, abssum) [nrows, n]."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    m, k = qa.shape
    n = qb.shape[0]
    ids = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nrows = m if ids is None else len(ids)
    d = np.zeros((nrows, n), dtype=np.float64)
    a = np.zeros((nrows, n), dtype=np.float64)
    lib().mxo_tw_gemm(_p(qa), _p(sa), _p(qb), _p(sb), m, n, k, _p(ids), nrows, _p(d), _p(a))
    return d, a


# ---------------------------------------------------------------- MoE expert layer

def moe_route(ids, num_experts: int, pad: int = 128):
    """Routing plan of a [T, topk] expert-id table (token-major entries).

    Returns (counts int32 [E], offsets int32 [E+1] padded to ``pad``, row
    int32 [T*topk] (-1 for an id outside [0, E)), dropped entries)."""
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(-1)
    counts = np.zeros(num_experts, dtype=np.int32)
    offsets = np.zeros(num_experts + 1, dtype=np.int32)
    row = np.zeros(ids.size, dtype=np.int32)
    bad = lib().mxo_moe_route(_p(ids), ids.size, num_experts, pad, _p(counts), _p(offsets), _p(row))
    return counts, offsets, row, int(bad)


def moe_peer_plan(ids_list, num_experts: int, pad: int = 128):
    """Expert-parallel placement of every rank's entries (rank r's ids are
    ids_list[r], token-major): on the owner of expert e (rank e // (E/R)), e's
    rows are rank 0's entries in order, then rank 1's, ...; each of the
    owner's groups padded to ``pad``.  Returns ([(dst_rank, dst_row)] per rank,
    counts_local int32 [R, E/R], offsets_local int32 [R, E/R+1])."""
    ranks = len(ids_list)
    flat = [np.ascontiguousarray(a, dtype=np.int32).reshape(-1) for a in ids_list]
    n_of = np.array([a.size for a in flat], dtype=np.int64)
    ids = np.ascontiguousarray(np.concatenate(flat) if flat else np.zeros(0, np.int32), dtype=np.int32)
    el = num_experts // ranks
    dst_rank = np.zeros(ids.size, dtype=np.int32)
    dst_row = np.zeros(ids.size, dtype=np.int32)
    counts = np.zeros((ranks, el), dtype=np.int32)
    offsets = np.zeros((ranks, el + 1), dtype=np.int32)
    lib().mxo_moe_peer_plan(_p(ids), _p(n_of), ranks, num_experts, pad, _p(dst_rank), _p(dst_row), _p(counts),
                            _p(offsets))
    per = []
    pos = 0
    for n in n_of:
        per.append((dst_rank[pos:pos + n], dst_row[pos:pos + n]))
        pos += n
    return per, counts, offsets


def moe_dispatch(x, row, topk: int, m_rows: int):
    """Token rows x BF16 [T, k] -> (q uint8 [m_rows, k], sf uint8 row-major
    [m_rows, k/32]): each token's MXFP8 row at every row it is routed to,
    zero (E4M3 0, scale code 0) elsewhere."""
    xb = _u16(x)
    T, k = xb.shape
    row = np.ascontiguousarray(row, dtype=np.int32).reshape(-1)
    assert row.size == T * topk and k % 32 == 0
    q = np.zeros((m_rows, k), dtype=np.uint8)
    sf = np.zeros((m_rows, k // 32), dtype=np.uint8)
    lib().mxo_moe_dispatch(_p(xb), T, k, _p(row), topk, m_rows, _p(q), _p(sf))
    return q, sf


def moe_combine(y, row, w):
    """out[t] = sum_j w[t, j] * y[row[t, j]] (fp64); y BF16 [*, n], w float32
    [T, topk].  Returns (out, abssum) float64 [T, n]."""
    yb = _u16(y)
    n = yb.shape[-1]
    w = np.ascontiguousarray(w, dtype=np.float32)
    T, topk = w.shape
    row = np.ascontiguousarray(row, dtype=np.int32).reshape(-1)
    assert row.size == T * topk
    out = np.zeros((T, n), dtype=np.float64)
    a = np.zeros((T, n), dtype=np.float64)
    lib().mxo_moe_combine(_p(yb), n, _p(row), _p(w), T, topk, _p(out), _p(a))
    return out, a


def num_threads() -> int:
    return lib().mxo_num_threads()
