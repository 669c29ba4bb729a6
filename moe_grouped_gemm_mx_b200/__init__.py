"""MXFP8 quantisation, dense GEMM and MoE grouped GEMMs on B200 (sm_100a).

A thin ctypes binding over ``libmx.so`` (declared in ``include/mx.h``): it
only checks tensor dtypes/devices, allocates outputs with torch when the
caller does not pass them, and forwards raw device pointers plus the current
CUDA stream.  Every arithmetic step runs in the library's CUDA kernels; there
is no CPU or PyTorch fallback -- if the library is missing, importing this
package raises.

Function names match the C ABI:

    q, sf = mx_quantize_bf16_to_e4m3(x)                 # x: bf16 [..., K] (3-D -> per-group scales)
    d     = mx_gemm(qa, sfa, qb, sfb)                   # D = A B^T, bf16 [M, N]
    d     = mx_grouped_gemm_contiguous(qa, sfa, qb, sfb, group_offsets)
    d     = mx_grouped_gemm_masked(qa, sfa, qb, sfb, masked_m)
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MXError", "lib_path", "scale_bytes", "mx_quantize_bf16_to_e4m3", "mx_quantize_bf16_to_e4m3_multi",
    "mx_gemm",
    "mx_grouped_gemm_contiguous", "mx_grouped_gemm_masked", "mx_gemm_swiglu_quant",
    "mx_grouped_gemm_contiguous_swiglu_quant", "mx_grouped_gemm_masked_swiglu_quant",
    "mx_quantize_bf16_to_e4m3_transposed", "mx_grouped_gemm_kgrouped", "mx_quantize_bf16_to_e4m3_tile1x128",
    "mx_quantize_bf16_to_e4m3_block128x128", "mx_gemm_tilewise", "mx_grouped_gemm_contiguous_tilewise",
    "mx_moe_max_rows", "mx_moe_route", "mx_moe_dispatch_quant", "mx_moe_scatter_rows", "mx_gather_rows",
    "mx_moe_combine", "mx_moe_peer_plan", "mx_moe_dispatch_quant_peer", "mx_moe_combine_peer",
    "read_internal_status", "MX_DEV_BAD_OFFSETS", "MX_DEV_BAD_MASK", "MX_DEV_TIMEOUT", "MX_DEV_BAD_INDEX",
    "C_SYMBOLS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libmx.so")

MX_DEV_BAD_OFFSETS = 0x1
MX_DEV_BAD_MASK = 0x2
MX_DEV_TIMEOUT = 0x4
MX_DEV_BAD_INDEX = 0x8

# every symbol include/mx.h declares
C_SYMBOLS = [
    "mx_status_string", "mx_scale_bytes", "mx_quantize_bf16_to_e4m3",
    "mx_quantize_bf16_to_e4m3_grouped", "mx_quantize_bf16_to_e4m3_multi", "mx_quantize_bf16_to_e4m3_multi_lean",
    "mx_gemm",
    "mx_grouped_gemm_contiguous",
    "mx_grouped_gemm_masked", "mx_read_internal_status", "mx_gemm_swiglu_quant",
    "mx_grouped_gemm_contiguous_swiglu_quant", "mx_grouped_gemm_masked_swiglu_quant",
    "mx_quantize_bf16_to_e4m3_transposed", "mx_grouped_gemm_kgrouped", "mx_quantize_bf16_to_e4m3_tile1x128",
    "mx_quantize_bf16_to_e4m3_block128x128", "mx_gemm_tilewise", "mx_grouped_gemm_contiguous_tilewise",
    "mx_moe_max_rows", "mx_moe_route", "mx_moe_dispatch_quant", "mx_moe_scatter_rows", "mx_gather_rows",
    "mx_moe_combine", "mx_moe_peer_plan", "mx_moe_dispatch_quant_peer", "mx_moe_combine_peer",
    "mx_set_wait_limit_ns", "mx_wait_limit_ns", "mx_gemm_batch",
]

MX_GEMM_BATCH_MAX = 4


class _QuantJob(ctypes.Structure):
    _fields_ = [("x_bf16", ctypes.c_void_p), ("groups", ctypes.c_int64), ("rows", ctypes.c_int64),
                ("k", ctypes.c_int64), ("q_e4m3", ctypes.c_void_p), ("sf_ue8m0", ctypes.c_void_p)]


class _GemmProblem(ctypes.Structure):
    _fields_ = [("qa", ctypes.c_void_p), ("sfa", ctypes.c_void_p), ("qb", ctypes.c_void_p),
                ("sfb", ctypes.c_void_p), ("d_bf16", ctypes.c_void_p), ("m", ctypes.c_int64),
                ("n", ctypes.c_int64), ("k", ctypes.c_int64)]


class MXError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_lib.mx_status_string(status).decode()} ({status})")


def _load():
    if not os.path.exists(lib_path):
        raise ImportError(
            f"moe_grouped_gemm_mx_b200: CUDA library {lib_path} is missing; build it with "
            "`python moe_grouped_gemm_mx_b200/_build.py` (or __graft_entry__.build())")
    L = ctypes.CDLL(lib_path)
    P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    L.mx_status_string.argtypes = [ctypes.c_int]
    L.mx_status_string.restype = ctypes.c_char_p
    L.mx_scale_bytes.argtypes = [I64, I64]
    L.mx_scale_bytes.restype = ctypes.c_size_t
    L.mx_quantize_bf16_to_e4m3.argtypes = [P, I64, I64, P, P, P]
    L.mx_quantize_bf16_to_e4m3.restype = ctypes.c_int
    L.mx_quantize_bf16_to_e4m3_grouped.argtypes = [P, I64, I64, I64, P, P, P]
    L.mx_quantize_bf16_to_e4m3_grouped.restype = ctypes.c_int
    L.mx_quantize_bf16_to_e4m3_multi.argtypes = [ctypes.POINTER(_QuantJob), I32, P]
    L.mx_quantize_bf16_to_e4m3_multi.restype = ctypes.c_int
    L.mx_quantize_bf16_to_e4m3_multi_lean.argtypes = [ctypes.POINTER(_QuantJob), I32, P]
    L.mx_quantize_bf16_to_e4m3_multi_lean.restype = ctypes.c_int
    L.mx_gemm.argtypes = [P, P, P, P, P, I64, I64, I64, P, P]
    L.mx_gemm.restype = ctypes.c_int
    L.mx_grouped_gemm_contiguous.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P]
    L.mx_grouped_gemm_contiguous.restype = ctypes.c_int
    L.mx_grouped_gemm_masked.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P]
    L.mx_grouped_gemm_masked.restype = ctypes.c_int
    L.mx_gemm_swiglu_quant.argtypes = [P, P, P, P, P, P, I64, I64, I64, P, P]
    L.mx_gemm_swiglu_quant.restype = ctypes.c_int
    L.mx_grouped_gemm_contiguous_swiglu_quant.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P, P]
    L.mx_grouped_gemm_contiguous_swiglu_quant.restype = ctypes.c_int
    L.mx_grouped_gemm_masked_swiglu_quant.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P, P]
    L.mx_grouped_gemm_masked_swiglu_quant.restype = ctypes.c_int
    L.mx_quantize_bf16_to_e4m3_transposed.argtypes = [P, I64, I64, I64, P, P, P]
    L.mx_quantize_bf16_to_e4m3_transposed.restype = ctypes.c_int
    L.mx_grouped_gemm_kgrouped.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P]
    L.mx_grouped_gemm_kgrouped.restype = ctypes.c_int
    L.mx_quantize_bf16_to_e4m3_tile1x128.argtypes = [P, I64, I64, P, P, P]
    L.mx_quantize_bf16_to_e4m3_tile1x128.restype = ctypes.c_int
    L.mx_quantize_bf16_to_e4m3_block128x128.argtypes = [P, I64, I64, P, P, P]
    L.mx_quantize_bf16_to_e4m3_block128x128.restype = ctypes.c_int
    L.mx_gemm_tilewise.argtypes = [P, P, P, P, P, I64, I64, I64, P, P]
    L.mx_gemm_tilewise.restype = ctypes.c_int
    L.mx_grouped_gemm_contiguous_tilewise.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P]
    L.mx_grouped_gemm_contiguous_tilewise.restype = ctypes.c_int
    L.mx_moe_max_rows.argtypes = [I64, I32, I32]
    L.mx_moe_max_rows.restype = I64
    L.mx_moe_route.argtypes = [P, I64, I32, I32, P, P, P, P, P]
    L.mx_moe_route.restype = ctypes.c_int
    L.mx_moe_dispatch_quant.argtypes = [P, I64, I64, P, I32, P, P, I32, I32, I64, P, P, I32, P, P]
    L.mx_moe_dispatch_quant.restype = ctypes.c_int
    L.mx_moe_scatter_rows.argtypes = [P, P, I64, I64, P, P, P, I32, I32, I64, P, P, P, P]
    L.mx_moe_scatter_rows.restype = ctypes.c_int
    L.mx_gather_rows.argtypes = [P, I64, I64, P, I64, P, P, P]
    L.mx_gather_rows.restype = ctypes.c_int
    L.mx_moe_combine.argtypes = [P, I64, I64, P, P, I64, I32, P, P, P]
    L.mx_moe_combine.restype = ctypes.c_int
    L.mx_moe_peer_plan.argtypes = [P, P, I64, P, I32, I32, I32, I32, P, P, P, P, P, P]
    L.mx_moe_peer_plan.restype = ctypes.c_int
    L.mx_moe_dispatch_quant_peer.argtypes = [P, I64, I64, P, P, I32, P, P, I32, I64, P, P, P, P, I32, I32, P, P]
    L.mx_moe_dispatch_quant_peer.restype = ctypes.c_int
    L.mx_moe_combine_peer.argtypes = [P, I32, I64, I64, P, P, P, I64, I32, P, P, P]
    L.mx_moe_combine_peer.restype = ctypes.c_int
    L.mx_read_internal_status.argtypes = [ctypes.POINTER(ctypes.c_int32), ctypes.c_int]
    L.mx_read_internal_status.restype = ctypes.c_int
    L.mx_gemm_batch.argtypes = [ctypes.POINTER(_GemmProblem), I32, P, P]
    L.mx_gemm_batch.restype = ctypes.c_int
    L.mx_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    L.mx_set_wait_limit_ns.restype = ctypes.c_int
    L.mx_wait_limit_ns.argtypes = []
    L.mx_wait_limit_ns.restype = ctypes.c_uint64
    return L


_lib = _load()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _check(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _raise(st: int, what: str):
    if st != 0:
        raise MXError(st, what)


def scale_bytes(rows: int, k: int) -> int:
    """Bytes of the tiled UE8M0 scale region of a [rows, k] operand."""
    return int(_lib.mx_scale_bytes(rows, k))


def mx_quantize_bf16_to_e4m3(x: torch.Tensor, q: torch.Tensor | None = None,
                             sf: torch.Tensor | None = None, stream=None):
    """BF16 [rows, K] or [groups, rows, K] -> (q uint8 same shape, sf uint8 tiled).

    For a 3-D input the scales are stored per group (each group a
    ``scale_bytes(rows, K)`` region, back to back)."""
    _check(x, torch.bfloat16, "x")
    if x.dim() not in (2, 3):
        raise ValueError("x must be 2-D [rows, K] or 3-D [groups, rows, K]")
    groups = 1 if x.dim() == 2 else x.shape[0]
    rows, k = x.shape[-2], x.shape[-1]
    if q is None:
        q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(groups * scale_bytes(rows, k), dtype=torch.uint8, device=x.device)
    _check(q, torch.uint8, "q")
    _check(sf, torch.uint8, "sf")
    if q.numel() != x.numel() or sf.numel() < groups * scale_bytes(rows, k):
        raise ValueError("output buffers too small")
    if x.dim() == 2:
        st = _lib.mx_quantize_bf16_to_e4m3(_ptr(x), rows, k, _ptr(q), _ptr(sf), _stream(stream))
    else:
        st = _lib.mx_quantize_bf16_to_e4m3_grouped(_ptr(x), groups, rows, k, _ptr(q), _ptr(sf),
                                                   _stream(stream))
    _raise(st, "mx_quantize_bf16_to_e4m3")
    return q, sf


def mx_quantize_bf16_to_e4m3_multi(xs, outs=None, stream=None, lean=False):
    """Quantise several BF16 tensors ([rows, K] or [groups, rows, K]) in one
    kernel launch.  ``outs`` optionally gives a (q, sf) pair per tensor.
    ``lean`` selects mx_quantize_bf16_to_e4m3_multi_lean (the same bytes from
    a form without shared memory, one CTA per SM, to run beside a GEMM on
    another stream).  Returns the list of (q, sf)."""
    xs = list(xs)
    res = []
    jobs = (_QuantJob * max(1, len(xs)))()
    for i, x in enumerate(xs):
        _check(x, torch.bfloat16, f"xs[{i}]")
        if x.dim() not in (2, 3):
            raise ValueError("each tensor must be 2-D or 3-D")
        groups = 1 if x.dim() == 2 else x.shape[0]
        rows, k = x.shape[-2], x.shape[-1]
        if outs is not None:
            q, sf = outs[i]
        else:
            q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
            sf = torch.empty(groups * scale_bytes(rows, k), dtype=torch.uint8, device=x.device)
        _check(q, torch.uint8, f"q[{i}]")
        _check(sf, torch.uint8, f"sf[{i}]")
        if q.numel() != x.numel() or sf.numel() < groups * scale_bytes(rows, k):
            raise ValueError("output buffers too small")
        jobs[i] = _QuantJob(_ptr(x), groups, rows, k, _ptr(q), _ptr(sf))
        res.append((q, sf))
    name = "mx_quantize_bf16_to_e4m3_multi_lean" if lean else "mx_quantize_bf16_to_e4m3_multi"
    _raise(getattr(_lib, name)(jobs, len(xs), _stream(stream)), name)
    return res


def mx_quantize_bf16_to_e4m3_transposed(x: torch.Tensor, q: torch.Tensor | None = None,
                                        sf: torch.Tensor | None = None, stream=None):
    """Quantise along the ROWS of x ([rows, cols] or [groups, rows, cols] BF16)
    into the transposed layout: q uint8 [cols, rows] / [groups, cols, rows] and
    per-group tiled scales of the [cols, rows] operand."""
    _check(x, torch.bfloat16, "x")
    if x.dim() not in (2, 3):
        raise ValueError("x must be 2-D [rows, cols] or 3-D [groups, rows, cols]")
    groups = 1 if x.dim() == 2 else x.shape[0]
    rows, cols = x.shape[-2], x.shape[-1]
    shape = (cols, rows) if x.dim() == 2 else (groups, cols, rows)
    if q is None:
        q = torch.empty(shape, dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(groups * scale_bytes(cols, rows), dtype=torch.uint8, device=x.device)
    _check(q, torch.uint8, "q")
    _check(sf, torch.uint8, "sf")
    if q.numel() != x.numel() or sf.numel() < groups * scale_bytes(cols, rows):
        raise ValueError("output buffers too small")
    st = _lib.mx_quantize_bf16_to_e4m3_transposed(_ptr(x), groups, rows, cols, _ptr(q), _ptr(sf), _stream(stream))
    _raise(st, "mx_quantize_bf16_to_e4m3_transposed")
    return q, sf


def _status_arg(dev_status):
    if dev_status is None:
        return None
    _check(dev_status, torch.int32, "dev_status")
    return dev_status.data_ptr()


def mx_gemm(qa, sfa, qb, sfb, d: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
            stream=None) -> torch.Tensor:
    """D = deq(A) deq(B)^T, qa uint8 [M, K], qb uint8 [N, K] -> bf16 [M, N]."""
    for t, nm in ((qa, "qa"), (sfa, "sfa"), (qb, "qb"), (sfb, "sfb")):
        _check(t, torch.uint8, nm)
    m, k = qa.shape
    n = qb.shape[0]
    if qb.shape[1] != k:
        raise ValueError("K mismatch")
    if d is None:
        d = torch.empty((m, n), dtype=torch.bfloat16, device=qa.device)
    _check(d, torch.bfloat16, "d")
    st = _lib.mx_gemm(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), _ptr(d), m, n, k,
                      _status_arg(dev_status), _stream(stream))
    _raise(st, "mx_gemm")
    return d


def mx_gemm_batch(problems, outs=None, dev_status: torch.Tensor | None = None, stream=None):
    """Up to MX_GEMM_BATCH_MAX independent dense GEMMs in one launch.
    problems: sequence of (qa, sfa, qb, sfb) as for mx_gemm; outs: optional
    BF16 [M_i, N_i] outputs.  Returns the list of D_i."""
    count = len(problems)
    if not 1 <= count <= MX_GEMM_BATCH_MAX:
        raise ValueError(f"1 to {MX_GEMM_BATCH_MAX} problems per batch")
    arr = (_GemmProblem * count)()
    ds = []
    for i, (qa, sfa, qb, sfb) in enumerate(problems):
        for t, nm in ((qa, "qa"), (sfa, "sfa"), (qb, "qb"), (sfb, "sfb")):
            _check(t, torch.uint8, nm)
        m, k = qa.shape
        n = qb.shape[0]
        if qb.shape[1] != k:
            raise ValueError(f"problem {i}: K mismatch")
        d = outs[i] if outs is not None else torch.empty((m, n), dtype=torch.bfloat16, device=qa.device)
        _check(d, torch.bfloat16, "d")
        if tuple(d.shape) != (m, n):
            raise ValueError(f"problem {i}: D must be [{m}, {n}]")
        arr[i] = _GemmProblem(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), _ptr(d), m, n, k)
        ds.append(d)
    _raise(_lib.mx_gemm_batch(arr, count, _status_arg(dev_status), _stream(stream)), "mx_gemm_batch")
    return ds


def mx_grouped_gemm_contiguous(qa, sfa, qb, sfb, group_offsets: torch.Tensor,
                               d: torch.Tensor | None = None,
                               dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """qa uint8 [M_total, K], qb uint8 [E, N, K], group_offsets int32 [E+1] (device)."""
    for t, nm in ((qa, "qa"), (sfa, "sfa"), (qb, "qb"), (sfb, "sfb")):
        _check(t, torch.uint8, nm)
    _check(group_offsets, torch.int32, "group_offsets")
    m_total, k = qa.shape
    groups, n, kb = qb.shape
    if kb != k or group_offsets.numel() != groups + 1:
        raise ValueError("shape mismatch")
    if d is None:
        d = torch.empty((m_total, n), dtype=torch.bfloat16, device=qa.device)
    _check(d, torch.bfloat16, "d")
    st = _lib.mx_grouped_gemm_contiguous(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), _ptr(group_offsets),
                                         groups, m_total, n, k, _ptr(d), _status_arg(dev_status),
                                         _stream(stream))
    _raise(st, "mx_grouped_gemm_contiguous")
    return d


def mx_grouped_gemm_masked(qa, sfa, qb, sfb, masked_m: torch.Tensor, d: torch.Tensor | None = None,
                           dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """qa uint8 [E, max_m, K], qb uint8 [E, N, K], masked_m int32 [E] (device)."""
    for t, nm in ((qa, "qa"), (sfa, "sfa"), (qb, "qb"), (sfb, "sfb")):
        _check(t, torch.uint8, nm)
    _check(masked_m, torch.int32, "masked_m")
    groups, max_m, k = qa.shape
    g2, n, kb = qb.shape
    if g2 != groups or kb != k or masked_m.numel() != groups:
        raise ValueError("shape mismatch")
    if d is None:
        d = torch.empty((groups, max_m, n), dtype=torch.bfloat16, device=qa.device)
    _check(d, torch.bfloat16, "d")
    st = _lib.mx_grouped_gemm_masked(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), _ptr(masked_m), groups,
                                     max_m, n, k, _ptr(d), _status_arg(dev_status), _stream(stream))
    _raise(st, "mx_grouped_gemm_masked")
    return d


def mx_grouped_gemm_kgrouped(qa, sfa, qb, sfb, group_offsets: torch.Tensor, groups: int | None = None,
                             d: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                             stream=None) -> torch.Tensor:
    """K-grouped MoE GEMM (weight gradient): qa uint8 [M, K_total], qb uint8
    [N, K_total], group_offsets int32 [E+1] along K -> bf16 [E, M, N] with
    D[e] = deq(A[:, off[e]:off[e+1]]) deq(B[:, off[e]:off[e+1]])^T."""
    for t, nm in ((qa, "qa"), (sfa, "sfa"), (qb, "qb"), (sfb, "sfb")):
        _check(t, torch.uint8, nm)
    _check(group_offsets, torch.int32, "group_offsets")
    m, k_total = qa.shape
    n, kb = qb.shape
    if kb != k_total:
        raise ValueError("K mismatch")
    groups = group_offsets.numel() - 1 if groups is None else groups
    if group_offsets.numel() != groups + 1:
        raise ValueError("group_offsets must hold groups + 1 entries")
    if d is None:
        d = torch.empty((groups, m, n), dtype=torch.bfloat16, device=qa.device)
    _check(d, torch.bfloat16, "d")
    st = _lib.mx_grouped_gemm_kgrouped(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), _ptr(group_offsets), groups,
                                       m, n, k_total, _ptr(d), _status_arg(dev_status), _stream(stream))
    _raise(st, "mx_grouped_gemm_kgrouped")
    return d


def _tw_quant(fn, name, x, q, s, scale_shape, stream):
    _check(x, torch.bfloat16, "x")
    if x.dim() != 2:
        raise ValueError("x must be 2-D [rows, K]")
    rows, k = x.shape
    if q is None:
        q = torch.empty((rows, k), dtype=torch.uint8, device=x.device)
    if s is None:
        s = torch.empty(scale_shape, dtype=torch.float32, device=x.device)
    _check(q, torch.uint8, "q")
    _check(s, torch.float32, "scales")
    if q.numel() != x.numel() or s.numel() < int(torch.tensor(scale_shape).prod()):
        raise ValueError("output buffers too small")
    _raise(fn(_ptr(x), rows, k, _ptr(q), _ptr(s), _stream(stream)), name)
    return q, s


def mx_quantize_bf16_to_e4m3_tile1x128(x: torch.Tensor, q=None, s=None, stream=None):
    """BF16 [rows, K] -> (q uint8 [rows, K], s float32 [K/128, rows]): one FP32
    scale per row and 128-element K tile (s = amax/448)."""
    rows, k = x.shape
    return _tw_quant(_lib.mx_quantize_bf16_to_e4m3_tile1x128, "mx_quantize_bf16_to_e4m3_tile1x128", x, q, s,
                     (k // 128, rows), stream)


def mx_quantize_bf16_to_e4m3_block128x128(x: torch.Tensor, q=None, s=None, stream=None):
    """BF16 [rows, K] -> (q uint8 [rows, K], s float32 [ceil(rows/128), K/128]): one
    FP32 scale per 128 x 128 block (s = amax/448)."""
    rows, k = x.shape
    return _tw_quant(_lib.mx_quantize_bf16_to_e4m3_block128x128, "mx_quantize_bf16_to_e4m3_block128x128", x, q, s,
                     ((rows + 127) // 128, k // 128), stream)


def mx_gemm_tilewise(qa, sa, qb, sb, d: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Tile-wise FP32-scaled FP8 GEMM: qa uint8 [M, K] with sa float32 [K/128, M],
    qb uint8 [N, K] with sb float32 [ceil(N/128), K/128] -> bf16 [M, N]."""
    for t, nm in ((qa, "qa"), (qb, "qb")):
        _check(t, torch.uint8, nm)
    for t, nm in ((sa, "sa"), (sb, "sb")):
        _check(t, torch.float32, nm)
    m, k = qa.shape
    n = qb.shape[0]
    if d is None:
        d = torch.empty((m, n), dtype=torch.bfloat16, device=qa.device)
    _check(d, torch.bfloat16, "d")
    _raise(_lib.mx_gemm_tilewise(_ptr(qa), _ptr(sa), _ptr(qb), _ptr(sb), _ptr(d), m, n, k, _status_arg(dev_status),
                                 _stream(stream)), "mx_gemm_tilewise")
    return d


def mx_grouped_gemm_contiguous_tilewise(qa, sa, qb, sb, group_offsets: torch.Tensor, d: torch.Tensor | None = None,
                                        dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Contiguous grouped form: qa [M_total, K], sa [K/128, M_total], qb [E, N, K],
    sb [E, ceil(N/128), K/128], group_offsets int32 [E+1] -> bf16 [M_total, N]."""
    for t, nm in ((qa, "qa"), (qb, "qb")):
        _check(t, torch.uint8, nm)
    for t, nm in ((sa, "sa"), (sb, "sb")):
        _check(t, torch.float32, nm)
    _check(group_offsets, torch.int32, "group_offsets")
    m_total, k = qa.shape
    groups, n, kb = qb.shape
    if kb != k or group_offsets.numel() != groups + 1:
        raise ValueError("shape mismatch")
    if d is None:
        d = torch.empty((m_total, n), dtype=torch.bfloat16, device=qa.device)
    _check(d, torch.bfloat16, "d")
    _raise(_lib.mx_grouped_gemm_contiguous_tilewise(_ptr(qa), _ptr(sa), _ptr(qb), _ptr(sb), _ptr(group_offsets),
                                                    groups, m_total, n, k, _ptr(d), _status_arg(dev_status),
                                                    _stream(stream)), "mx_grouped_gemm_contiguous_tilewise")
    return d


def _swiglu_out(rows_shape, i_dim, groups, rows_per_group, qh, sfh, device):
    if qh is None:
        qh = torch.empty(rows_shape + (i_dim,), dtype=torch.uint8, device=device)
    if sfh is None:
        sfh = torch.empty(groups * scale_bytes(rows_per_group, i_dim), dtype=torch.uint8, device=device)
    _check(qh, torch.uint8, "qh")
    _check(sfh, torch.uint8, "sfh")
    if qh.numel() != int(torch.tensor(rows_shape).prod()) * i_dim or \
            sfh.numel() < groups * scale_bytes(rows_per_group, i_dim):
        raise ValueError("output buffers too small")
    return qh, sfh


def mx_gemm_swiglu_quant(qa, sfa, qb, sfb, qh: torch.Tensor | None = None, sfh: torch.Tensor | None = None,
                         dev_status: torch.Tensor | None = None, stream=None):
    """Fused gate/up GEMM + SwiGLU + MXFP8: qa uint8 [M, K], qb uint8
    [2I, K] = [gate; up] -> (qh uint8 [M, I], sfh tiled scales)."""
    for t, nm in ((qa, "qa"), (sfa, "sfa"), (qb, "qb"), (sfb, "sfb")):
        _check(t, torch.uint8, nm)
    m, k = qa.shape
    n2, kb = qb.shape
    if kb != k or n2 % 2:
        raise ValueError("shape mismatch")
    i_dim = n2 // 2
    qh, sfh = _swiglu_out((m,), i_dim, 1, m, qh, sfh, qa.device)
    st = _lib.mx_gemm_swiglu_quant(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), _ptr(qh), _ptr(sfh), m, i_dim, k,
                                   _status_arg(dev_status), _stream(stream))
    _raise(st, "mx_gemm_swiglu_quant")
    return qh, sfh


def mx_grouped_gemm_contiguous_swiglu_quant(qa, sfa, qb, sfb, group_offsets: torch.Tensor,
                                            qh: torch.Tensor | None = None, sfh: torch.Tensor | None = None,
                                            dev_status: torch.Tensor | None = None, stream=None):
    """Contiguous layout: qa uint8 [M_total, K], qb uint8 [E, 2I, K] ([gate; up]
    per expert), group_offsets int32 [E+1] -> (qh uint8 [M_total, I], sfh)."""
    for t, nm in ((qa, "qa"), (sfa, "sfa"), (qb, "qb"), (sfb, "sfb")):
        _check(t, torch.uint8, nm)
    _check(group_offsets, torch.int32, "group_offsets")
    m_total, k = qa.shape
    groups, n2, kb = qb.shape
    if kb != k or n2 % 2 or group_offsets.numel() != groups + 1:
        raise ValueError("shape mismatch")
    i_dim = n2 // 2
    qh, sfh = _swiglu_out((m_total,), i_dim, 1, m_total, qh, sfh, qa.device)
    st = _lib.mx_grouped_gemm_contiguous_swiglu_quant(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), _ptr(group_offsets),
                                                      groups, m_total, i_dim, k, _ptr(qh), _ptr(sfh),
                                                      _status_arg(dev_status), _stream(stream))
    _raise(st, "mx_grouped_gemm_contiguous_swiglu_quant")
    return qh, sfh


def mx_grouped_gemm_masked_swiglu_quant(qa, sfa, qb, sfb, masked_m: torch.Tensor,
                                        qh: torch.Tensor | None = None, sfh: torch.Tensor | None = None,
                                        dev_status: torch.Tensor | None = None, stream=None):
    """Masked layout: qa uint8 [E, max_m, K], qb uint8 [E, 2I, K], masked_m int32
    [E] -> (qh uint8 [E, max_m, I], sfh with one scale region per expert)."""
    for t, nm in ((qa, "qa"), (sfa, "sfa"), (qb, "qb"), (sfb, "sfb")):
        _check(t, torch.uint8, nm)
    _check(masked_m, torch.int32, "masked_m")
    groups, max_m, k = qa.shape
    g2, n2, kb = qb.shape
    if g2 != groups or kb != k or n2 % 2 or masked_m.numel() != groups:
        raise ValueError("shape mismatch")
    i_dim = n2 // 2
    qh, sfh = _swiglu_out((groups, max_m), i_dim, groups, max_m, qh, sfh, qa.device)
    st = _lib.mx_grouped_gemm_masked_swiglu_quant(_ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), _ptr(masked_m),
                                                  groups, max_m, i_dim, k, _ptr(qh), _ptr(sfh),
                                                  _status_arg(dev_status), _stream(stream))
    _raise(st, "mx_grouped_gemm_masked_swiglu_quant")
    return qh, sfh


# ---------------------------------------------------------------- MoE expert layer

def mx_moe_max_rows(n: int, experts: int, pad: int) -> int:
    """Rows to allocate for the grouped operand of a routing plan of ``n``
    entries (every group padded to ``pad``), rounded up to 128."""
    return int(_lib.mx_moe_max_rows(n, experts, pad))


def mx_moe_route(ids: torch.Tensor, experts: int, pad: int = 128, counts=None, offsets=None, row=None,
                 dropped=None, stream=None):
    """Routing plan of an int32 expert-id table ([tokens, topk] or flat,
    token-major).  Returns (counts [E], offsets [E+1], row [n], dropped [1]),
    int32 device tensors: expert e's rows are its entries in entry order from
    offsets[e], groups padded to ``pad`` rows; row = -1 for an id outside
    [0, experts)."""
    _check(ids, torch.int32, "ids")
    n = ids.numel()
    dev = ids.device
    counts = torch.empty(experts, dtype=torch.int32, device=dev) if counts is None else counts
    offsets = torch.empty(experts + 1, dtype=torch.int32, device=dev) if offsets is None else offsets
    row = torch.empty(n, dtype=torch.int32, device=dev) if row is None else row
    dropped = torch.empty(1, dtype=torch.int32, device=dev) if dropped is None else dropped
    for t, nm, size in ((counts, "counts", experts), (offsets, "offsets", experts + 1), (row, "row", n),
                        (dropped, "dropped", 1)):
        _check(t, torch.int32, nm)
        if t.numel() < size:
            raise ValueError(f"{nm} too small")
    _raise(_lib.mx_moe_route(_ptr(ids), n, experts, pad, _ptr(counts), _ptr(offsets), _ptr(row), _ptr(dropped),
                             _stream(stream)), "mx_moe_route")
    return counts, offsets, row, dropped


def mx_moe_dispatch_quant(x: torch.Tensor, row: torch.Tensor, topk: int, counts: torch.Tensor,
                          offsets: torch.Tensor, pad: int, m_rows: int, q=None, sf=None, sf_row_major=False,
                          dev_status=None, stream=None):
    """Quantise each token of x (BF16 [tokens, K]) once and write its MXFP8
    row at every row it is routed to (``row`` from mx_moe_route).  Returns
    (q uint8 [m_rows, K], sf): sf tiled (the GEMM operand) or row-major
    [m_rows, K/32].  Group padding rows (pad > 1) are zero rows."""
    _check(x, torch.bfloat16, "x")
    _check(row, torch.int32, "row")
    tokens, k = x.shape
    if row.numel() != tokens * topk:
        raise ValueError("row must hold tokens*topk entries")
    experts = counts.numel() if counts is not None else 0
    if counts is not None:
        _check(counts, torch.int32, "counts")
        _check(offsets, torch.int32, "offsets")
    sf_bytes = m_rows * (k // 32) if sf_row_major else scale_bytes(m_rows, k)
    q = torch.empty((m_rows, k), dtype=torch.uint8, device=x.device) if q is None else q
    sf = torch.empty(sf_bytes, dtype=torch.uint8, device=x.device) if sf is None else sf
    _check(q, torch.uint8, "q")
    _check(sf, torch.uint8, "sf")
    if q.numel() < m_rows * k or sf.numel() < sf_bytes:
        raise ValueError("output buffers too small")
    _raise(_lib.mx_moe_dispatch_quant(_ptr(x), tokens, k, _ptr(row), topk, _ptr(counts), _ptr(offsets), experts,
                                      pad, m_rows, _ptr(q), _ptr(sf), 1 if sf_row_major else 0, _ptr(dev_status),
                                      _stream(stream)), "mx_moe_dispatch_quant")
    return q, sf


def mx_moe_scatter_rows(q_src: torch.Tensor, sf_src: torch.Tensor, dst_row: torch.Tensor, counts: torch.Tensor,
                        offsets: torch.Tensor, pad: int, m_rows: int, q=None, sf=None, dev_status=None,
                        stream=None):
    """Place quantised rows (q_src uint8 [n, K], row-major scales sf_src
    [n, K/32]) at dst_row of a grouped operand (q [m_rows, K], tiled sf),
    clearing the group padding rows.  Returns (q, sf)."""
    _check(q_src, torch.uint8, "q_src")
    _check(sf_src, torch.uint8, "sf_src")
    _check(dst_row, torch.int32, "dst_row")
    n, k = q_src.shape
    if dst_row.numel() != n or sf_src.numel() < n * (k // 32):
        raise ValueError("dst_row / sf_src do not match q_src")
    _check(counts, torch.int32, "counts")
    _check(offsets, torch.int32, "offsets")
    q = torch.empty((m_rows, k), dtype=torch.uint8, device=q_src.device) if q is None else q
    sf = torch.empty(scale_bytes(m_rows, k), dtype=torch.uint8, device=q_src.device) if sf is None else sf
    _check(q, torch.uint8, "q")
    _check(sf, torch.uint8, "sf")
    if q.numel() < m_rows * k or sf.numel() < scale_bytes(m_rows, k):
        raise ValueError("output buffers too small")
    _raise(_lib.mx_moe_scatter_rows(_ptr(q_src), _ptr(sf_src), n, k, _ptr(dst_row), _ptr(counts), _ptr(offsets),
                                    counts.numel(), pad, m_rows, _ptr(q), _ptr(sf), _ptr(dev_status),
                                    _stream(stream)), "mx_moe_scatter_rows")
    return q, sf


def mx_gather_rows(src: torch.Tensor, idx: torch.Tensor, out=None, dev_status=None, stream=None):
    """out[i] = src[idx[i]] for the rows of a 2-D contiguous tensor (row size a
    multiple of 16 bytes); an out-of-range index gives a zero row."""
    if src.dim() != 2 or not src.is_contiguous() or src.device.type != "cuda":
        raise ValueError("src must be a contiguous 2-D CUDA tensor")
    _check(idx, torch.int32, "idx")
    n = idx.numel()
    out = torch.empty((n, src.shape[1]), dtype=src.dtype, device=src.device) if out is None else out
    if out.dtype != src.dtype or not out.is_contiguous() or out.shape[1:] != src.shape[1:] or out.shape[0] < n:
        raise ValueError("out does not match src")
    row_bytes = src.shape[1] * src.element_size()
    _raise(_lib.mx_gather_rows(_ptr(src), src.shape[0], row_bytes, _ptr(idx), n, _ptr(out), _ptr(dev_status),
                               _stream(stream)), "mx_gather_rows")
    return out


def mx_moe_combine(y: torch.Tensor, row: torch.Tensor, w: torch.Tensor, out=None, dev_status=None, stream=None):
    """out[t] = sum_j w[t, j] * y[row[t, j]] (FP32 in j order, BF16 out);
    y BF16 [rows, N], w float32 [tokens, topk], row int32 [tokens*topk]."""
    _check(y, torch.bfloat16, "y")
    _check(w, torch.float32, "w")
    _check(row, torch.int32, "row")
    tokens, topk = w.shape
    if row.numel() != tokens * topk:
        raise ValueError("row must hold tokens*topk entries")
    n = y.shape[1]
    out = torch.empty((tokens, n), dtype=torch.bfloat16, device=y.device) if out is None else out
    _check(out, torch.bfloat16, "out")
    if out.numel() < tokens * n:
        raise ValueError("out too small")
    _raise(_lib.mx_moe_combine(_ptr(y), y.shape[0], n, _ptr(row), _ptr(w), tokens, topk, _ptr(out),
                               _ptr(dev_status), _stream(stream)), "mx_moe_combine")
    return out


def _ptr_table(t: torch.Tensor, ranks: int, name: str):
    """A device int64 tensor of ``ranks`` buffer addresses (a peer pointer table)."""
    if t.dtype != torch.int64 or t.device.type != "cuda" or not t.is_contiguous() or t.numel() != ranks:
        raise ValueError(f"{name} must be a contiguous int64 CUDA tensor of {ranks} addresses")
    return _ptr(t)


def mx_moe_peer_plan(ids: torch.Tensor, row_send: torch.Tensor, count_table: torch.Tensor, rank: int,
                     experts: int, pad: int = 128, dst_rank=None, dst_row=None, counts_local=None,
                     offsets_local=None, dev_status=None, stream=None):
    """Where each of this rank's entries goes under expert parallelism over
    peer memory.  ids int32 [tokens*topk] (global expert ids), row_send the
    row output of mx_moe_route(ids, experts, pad=1), count_table int32
    [ranks, experts] every rank's counts of that route.  Returns (dst_rank,
    dst_row, counts_local [E/R], offsets_local [E/R+1]) int32 device tensors:
    the owner and the row in its receive buffer per entry, and this rank's own
    receive plan (group offsets of its local experts, padded to ``pad``)."""
    _check(ids, torch.int32, "ids")
    _check(row_send, torch.int32, "row_send")
    _check(count_table, torch.int32, "count_table")
    n = ids.numel()
    ranks = count_table.shape[0]
    if count_table.dim() != 2 or count_table.shape[1] != experts or row_send.numel() != n:
        raise ValueError("count_table must be [ranks, experts] and row_send match ids")
    if experts % ranks:
        raise ValueError("the experts must divide evenly over the ranks")
    el = experts // ranks
    dev = ids.device
    dst_rank = torch.empty(n, dtype=torch.int32, device=dev) if dst_rank is None else dst_rank
    dst_row = torch.empty(n, dtype=torch.int32, device=dev) if dst_row is None else dst_row
    counts_local = torch.empty(el, dtype=torch.int32, device=dev) if counts_local is None else counts_local
    offsets_local = torch.empty(el + 1, dtype=torch.int32, device=dev) if offsets_local is None else offsets_local
    for t, nm, size in ((dst_rank, "dst_rank", n), (dst_row, "dst_row", n), (counts_local, "counts_local", el),
                        (offsets_local, "offsets_local", el + 1)):
        _check(t, torch.int32, nm)
        if t.numel() < size:
            raise ValueError(f"{nm} too small")
    _raise(_lib.mx_moe_peer_plan(_ptr(ids), _ptr(row_send), n, _ptr(count_table), ranks, rank, experts, pad,
                                 _ptr(dst_rank), _ptr(dst_row), _ptr(counts_local), _ptr(offsets_local),
                                 _ptr(dev_status), _stream(stream)), "mx_moe_peer_plan")
    return dst_rank, dst_row, counts_local, offsets_local


def mx_moe_dispatch_quant_peer(x: torch.Tensor, dst_rank: torch.Tensor, dst_row: torch.Tensor, topk: int,
                               q_ptrs: torch.Tensor, sf_ptrs: torch.Tensor, m_rows: int, q_local: torch.Tensor,
                               sf_local: torch.Tensor, counts_local: torch.Tensor, offsets_local: torch.Tensor,
                               pad: int = 128, dev_status=None, stream=None):
    """Quantise each token of x (BF16 [tokens, K]) once and store its MXFP8
    row (tiled scales) at row dst_row of rank dst_rank's receive buffer, the
    buffers given by device address tables q_ptrs / sf_ptrs (int64 [ranks]);
    this rank's own receive buffer (q_local [m_rows, K], sf_local) gets the
    padding rows of its plan cleared."""
    _check(x, torch.bfloat16, "x")
    _check(dst_rank, torch.int32, "dst_rank")
    _check(dst_row, torch.int32, "dst_row")
    _check(q_local, torch.uint8, "q_local")
    _check(sf_local, torch.uint8, "sf_local")
    _check(counts_local, torch.int32, "counts_local")
    _check(offsets_local, torch.int32, "offsets_local")
    tokens, k = x.shape
    ranks = q_ptrs.numel()
    if dst_row.numel() != tokens * topk or dst_rank.numel() != tokens * topk:
        raise ValueError("dst_rank / dst_row must hold tokens*topk entries")
    if q_local.numel() < m_rows * k or sf_local.numel() < scale_bytes(m_rows, k):
        raise ValueError("local receive buffers too small")
    _raise(_lib.mx_moe_dispatch_quant_peer(_ptr(x), tokens, k, _ptr(dst_rank), _ptr(dst_row), topk,
                                           _ptr_table(q_ptrs, ranks, "q_ptrs"), _ptr_table(sf_ptrs, ranks, "sf_ptrs"),
                                           ranks, m_rows, _ptr(q_local), _ptr(sf_local), _ptr(counts_local),
                                           _ptr(offsets_local), counts_local.numel(), pad, _ptr(dev_status),
                                           _stream(stream)), "mx_moe_dispatch_quant_peer")


def mx_moe_combine_peer(y_ptrs: torch.Tensor, y_rows: int, n: int, src_rank: torch.Tensor, src_row: torch.Tensor,
                        w: torch.Tensor, out=None, dev_status=None, stream=None):
    """out[t] = sum_j w[t, j] * (rank src_rank[t, j]'s output)[src_row[t, j]]
    (FP32 in j order, BF16 out); every rank's output is BF16 [y_rows, n],
    addressed by the device table y_ptrs (int64 [ranks])."""
    _check(w, torch.float32, "w")
    _check(src_rank, torch.int32, "src_rank")
    _check(src_row, torch.int32, "src_row")
    tokens, topk = w.shape
    if src_row.numel() != tokens * topk or src_rank.numel() != tokens * topk:
        raise ValueError("src_rank / src_row must hold tokens*topk entries")
    ranks = y_ptrs.numel()
    out = torch.empty((tokens, n), dtype=torch.bfloat16, device=w.device) if out is None else out
    _check(out, torch.bfloat16, "out")
    if out.numel() < tokens * n:
        raise ValueError("out too small")
    _raise(_lib.mx_moe_combine_peer(_ptr_table(y_ptrs, ranks, "y_ptrs"), ranks, y_rows, n, _ptr(src_rank),
                                    _ptr(src_row), _ptr(w), tokens, topk, _ptr(out), _ptr(dev_status),
                                    _stream(stream)), "mx_moe_combine_peer")
    return out


def read_internal_status(clear: bool = True) -> int:
    """Device-status bits accumulated by calls made without ``dev_status``."""
    out = ctypes.c_int32(0)
    _raise(_lib.mx_read_internal_status(ctypes.byref(out), int(clear)), "mx_read_internal_status")
    return int(out.value)


def mx_set_wait_limit_ns(ns: int) -> None:
    """Bound, in nanoseconds, of every wait inside the GEMM kernels launched
    from now on (0 restores the default of 2 s).  A wait that runs longer
    makes the kernel give up cleanly and set MX_DEV_TIMEOUT; a limit below a
    kernel's legitimate waits is how that failure path is exercised."""
    _raise(_lib.mx_set_wait_limit_ns(int(ns)), "mx_set_wait_limit_ns")


def mx_wait_limit_ns() -> int:
    """The current wait bound in nanoseconds."""
    return int(_lib.mx_wait_limit_ns())
