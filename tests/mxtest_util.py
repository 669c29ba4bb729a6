"""Helpers shared by the GPU parity tests: oracle-side reference computation and
the element-wise GEMM tolerance

    |D_gpu - D_ref| <= 1e-2 * sum_k |a_ik * b_jk| + 1e-3

with D_ref the oracle's exact fp64 sum over the dequantised operands."""
import numpy as np
import torch

RTOL_ABS = 1e-2
ATOL = 1e-3


def bf16_bits_np(x: torch.Tensor) -> np.ndarray:
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_quantize(oracle, x: torch.Tensor):
    """(q [rows, k] uint8, sf row-major [rows, k/32]) of a [..., k] BF16 tensor."""
    return oracle.quantize(bf16_bits_np(x.reshape(-1, x.shape[-1])))


def gpu_sf_rowmajor(oracle, sf_tiled: torch.Tensor, groups: int, rows: int, k: int) -> np.ndarray:
    """Undo the tiled scale layout (per group) with the oracle's permutation."""
    t = sf_tiled.detach().cpu().numpy()
    per = oracle.scale_bytes(rows, k)
    parts = [oracle.sf_untile(t[g * per:(g + 1) * per], rows, k) for g in range(groups)]
    return np.concatenate(parts, axis=0)


def assert_gemm_close(d_gpu: np.ndarray, d_ref: np.ndarray, abssum: np.ndarray, what: str = ""):
    d_gpu = np.asarray(d_gpu, dtype=np.float64)
    assert d_gpu.shape == d_ref.shape, (d_gpu.shape, d_ref.shape)
    assert np.all(np.isfinite(d_gpu)), f"{what}: non-finite output"
    err = np.abs(d_gpu - d_ref)
    tol = RTOL_ABS * abssum + ATOL
    bad = err > tol
    if bad.any():
        idx = np.argwhere(bad)[:5]
        msg = "; ".join(f"{tuple(i)} gpu={d_gpu[tuple(i)]:.6g} ref={d_ref[tuple(i)]:.6g} tol={tol[tuple(i)]:.3g}"
                        for i in idx)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance: {msg}")


def to_np_f64(d: torch.Tensor) -> np.ndarray:
    return d.detach().float().cpu().numpy().astype(np.float64)


SENTINEL_BITS = 0x7F7F  # BF16 3.39e38: a pattern no tested product can produce


def sentinel_fill(shape, device="cuda") -> torch.Tensor:
    return torch.full(shape, SENTINEL_BITS, dtype=torch.int16, device=device).view(torch.bfloat16)


def is_sentinel(d: torch.Tensor) -> torch.Tensor:
    return d.contiguous().view(torch.int16) == SENTINEL_BITS
