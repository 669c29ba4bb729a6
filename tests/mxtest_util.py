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


# ---------------------------------------------------------------- fused SwiGLU + MXFP8 output

def e4m3_spacing(vabs_scaled: np.ndarray) -> np.ndarray:
    """Distance between adjacent E4M3 magnitudes around |v'| (already scaled by
    2^-X): 2^(e-3) in the binade [2^e, 2^(e+1)), e >= -6; 2^-9 below 2^-6."""
    v = np.maximum(np.asarray(vabs_scaled, dtype=np.float64), 2.0 ** -6)
    e = np.floor(np.log2(v))
    return np.exp2(np.minimum(e, 8.0) - 3.0)


def check_swiglu_quant(oracle, qh: np.ndarray, sf_rm: np.ndarray, g_ref, u_ref, g_abs, u_abs, what=""):
    """Compare a GPU H = MXFP8(silu(G) * U) with the oracle.

    qh uint8 [rows, i] and sf_rm uint8 [rows, i/32] (un-tiled) from the GPU;
    g_ref/u_ref the oracle's exact fp64 gate/up GEMMs, g_abs/u_abs their
    sum_k |a*b|.  The GPU's G and U may each differ from the exact values by
    the GEMM tolerance 1e-2 * sum|a*b| + 1e-3; that error is carried through
    h = silu(g) * u to first order (|dh/dg| <= |u| * max|silu'| with
    max|silu'| < 1.1, |dh/du| = |silu(g)|), and the requantised value may then
    sit one E4M3 step (at the block's own scale) from the perturbed h.
    Also checked: every block's scale is the one the rule gives for some amax
    within that error of the oracle's amax, every block whose largest element
    scales to [256, 448] shows it as a code >= 0x78, and almost every element
    code equals the oracle's own quantisation of the exact h."""
    rows, i_dim = qh.shape
    h_ref = oracle.swiglu(g_ref, u_ref)
    tol_g = RTOL_ABS * g_abs + ATOL
    tol_u = RTOL_ABS * u_abs + ATOL
    silu_abs = np.abs(oracle.swiglu(g_ref, np.ones_like(g_ref)))
    dh = 1.1 * (np.abs(u_ref) + tol_u) * tol_g + (silu_abs + 1.1 * tol_g) * tol_u
    table = oracle.e4m3_table()
    codes = table[qh]
    assert sf_rm.shape == (rows, i_dim // 32)
    assert np.all(sf_rm != 0xFF), f"{what}: NaN scale in a valid row"
    assert np.all((qh & 0x7F) != 0x7F), f"{what}: NaN element in a valid row"
    X = sf_rm.astype(np.int64) - 127
    Xe = np.repeat(X, 32, axis=1)
    deq = codes * np.exp2(Xe)
    # element bound: one E4M3 step at the GPU's block scale plus the carried GEMM error
    step = e4m3_spacing(np.maximum(np.abs(h_ref) + dh, np.abs(deq)) * np.exp2(-Xe)) * np.exp2(Xe)
    sat = np.maximum(np.abs(h_ref) - 448.0 * np.exp2(Xe), 0.0)  # values in (448, 512) * 2^X saturate
    err = np.abs(deq - h_ref)
    bound = step + dh + sat + 1e-30
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        msg = "; ".join(f"{tuple(j)} gpu={deq[tuple(j)]:.6g} ref={h_ref[tuple(j)]:.6g} bound={bound[tuple(j)]:.3g}"
                        for j in idx)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} H elements outside bound: {msg}")
    # scale: the rule's X for some amax in [amax_ref - dh_blk, amax_ref + dh_blk]
    hb = np.abs(h_ref).reshape(rows, i_dim // 32, 32)
    db = dh.reshape(rows, i_dim // 32, 32)
    amax_hi = (hb + db).max(axis=2)
    amax_lo = np.maximum(hb - db, 0.0).max(axis=2)

    def rule_x(a):
        with np.errstate(divide="ignore"):
            x = np.floor(np.log2(np.where(a > 0, a, 1.0))) - 8
        return np.clip(np.where(a > 0, x, -127), -127, 127)

    ok = (X >= rule_x(amax_lo)) & (X <= rule_x(amax_hi))
    assert ok.all(), f"{what}: {(~ok).sum()} block scales inconsistent with the block amax"
    top = (qh & 0x7F).reshape(rows, i_dim // 32, 32).max(axis=2)
    live = X > -127
    assert np.all(top[live] >= 0x78), f"{what}: a block's largest element is not in [256, 448] after scaling"
    # almost every code matches the oracle's own quantisation of the exact h (as FP32)
    q_ref, s_ref = oracle.quantize_f32(h_ref.astype(np.float32))
    same = (q_ref == qh) & np.repeat(s_ref == sf_rm, 32, axis=1)
    assert same.mean() > 0.97, f"{what}: only {same.mean():.4f} of H codes equal the oracle's"
    return h_ref


def sampled_rows(m_end, n_random, seed=0, tile=128, extra=()):
    """Row indices for a full-size parity check: ``n_random`` distinct random
    rows of [0, m_end), the first and last row of every ``tile``-row block
    (where a tile of the GEMM, and each CTA's half of a pair tile, starts and
    ends), and ``extra``; sorted int64."""
    import numpy as np
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(m_end, min(n_random, m_end), replace=False).tolist())
    for t0 in range(0, m_end, tile):
        rows.update([t0, min(t0 + tile, m_end) - 1])
    rows.update(int(r) for r in extra if 0 <= int(r) < m_end)
    return np.array(sorted(rows), dtype=np.int64)
