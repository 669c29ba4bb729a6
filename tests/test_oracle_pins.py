"""Pins for the CPU oracle: each check ties the oracle to something other than
itself -- hand-derived golden blocks, torch's own float8_e4m3fn codec, the
BF16 bit layout, closed forms, invariants and brute force on tiny inputs.

No GPU is needed; these run in the CPU suite.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "blocks.txt")


def _expand(items):
    out = []
    i = 0
    while i < len(items):
        tok = items[i]
        if i + 1 < len(items) and items[i + 1].startswith("x") and items[i + 1][1:].isdigit():
            out.extend([tok] * int(items[i + 1][1:]))
            i += 2
        else:
            out.append(tok)
            i += 1
    return out


def load_golden_blocks():
    cases, cur = [], None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, val = line.partition(":")
        val = val.strip()
        if key == "case":
            cur = {"name": val}
            cases.append(cur)
        elif key == "input":
            cur["input"] = [float(t) for t in _expand(val.split())]
        elif key == "scale":
            cur["scale"] = int(val, 16)
        elif key == "codes":
            cur["codes"] = [int(t, 16) for t in _expand(val.split())]
    for c in cases:
        assert len(c["input"]) == 32 and len(c["codes"]) == 32, c["name"]
    return cases


def bf16_bits(values):
    t = torch.tensor(values, dtype=torch.float64).to(torch.bfloat16)
    assert torch.equal(t.double().isnan(), torch.tensor(values, dtype=torch.float64).isnan())
    return t.view(torch.int16).numpy().view(np.uint16)


def all_bf16():
    """Every BF16 bit pattern as (uint16 bits, float64 values)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    return bits, vals


# ---------------------------------------------------------------- E4M3 table

def test_e4m3_table_matches_torch_float8(oracle):
    tab = oracle.e4m3_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(tab), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(tab[fin], ref[fin])
    assert np.array_equal(np.signbit(tab[fin]), np.signbit(ref[fin]))


def test_e4m3_table_landmarks(oracle):
    tab = oracle.e4m3_table()
    assert tab[0x7E] == 448.0
    assert tab[0x78] == 256.0
    assert tab[0x01] == 2.0 ** -9
    assert tab[0x08] == 2.0 ** -6          # smallest normal
    assert tab[0x07] == 7 * 2.0 ** -9      # largest subnormal
    assert tab[0x80] == 0.0 and math.copysign(1.0, tab[0x80]) == -1.0
    assert math.isnan(tab[0x7F]) and math.isnan(tab[0xFF])
    assert np.sum(np.isnan(tab)) == 2
    pos = tab[0x00:0x7F]
    assert np.all(np.diff(pos) > 0)        # strictly increasing 0x00..0x7E
    assert np.array_equal(tab[0x80:0xFF], -pos)


def test_e4m3_roundtrip_all_finite_codes(oracle):
    for c in list(range(0x00, 0x7F)) + list(range(0x80, 0xFF)):
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c, hex(c)


def test_e4m3_encode_matches_torch_cast_exhaustive(oracle):
    """Every BF16 value v, scaled by 2^j for several j, encoded by the oracle
    equals torch's RNE float->float8_e4m3fn cast wherever torch does not
    overflow (|v| <= 464); above that the oracle saturates to +-448."""
    bits, vals = all_bf16()
    fin = np.isfinite(vals)
    for j in (0, -8, 4, 9):
        v = np.ldexp(vals[fin], j)
        ours = np.array([oracle.e4m3_encode(float(x)) for x in v[::7]], dtype=np.uint8)
        vs = v[::7]
        small = np.abs(vs) <= 464.0
        ref = torch.from_numpy(vs[small]).float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(ours[small], ref), f"j={j}"
        big = ~small
        assert np.all(ours[big] == np.where(np.signbit(vs[big]), 0xFE, 0x7E))


def test_e4m3_encode_dense_sweep_against_torch(oracle):
    """Values on a grid finer than the E4M3 spacing over the full range,
    including exact midpoints (ties) between neighbouring codes."""
    tab = oracle.e4m3_table()
    pos = tab[0x00:0x7F]
    mids = (pos[:-1] + pos[1:]) / 2
    grid = np.concatenate([pos, mids, mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20)])
    grid = np.concatenate([grid, -grid])
    ours = np.array([oracle.e4m3_encode(float(x)) for x in grid], dtype=np.uint8)
    ref = torch.from_numpy(grid).float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # float32 conversion of the grid is exact for pos/mids; the +-2^-20 nudges
    # stay on their side of the midpoint in float32 too.
    assert np.array_equal(ours, ref)


# ---------------------------------------------------------------- scale

def test_ue8m0_decode(oracle):
    assert oracle.ue8m0_decode(127) == 1.0
    assert oracle.ue8m0_decode(0) == 2.0 ** -127
    assert oracle.ue8m0_decode(254) == 2.0 ** 127
    assert math.isnan(oracle.ue8m0_decode(255))


def test_floor_log2_matches_bf16_exponent_field(oracle):
    """floor(log2 |v|) for every positive finite BF16 value, against the
    value's own bit fields: exponent-127 for normals, and for subnormals
    (m * 2^-133) the index of m's top bit minus 133."""
    bits, vals = all_bf16()
    sel = (vals > 0) & np.isfinite(vals)
    for b, v in zip(bits[sel][::3], vals[sel][::3]):
        e = (int(b) >> 7) & 0xFF
        m = int(b) & 0x7F
        want = e - 127 if e > 0 else m.bit_length() - 1 - 133
        assert oracle.floor_log2(float(v)) == want, (hex(b), v)


@pytest.mark.parametrize("case", load_golden_blocks(), ids=lambda c: c["name"])
def test_golden_blocks(oracle, case):
    q, s = oracle.quantize_block(bf16_bits(case["input"]))
    assert s == case["scale"]
    assert q.tolist() == case["codes"]


def test_scale_invariance_power_of_two(oracle):
    """Multiplying a block by 2^j (no clamping) keeps every element code and
    shifts the scale code by +j."""
    rng = np.random.default_rng(0)
    for t in range(200):
        x = rng.standard_normal(32) * 2.0 ** rng.integers(-20, 20)
        base = bf16_bits(list(x))
        xb = torch.from_numpy(base.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
        q0, s0 = oracle.quantize_block(base)
        for j in (-30, -5, 1, 7, 40):
            xs = np.ldexp(xb, j)
            if not (1e-30 < np.max(np.abs(xs)) < 1e30):
                continue
            q1, s1 = oracle.quantize_block(bf16_bits(list(xs)))
            if 0 < s0 + j < 255 and s0 != 0:
                assert s1 == s0 + j
                assert np.array_equal(q1, q0)


def test_roundtrip_exactly_representable_blocks(oracle):
    """Blocks built as e4m3(c_i) * 2^X with amax in [256, 448]*2^X quantise
    back to exactly (c_i, X+127)."""
    rng = np.random.default_rng(1)
    tab = oracle.e4m3_table()
    for t in range(300):
        X = int(rng.integers(-100, 100))
        codes = rng.integers(0, 0x7F, size=32).astype(np.uint8)
        codes[rng.integers(0, 32)] = rng.integers(0x78, 0x7F)  # amax in [256, 448]
        signs = rng.integers(0, 2, size=32).astype(np.uint8) << 7
        codes = codes | signs
        vals = np.ldexp(tab[codes], X)
        q, s = oracle.quantize_block(bf16_bits(list(vals)))
        assert s == X + 127
        # -0 and +0 both decode to 0; the sign survives
        assert np.array_equal(q, codes)


def test_dequantised_error_bound(oracle):
    """|deq(q) - v| <= half an E4M3 ulp at v's binade (relative 2^-4), or the
    subnormal spacing 2^(X-10), except for saturated elements."""
    rng = np.random.default_rng(2)
    tab = oracle.e4m3_table()
    x = torch.from_numpy(rng.standard_normal((64, 256)) * 3).to(torch.bfloat16)
    q, sf = oracle.quantize(x)
    v = x.double().numpy()
    deq = tab[q] * np.ldexp(1.0, sf.astype(np.int64) - 127).repeat(32, axis=1)
    X = sf.astype(np.int64).repeat(32, axis=1) - 127
    err = np.abs(deq - v)
    sat = np.abs(v) * np.ldexp(1.0, -X) >= 448
    bound = np.maximum(np.abs(v) * 2.0 ** -4, np.ldexp(1.0, X - 10))
    assert np.all(err[~sat] <= bound[~sat])


# ---------------------------------------------------------------- layout

def test_scale_layout_is_bijection(oracle):
    for rows, k in [(1, 32), (128, 128), (129, 160), (300, 512), (64, 7168)]:
        kb = k // 32
        nbytes = oracle.scale_bytes(rows, k)
        assert nbytes == ((rows + 127) // 128 * 128) * ((kb + 3) // 4 * 4)
        rpad = (rows + 127) // 128 * 128
        kbpad = (kb + 3) // 4 * 4
        offs = {oracle.sf_offset(r, c, k) for r in range(rpad) for c in range(kbpad)}
        assert offs == set(range(nbytes))


def test_scale_layout_tile_geometry(oracle):
    """Inside a 128x4 tile: 4 consecutive K-blocks of one row are 4
    consecutive bytes; rows r, r+32, r+64, r+96 share one 16-byte line."""
    k = 512
    for r in range(128):
        base = oracle.sf_offset(r, 0, k)
        assert [oracle.sf_offset(r, c, k) - base for c in range(4)] == [0, 1, 2, 3]
        assert base // 16 == r % 32
        assert (base % 16) // 4 == r // 32
    assert oracle.sf_offset(0, 4, k) == 512            # next K tile
    assert oracle.sf_offset(128, 0, k) == 512 * 4      # next row block (kb=16 -> 4 K tiles)


def test_scale_tile_untile_roundtrip(oracle):
    rng = np.random.default_rng(3)
    for rows, k in [(1, 32), (130, 96), (256, 512)]:
        sf = rng.integers(0, 256, size=(rows, k // 32)).astype(np.uint8)
        t = oracle.sf_tile(sf, rows, k)
        assert np.array_equal(oracle.sf_untile(t, rows, k), sf)
        mask = np.zeros(t.shape, bool)
        for r in range(rows):
            for c in range(k // 32):
                mask[oracle.sf_offset(r, c, k)] = True
        assert np.all(t[~mask] == 0)


# ---------------------------------------------------------------- GEMM

def _int_block_matrix(rng, rows, k):
    """Integers in [-4, 4] with a +-4 in every 32-block (so X = 2-8 = -6 and
    every element v*64 is an exact E4M3 value)."""
    m = rng.integers(-4, 5, size=(rows, k)).astype(np.float64)
    for c in range(k // 32):
        m[np.arange(rows), c * 32 + rng.integers(0, 32, size=rows)] = 4.0 * rng.choice([-1, 1], size=rows)
    return m


def test_gemm_exact_on_small_integers(oracle):
    rng = np.random.default_rng(4)
    for m, n, k in [(5, 7, 32), (16, 9, 64), (3, 33, 96)]:
        a = _int_block_matrix(rng, m, k)
        b = _int_block_matrix(rng, n, k)
        qa, sfa = oracle.quantize(torch.from_numpy(a).to(torch.bfloat16))
        qb, sfb = oracle.quantize(torch.from_numpy(b).to(torch.bfloat16))
        assert np.all(sfa == 121) and np.all(sfb == 121)
        d, absd = oracle.gemm(qa, sfa, qb, sfb)
        want = a.astype(np.int64) @ b.astype(np.int64).T
        assert np.array_equal(d, want.astype(np.float64))
        assert np.array_equal(absd, (np.abs(a) @ np.abs(b).T))


def test_gemm_identity_and_permutation(oracle):
    rng = np.random.default_rng(5)
    k = 64
    b = torch.from_numpy(rng.standard_normal((10, k))).to(torch.bfloat16)
    qb, sfb = oracle.quantize(b)
    tab = oracle.e4m3_table()
    deq_b = tab[qb] * np.ldexp(1.0, sfb.astype(np.int64) - 127).repeat(32, axis=1)
    perm = rng.permutation(k)[:7]
    a = np.zeros((7, k))
    a[np.arange(7), perm] = 1.0
    qa, sfa = oracle.quantize(torch.from_numpy(a).to(torch.bfloat16))
    d, _ = oracle.gemm(qa, sfa, qb, sfb)
    assert np.array_equal(d, deq_b[:, perm].T)


def test_gemm_matches_torch_matmul_fp64(oracle):
    rng = np.random.default_rng(6)
    m, n, k = 33, 40, 160
    a = torch.from_numpy(rng.standard_normal((m, k)) * 3).to(torch.bfloat16)
    b = torch.from_numpy(rng.standard_normal((n, k)) * 0.02).to(torch.bfloat16)
    qa, sfa = oracle.quantize(a)
    qb, sfb = oracle.quantize(b)
    tab = oracle.e4m3_table()
    da = tab[qa] * np.ldexp(1.0, sfa.astype(np.int64) - 127).repeat(32, axis=1)
    db = tab[qb] * np.ldexp(1.0, sfb.astype(np.int64) - 127).repeat(32, axis=1)
    want = (torch.from_numpy(da) @ torch.from_numpy(db).T).numpy()
    d, absd = oracle.gemm(qa, sfa, qb, sfb)
    assert np.allclose(d, want, rtol=0, atol=1e-12 * np.max(absd))
    # a row subset gives the same rows
    rows = np.array([0, 5, 32])
    d2, _ = oracle.gemm(qa, sfa, qb, sfb, rows=rows)
    assert np.array_equal(d2, d[rows])


def test_gemm_quantisation_error_within_stated_tolerance(oracle):
    """The oracle's MXFP8 product stays within 1e-2*sum|a*b| + 1e-3 of the
    unquantised BF16 product for this data -- a loose sanity pin that a
    wrong scale sign or a dropped 2^X would break by orders of magnitude."""
    rng = np.random.default_rng(7)
    a = torch.from_numpy(rng.standard_normal((20, 256))).to(torch.bfloat16)
    b = torch.from_numpy(rng.standard_normal((24, 256)) * 0.02).to(torch.bfloat16)
    qa, sfa = oracle.quantize(a)
    qb, sfb = oracle.quantize(b)
    d, absd = oracle.gemm(qa, sfa, qb, sfb)
    exact = a.double().numpy() @ b.double().numpy().T
    assert np.all(np.abs(d - exact) <= 0.1 * absd + 1e-3)


# ---------------------------------------------------------------- grouped

def test_grouped_contiguous_equals_dense_per_group(oracle):
    rng = np.random.default_rng(8)
    k, n = 64, 24
    counts = [3, 0, 130, 1]
    off = [0]
    for c in counts:
        off.append(off[-1] + (c + 127) // 128 * 128)
    m_total = off[-1]
    a = torch.from_numpy(rng.standard_normal((m_total, k))).to(torch.bfloat16)
    b = torch.from_numpy(rng.standard_normal((len(counts), n, k)) * 0.02).to(torch.bfloat16)
    qa, sfa = oracle.quantize(a)
    qb, sfb = oracle.quantize(b)
    qb = qb.reshape(len(counts), n, k)
    d, _ = oracle.grouped_contiguous(qa, sfa, qb, sfb, np.array(off, np.int32))
    sfb3 = sfb.reshape(len(counts), n, k // 32)
    for e in range(len(counts)):
        lo, hi = off[e], off[e + 1]
        if hi == lo:
            continue
        de, _ = oracle.gemm(qa[lo:hi], sfa[lo:hi], qb[e], sfb3[e])
        assert np.array_equal(d[lo:hi], de)
    # one group == dense
    d1, _ = oracle.grouped_contiguous(qa[:128], sfa[:128], qb[:1], sfb3[:1].reshape(-1, k // 32),
                                      np.array([0, 128], np.int32))
    dd, _ = oracle.gemm(qa[:128], sfa[:128], qb[0], sfb3[0])
    assert np.array_equal(d1, dd)


def test_grouped_masked_equals_dense_per_group(oracle):
    rng = np.random.default_rng(9)
    E, max_m, n, k = 3, 40, 16, 96
    mm = np.array([0, 40, 7], np.int32)
    a = torch.from_numpy(rng.standard_normal((E, max_m, k))).to(torch.bfloat16)
    b = torch.from_numpy(rng.standard_normal((E, n, k)) * 0.02).to(torch.bfloat16)
    qa, sfa = oracle.quantize(a)
    qb, sfb = oracle.quantize(b)
    qa3, sfa3 = qa.reshape(E, max_m, k), sfa.reshape(E, max_m, k // 32)
    qb3, sfb3 = qb.reshape(E, n, k), sfb.reshape(E, n, k // 32)
    d, _ = oracle.grouped_masked(qa3, sfa, qb3, sfb, mm)
    for e in range(E):
        assert np.all(np.isnan(d[e, mm[e]:]))
        if mm[e]:
            de, _ = oracle.gemm(qa3[e, :mm[e]], sfa3[e, :mm[e]], qb3[e], sfb3[e])
            assert np.array_equal(d[e, :mm[e]], de)


# ---------------------------------------------------------------- SwiGLU and the FP32 quantiser
# (the fused MoE expert MLP: gate/up GEMM -> silu(gate) * up -> MXFP8 -> down GEMM)

@pytest.mark.parametrize("x", [0.1, 0.5, 1.0, 2.5, 7.0, 19.0, 60.0])
def test_silu_odd_part_identity(oracle, x):
    """silu(x) - silu(-x) = x * (sigmoid(x) + sigmoid(-x)) = x exactly."""
    assert oracle.silu(x) - oracle.silu(-x) == pytest.approx(x, rel=1e-15, abs=1e-300)


def test_silu_closed_forms(oracle):
    assert oracle.silu(0.0) == 0.0
    # sigmoid(ln 3) = 3/4
    assert oracle.silu(math.log(3.0)) == pytest.approx(0.75 * math.log(3.0), rel=1e-15)
    # sigmoid(-ln 3) = 1/4
    assert oracle.silu(-math.log(3.0)) == pytest.approx(-0.25 * math.log(3.0), rel=1e-15)
    # saturation: silu(x) -> x for large x, -> 0- for very negative x
    assert oracle.silu(40.0) == pytest.approx(40.0, rel=1e-15)
    assert -1e-15 < oracle.silu(-40.0) < 0.0
    # minimum of silu is about -0.2785 at x about -1.2785 (W(1/e) + 1 solution)
    xs = np.linspace(-3, 0, 30001)
    vals = np.array([oracle.silu(float(v)) for v in xs])
    assert vals.min() == pytest.approx(-0.278464542761074, abs=1e-9)


def test_swiglu_definition(oracle):
    rng = np.random.default_rng(5)
    g = rng.standard_normal(1000) * 3
    u = rng.standard_normal(1000)
    h = oracle.swiglu(g, u)
    # u = 1 gives silu; u = 0 gives zeros; the gate and up roles are not symmetric
    np.testing.assert_array_equal(oracle.swiglu(g, np.ones_like(g)), [oracle.silu(float(v)) for v in g])
    assert not oracle.swiglu(g, np.zeros_like(g)).any()
    assert np.abs(oracle.swiglu(u, g) - h).max() > 0.1
    assert oracle.swiglu(np.array([math.log(3.0)]), np.array([2.0]))[0] == pytest.approx(1.5 * math.log(3.0),
                                                                                        rel=1e-15)


def test_quantize_f32_equals_bf16_quantiser_on_bf16_values(oracle):
    """On values exactly representable in BF16 the FP32 quantiser must give the
    BF16 quantiser's bytes (one rule for both input precisions)."""
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(64, 256, generator=g) * torch.exp2(torch.randint(-20, 20, (64, 1), generator=g).float()))
    x = x.to(torch.bfloat16)
    x[3, 5] = 0.0
    x[7, :32] = 0.0
    x[9, 40] = float("nan")
    x[10, 70] = float("-inf")
    q16, s16 = oracle.quantize(x)
    q32, s32 = oracle.quantize_f32(x.float().numpy())
    np.testing.assert_array_equal(q32, q16)
    np.testing.assert_array_equal(s32, s16)


def test_quantize_f32_keeps_fp32_precision(oracle):
    """A tie at BF16 precision is broken by the extra FP32 bits: with amax 1.75
    (X = -8), 1.0625 scales to 272, exactly between the E4M3 values 256 and
    288, and ties to the even code 0x78; 1.0625 * (1 + 2^-20) scales just above
    the tie and must round up to 0x79.  Both inputs are exact FP32 values."""
    blk = np.full(32, 0.5, dtype=np.float32)
    blk[0] = 1.75
    blk[1] = 1.0625
    blk[2] = np.float32(1.0625 * (1.0 + 2.0 ** -20))
    blk[3] = -np.float32(1.0625 * (1.0 + 2.0 ** -20))
    q, s = oracle.quantize_block_f32(blk)
    assert s == 127 - 8
    assert q[0] == 0x7E  # 1.75 * 256 = 448, the largest finite E4M3 value
    assert q[1] == 0x78
    assert q[2] == 0x79
    assert q[3] == 0xF9


def test_quantize_f32_special_blocks(oracle):
    # FP32 subnormals: amax = 2^-130 < 2^-126 -> X clamps to -127, so values
    # scale by 2^127: 2^-130 -> 2^-3 (code 0x20), 2^-140 -> 2^-13, below half
    # the smallest E4M3 subnormal 2^-9, -> +0
    blk = np.zeros(32, dtype=np.float32)
    blk[0] = np.float32(2.0 ** -130)
    blk[1] = np.float32(2.0 ** -140)
    q, s = oracle.quantize_block_f32(blk)
    assert s == 0
    assert q[0] == 0x20 and oracle.e4m3_decode(0x20) == 2.0 ** -3
    assert q[1] == 0x00
    # non-finite FP32 -> scale 0xFF, elements 0x7F
    blk = np.ones(32, dtype=np.float32)
    blk[31] = np.float32("inf")
    q, s = oracle.quantize_block_f32(blk)
    assert s == 0xFF and (q == 0x7F).all()
    # large FP32 magnitudes: amax = 2^100 -> X = 92
    blk = np.full(32, 2.0 ** 100, dtype=np.float32)
    q, s = oracle.quantize_block_f32(blk)
    assert s == 127 + 92 and (q == 0x78).all()


# ---------------------------------------------------------------- training-side GEMMs
# (quantisation along the token dimension and the K-grouped weight-gradient GEMM)

def test_quantize_transposed_hand_example(oracle):
    """Blocks run down a column: x [64, 3]; column 0 all ones (amax 1 -> X = -8,
    scale 0x77, elements 256 -> 0x78); column 1 = row index r in rows 0..31
    (amax 31 -> X = -4, r*16: 0..496, 31*16 = 496 saturates to 448 = 0x7E)
    and zeros in rows 32..63 (scale 0x00, codes 0x00); column 2 = -2 everywhere
    (X = -7, -256 -> 0xF8).  Output layout: q[c, r] is the code of x[r, c]."""
    x = np.zeros((64, 3), dtype=np.float32)
    x[:, 0] = 1.0
    x[:32, 1] = np.arange(32)
    x[:, 2] = -2.0
    q, sf = oracle.quantize_transposed(torch.from_numpy(x).to(torch.bfloat16))
    assert q.shape == (3, 64) and sf.shape == (3, 2)
    assert list(sf[0]) == [0x77, 0x77] and np.all(q[0] == 0x78)
    assert list(sf[1]) == [127 - 4, 0x00]
    assert q[1, 1] == oracle.e4m3_encode(16.0) and q[1, 31] == 0x7E and q[1, 30] == oracle.e4m3_encode(480.0)
    assert np.all(q[1, 32:] == 0x00)
    assert list(sf[2]) == [127 - 7, 127 - 7] and np.all(q[2] == 0xF8)


def _kgrouped_operands(oracle, rng, m, n, tokens):
    a = _int_block_matrix(rng, m, tokens)   # [m, tokens], blocks of 32 tokens share amax 4
    b = _int_block_matrix(rng, n, tokens)
    qa, sfa = oracle.quantize(torch.from_numpy(a).to(torch.bfloat16))
    qb, sfb = oracle.quantize(torch.from_numpy(b).to(torch.bfloat16))
    return a, b, qa, sfa, qb, sfb


def test_kgrouped_exact_on_small_integers(oracle):
    """Integer operands whose every 32-token block has amax 4 are exact in
    MXFP8, and all partial sums are small integers: each expert's result must
    equal the integer matmul over its own token range."""
    rng = np.random.default_rng(21)
    a, b, qa, sfa, qb, sfb = _kgrouped_operands(oracle, rng, 6, 5, 256)
    off = np.array([0, 64, 64, 96, 256], dtype=np.int32)   # expert 1 has no tokens
    d, absd = oracle.grouped_kgrouped(qa, sfa, qb, sfb, off)
    for e in range(4):
        s0, s1 = off[e], off[e + 1]
        want = a[:, s0:s1].astype(np.int64) @ b[:, s0:s1].astype(np.int64).T
        assert np.array_equal(d[e], want.astype(np.float64)), e
        assert np.array_equal(absd[e], np.abs(a[:, s0:s1]) @ np.abs(b[:, s0:s1]).T)
    assert not d[1].any()


def test_kgrouped_one_group_equals_dense_and_sum_over_groups(oracle):
    g = torch.Generator().manual_seed(5)
    a = torch.randn(40, 384, generator=g).to(torch.bfloat16)
    b = (torch.randn(24, 384, generator=g) * 0.3).to(torch.bfloat16)
    qa, sfa = oracle.quantize(a)
    qb, sfb = oracle.quantize(b)
    dense, dabs = oracle.gemm(qa, sfa, qb, sfb)
    one, oabs = oracle.grouped_kgrouped(qa, sfa, qb, sfb, np.array([0, 384], dtype=np.int32))
    np.testing.assert_array_equal(one[0], dense)
    np.testing.assert_array_equal(oabs[0], dabs)
    # the experts partition the tokens, so their gradients sum to the dense product
    parts, _ = oracle.grouped_kgrouped(qa, sfa, qb, sfb, np.array([0, 128, 160, 160, 384], dtype=np.int32))
    np.testing.assert_allclose(parts.sum(axis=0), dense, rtol=1e-12, atol=1e-12)
    # sampled rows (flat e*m + i) agree with the full result
    ids = np.array([0, 39, 40 + 7, 3 * 40 + 39], dtype=np.int64)
    sub, _ = oracle.grouped_kgrouped(qa, sfa, qb, sfb, np.array([0, 128, 160, 160, 384], dtype=np.int32), rows=ids)
    np.testing.assert_array_equal(sub, parts.reshape(-1, 24)[ids])


# ---------------------------------------------------------------- tile-wise FP32-scaled FP8 (DeepGEMM format)

def test_tw_quantize_power_of_two_scales_are_exact(oracle):
    """amax = 448 * 2^j gives s = 2^j exactly, so every BF16 value that is an
    E4M3 value times 2^j quantises to that E4M3 code."""
    table = oracle.e4m3_table()
    finite = [c for c in range(0x7F) if c not in (0x7F,)]
    rng = np.random.default_rng(3)
    for j in (-10, -3, 0, 4, 20):
        codes = rng.choice(finite, size=128).astype(np.uint8)
        codes[5] = 0x7E                     # amax = 448 * 2^j
        signs = rng.choice([0, 0x80], size=128).astype(np.uint8)
        vals = np.array([table[c] for c in codes]) * 2.0 ** j
        vals = np.where(signs == 0x80, -vals, vals)
        x = torch.from_numpy(vals).to(torch.bfloat16)
        q, s = oracle.tw_quantize_rows(x.reshape(1, 128))
        assert s[0, 0] == np.float32(2.0 ** j)
        want = codes | signs
        want[(codes == 0) & (signs == 0x80)] = 0x80   # -0 keeps its sign
        assert np.array_equal(q[0], want), j


def test_tw_quantize_matches_torch_division_and_cast(oracle):
    """Independent path: FP32 division in torch and torch's own float8_e4m3fn
    cast of the quotient give the oracle's codes; s is amax / 448 in FP32."""
    g = torch.Generator().manual_seed(8)
    x = (torch.randn(64, 512, generator=g) * torch.exp2(torch.randint(-8, 8, (64, 1), generator=g).float())
         ).to(torch.bfloat16)
    q, s = oracle.tw_quantize_rows(x)
    xf = x.float().reshape(64, 4, 128)
    amax = xf.abs().amax(dim=2)
    s_t = amax / torch.tensor(448.0)
    assert np.array_equal(s.T, s_t.numpy())
    codes = (xf / s_t[:, :, None]).to(torch.float8_e4m3fn).view(torch.uint8).reshape(64, 512).numpy()
    assert np.array_equal(q, codes)
    # every tile's largest element lands on +-448
    assert np.all((q.reshape(64, 4, 128) & 0x7F).max(axis=2) == 0x7E)


def test_tw_quantize_blocks_and_special_tiles(oracle):
    g = torch.Generator().manual_seed(9)
    x = torch.randn(200, 256, generator=g).to(torch.bfloat16)   # 2 row blocks (128 + 72) x 2 K tiles
    x[128:, 128:] = 0.0                                         # an all-zero block
    x[3, 7] = float("inf")                                      # a non-finite block
    q, s = oracle.tw_quantize_blocks(x)
    assert s.shape == (2, 2)
    assert np.isnan(s[0, 0]) and np.all(q[:128, :128] == 0x7F)
    assert s[1, 1] == 1.0 and np.all((q[128:, 128:] & 0x7F) == 0)
    blk = x[:128, 128:].float()
    assert s[0, 1] == np.float32(blk.abs().max().item()) / np.float32(448.0)
    assert s[1, 0] == np.float32(x[128:, :128].float().abs().max().item()) / np.float32(448.0)


def test_tw_gemm_equals_mxfp8_gemm_on_power_of_two_scales(oracle):
    """With tile scales that are powers of two the tile-wise dequantisation is
    an MXFP8 dequantisation with the same exponent in every 32-block of the
    tile, so the two oracle GEMMs must agree exactly."""
    rng = np.random.default_rng(12)
    m, n, k = 9, 140, 256
    qa = rng.integers(0, 0x7F, size=(m, k)).astype(np.uint8) | rng.choice([0, 0x80], size=(m, k)).astype(np.uint8)
    qb = rng.integers(0, 0x7F, size=(n, k)).astype(np.uint8)
    ja = rng.integers(-6, 6, size=(k // 128, m))
    jb = rng.integers(-6, 6, size=((n + 127) // 128, k // 128))
    sa = np.exp2(ja).astype(np.float32)
    sb = np.exp2(jb).astype(np.float32)
    d_tw, a_tw = oracle.tw_gemm(qa, sa, qb, sb)
    sfa = (127 + np.repeat(ja.T, 4, axis=1)).astype(np.uint8)                    # [m, k/32]
    sfb = (127 + np.repeat(np.repeat(jb, 128, axis=0)[:n], 4, axis=1)).astype(np.uint8)  # [n, k/32]
    d_mx, a_mx = oracle.gemm(qa, sfa, qb, sfb)
    assert np.array_equal(d_tw, d_mx) and np.array_equal(a_tw, a_mx)
