"""CPU-only checks of the C ABI: the library loads without a GPU, exports
every function include/mx.h declares, and rejects bad arguments on the host
before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mx.h")
LIB = os.path.join(ROOT, "moe_grouped_gemm_mx_b200", "libmx.so")

MX_OK, MX_ERR_INVALID_ARGUMENT, MX_ERR_UNSUPPORTED_SHAPE, MX_ERR_MISALIGNED = 0, 1, 2, 3


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mx_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        import __graft_entry__
        __graft_entry__.build()
    L = ctypes.CDLL(LIB)
    P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    L.mx_scale_bytes.argtypes = [I64, I64]
    L.mx_scale_bytes.restype = ctypes.c_size_t
    L.mx_status_string.argtypes = [ctypes.c_int]
    L.mx_status_string.restype = ctypes.c_char_p
    L.mx_quantize_bf16_to_e4m3.argtypes = [P, I64, I64, P, P, P]
    L.mx_quantize_bf16_to_e4m3_grouped.argtypes = [P, I64, I64, I64, P, P, P]
    L.mx_quantize_bf16_to_e4m3_multi.argtypes = [P, I32, P]
    L.mx_gemm.argtypes = [P, P, P, P, P, I64, I64, I64, P, P]
    L.mx_grouped_gemm_contiguous.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P]
    L.mx_grouped_gemm_masked.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P]
    L.mx_gemm_swiglu_quant.argtypes = [P, P, P, P, P, P, I64, I64, I64, P, P]
    L.mx_quantize_bf16_to_e4m3_transposed.argtypes = [P, I64, I64, I64, P, P, P]
    L.mx_grouped_gemm_kgrouped.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P]
    L.mx_quantize_bf16_to_e4m3_tile1x128.argtypes = [P, I64, I64, P, P, P]
    L.mx_quantize_bf16_to_e4m3_block128x128.argtypes = [P, I64, I64, P, P, P]
    L.mx_gemm_tilewise.argtypes = [P, P, P, P, P, I64, I64, I64, P, P]
    L.mx_grouped_gemm_contiguous_tilewise.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P]
    L.mx_grouped_gemm_contiguous_swiglu_quant.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P, P]
    L.mx_grouped_gemm_masked_swiglu_quant.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P, P]
    L.mx_moe_max_rows.argtypes = [I64, I32, I32]
    L.mx_moe_max_rows.restype = I64
    L.mx_moe_route.argtypes = [P, I64, I32, I32, P, P, P, P, P]
    L.mx_moe_dispatch_quant.argtypes = [P, I64, I64, P, I32, P, P, I32, I32, I64, P, P, I32, P, P]
    L.mx_moe_scatter_rows.argtypes = [P, P, I64, I64, P, P, P, I32, I32, I64, P, P, P, P]
    L.mx_gather_rows.argtypes = [P, I64, I64, P, I64, P, P, P]
    L.mx_moe_combine.argtypes = [P, I64, I64, P, P, I64, I32, P, P, P]
    L.mx_moe_peer_plan.argtypes = [P, P, I64, P, I32, I32, I32, I32, P, P, P, P, P, P]
    L.mx_moe_dispatch_quant_peer.argtypes = [P, I64, I64, P, P, I32, P, P, I32, I64, P, P, P, P, I32, I32, P, P]
    L.mx_moe_combine_peer.argtypes = [P, I32, I64, I64, P, P, P, I64, I32, P, P, P]
    return L


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "mx_gemm" in names and "mx_grouped_gemm_masked" in names
    for name in names:
        assert hasattr(lib, name), name
    import moe_grouped_gemm_mx_b200 as mx
    assert sorted(mx.C_SYMBOLS) == names


def test_scale_bytes_matches_oracle(lib, oracle):
    for rows, k in [(1, 32), (128, 512), (129, 160), (64, 7168), (2112, 7168), (300, 96)]:
        assert lib.mx_scale_bytes(rows, k) == oracle.scale_bytes(rows, k)
    assert lib.mx_scale_bytes(0, 128) == 0
    assert lib.mx_scale_bytes(-1, 128) == 0


def test_status_strings(lib):
    assert lib.mx_status_string(0) == b"MX_OK"
    assert lib.mx_status_string(3) == b"MX_ERR_MISALIGNED"
    assert lib.mx_status_string(99) == b"MX_ERR_UNKNOWN"


FAKE = 0x10000  # a 16-byte aligned non-null value; never dereferenced by these calls


def test_quantize_argument_checks(lib):
    q = lib.mx_quantize_bf16_to_e4m3
    assert q(FAKE, 4, 33, FAKE, FAKE, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert q(FAKE, -1, 32, FAKE, FAKE, None) == MX_ERR_INVALID_ARGUMENT
    assert q(None, 4, 32, FAKE, FAKE, None) == MX_ERR_INVALID_ARGUMENT
    assert q(FAKE + 8, 4, 32, FAKE, FAKE, None) == MX_ERR_MISALIGNED
    assert q(None, 0, 32, None, None, None) == MX_OK  # empty is a no-op
    g = lib.mx_quantize_bf16_to_e4m3_grouped
    assert g(FAKE, -2, 4, 32, FAKE, FAKE, None) == MX_ERR_INVALID_ARGUMENT
    assert g(None, 0, 4, 32, None, None, None) == MX_OK


def test_gemm_argument_checks(lib):
    f = lib.mx_gemm
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 100, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 24, 128, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 0, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert f(FAKE, FAKE, None, FAKE, FAKE, 128, 256, 128, None, None) == MX_ERR_INVALID_ARGUMENT
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE + 4, 128, 256, 128, None, None) == MX_ERR_MISALIGNED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, -1, 256, 128, None, None) == MX_ERR_INVALID_ARGUMENT
    assert f(None, None, None, None, None, 0, 256, 128, None, None) == MX_OK


def test_grouped_argument_checks(lib):
    c = lib.mx_grouped_gemm_contiguous
    assert c(FAKE, FAKE, FAKE, FAKE, None, 4, 512, 256, 128, FAKE, None, None) == MX_ERR_INVALID_ARGUMENT
    assert c(FAKE, FAKE, FAKE, FAKE, FAKE, 2000, 512, 256, 128, FAKE, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert c(FAKE, FAKE, FAKE, FAKE, FAKE + 2, 4, 512, 256, 128, FAKE, None, None) == MX_ERR_MISALIGNED
    assert c(None, None, None, None, None, 0, 512, 256, 128, None, None, None) == MX_OK
    m = lib.mx_grouped_gemm_masked
    assert m(FAKE, FAKE, FAKE, FAKE, None, 4, 256, 256, 128, FAKE, None, None) == MX_ERR_INVALID_ARGUMENT
    assert m(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 256, 250, 128, FAKE, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert m(None, None, None, None, None, 4, 0, 256, 128, None, None, None) == MX_OK


def test_quantize_multi_argument_checks(lib):
    import moe_grouped_gemm_mx_b200 as mx
    J = mx._QuantJob
    f = lib.mx_quantize_bf16_to_e4m3_multi
    jobs = (J * 3)(J(FAKE, 1, 4, 64, FAKE, FAKE), J(FAKE, 1, 4, 48, FAKE, FAKE), J(FAKE, 1, 4, 64, FAKE, FAKE))
    addr = ctypes.addressof(jobs)
    assert f(addr, 3, None) == MX_ERR_UNSUPPORTED_SHAPE          # second job: k % 32 != 0, nothing launched
    jobs[1] = J(FAKE + 8, 1, 4, 64, FAKE, FAKE)
    assert f(addr, 3, None) == MX_ERR_MISALIGNED
    assert f(None, 2, None) == MX_ERR_INVALID_ARGUMENT
    assert f(addr, -1, None) == MX_ERR_INVALID_ARGUMENT
    assert f(None, 0, None) == MX_OK
    empty = (J * 2)(J(None, 0, 4, 64, None, None), J(None, 1, 0, 64, None, None))
    assert f(ctypes.addressof(empty), 2, None) == MX_OK


def test_swiglu_quant_argument_checks(lib):
    f = lib.mx_gemm_swiglu_quant
    # i_dim must be a positive multiple of 128 (the fused epilogue's column block)
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 192, 256, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 0, 256, None, None) == MX_ERR_INVALID_ARGUMENT
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 96, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, 128, 256, 256, None, None) == MX_ERR_INVALID_ARGUMENT
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4, 128, 256, 256, None, None) == MX_ERR_MISALIGNED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE + 8, FAKE, 128, 256, 256, None, None) == MX_ERR_MISALIGNED
    assert f(None, None, None, None, None, None, 0, 256, 256, None, None) == MX_OK
    c = lib.mx_grouped_gemm_contiguous_swiglu_quant
    assert c(FAKE, FAKE, FAKE, FAKE, None, 4, 512, 256, 128, FAKE, FAKE, None, None) == MX_ERR_INVALID_ARGUMENT
    assert c(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 512, 200, 128, FAKE, FAKE, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert c(FAKE, FAKE, FAKE, FAKE, FAKE + 2, 4, 512, 256, 128, FAKE, FAKE, None, None) == MX_ERR_MISALIGNED
    assert c(None, None, None, None, None, 0, 512, 256, 128, None, None, None, None) == MX_OK
    m = lib.mx_grouped_gemm_masked_swiglu_quant
    assert m(FAKE, FAKE, FAKE, FAKE, None, 4, 256, 256, 128, FAKE, FAKE, None, None) == MX_ERR_INVALID_ARGUMENT
    assert m(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 256, 256, 130, FAKE, FAKE, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert m(None, None, None, None, None, 4, 0, 256, 128, None, None, None, None) == MX_OK


def test_training_side_argument_checks(lib):
    t = lib.mx_quantize_bf16_to_e4m3_transposed
    assert t(FAKE, 1, 48, 64, FAKE, FAKE, None) == MX_ERR_UNSUPPORTED_SHAPE   # rows % 32
    assert t(FAKE, 1, 64, 60, FAKE, FAKE, None) == MX_ERR_UNSUPPORTED_SHAPE   # cols % 8
    assert t(FAKE, -1, 64, 64, FAKE, FAKE, None) == MX_ERR_INVALID_ARGUMENT
    assert t(None, 1, 64, 64, FAKE, FAKE, None) == MX_ERR_INVALID_ARGUMENT
    assert t(FAKE, 1, 64, 64, FAKE + 8, FAKE, None) == MX_ERR_MISALIGNED
    assert t(None, 0, 64, 64, None, None, None) == MX_OK
    k = lib.mx_grouped_gemm_kgrouped
    assert k(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 256, 256, 200, FAKE, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert k(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 256, 256, 0, FAKE, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert k(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 256, 250, 256, FAKE, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert k(FAKE, FAKE, FAKE, FAKE, None, 4, 256, 256, 256, FAKE, None, None) == MX_ERR_INVALID_ARGUMENT
    assert k(FAKE, FAKE, FAKE, FAKE, FAKE + 2, 4, 256, 256, 256, FAKE, None, None) == MX_ERR_MISALIGNED
    assert k(None, None, None, None, None, 0, 256, 256, 256, None, None, None) == MX_OK


def test_tilewise_argument_checks(lib):
    for q in (lib.mx_quantize_bf16_to_e4m3_tile1x128, lib.mx_quantize_bf16_to_e4m3_block128x128):
        assert q(FAKE, 4, 96, FAKE, FAKE, None) == MX_ERR_UNSUPPORTED_SHAPE       # k % 128
        assert q(FAKE, -1, 128, FAKE, FAKE, None) == MX_ERR_INVALID_ARGUMENT
        assert q(FAKE, 4, 128, FAKE, None, None) == MX_ERR_INVALID_ARGUMENT
        assert q(FAKE, 4, 128, FAKE, FAKE + 2, None) == MX_ERR_MISALIGNED
        assert q(None, 0, 128, None, None, None) == MX_OK
        # more than 2^32 - 16 groups of 8 rows x 128 columns
        assert q(FAKE, (1 << 31) - 1, 1 << 30, FAKE, FAKE, None) == MX_ERR_UNSUPPORTED_SHAPE
    g = lib.mx_gemm_tilewise
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 96, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 24, 128, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert g(FAKE, None, FAKE, FAKE, FAKE, 128, 256, 128, None, None) == MX_ERR_INVALID_ARGUMENT
    assert g(FAKE, FAKE + 2, FAKE, FAKE, FAKE, 128, 256, 128, None, None) == MX_ERR_MISALIGNED
    assert g(None, None, None, None, None, 0, 256, 128, None, None) == MX_OK
    c = lib.mx_grouped_gemm_contiguous_tilewise
    assert c(FAKE, FAKE, FAKE, FAKE, None, 4, 512, 256, 128, FAKE, None, None) == MX_ERR_INVALID_ARGUMENT
    assert c(FAKE, FAKE, FAKE, FAKE, FAKE, 2000, 512, 256, 128, FAKE, None, None) == MX_ERR_UNSUPPORTED_SHAPE


def test_moe_argument_checks(lib):
    A, B, C, D, E = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000
    assert lib.mx_moe_max_rows(65536, 32, 128) == 69632          # 65536 + 32*127 -> 69600 -> x128
    assert lib.mx_moe_max_rows(10, 4, 1) == 128
    assert lib.mx_moe_max_rows(-1, 4, 1) == 0
    # route: experts in [1, 1024], pad in [1, 128], 4-byte aligned pointers
    assert lib.mx_moe_route(A, 16, 0, 128, B, C, D, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_moe_route(A, 16, 1025, 128, B, C, D, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_moe_route(A, 16, 8, 0, B, C, D, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_moe_route(A, 16, 8, 129, B, C, D, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_moe_route(None, 16, 8, 128, B, C, D, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_moe_route(A + 2, 16, 8, 128, B, C, D, None, None) == MX_ERR_MISALIGNED
    # dispatch: k % 128, m_rows % 128 for tiled scales, topk in [1, 64], alignment
    assert lib.mx_moe_dispatch_quant(A, 4, 96, B, 2, C, D, 8, 128, 128, E, E, 0, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert lib.mx_moe_dispatch_quant(A, 4, 128, B, 2, C, D, 8, 128, 100, E, E, 0, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert lib.mx_moe_dispatch_quant(A, 4, 128, B, 0, C, D, 8, 128, 128, E, E, 0, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_moe_dispatch_quant(A, 4, 128, B, 2, None, None, 8, 128, 128, E, E, 0, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_moe_dispatch_quant(A + 8, 4, 128, B, 2, C, D, 8, 128, 128, E, E, 0, None, None) == MX_ERR_MISALIGNED
    assert lib.mx_moe_dispatch_quant(A, 4, 128, None, 2, C, D, 8, 128, 128, E, E, 0, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_moe_dispatch_quant(A, 0, 128, None, 2, None, None, 0, 1, 0, None, None, 1, None, None) == MX_OK
    # scatter: same rules, plus the source scales
    assert lib.mx_moe_scatter_rows(A, None, 4, 128, B, C, D, 8, 128, 128, E, E, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_moe_scatter_rows(A, A, 4, 64, B, C, D, 8, 128, 128, E, E, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    # gather: rows of a multiple of 16 bytes, aligned
    assert lib.mx_gather_rows(A, 8, 24, B, 4, C, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert lib.mx_gather_rows(A + 4, 8, 32, B, 4, C, None, None) == MX_ERR_MISALIGNED
    assert lib.mx_gather_rows(A, 8, 32, None, 4, C, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_gather_rows(A, 8, 32, B, 0, C, None, None) == MX_OK
    # combine: n_cols % 8, topk in [1, 64], aligned y/out and 4-byte w/row
    assert lib.mx_moe_combine(A, 8, 12, B, C, 4, 2, D, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert lib.mx_moe_combine(A, 8, 16, B, C, 4, 0, D, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_moe_combine(A, 8, 16, B, C, 4, 65, D, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_moe_combine(A, 8, 16, B, C + 2, 4, 2, D, None, None) == MX_ERR_MISALIGNED
    assert lib.mx_moe_combine(A, 8, 16, None, C, 4, 2, D, None, None) == MX_ERR_INVALID_ARGUMENT
    assert lib.mx_moe_combine(A, 8, 16, B, C, 0, 2, D, None, None) == MX_OK


def test_moe_peer_argument_checks(lib):
    A, B, C, D, E, F, G = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000, 0x70000
    plan = lib.mx_moe_peer_plan
    # ranks in [1, 1024], rank in [0, ranks), experts % ranks == 0, pad in [1, 128]
    assert plan(A, B, 16, C, 0, 0, 8, 128, D, E, F, G, None, None) == MX_ERR_INVALID_ARGUMENT
    assert plan(A, B, 16, C, 2, 2, 8, 128, D, E, F, G, None, None) == MX_ERR_INVALID_ARGUMENT
    assert plan(A, B, 16, C, 3, 0, 8, 128, D, E, F, G, None, None) == MX_ERR_INVALID_ARGUMENT
    assert plan(A, B, 16, C, 2, 0, 8, 0, D, E, F, G, None, None) == MX_ERR_INVALID_ARGUMENT
    assert plan(A, B, 16, None, 2, 0, 8, 128, D, E, F, G, None, None) == MX_ERR_INVALID_ARGUMENT
    assert plan(A, B, 16, C, 2, 0, 8, 128, None, E, F, G, None, None) == MX_ERR_INVALID_ARGUMENT
    assert plan(A + 2, B, 16, C, 2, 0, 8, 128, D, E, F, G, None, None) == MX_ERR_MISALIGNED
    assert plan(A, B, 1 << 30, C, 4, 0, 8, 128, D, E, F, G, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    # entries fit in int32 but the padded offsets could not: every expert
    # adds up to pad - 1 rows
    n_edge = ((1 << 31) - 1 - 1024 * 127) // 2
    assert plan(A, B, n_edge + 1, C, 2, 0, 1024, 128, D, E, F, G, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert plan(A, B, n_edge, C, 2, 0, 1024, 128, None, E, F, G, None, None) == MX_ERR_INVALID_ARGUMENT
    disp = lib.mx_moe_dispatch_quant_peer
    # the dispatch's rules, plus ranks and 8-byte aligned pointer tables
    assert disp(A, 4, 128, B, C, 2, D, E, 0, 128, F, G, A, B, 4, 128, None, None) == MX_ERR_INVALID_ARGUMENT
    assert disp(A, 4, 96, B, C, 2, D, E, 2, 128, F, G, A, B, 4, 128, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert disp(A, 4, 128, B, C, 2, D, E, 2, 100, F, G, A, B, 4, 128, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert disp(A, 4, 128, B, C, 2, None, E, 2, 128, F, G, A, B, 4, 128, None, None) == MX_ERR_INVALID_ARGUMENT
    assert disp(A, 4, 128, None, C, 2, D, E, 2, 128, F, G, A, B, 4, 128, None, None) == MX_ERR_INVALID_ARGUMENT
    assert disp(A, 4, 128, B, C, 2, D + 4, E, 2, 128, F, G, A, B, 4, 128, None, None) == MX_ERR_MISALIGNED
    assert disp(A, 4, 128, B, C, 2, D, E, 2, 128, F, G, None, None, 4, 128, None, None) == MX_ERR_INVALID_ARGUMENT
    comb = lib.mx_moe_combine_peer
    assert comb(A, 0, 8, 16, B, C, D, 4, 2, E, None, None) == MX_ERR_INVALID_ARGUMENT
    assert comb(A, 2, 8, 12, B, C, D, 4, 2, E, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    assert comb(A, 2, 8, 16, B, C, D, 4, 65, E, None, None) == MX_ERR_INVALID_ARGUMENT
    assert comb(None, 2, 8, 16, B, C, D, 4, 2, E, None, None) == MX_ERR_INVALID_ARGUMENT
    assert comb(A + 4, 2, 8, 16, B, C, D, 4, 2, E, None, None) == MX_ERR_MISALIGNED
    assert comb(A, 2, 8, 16, B, C, D, 0, 2, E, None, None) == MX_OK


def test_wait_limit_setter(lib):
    """The GEMM kernels' wait bound: 2 s by default, settable, 0 restores the
    default (host-side state; no GPU needed)."""
    lib.mx_wait_limit_ns.restype = ctypes.c_uint64
    lib.mx_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    assert lib.mx_wait_limit_ns() == 2_000_000_000
    assert lib.mx_set_wait_limit_ns(1000) == MX_OK
    assert lib.mx_wait_limit_ns() == 1000
    assert lib.mx_set_wait_limit_ns(0) == MX_OK
    assert lib.mx_wait_limit_ns() == 2_000_000_000


class _Prob(ctypes.Structure):
    _fields_ = [("qa", ctypes.c_void_p), ("sfa", ctypes.c_void_p), ("qb", ctypes.c_void_p),
                ("sfb", ctypes.c_void_p), ("d_bf16", ctypes.c_void_p), ("m", ctypes.c_int64),
                ("n", ctypes.c_int64), ("k", ctypes.c_int64)]


def test_gemm_batch_argument_checks(lib):
    """mx_gemm_batch: 1..4 problems, each with mx_gemm's rules; every problem
    is checked before anything is launched; an all-empty batch is a no-op
    (no GPU needed for any of these)."""
    f = lib.mx_gemm_batch
    f.argtypes = [ctypes.POINTER(_Prob), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
    A, B, C, D, E = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000
    good = _Prob(A, B, C, D, E, 64, 256, 512)
    arr = (_Prob * 5)(*([good] * 5))
    assert f(arr, 0, None, None) == MX_ERR_INVALID_ARGUMENT
    assert f(arr, 5, None, None) == MX_ERR_INVALID_ARGUMENT
    assert f(None, 1, None, None) == MX_ERR_INVALID_ARGUMENT
    bad = (_Prob * 2)(good, _Prob(A, B, C, D, E, 64, 256, 500))           # second problem: k % 128
    assert f(bad, 2, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    bad = (_Prob * 2)(good, _Prob(A, B, C, D, E, 64, 250, 512))           # n % 16
    assert f(bad, 2, None, None) == MX_ERR_UNSUPPORTED_SHAPE
    bad = (_Prob * 2)(good, _Prob(A + 8, B, C, D, E, 64, 256, 512))       # misaligned A
    assert f(bad, 2, None, None) == MX_ERR_MISALIGNED
    bad = (_Prob * 2)(good, _Prob(None, B, C, D, E, 64, 256, 512))        # null A
    assert f(bad, 2, None, None) == MX_ERR_INVALID_ARGUMENT
    bad = (_Prob * 1)(_Prob(A, B, C, D, E, -1, 256, 512))
    assert f(bad, 1, None, None) == MX_ERR_INVALID_ARGUMENT
    empty = (_Prob * 2)(_Prob(None, None, None, None, None, 0, 256, 512),
                        _Prob(None, None, None, None, None, 64, 0, 512))
    assert f(empty, 2, None, None) == MX_OK
