"""GPU quantiser vs the CPU oracle: element bytes and scales must match
bit for bit, on every BF16 bit pattern and on the workloads' shapes, with the
scale-tile padding written as 0x00 and nothing written outside the outputs."""
import numpy as np
import pytest
import torch

import mx_inputs
from mxtest_util import bf16_bits_np, gpu_sf_rowmajor, oracle_quantize

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    import moe_grouped_gemm_mx_b200 as m
    return m


def run_gpu_quant(mx, x_cpu: torch.Tensor, guard: int = 4096):
    """Quantise on the GPU into sentinel-filled buffers with guard bytes."""
    dev = torch.device("cuda")
    x = x_cpu.to(dev)
    groups = 1 if x.dim() == 2 else x.shape[0]
    rows, k = x.shape[-2], x.shape[-1]
    nq = x.numel()
    nsf = groups * mx.scale_bytes(rows, k)
    qbuf = torch.full((nq + guard,), 0xA5, dtype=torch.uint8, device=dev)
    sfbuf = torch.full((nsf + guard,), 0xA5, dtype=torch.uint8, device=dev)
    q, sf = mx.mx_quantize_bf16_to_e4m3(x, q=qbuf[:nq].view(x.shape), sf=sfbuf[:nsf])
    torch.cuda.synchronize()
    assert torch.all(qbuf[nq:] == 0xA5), "quantiser wrote past the end of q"
    assert torch.all(sfbuf[nsf:] == 0xA5), "quantiser wrote past the end of sf"
    return q.cpu().numpy().reshape(-1, k), sf.cpu()


def check_against_oracle(mx, oracle, x_cpu: torch.Tensor):
    groups = 1 if x_cpu.dim() == 2 else x_cpu.shape[0]
    rows, k = x_cpu.shape[-2], x_cpu.shape[-1]
    q_gpu, sf_gpu_tiled = run_gpu_quant(mx, x_cpu)
    q_ref, sf_ref = oracle_quantize(oracle, x_cpu)
    assert np.array_equal(q_gpu, q_ref), f"element bytes differ at {np.argwhere(q_gpu != q_ref)[:5]}"
    sf_gpu = gpu_sf_rowmajor(oracle, sf_gpu_tiled, groups, rows, k)
    assert np.array_equal(sf_gpu, sf_ref), f"scales differ at {np.argwhere(sf_gpu != sf_ref)[:5]}"
    # the whole tiled region, padding included, equals the oracle's tiling
    per = oracle.scale_bytes(rows, k)
    want = np.concatenate([oracle.sf_tile(sf_ref[g * rows:(g + 1) * rows], rows, k) for g in range(groups)])
    assert np.array_equal(sf_gpu_tiled.numpy(), want)


def all_patterns_blocks(seed: int, control=None) -> torch.Tensor:
    """Every BF16 bit pattern once, shuffled into rows of 32-element blocks;
    with `control`, element 0 of every block is replaced by that value."""
    g = torch.Generator().manual_seed(seed)
    bits = torch.randperm(65536, generator=g).to(torch.int32)
    bits = torch.where(bits >= 32768, bits - 65536, bits).to(torch.int16)
    x = bits.view(torch.bfloat16).reshape(-1, 512)  # 128 rows x 512 (16 blocks per row)
    if control is not None:
        x = x.clone().reshape(-1, 32)
        x[:, 0] = control
        x = x.reshape(-1, 512)
    return x


def test_all_bf16_patterns_natural_blocks(mx, oracle):
    check_against_oracle(mx, oracle, all_patterns_blocks(0))


@pytest.mark.parametrize("control", [2.0 ** 126, 1.5 * 2.0 ** 40, 448.0, 1.0, 2.0 ** -20, 2.0 ** -119, 2.0 ** -130])
def test_all_bf16_patterns_with_controlling_amax(mx, oracle, control):
    """Element 0 = control; finite patterns with larger magnitude raise amax,
    the rest probe rounding (ties, subnormals, underflow) at that scale."""
    check_against_oracle(mx, oracle, all_patterns_blocks(1, control))


def test_all_patterns_small_magnitudes(mx, oracle):
    """All patterns with |v| <= 1 next to a controlling 1.0, so every block
    scale is X = -8 and every pattern is converted at the same scale."""
    bits = torch.arange(65536, dtype=torch.int32)
    bits = torch.where(bits >= 32768, bits - 65536, bits).to(torch.int16)
    v = bits.view(torch.bfloat16)
    keep = v.float().abs() <= 1.0
    v = v[keep]
    n = (v.numel() + 30) // 31 * 31
    pad = torch.zeros(n - v.numel(), dtype=torch.bfloat16)
    blocks = torch.cat([v, pad]).reshape(-1, 31)
    x = torch.cat([torch.ones(blocks.shape[0], 1, dtype=torch.bfloat16), blocks], dim=1)
    rows = (x.shape[0] + 15) // 16 * 16
    x = torch.cat([x, torch.zeros(rows - x.shape[0], 32, dtype=torch.bfloat16)]).reshape(-1, 512)
    check_against_oracle(mx, oracle, x)


@pytest.mark.parametrize("rows,k", [(1, 32), (3, 96), (63, 160), (64, 7168), (128, 512), (129, 128),
                                    (256, 512), (300, 224), (2112, 256)])
def test_shapes_random(mx, oracle, rows, k):
    x = mx_inputs.outlier_bf16((rows, k), seed=rows * 7 + k)
    check_against_oracle(mx, oracle, x)


def test_grouped_3d_with_ragged_rows(mx, oracle):
    x = mx_inputs.normal_bf16((3, 130, 160), 1.0, seed=5)
    check_against_oracle(mx, oracle, x)


def test_nan_padding_rows(mx, oracle):
    p = mx_inputs.masked_problem(n=64, k=256, experts=4, max_m=40, seed=3)
    check_against_oracle(mx, oracle, p.a)


def test_page_shapes_full(mx, oracle):
    """Operands of the dense page shapes, full tensors, bit-exact."""
    for (m, n, k) in mx_inputs.PAGE_SHAPES:
        a, b = mx_inputs.dense_problem(m, n, k, seed=0, kind="outlier")
        check_against_oracle(mx, oracle, a)
        check_against_oracle(mx, oracle, b)


def test_multi_matches_single_and_oracle(mx, oracle):
    """Nine tensors of assorted shapes (2-D, 3-D, ragged K, one empty) in one
    batched call: every output bit-identical to the one-tensor call and to
    the oracle (more than 8 tensors exercises the split into two launches)."""
    shapes = [(64, 7168), (2112, 256), (3, 130, 160), (1, 32), (0, 64), (300, 224), (129, 96),
              (2, 128, 512), (5, 7168)]
    xs = [mx_inputs.outlier_bf16(s, seed=i).cuda() for i, s in enumerate(shapes)]
    outs = mx.mx_quantize_bf16_to_e4m3_multi(xs)
    torch.cuda.synchronize()
    for x, (q, sf) in zip(xs, outs):
        if x.numel() == 0:
            continue
        q1, sf1 = mx.mx_quantize_bf16_to_e4m3(x)
        torch.cuda.synchronize()
        assert torch.equal(q, q1) and torch.equal(sf, sf1)
        groups = 1 if x.dim() == 2 else x.shape[0]
        rows, k = x.shape[-2], x.shape[-1]
        q_ref, sf_ref = oracle_quantize(oracle, x.cpu())
        assert np.array_equal(q.cpu().numpy().reshape(-1, k), q_ref)
        assert np.array_equal(gpu_sf_rowmajor(oracle, sf, groups, rows, k), sf_ref)


def test_multi_lean_matches_normal_form(mx, oracle):
    """The lean form (no shared memory, one CTA per SM) writes the same bytes
    as the normal form: the nine assorted tensors of the test above (outputs
    small enough to be kept in L2), and the contiguous MoE's down operands
    ([67,456 x 2048] tokens and 8 experts of [7168 x 2048]: outputs larger
    than L2, streamed), scale padding included (buffers pre-filled with a
    sentinel)."""
    shapes = [(64, 7168), (2112, 256), (3, 130, 160), (1, 32), (0, 64), (300, 224), (129, 96),
              (2, 128, 512), (5, 7168)]
    for case in (shapes, [(67456, 2048), (8, 7168, 2048)]):
        xs = [mx_inputs.outlier_bf16(s, seed=30 + i).cuda() if len(case) > 2 else
              mx_inputs.normal_bf16(s, 1.0 if i == 0 else 0.02, 30 + i).cuda() for i, s in enumerate(case)]
        outs = []
        for x in xs:
            groups = 1 if x.dim() == 2 else x.shape[0]
            rows, k = x.shape[-2], x.shape[-1]
            outs.append((torch.full(x.shape, 0xAB, dtype=torch.uint8, device="cuda"),
                         torch.full((groups * mx.scale_bytes(rows, k),), 0xCD, dtype=torch.uint8, device="cuda")))
        mx.mx_quantize_bf16_to_e4m3_multi(xs, outs, lean=True)
        ref = mx.mx_quantize_bf16_to_e4m3_multi(xs)
        torch.cuda.synchronize()
        for (q, sf), (q1, sf1) in zip(outs, ref):
            assert torch.equal(q, q1) and torch.equal(sf, sf1)
    x = xs[0][:4096]
    q_ref, sf_ref = oracle_quantize(oracle, x.cpu())
    assert np.array_equal(outs[0][0][:4096].cpu().numpy(), q_ref)


def test_empty_is_noop(mx):
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q, sf = mx.mx_quantize_bf16_to_e4m3(x)
    assert q.numel() == 0 and sf.numel() == 0


def test_rejects_bad_k(mx):
    x = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mx.MXError):
        mx.mx_quantize_bf16_to_e4m3(x)
