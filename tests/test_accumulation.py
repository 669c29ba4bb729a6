"""Accumulation precision of the GPU GEMMs, on hand-built MXFP8 operands whose
exact results survive only with FP32 accumulation.

The DeepGEMM pages explain that Hopper's FP8 tensor-core accumulation loses
precision, which DeepGEMM repairs by promoting partial sums to FP32 on CUDA
cores ("two-level accumulation").  The kernels here accumulate in the tensor
core's FP32 TMEM accumulator with no promotion step; these tests check that
nothing is lost at that level:

* across 32-element blocks (successive MMAs into the accumulator): the blocks
  contribute +2^23, +1 and -2^23 in K order, so the exact result 1 needs 24
  significant bits in the running sum;
* inside one 32-element block (one MMA's own reduction): fifteen products of
  +2^16, fifteen of -2^16, one zero and one product of exactly 1 (2^-8 x 256)
  whose position moves with the row, so whatever order the hardware reduces
  in, some partial sum of magnitude up to 2^19.9 must carry the 1.

The operands are built directly as E4M3 bytes and UE8M0 scale codes; the
results are checked against the oracle and against the hand value 1."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

E4M3_ONE = 0x38     # 1.0
E4M3_P256 = 0x78    # +256 = 2^8
E4M3_M256 = 0xF8    # -256
E4M3_2M8 = 0x02     # 2^-8 (subnormal: 2/8 * 2^-6)


@pytest.fixture(scope="module")
def mx():
    import moe_grouped_gemm_mx_b200 as m
    return m


def run(mx, oracle, qa, sa, qb, sb):
    """qa [m, k] / qb [n, k] E4M3 bytes, sa / sb row-major scale codes [., k/32]."""
    m, k = qa.shape
    n = qb.shape[0]
    dev = torch.device("cuda")
    ta = torch.from_numpy(oracle.sf_tile(sa, m, k)).to(dev)
    tb = torch.from_numpy(oracle.sf_tile(sb, n, k)).to(dev)
    d = mx.mx_gemm(torch.from_numpy(qa).to(dev), ta, torch.from_numpy(qb).to(dev), tb)
    torch.cuda.synchronize()
    ref, _ = oracle.gemm(qa, sa, qb, sb)
    return d.float().cpu().numpy().astype(np.float64), ref


def operands(m, n, k):
    kb = k // 32
    return (np.zeros((m, k), dtype=np.uint8), np.full((m, kb), 127, dtype=np.uint8),
            np.zeros((n, k), dtype=np.uint8), np.full((n, kb), 127, dtype=np.uint8))


@pytest.mark.parametrize("m,n,k", [(128, 256, 256), (64, 2112, 7168), (8192, 256, 512), (8192, 2048, 256)])
def test_cross_block_fp32_accumulation(mx, oracle, m, n, k):
    qa, sa, qb, sb = operands(m, n, k)
    # block 0: 32 products of (256 * 2^2) * 256 = 2^18 -> +2^23
    qa[:, 0:32] = E4M3_P256
    sa[:, 0] = 127 + 2
    qb[:, 0:32] = E4M3_P256
    # block 1: one product 1 * 1
    qa[:, 32] = E4M3_ONE
    qb[:, 32] = E4M3_ONE
    # block 2: 32 products of -(2^18) -> -2^23
    qa[:, 64:96] = E4M3_M256
    sa[:, 2] = 127 + 2
    qb[:, 64:96] = E4M3_P256
    d, ref = run(mx, oracle, qa, sa, qb, sb)
    assert np.all(ref == 1.0)
    bad = d != 1.0
    assert not bad.any(), f"{bad.sum()} of {d.size} outputs lost the +1 (values {np.unique(d[bad])[:5]})"


@pytest.mark.parametrize("m,n,k", [(128, 256, 128), (256, 4096, 256), (64, 528, 1024), (8192, 2048, 256)])
def test_in_block_fp32_accumulation(mx, oracle, m, n, k):
    qa, sa, qb, sb = operands(m, n, k)
    qb[:, 0:32] = E4M3_P256                  # every B element of block 0 is 256
    for r in range(m):
        p = r % 32                           # where this row's residue sits
        others = [j for j in range(32) if j != p]
        signs = np.array([E4M3_P256] * 15 + [E4M3_M256] * 15 + [0x00], dtype=np.uint8)
        qa[r, others] = np.roll(signs, r // 32)   # vary the arrangement of the +-2^16 products too
        qa[r, p] = E4M3_2M8                  # 2^-8 * 256 = 1
    d, ref = run(mx, oracle, qa, sa, qb, sb)
    assert np.all(ref == 1.0)
    bad = d != 1.0
    assert not bad.any(), f"{bad.sum()} of {d.size} outputs lost the +1 (values {np.unique(d[bad])[:5]})"
