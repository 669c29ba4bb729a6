"""The expert-parallel layer over peer memory on real GPUs, one process per
GPU: buffers in torch's symmetric memory (no multicast object), the
dispatch kernel storing MXFP8 rows into the owners' buffers over NVLink, the
combine kernel loading the owners' outputs, NCCL stream barriers between the
phases.  Every rank's output must equal, bit for bit, the same layer with
all ranks emulated on one GPU (tests/test_ep_peer.py shows that one equals
the single-GPU layer).  Needs two GPUs; skipped otherwise."""
import os
import socket
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))

CHILD = r"""
import datetime, os, sys
import numpy as np, torch
import torch.distributed as dist
sys.path[:0] = [sys.argv[1], sys.argv[2]]
import moe_grouped_gemm_mx_b200 as mx, mx_inputs
from moe_grouped_gemm_mx_b200.ep import PeerBuffers, ep_moe_layer_peer, ep_moe_layer_peer_emulated
rank, world, out = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"]), sys.argv[3]
torch.cuda.set_device(rank)
dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=60))
E, TOPK, H, I, N, PAD = 8, 4, 256, 256, 256, 128
tokens = [300, 211][:world] + [128] * max(0, world - 2)
dev = torch.device("cuda", rank)
ids_l = [mx_inputs.topk_ids(tokens[r], TOPK, E, seed=40 + r) for r in range(world)]
xs = [mx_inputs.normal_bf16((tokens[r], H), 1.0, 60 + r).to(dev) for r in range(world)]
gws = [torch.from_numpy(mx_inputs.gate_weights(tokens[r], TOPK, seed=70 + r)).to(dev) for r in range(world)]
w13 = mx_inputs.normal_bf16((E, 2 * I, H), 0.05, 80).to(dev)
w2 = mx_inputs.normal_bf16((E, N, I), 0.05, 81).to(dev)
q13, sf13 = mx.mx_quantize_bf16_to_e4m3(w13)
q2, sf2 = mx.mx_quantize_bf16_to_e4m3(w2)
el = E // world
p13, p2 = mx.scale_bytes(2 * I, H), mx.scale_bytes(N, I)
wts = [(q13[r * el:(r + 1) * el], sf13[r * el * p13:(r + 1) * el * p13], q2[r * el:(r + 1) * el],
        sf2[r * el * p2:(r + 1) * el * p2]) for r in range(world)]
m_cap = mx.mx_moe_max_rows(sum(tokens) * TOPK, el, PAD)
bufs = PeerBuffers.symmetric(m_cap, H, N)
y = ep_moe_layer_peer(xs[rank], torch.from_numpy(ids_l[rank]).to(dev), gws[rank], E, *wts[rank], bufs, pad=PAD)
torch.cuda.synchronize()
ebufs = PeerBuffers.emulated(world, m_cap, H, N, dev)
ref = ep_moe_layer_peer_emulated(xs, [torch.from_numpy(i).to(dev) for i in ids_l], gws, E, wts, ebufs, pad=PAD)
torch.cuda.synchronize()
np.save(out + f".{rank}.npy", np.array([int(torch.equal(y.view(torch.int16), ref[rank].view(torch.int16)))]))
dist.barrier()
del bufs
dist.destroy_process_group()
"""


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2, reason="needs two GPUs")
def test_peer_layer_two_gpus_matches_emulated():
    world = 2
    with tempfile.TemporaryDirectory() as td:
        out = os.path.join(td, "eq")
        port = _free_port()
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                   NCCL_NVLS_ENABLE="0", TORCH_SYMM_MEM_DISABLE_MULTICAST="1")
        procs = [subprocess.Popen([sys.executable, "-c", CHILD, ROOT, TESTS, out],
                                  env=dict(env, RANK=str(r), LOCAL_RANK=str(r)), stdout=subprocess.PIPE,
                                  stderr=subprocess.PIPE, text=True) for r in range(world)]
        errs = []
        for p in procs:
            try:
                _, err = p.communicate(timeout=300)
            except subprocess.TimeoutExpired:
                p.kill()
                _, err = p.communicate()
            errs.append((p.returncode, err[-2000:]))
        for r, (rc, err) in enumerate(errs):
            assert rc == 0, f"rank {r}: {err}"
        for r in range(world):
            assert int(np.load(out + f".{r}.npy")[0]) == 1, f"rank {r}: output differs from the emulated layer"
