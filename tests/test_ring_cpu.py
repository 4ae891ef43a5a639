"""The sequence-parallel ring's host logic on CPU: gloo ranks exchange key/value
blocks and travelling dK/dV accumulators exactly as on GPUs, with each block step
computed by the fp64 oracle's key-block functions instead of the kernels. Every
rank's output block must equal the full oracle's on the whole sequence."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleBlockOps:
    """Block steps from the oracle (fp64), with the ring's calling convention."""

    def __init__(self, scale):
        self.scale = scale

    def new_acc(self, q):
        return (torch.zeros(q.shape, dtype=torch.float64), torch.full(q.shape[:3], -math.inf, dtype=torch.float64))

    def fwd_block(self, q, k, v, causal):
        import oracle
        B, H = q.shape[:2]
        o = torch.zeros(q.shape, dtype=torch.float64)
        lse = torch.zeros(q.shape[:3], dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                ob, lb = oracle.attn_fwd_block_ref(q[b, h], k[b, h], v[b, h], self.scale, causal)
                o[b, h], lse[b, h] = torch.from_numpy(ob), torch.from_numpy(lb)
        return o, lse

    def merge(self, acc, part):
        a, b = acc[1].numpy(), part[1].numpy()
        lse = np.logaddexp(a, b)
        fin = np.isfinite(lse)
        wa = np.where(fin, np.exp(np.where(fin, a - lse, 0.0)), 0.0)
        wb = np.where(fin, np.exp(np.where(fin, b - lse, 0.0)), 0.0)
        o = acc[0].numpy() * wa[..., None] + part[0].numpy() * wb[..., None]
        acc[0].copy_(torch.from_numpy(o))
        acc[1].copy_(torch.from_numpy(lse))

    def finish_o(self, acc):
        return acc[0].clone(), acc[1].clone()

    def bwd_prepare(self, q, o, lse, do):
        return {"lse": lse, "D": (do * o).sum(-1)}

    def bwd_block(self, st, q, k, v, do, causal):
        import oracle
        B, H = q.shape[:2]
        out = [torch.zeros(q.shape, dtype=torch.float64) for _ in range(3)]
        for b in range(B):
            for h in range(H):
                g = oracle.attn_bwd_block_ref(q[b, h], k[b, h], v[b, h], do[b, h], st["lse"][b, h], st["D"][b, h],
                                              self.scale, causal)
                for t, x in zip(out, g):
                    t[b, h] = torch.from_numpy(x)
        return out

    def zeros_f32(self, x):
        return torch.zeros(x.shape, dtype=torch.float64)

    def accumulate(self, acc, x):
        acc += x

    def to_out(self, acc):
        return acc.clone()


def _worker(rank, world, port, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from exact_tiled_attention_34_b200 import ring
        B, H, n, d, scale = 1, 2, 5, 3, 0.7
        N = world * n
        g = torch.Generator().manual_seed(11)
        q, k, v, do = (torch.randn((B, H, N, d), generator=g, dtype=torch.float64) for _ in range(4))
        blk = lambda x: x[:, :, rank * n:(rank + 1) * n].contiguous()
        ops = OracleBlockOps(scale)
        rg = ring.ProcessGroupRing()
        o, lse = ring.ring_forward(blk(q), blk(k), blk(v), causal, scale, rg, ops)
        dq, dk, dv = ring.ring_backward(blk(q), blk(k), blk(v), o, lse, blk(do), causal, scale, rg, ops)
        full = oracle.attn_bwd_ref(q, k, v, do, causal, scale)
        errs = {}
        for name, x in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            ref = full[name][:, :, rank * n:(rank + 1) * n]
            errs[name] = float(np.max(np.abs(x.numpy() - ref)))
        # the autograd wrapper: same blocks, gradients through torch.autograd
        qa, ka, va = (blk(x).requires_grad_(True) for x in (q, k, v))
        oa = ring.ring_attention(qa, ka, va, causal, scale, rg, ops)
        oa.backward(blk(do))
        errs["autograd_o"] = float((oa.detach() - o).abs().max())
        for name, x in (("autograd_dq", qa), ("autograd_dk", ka), ("autograd_dv", va)):
            errs[name] = float(np.max(np.abs(x.grad.numpy() - full[name[-2:]][:, :, rank * n:(rank + 1) * n])))
        out[rank] = errs
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_matches_full_attention(world, causal):
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, causal, out), nprocs=world, start_method="spawn", join=True)
    for rank in range(world):
        errs = out[rank]
        assert max(errs.values()) < 1e-12, (rank, errs)
