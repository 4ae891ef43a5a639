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
    """Block steps from the oracle (fp64), with the ring's calling convention: the
    oracle's key-block functions take the chunks' global offsets and apply the causal
    rule themselves."""

    def __init__(self, scale):
        self.scale = scale

    def new_acc(self, q):
        return (torch.zeros(q.shape, dtype=torch.float64), torch.full(q.shape[:3], -math.inf, dtype=torch.float64))

    def fwd_pair(self, acc, q, k, v, q_off, k_off, causal):
        import oracle
        B, H = q.shape[:2]
        o = torch.zeros(q.shape, dtype=torch.float64)
        lse = torch.zeros(q.shape[:3], dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                ob, lb = oracle.attn_fwd_block_ref(q[b, h], k[b, h], v[b, h], self.scale, causal, q_off, k_off)
                o[b, h], lse[b, h] = torch.from_numpy(ob), torch.from_numpy(lb)
        a, bb = acc[1].numpy(), lse.numpy()
        new = np.logaddexp(a, bb)
        fin = np.isfinite(new)
        wa = np.where(fin, np.exp(np.where(fin, a - new, 0.0)), 0.0)
        wb = np.where(fin, np.exp(np.where(fin, bb - new, 0.0)), 0.0)
        acc[0].copy_(torch.from_numpy(acc[0].numpy() * wa[..., None] + o.numpy() * wb[..., None]))
        acc[1].copy_(torch.from_numpy(new))

    def finish_o(self, acc):
        return acc[0].clone(), acc[1].clone()

    def bwd_prepare(self, q, o, lse, do):
        return {"lse": lse, "D": (do * o).sum(-1), "dq": torch.zeros(q.shape, dtype=torch.float64)}

    def bwd_pair(self, st, q, k, v, do, q_off, k_off, causal):
        import oracle
        B, H = q.shape[:2]
        dk = torch.zeros(k.shape, dtype=torch.float64)
        dv = torch.zeros(v.shape, dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                gq, gk, gv = oracle.attn_bwd_block_ref(q[b, h], k[b, h], v[b, h], do[b, h], st["lse"][b, h],
                                                       st["D"][b, h], self.scale, causal, q_off, k_off)
                st["dq"][b, h] += torch.from_numpy(gq)
                dk[b, h], dv[b, h] = torch.from_numpy(gk), torch.from_numpy(gv)
        return dk, dv

    def finish_dq(self, st):
        return st["dq"].clone()

    def zeros_acc(self, x):
        return torch.zeros(x.shape, dtype=torch.float64)

    def accumulate(self, acc, x):
        acc += x

    def to_out(self, acc):
        return acc.clone()


def zigzag_rows(rank, world, n):
    """Global rows of a rank's block with zig-zag chunks (chunks r and 2R - 1 - r)."""
    from exact_tiled_attention_34_b200 import ring
    c = n // 2
    return np.concatenate([np.arange(o, o + c) for o in ring.chunk_offsets(rank, world, n, True)])


def _worker(rank, world, port, causal, zigzag, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from exact_tiled_attention_34_b200 import ring
        B, H, n, d, scale = 1, 2, 6, 3, 0.7
        N = world * n
        g = torch.Generator().manual_seed(11)
        q, k, v, do = (torch.randn((B, H, N, d), generator=g, dtype=torch.float64) for _ in range(4))
        rows = zigzag_rows(rank, world, n) if zigzag else np.arange(rank * n, (rank + 1) * n)
        idx = torch.as_tensor(rows)
        blk = lambda x: x[:, :, idx].contiguous()
        ops = OracleBlockOps(scale)
        rg = ring.ProcessGroupRing()
        o, lse = ring.ring_forward(blk(q), blk(k), blk(v), causal, scale, rg, ops, zigzag)
        dq, dk, dv = ring.ring_backward(blk(q), blk(k), blk(v), o, lse, blk(do), causal, scale, rg, ops, zigzag)
        full = oracle.attn_bwd_ref(q, k, v, do, causal, scale)
        errs = {}
        for name, x in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            ref = full[name][:, :, rows]
            errs[name] = float(np.max(np.abs(x.numpy() - ref)))
        # the autograd wrapper: same blocks, gradients through torch.autograd
        qa, ka, va = (blk(x).requires_grad_(True) for x in (q, k, v))
        oa = ring.ring_attention(qa, ka, va, causal, scale, rg, ops, zigzag)
        oa.backward(blk(do))
        errs["autograd_o"] = float((oa.detach() - o).abs().max())
        for name, x in (("autograd_dq", qa), ("autograd_dk", ka), ("autograd_dv", va)):
            errs[name] = float(np.max(np.abs(x.grad.numpy() - full[name[-2:]][:, :, rows])))
        out[rank] = errs
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal,zigzag", [(False, False), (True, False), (True, True)])
def test_ring_matches_full_attention(world, causal, zigzag):
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, causal, zigzag, out), nprocs=world, start_method="spawn",
                       join=True)
    for rank in range(world):
        errs = out[rank]
        assert max(errs.values()) < 1e-12, (rank, errs)


def test_zigzag_balances_causal_work():
    """With zig-zag chunks every rank computes the same number of visible (query chunk,
    key chunk) pairs, 2R + 1 for R ranks; with plain blocks rank r computes r + 1."""
    from exact_tiled_attention_34_b200 import ring
    for R in (2, 3, 4, 8):
        plain = [sum(1 for s in range(R) if (r - s) % R <= r) for r in range(R)]
        assert plain == [r + 1 for r in range(R)]
        counts = []
        for r in range(R):
            c = 0
            for s in range(R):
                src = (r - s) % R
                for qo in ring.chunk_offsets(r, R, 2, True):
                    for ko in ring.chunk_offsets(src, R, 2, True):
                        c += ring._pair_kind(True, qo, ko) is not None
            counts.append(c)
        assert len(set(counts)) == 1 and counts[0] == 2 * R + 1, counts
