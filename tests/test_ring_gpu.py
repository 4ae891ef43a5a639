"""The sequence-parallel ring with the library's kernels on one GPU: R ranks are
emulated by host threads that hand each other tensors through queues (no kernel waits
for another; all launches share one stream in the order the ranks make them). The
output blocks are compared with the fp64 oracle on the whole sequence. Also the merge
kernel on its own: two key halves merged equal attention over all keys.

The autograd wrapper is not run here: torch's autograd engine executes CUDA backward
nodes on one worker thread per device, so emulated ranks blocking on each other inside
their backward would wait forever; separate processes (the real setting) do not share
that thread, and the wrapper is tested that way on gloo ranks."""
import math
import queue
import threading

import numpy as np
import pytest
import torch

import exact_tiled_attention_34_b200 as fa
import oracle
from exact_tiled_attention_34_b200 import ring
from exact_tiled_attention_34_b200.inputs import make_qkv
from tests.parity import assert_fwd_close, assert_grad_close

pytestmark = pytest.mark.gpu


class ThreadRing:
    """Ring neighbours among threads; message k sent to a rank is its k-th receive."""

    def __init__(self, rank, world, inboxes):
        self.rank, self.world, self.inboxes = rank, world, inboxes
        self.sent = 0
        self.posted = 0
        self.arrived = {}

    def start(self, tensors):
        self.inboxes[(self.rank + 1) % self.world].put((self.sent, [t.clone() for t in tensors]))
        self.sent += 1
        self.posted += 1
        return self.posted - 1

    def finish(self, seq):
        while seq not in self.arrived:
            k, ts = self.inboxes[self.rank].get(timeout=120)
            self.arrived[k] = ts
        return self.arrived.pop(seq)

    def exchange(self, tensors):
        return self.finish(self.start(tensors))


def _run_ring(q, k, v, do, world, causal, scale):
    n = q.shape[2] // world
    blk = lambda x, r: x[:, :, r * n:(r + 1) * n].contiguous()
    inboxes = [queue.Queue() for _ in range(world)]
    res, errs = {}, []

    def rank_main(r):
        try:
            rg = ThreadRing(r, world, inboxes)
            o, lse = ring.ring_forward(blk(q, r), blk(k, r), blk(v, r), causal, scale, rg)
            g = ring.ring_backward(blk(q, r), blk(k, r), blk(v, r), o, lse, blk(do, r), causal, scale, rg)
            res[r] = (o, lse) + tuple(g)
        except Exception as e:  # reported below
            errs.append(e)

    ts = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in ts:
        t.start()
    for t in ts:
        t.join(timeout=300)
    assert not errs, errs
    torch.cuda.synchronize()
    cat = lambda i: torch.cat([res[r][i] for r in range(world)], dim=2)
    return [cat(i) for i in range(5)]


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_parity(cuda_device, world, d, causal):
    B, H, n = 1, 2, 256
    N = world * n
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=40 + world + d).items()}
    sc = 1.0 / math.sqrt(d)
    o, lse, dq, dk, dv = _run_ring(t["q"], t["k"], t["v"], t["do"], world, causal, sc)
    assert fa.device_status() == (0, 0)
    ref = oracle.attn_bwd_ref(t["q"].cpu(), t["k"].cpu(), t["v"].cpu(), t["do"].cpu(), causal, sc)
    what = f"ring R={world} d={d} causal={causal}"
    assert_fwd_close(o.cpu(), lse.cpu(), ref["o"], ref["lse"], what)
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert_grad_close(g.cpu(), ref[name], name, what)


@pytest.mark.parametrize("d", [64, 128])
def test_merge_of_key_halves_is_full_attention(cuda_device, d):
    B, H, N = 2, 3, 384
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=7, with_do=False).items()}
    sc = 1.0 / math.sqrt(d)
    acc = torch.zeros((B, H, N, d), dtype=torch.float32, device=cuda_device)
    lse = torch.full((B, H, N), -math.inf, dtype=torch.float32, device=cuda_device)
    for sl in (slice(0, 128), slice(128, N)):
        k, v = t["k"][:, :, sl].contiguous(), t["v"][:, :, sl].contiguous()
        o_p, l_p = fa.forward(t["q"], k, v, scale=sc)
        fa.merge_partial(acc, lse, o_p, l_p)
    o = fa.to_bf16(acc)
    o_ref, l_ref = oracle.attn_fwd_ref(t["q"].cpu(), t["k"].cpu(), t["v"].cpu(), False, sc)
    assert_fwd_close(o.cpu(), lse.cpu(), o_ref, l_ref, f"merged halves d={d}")


def test_merge_handles_empty_rows(cuda_device):
    """lse = -inf on both sides keeps O = 0 and lse = -inf; on one side takes the other."""
    rows, d = 64, 64
    acc = torch.zeros((1, 1, rows, d), dtype=torch.float32, device=cuda_device)
    lse = torch.full((1, 1, rows), -math.inf, dtype=torch.float32, device=cuda_device)
    part = torch.randn((1, 1, rows, d), device=cuda_device).to(torch.bfloat16)
    lp = torch.full((1, 1, rows), -math.inf, dtype=torch.float32, device=cuda_device)
    lp[..., ::2] = 1.5
    fa.merge_partial(acc, lse, part, lp)
    torch.cuda.synchronize()
    assert torch.all(acc[..., 1::2, :] == 0) and torch.all(torch.isneginf(lse[..., 1::2]))
    assert torch.equal(acc[..., ::2, :], part[..., ::2, :].float()) and torch.all(lse[..., ::2] == 1.5)


def test_accumulate_and_convert(cuda_device):
    x = torch.randn(4096, device=cuda_device).to(torch.bfloat16)
    acc = torch.full((4096,), 2.0, device=cuda_device)
    fa.accumulate_bf16(acc, x)
    assert torch.equal(acc, 2.0 + x.float())
    fa.accumulate_bf16(acc, x, overwrite=True)
    assert torch.equal(acc, x.float())
    y = torch.randn(4096, device=cuda_device)
    assert torch.equal(fa.to_bf16(y), y.to(torch.bfloat16))
