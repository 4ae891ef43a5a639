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


def _run_ring(q, k, v, do, world, causal, scale, zigzag=False):
    """The ring's outputs, put back in global row order."""
    n = q.shape[2] // world
    rows = {r: (np.concatenate([np.arange(o, o + n // 2) for o in ring.chunk_offsets(r, world, n, True)])
                if zigzag else np.arange(r * n, (r + 1) * n)) for r in range(world)}
    blk = lambda x, r: x[:, :, torch.as_tensor(rows[r], device=x.device)].contiguous()
    inboxes = [queue.Queue() for _ in range(world)]
    res, errs = {}, []

    def rank_main(r):
        try:
            rg = ThreadRing(r, world, inboxes)
            o, lse = ring.ring_forward(blk(q, r), blk(k, r), blk(v, r), causal, scale, rg, zigzag=zigzag)
            g = ring.ring_backward(blk(q, r), blk(k, r), blk(v, r), o, lse, blk(do, r), causal, scale, rg,
                                   zigzag=zigzag)
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
    order = torch.as_tensor(np.argsort(np.concatenate([rows[r] for r in range(world)])), device=q.device)
    cat = lambda i: torch.cat([res[r][i] for r in range(world)], dim=2)[:, :, order]
    return [cat(i) for i in range(5)]


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal,zigzag", [(False, False), (True, False), (True, True)])
def test_ring_parity(cuda_device, world, d, causal, zigzag):
    B, H, n = 1, 2, 256
    N = world * n
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=40 + world + d).items()}
    sc = 1.0 / math.sqrt(d)
    o, lse, dq, dk, dv = _run_ring(t["q"], t["k"], t["v"], t["do"], world, causal, sc, zigzag)
    assert fa.device_status() == (0, 0)
    ref = oracle.attn_bwd_ref(t["q"].cpu(), t["k"].cpu(), t["v"].cpu(), t["do"].cpu(), causal, sc)
    what = f"ring R={world} d={d} causal={causal}"
    assert_fwd_close(o.cpu(), lse.cpu(), ref["o"], ref["lse"], what)
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert_grad_close(g.cpu(), ref[name], name, what)


@pytest.mark.parametrize("causal,zigzag", [(True, False), (True, True), (False, False)])
def test_ring_eight_ranks_long_blocks(cuda_device, causal, zigzag):
    """R = 8 ranks of 1024 positions each (N = 8192), d = 128: the whole sequence against
    the oracle; the fp32 accumulation of partial results keeps the error within the
    single-GPU tolerances."""
    world, B, H, n, d = 8, 1, 2, 1024, 128
    N = world * n
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=48).items()}
    sc = 1.0 / math.sqrt(d)
    o, lse, dq, dk, dv = _run_ring(t["q"], t["k"], t["v"], t["do"], world, causal, sc, zigzag)
    assert fa.device_status() == (0, 0)
    c = {k: x.cpu() for k, x in t.items()}
    for h in range(H):
        ref = oracle.attn_bwd_ref(c["q"][:, h:h + 1], c["k"][:, h:h + 1], c["v"][:, h:h + 1], c["do"][:, h:h + 1],
                                  causal, sc)
        what = f"ring R=8 n=1024 causal={causal} zigzag={zigzag} h={h}"
        assert_fwd_close(o[:, h:h + 1].cpu(), lse[:, h:h + 1].cpu(), ref["o"], ref["lse"], what)
        for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
            assert_grad_close(g[:, h:h + 1].cpu(), ref[name], name, what)


@pytest.mark.parametrize("d", [64, 128])
def test_forward_merge_of_key_blocks(cuda_device, d):
    """The merging forward over four key blocks (one on the causal diagonal) equals causal
    attention of the last query block over all keys; rows are merged in fp32."""
    B, H, c = 2, 3, 256
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, 4 * c, d, seed=8, with_do=False).items()}
    sc = 1.0 / math.sqrt(d)
    q = t["q"][:, :, 3 * c:].contiguous()
    acc = torch.zeros(q.shape, dtype=torch.float32, device=cuda_device)
    lse = torch.full(q.shape[:3], -math.inf, dtype=torch.float32, device=cuda_device)
    for b in range(4):
        sl = slice(b * c, (b + 1) * c)
        fa.forward_merge(q, t["k"][:, :, sl].contiguous(), t["v"][:, :, sl].contiguous(), acc, lse, causal=b == 3,
                         scale=sc)
    torch.cuda.synchronize()
    assert fa.device_status() == (0, 0)
    rows = np.arange(3 * c, 4 * c)
    for bb in range(B):
        for h in range(H):
            o_ref, l_ref = oracle.attn_fwd_rows_ref(t["q"][bb, h].cpu()[3 * c:], rows, t["k"][bb, h].cpu(),
                                                    t["v"][bb, h].cpu(), True, sc)
            assert_fwd_close(acc[bb, h].cpu().numpy(), lse[bb, h].cpu().numpy(), o_ref, l_ref, f"merge d={d}")


@pytest.mark.parametrize("d", [64, 128])
def test_fused_f32_shares_sum_to_full(cuda_device, d):
    """The sequence split into two halves: for every (query half, key half) pair the fused
    kernel's fp32 dK, dV shares (with the whole sequence's row statistics), summed in fp32
    over the query halves, and the dQ shares added in each query half's accumulator, give
    the full gradients."""
    B, H, N = 1, 2, 512
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=9).items()}
    sc = 1.0 / math.sqrt(d)
    o, lse = fa.forward(t["q"], t["k"], t["v"], scale=sc)
    half = lambda x, a: x[:, :, a * (N // 2):(a + 1) * (N // 2)].contiguous()
    wss = []
    for a in range(2):
        ws = torch.empty(fa.bwd_workspace_bytes(B, H, N // 2, d, deterministic=False), dtype=torch.uint8,
                         device=cuda_device)
        fa.bwd_fused_preprocess(half(o, a), half(t["do"], a), half(lse, a), ws)
        wss.append(ws)
    acc = {n: [torch.zeros((B, H, N // 2, d), dtype=torch.float32, device=cuda_device) for _ in range(2)]
           for n in ("dk", "dv")}
    for a in range(2):
        for b in range(2):
            dk, dv = (torch.empty((B, H, N // 2, d), dtype=torch.float32, device=cuda_device) for _ in range(2))
            fa.bwd_fused_main_f32(half(t["q"], a), half(t["k"], b), half(t["v"], b), half(t["do"], a), dk, dv, wss[a],
                                  scale=sc)
            fa.accumulate_f32(acc["dk"][b], dk)
            fa.accumulate_f32(acc["dv"][b], dv)
    dqs = []
    for a in range(2):
        dq = torch.empty((B, H, N // 2, d), dtype=torch.bfloat16, device=cuda_device)
        fa.bwd_fused_dq(dq, wss[a], scale=sc)
        dqs.append(dq)
    torch.cuda.synchronize()
    assert fa.device_status() == (0, 0)
    ref = oracle.attn_bwd_ref(t["q"].cpu(), t["k"].cpu(), t["v"].cpu(), t["do"].cpu(), False, sc)
    assert_grad_close(torch.cat(dqs, dim=2).cpu(), ref["dq"], "dq", f"fp32 shares d={d}")
    assert_grad_close(torch.cat(acc["dk"], dim=2).cpu().numpy(), ref["dk"], "dk", f"fp32 shares d={d}")
    assert_grad_close(torch.cat(acc["dv"], dim=2).cpu().numpy(), ref["dv"], "dv", f"fp32 shares d={d}")


def test_accumulate_f32(cuda_device):
    a = torch.randn(4096, device=cuda_device)
    x = torch.randn(4096, device=cuda_device)
    ref = a + x
    fa.accumulate_f32(a, x)
    assert torch.equal(a, ref)


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
