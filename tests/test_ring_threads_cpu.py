"""The thread-emulated ring used by the GPU ring test, run on CPU with the oracle's
block steps: checks the emulation's message ordering (several transfers in flight,
finished out of order) together with the ring's own logic, for R = 1 .. 4."""
import queue
import threading

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_34_b200 import ring
from tests.test_ring_cpu import OracleBlockOps, zigzag_rows
from tests.test_ring_gpu import ThreadRing


@pytest.mark.parametrize("world", [1, 2, 4, 8])
@pytest.mark.parametrize("causal,zigzag", [(False, False), (True, False), (True, True)])
def test_thread_ring_matches_full_attention(world, causal, zigzag):
    B, H, n, d, scale = 1, 2, 4, 3, 0.9
    N = world * n
    g = torch.Generator().manual_seed(3 + world)
    q, k, v, do = (torch.randn((B, H, N, d), generator=g, dtype=torch.float64) for _ in range(4))
    rows = {r: (zigzag_rows(r, world, n) if zigzag else np.arange(r * n, (r + 1) * n)) for r in range(world)}
    blk = lambda x, r: x[:, :, torch.as_tensor(rows[r])].contiguous()
    inboxes = [queue.Queue() for _ in range(world)]
    res, errs = {}, []

    def rank_main(r):
        try:
            rg = ThreadRing(r, world, inboxes)
            ops = OracleBlockOps(scale)
            o, lse = ring.ring_forward(blk(q, r), blk(k, r), blk(v, r), causal, scale, rg, ops, zigzag)
            res[r] = (o, lse) + tuple(ring.ring_backward(blk(q, r), blk(k, r), blk(v, r), o, lse, blk(do, r),
                                                          causal, scale, rg, ops, zigzag))
        except Exception as e:  # reported below
            errs.append(e)

    ts = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in ts:
        t.start()
    for t in ts:
        t.join(timeout=120)
    assert not errs, errs
    full = oracle.attn_bwd_ref(q, k, v, do, causal, scale)
    for i, name in enumerate(("o", "lse", "dq", "dk", "dv")):
        for r in range(world):
            assert np.max(np.abs(res[r][i].numpy() - full[name][:, :, rows[r]])) < 1e-12, (name, r)
