"""Sequence-parallel attention over a ring of ranks (one process per GPU).

The sequence of N positions is split into R equal blocks, rank r holding block r of
Q, K, V (and of dO, O, lse in the backward). The method's online softmax combines
partial results over key tiles through their log-sum-exp; here the same combination
runs over key BLOCKS that travel around the ring:

forward, rank r, steps s = 0 .. R-1 (block src = (r - s) mod R held at step s):
    partial (O_s, lse_s) = attention(Q_r, K_src, V_src)   [library forward kernel]
    (O, lse) <- merge((O, lse), (O_s, lse_s))             [library merge kernel]
    send (K_src, V_src) to rank r + 1, receive the next block from rank r - 1
With the causal mask (global positions), block src is skipped when src > r and is
the causal diagonal when src = r; earlier blocks are fully visible.

backward, rank r: the pre-pass forms D_r = rowsum(dO_r * O_r) and lse_r for the
rank's queries once (global O and lse, so each block's P = exp(S - lse) is the
block's share of the full softmax). At step s the dK/dV and dQ kernels give the
block's shares of dQ_r, dK_src, dV_src; dQ_r is accumulated locally, the dK, dV
shares are added into fp32 accumulators that travel with the block, and after R
steps each block's accumulators arrive back at their owner.

Transfers use torch.distributed point-to-point operations (NCCL over NVLink for CUDA
tensors), issued as one batch per step so that the sends and receives of a ring
step cannot deadlock; the next block's K/V transfer overlaps the current block's
kernels. Every step of the arithmetic runs in the library's kernels; this module
only orders calls and moves tensors.
"""
from __future__ import annotations

import math

__all__ = ["ProcessGroupRing", "CudaBlockOps", "ring_forward", "ring_backward", "ring_attention"]


class ProcessGroupRing:
    """Ring neighbours in a torch.distributed process group."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def _peer(self, r):
        import torch.distributed as dist
        r %= self.world
        return r if self.group is None else dist.get_global_rank(self.group, r)

    def start(self, tensors):
        """Send `tensors` to rank + 1 and receive tensors of the same shapes from rank - 1;
        returns a handle for ``finish``."""
        import torch
        import torch.distributed as dist
        recv = [torch.empty_like(t) for t in tensors]
        ops = [dist.P2POp(dist.isend, t, self._peer(self.rank + 1), self.group) for t in tensors]
        ops += [dist.P2POp(dist.irecv, t, self._peer(self.rank - 1), self.group) for t in recv]
        return dist.batch_isend_irecv(ops), recv

    def finish(self, handle):
        reqs, recv = handle
        for q in reqs:
            q.wait()
        return recv

    def exchange(self, tensors):
        return self.finish(self.start(tensors))


class CudaBlockOps:
    """The per-block steps, each a call into the library."""

    def __init__(self, scale):
        self.scale = scale

    def new_acc(self, q):
        import torch
        B, H, N, d = q.shape
        return (torch.zeros((B, H, N, d), dtype=torch.float32, device=q.device),
                torch.full((B, H, N), -math.inf, dtype=torch.float32, device=q.device))

    def fwd_block(self, q, k, v, causal):
        from . import forward
        return forward(q, k, v, causal=causal, scale=self.scale)

    def merge(self, acc, part):
        from . import merge_partial
        merge_partial(acc[0], acc[1], part[0], part[1])

    def finish_o(self, acc):
        from . import to_bf16
        return to_bf16(acc[0]), acc[1]

    def bwd_prepare(self, q, o, lse, do):
        import torch
        from . import bwd_preprocess, bwd_workspace_bytes
        B, H, N, d = q.shape
        ws = torch.empty(bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=q.device)
        bwd_preprocess(o, do, lse, ws)
        return {"ws": ws, "dq": torch.empty_like(q), "dk": torch.empty_like(q), "dv": torch.empty_like(q)}

    def bwd_block(self, state, q, k, v, do, causal):
        from . import bwd_dkdv, bwd_dq
        bwd_dkdv(q, k, v, do, state["dk"], state["dv"], state["ws"], causal=causal, scale=self.scale)
        bwd_dq(q, k, v, do, state["dq"], state["ws"], causal=causal, scale=self.scale)
        return state["dq"], state["dk"], state["dv"]

    def zeros_f32(self, x):
        import torch
        return torch.zeros(x.shape, dtype=torch.float32, device=x.device)

    def accumulate(self, acc, x):
        from . import accumulate_bf16
        accumulate_bf16(acc, x)

    def to_out(self, acc):
        from . import to_bf16
        return to_bf16(acc)


def _visible(causal, src, r):
    return (not causal) or src <= r


def _check_block_shapes(q, k, v, ops):
    """Reject, before any exchange is posted, what the library's per-block steps cannot
    take: the merge kernel handles head dims 64 and 128 only (the attention kernels also
    take 96), and every rank's key block must have the query block's shape."""
    if tuple(k.shape) != tuple(q.shape) or tuple(v.shape) != tuple(q.shape):
        raise ValueError("the ring needs q, k, v blocks of one shape [B, H, n, d]")
    if isinstance(ops, CudaBlockOps) and q.shape[-1] not in (64, 128):
        raise ValueError(f"head dim {q.shape[-1]}: the ring's merge step supports head dims 64 and 128")


def ring_forward(q, k, v, causal=False, scale=None, ring=None, ops=None):
    """(O_r, lse_r) for this rank's query block against every rank's key block.
    q, k, v: this rank's [B, H, n, d] blocks (n equal on all ranks)."""
    ring = ProcessGroupRing() if ring is None else ring
    ops = CudaBlockOps(1.0 / math.sqrt(q.shape[-1]) if scale is None else scale) if ops is None else ops
    _check_block_shapes(q, k, v, ops)
    R, r = ring.world, ring.rank
    acc = ops.new_acc(q)
    kv = [k, v]
    for s in range(R):
        src = (r - s) % R
        pending = ring.start(kv) if s < R - 1 else None  # the next block travels meanwhile
        if _visible(causal, src, r):
            ops.merge(acc, ops.fwd_block(q, kv[0], kv[1], causal and src == r))
        if pending is not None:
            kv = ring.finish(pending)
    return ops.finish_o(acc)


def ring_backward(q, k, v, o, lse, do, causal=False, scale=None, ring=None, ops=None):
    """(dQ_r, dK_r, dV_r) for this rank's blocks, given the ring forward's O_r, lse_r."""
    ring = ProcessGroupRing() if ring is None else ring
    ops = CudaBlockOps(1.0 / math.sqrt(q.shape[-1]) if scale is None else scale) if ops is None else ops
    _check_block_shapes(q, k, v, ops)
    R, r = ring.world, ring.rank
    state = ops.bwd_prepare(q, o, lse, do)
    dq = ops.zeros_f32(q)
    kv = [k, v]
    dkv = [ops.zeros_f32(k), ops.zeros_f32(v)]  # accumulators of the block held at step 0 (own)
    moving = None  # accumulators in flight to rank r + 1 (this step's arrive from rank r - 1)
    for s in range(R):
        src = (r - s) % R
        pending = ring.start(kv) if s < R - 1 else None
        shares = None
        if _visible(causal, src, r):
            shares = ops.bwd_block(state, q, kv[0], kv[1], do, causal and src == r)
            ops.accumulate(dq, shares[0])
        # The accumulators of block src travel with it: they arrive while this block's
        # kernels run, take its shares, and leave for the next rank; after the last
        # step that hop takes every block's accumulators home.
        if moving is not None:
            dkv = ring.finish(moving)
        if shares is not None:
            ops.accumulate(dkv[0], shares[1])
            ops.accumulate(dkv[1], shares[2])
        if R > 1:
            moving = ring.start(dkv)
        if pending is not None:
            kv = ring.finish(pending)
    if moving is not None:
        dkv = ring.finish(moving)
    return ops.to_out(dq), ops.to_out(dkv[0]), ops.to_out(dkv[1])


def _autograd_fn():
    import torch

    class _Ring(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v, causal, scale, ring, ops):
            o, lse = ring_forward(q, k, v, causal, scale, ring, ops)
            ctx.save_for_backward(q, k, v, o, lse)
            ctx.causal, ctx.scale, ctx.ring, ctx.ops = causal, scale, ring, ops
            return o

        @staticmethod
        def backward(ctx, do):
            q, k, v, o, lse = ctx.saved_tensors
            dq, dk, dv = ring_backward(q, k, v, o, lse, do.contiguous(), ctx.causal, ctx.scale, ctx.ring, ctx.ops)
            return dq, dk, dv, None, None, None, None

    return _Ring


_RING = None


def ring_attention(q, k, v, causal=False, scale=None, ring=None, ops=None):
    """Differentiable sequence-parallel attention over the ranks of `ring` (default: the
    default process group); q, k, v are this rank's [B, H, n, d] sequence blocks. `ops`
    are the per-block steps (default: the library's kernels)."""
    global _RING
    if _RING is None:
        _RING = _autograd_fn()
    return _RING.apply(q, k, v, bool(causal), scale, ProcessGroupRing() if ring is None else ring, ops)
