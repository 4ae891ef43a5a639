"""Sequence-parallel attention over a ring of ranks (one process per GPU).

The sequence of N positions is split into R equal blocks, rank r holding block r of
Q, K, V (and of dO, O, lse in the backward). The method's online softmax combines
partial results over key tiles through their log-sum-exp; here the same combination
runs over key BLOCKS that travel around the ring:

forward, rank r, steps s = 0 .. R-1 (block src = (r - s) mod R held at step s):
    (O, lse) <- (O, lse) merged with attention(Q_r, K_src, V_src)   [library kernel:
                the forward's epilogue merges into the running fp32 result]
    send (K_src, V_src) to rank r + 1, receive the next block from rank r - 1
With the causal mask (global positions) a key block after the query block is skipped,
the block on the diagonal uses the causal kernel and an earlier block the full one.

backward, rank r: one pre-pass forms D_r = rowsum(dO_r * O_r) and lse_r for the rank's
queries (from the global O and lse, so each block's P = exp(S - lse) is the block's
share of the full softmax) and zeroes an fp32 dQ accumulator. At step s the fused
backward kernel on (Q_r, K_src, V_src) adds dQ_r's share into that accumulator and
writes the block's dK_src, dV_src shares in fp32; those are added (fp32) into
accumulators that travel with the block, and after R steps each block's accumulators
arrive back at their owner. No partial result is rounded to bf16 before the end.

Causal balance (zigzag=True): with plain blocks rank r has r + 1 visible key blocks, so
the last rank does R times the work of the first. Zig-zag assignment splits the sequence
into 2R chunks and gives rank r chunks r and 2R - 1 - r (its q, k, v are those two
chunks, concatenated along the sequence); every rank then computes the same number of
visible (query chunk, key chunk) pairs.

Transfers use torch.distributed point-to-point operations (NCCL over NVLink for CUDA
tensors), issued as one batch per step so that the sends and receives of a ring step
cannot deadlock; the next block's K/V transfer overlaps the current block's kernels.
Every step of the arithmetic runs in the library's kernels; this module only orders
calls and moves tensors.
"""
from __future__ import annotations

import math

__all__ = ["ProcessGroupRing", "CudaBlockOps", "ring_forward", "ring_backward", "ring_attention", "chunk_offsets"]


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


def _pair_kind(causal, q_off, k_off):
    """How a query chunk sees a key chunk of the same length (chunk starts are multiples of
    the length): 'full', 'diag' (the causal diagonal) or None (no key visible)."""
    if not causal or k_off < q_off:
        return "full"
    return "diag" if k_off == q_off else None


class CudaBlockOps:
    """The per-block steps, each a call into the library."""

    def __init__(self, scale):
        self.scale = scale

    def new_acc(self, q):
        import torch
        B, H, N, d = q.shape
        return (torch.zeros((B, H, N, d), dtype=torch.float32, device=q.device),
                torch.full((B, H, N), -math.inf, dtype=torch.float32, device=q.device))

    def fwd_pair(self, acc, q, k, v, q_off, k_off, causal):
        from . import forward_merge
        kind = _pair_kind(causal, q_off, k_off)
        if kind is not None:
            forward_merge(q, k, v, acc[0], acc[1], causal=kind == "diag", scale=self.scale)

    def finish_o(self, acc):
        from . import to_bf16
        return to_bf16(acc[0]), acc[1]

    def bwd_prepare(self, q, o, lse, do):
        import torch
        from . import bwd_fused_preprocess, bwd_workspace_bytes
        B, H, N, d = q.shape
        ws = torch.empty(bwd_workspace_bytes(B, H, N, d, deterministic=False), dtype=torch.uint8, device=q.device)
        bwd_fused_preprocess(o, do, lse, ws)  # D, lse rows and the zeroed dQ accumulator
        return {"ws": ws, "shape": q.shape, "device": q.device}

    def bwd_pair(self, state, q, k, v, do, q_off, k_off, causal):
        """dK, dV shares (fp32) of key chunk (k, v) from query chunk q; dQ's share goes into
        the state's accumulator. None when no key of the chunk is visible."""
        import torch
        from . import bwd_fused_main_f32
        kind = _pair_kind(causal, q_off, k_off)
        if kind is None:
            return None
        dk = torch.empty(k.shape, dtype=torch.float32, device=k.device)
        dv = torch.empty(v.shape, dtype=torch.float32, device=v.device)
        bwd_fused_main_f32(q, k, v, do, dk, dv, state["ws"], causal=kind == "diag", scale=self.scale)
        return dk, dv

    def finish_dq(self, state):
        import torch
        from . import bwd_fused_dq
        dq = torch.empty(state["shape"], dtype=torch.bfloat16, device=state["device"])
        bwd_fused_dq(dq, state["ws"], scale=self.scale)
        return dq

    def zeros_acc(self, x):
        import torch
        return torch.zeros(x.shape, dtype=torch.float32, device=x.device)

    def accumulate(self, acc, x):
        from . import accumulate_f32
        accumulate_f32(acc, x)

    def to_out(self, acc):
        from . import to_bf16
        return to_bf16(acc)


def chunk_offsets(rank, world, n, zigzag):
    """Global start of each chunk a rank holds (its block is those chunks in order):
    one chunk [r n, (r + 1) n), or with zigzag two of n / 2: chunks r and 2R - 1 - r."""
    if not zigzag:
        return [rank * n]
    c = n // 2
    return [rank * c, (2 * world - 1 - rank) * c]


def _split(x, nch):
    if nch == 1:
        return [x]
    c = x.shape[2] // nch
    return [x[:, :, i * c:(i + 1) * c].contiguous() for i in range(nch)]


def _join(xs):
    import torch
    return xs[0] if len(xs) == 1 else torch.cat(xs, dim=2)


def _check_block_shapes(q, k, v, ops, zigzag):
    """Reject, before any exchange is posted, what the library's per-block steps cannot
    take: the merging forward handles head dims 64 and 128 only (the attention kernels
    also take 96 and 256), every rank's key block must have the query block's shape, and
    zig-zag chunks need an even block length."""
    if tuple(k.shape) != tuple(q.shape) or tuple(v.shape) != tuple(q.shape):
        raise ValueError("the ring needs q, k, v blocks of one shape [B, H, n, d]")
    if isinstance(ops, CudaBlockOps) and q.shape[-1] not in (64, 128):
        raise ValueError(f"head dim {q.shape[-1]}: the ring's merge step supports head dims 64 and 128")
    if zigzag and q.shape[2] % 2:
        raise ValueError("zig-zag chunks need an even block length")


def ring_forward(q, k, v, causal=False, scale=None, ring=None, ops=None, zigzag=False):
    """(O_r, lse_r) for this rank's query block against every rank's key block.
    q, k, v: this rank's [B, H, n, d] blocks (n equal on all ranks; with zigzag the two
    chunks of ``chunk_offsets``, concatenated)."""
    ring = ProcessGroupRing() if ring is None else ring
    ops = CudaBlockOps(1.0 / math.sqrt(q.shape[-1]) if scale is None else scale) if ops is None else ops
    _check_block_shapes(q, k, v, ops, zigzag)
    R, r, n = ring.world, ring.rank, q.shape[2]
    nch = 2 if zigzag else 1
    q_offs = chunk_offsets(r, R, n, zigzag)
    qs = _split(q, nch)
    acc = [ops.new_acc(x) for x in qs]
    kv = _split(k, nch) + _split(v, nch)
    for s in range(R):
        src = (r - s) % R
        pending = ring.start(kv) if s < R - 1 else None  # the next block travels meanwhile
        for a, qo in enumerate(q_offs):
            for b, ko in enumerate(chunk_offsets(src, R, n, zigzag)):
                ops.fwd_pair(acc[a], qs[a], kv[b], kv[nch + b], qo, ko, causal)
        if pending is not None:
            kv = ring.finish(pending)
    outs = [ops.finish_o(x) for x in acc]
    return _join([o for o, _ in outs]), _join([l for _, l in outs])


def ring_backward(q, k, v, o, lse, do, causal=False, scale=None, ring=None, ops=None, zigzag=False):
    """(dQ_r, dK_r, dV_r) for this rank's blocks, given the ring forward's O_r, lse_r."""
    ring = ProcessGroupRing() if ring is None else ring
    ops = CudaBlockOps(1.0 / math.sqrt(q.shape[-1]) if scale is None else scale) if ops is None else ops
    _check_block_shapes(q, k, v, ops, zigzag)
    R, r, n = ring.world, ring.rank, q.shape[2]
    nch = 2 if zigzag else 1
    q_offs = chunk_offsets(r, R, n, zigzag)
    qs, dos = _split(q, nch), _split(do, nch)
    lses = [lse[:, :, i * (n // nch):(i + 1) * (n // nch)].contiguous() for i in range(nch)]
    states = [ops.bwd_prepare(qs[a], x, lses[a], dos[a]) for a, x in enumerate(_split(o, nch))]
    kv = _split(k, nch) + _split(v, nch)
    dkv = [ops.zeros_acc(x) for x in kv]  # accumulators of the block held at step 0 (own)
    moving = None  # accumulators in flight to rank r + 1 (this step's arrive from rank r - 1)
    for s in range(R):
        src = (r - s) % R
        pending = ring.start(kv) if s < R - 1 else None
        shares = []
        for a, qo in enumerate(q_offs):
            for b, ko in enumerate(chunk_offsets(src, R, n, zigzag)):
                sh = ops.bwd_pair(states[a], qs[a], kv[b], kv[nch + b], dos[a], qo, ko, causal)
                if sh is not None:
                    shares.append((b, sh))
        # The accumulators of block src travel with it: they arrive while this block's
        # kernels run, take its shares, and leave for the next rank; after the last
        # step that hop takes every block's accumulators home.
        if moving is not None:
            dkv = ring.finish(moving)
        for b, (dk_s, dv_s) in shares:
            ops.accumulate(dkv[b], dk_s)
            ops.accumulate(dkv[nch + b], dv_s)
        if R > 1:
            moving = ring.start(dkv)
        if pending is not None:
            kv = ring.finish(pending)
    if moving is not None:
        dkv = ring.finish(moving)
    dq = _join([ops.finish_dq(st) for st in states])
    return dq, _join([ops.to_out(x) for x in dkv[:nch]]), _join([ops.to_out(x) for x in dkv[nch:]])


def _autograd_fn():
    import torch

    class _Ring(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v, causal, scale, ring, ops, zigzag):
            o, lse = ring_forward(q, k, v, causal, scale, ring, ops, zigzag)
            ctx.save_for_backward(q, k, v, o, lse)
            ctx.causal, ctx.scale, ctx.ring, ctx.ops, ctx.zigzag = causal, scale, ring, ops, zigzag
            return o

        @staticmethod
        def backward(ctx, do):
            q, k, v, o, lse = ctx.saved_tensors
            dq, dk, dv = ring_backward(q, k, v, o, lse, do.contiguous(), ctx.causal, ctx.scale, ctx.ring, ctx.ops,
                                       ctx.zigzag)
            return dq, dk, dv, None, None, None, None, None

    return _Ring


_RING = None


def ring_attention(q, k, v, causal=False, scale=None, ring=None, ops=None, zigzag=False):
    """Differentiable sequence-parallel attention over the ranks of `ring` (default: the
    default process group); q, k, v are this rank's [B, H, n, d] sequence blocks (with
    zigzag, the rank's two chunks of ``chunk_offsets``). `ops` are the per-block steps
    (default: the library's kernels)."""
    global _RING
    if _RING is None:
        _RING = _autograd_fn()
    return _RING.apply(q, k, v, bool(causal), scale, ProcessGroupRing() if ring is None else ring, ops,
                       bool(zigzag))
