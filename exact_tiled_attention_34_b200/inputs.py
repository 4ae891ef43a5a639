"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no attention arithmetic: it only draws random tensors and
names the workload shapes, so that the oracle and the CUDA path are fed the
very same bf16 values.

Recipe (one CPU ``torch.Generator`` per workload):
  * Q, K, V, dO are drawn in that order with ``torch.randn((B, H, N, d))`` in
    float32 from ``manual_seed(seed)``; dO is multiplied by ``do_scale`` (0.5 for
    the sequence-length sweep); each is then rounded to bfloat16 (nearest-even).
  * The block-sparse tile mask uses a separate generator seeded with ``seed + 1``:
    ``rand(nT, nT) < density`` with the diagonal forced to 1, stored as uint8
    [nT, nT] (1 = keep), shared by every (batch, head).
"""
from __future__ import annotations

import torch

# Workload shapes. "sweep" expands to the sequence-length sweep with B*N = 16384
# tokens and H = 2048 / d heads.
WORKLOADS = {
    "pr1": dict(B=1, H=2, N=128, d=64, causal=(False,), backward=False),
    "b8h16n2048d64": dict(B=8, H=16, N=2048, d=64, causal=(False, True), backward=True),
    "b2h16n8192d128_causal": dict(B=2, H=16, N=8192, d=128, causal=(True,), backward=True),
    "b1h16n16384d64_sparse": dict(B=1, H=16, N=16384, d=64, causal=(False,), backward=True,
                                  sparse_density=0.25),
    # Sequence lengths that are not a multiple of the 128-row tile (last tile partial).
    "b8h16n2000d64_ragged": dict(B=8, H=16, N=2000, d=64, causal=(False, True), backward=True),
    "b2h16n8000d128_ragged_causal": dict(B=2, H=16, N=8000, d=128, causal=(True,), backward=True),
    # Different query and key lengths: 512 new queries against 8192 keys (chunked
    # prefill), causal mask aligned bottom-right.
    "b4h16q512k8192d128_causal": dict(B=4, H=16, N=512, Nk=8192, d=128, causal=(True,), backward=True),
    # Head dim 96 (runs on the 128-wide kernels).
    "b4h16n4096d96": dict(B=4, H=16, N=4096, d=96, causal=(False, True), backward=True),
    # Head dim 256 (kernels of its own; the fused backward only).
    "b2h8n8192d256": dict(B=2, H=8, N=8192, d=256, causal=(False, True), backward=True),
    # Dropout on the probabilities (p = 0.1) on the shapes above.
    "b8h16n2048d64_dropout": dict(B=8, H=16, N=2048, d=64, causal=(False, True), backward=True, dropout_p=0.1),
    "b2h16n8192d128_causal_dropout": dict(B=2, H=16, N=8192, d=128, causal=(True,), backward=True,
                                          dropout_p=0.1),
}

SWEEP_N = (512, 1024, 2048, 4096, 8192, 16384)
SWEEP_D = (64, 128)


def sweep_shape(N: int, d: int):
    """(B, H) of the sweep point at sequence length N and head dim d."""
    return 16384 // N, 2048 // d


def make_qkv(B: int, H: int, N: int, d: int, seed: int = 0, with_do: bool = True,
             do_scale: float = 1.0):
    """Q, K, V (and dO) as contiguous CPU bf16 tensors of shape [B, H, N, d]."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    shape = (B, H, N, d)
    out = {}
    for name in ("q", "k", "v"):
        out[name] = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    if with_do:
        do = torch.randn(shape, generator=g, dtype=torch.float32)
        if do_scale != 1.0:
            do = do * do_scale
        out["do"] = do.to(torch.bfloat16)
    return out


def make_tile_mask(n_tiles: int, seed: int = 0, density: float = 0.25) -> torch.Tensor:
    """uint8 [n_tiles, n_tiles] Bernoulli(density) keep-mask with the diagonal kept."""
    g = torch.Generator(device="cpu").manual_seed(seed + 1)
    m = torch.rand((n_tiles, n_tiles), generator=g) < density
    m.fill_diagonal_(True)
    return m.to(torch.uint8).contiguous()
