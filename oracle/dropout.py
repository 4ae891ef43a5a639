"""Plain fp64 CPU oracle for attention with dropout on the attention probabilities.

TEST INFRASTRUCTURE ONLY (same rules as ``oracle.attention``): only the tests, the
smoke check and the CPU legs of ``bench.py`` may import it; it shares nothing with
the CUDA library.

The pages name dropout only in passing, as one of the O(N^2) element-wise operations
of standard attention next to scaling, masking and softmax (the PagedAttention page,
section on bandwidth constraints). Everything below is this library's reading of
that one word, the usual one for attention dropout:

    P       = softmax_rows(S)                      (as without dropout; lse unchanged)
    P~_ij   = P_ij * M_ij / q_keep                  (M_ij in {0, 1}: keep or drop)
    O       = P~ V

and for L = sum(O * dO):

    dV = P~^T dO,   dP~ = dO V^T,   dP_ij = dP~_ij * M_ij / q_keep,
    D_i = sum_j P_ij dP_ij   (= sum_c dO_ic O_ic, since O = P~ V),
    dS = P * (dP - D),   dQ = scale dS K,   dK = scale dS^T Q.

The keep mask M is a function of (batch*head, query row, key column, seed, offset)
only, drawn from the Philox4x32-10 counter-based generator (Salmon, Moraes, Dror and
Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011), so that a forward and
its backward see the same mask without storing it:

  * one Philox call covers a 4 x 4 block of the score matrix: counter
    (key column // 4, query row // 4, b * H + h, offset), key (seed mod 2^32,
    seed // 2^32);
  * output word w (of four 32-bit words) belongs to query row 4 * (i // 4) + w, and
    byte e of that word (least significant first) to key column 4 * (j // 4) + e;
  * an element is kept iff its byte is below the keep threshold t = round(256 q_keep)
    with q_keep = 1 - p requested; the keep probability is then exactly t / 256 and
    the kept entries are scaled by 256 / t (so the drop probability is p rounded to a
    multiple of 1/256; t must be at least 1).

Parity status: pinned by tests/test_oracle_dropout.py (the generator against its
published known-answer vectors; the mask layout against a scalar re-derivation; p = 0
against plain attention; keep statistics; finite differences of the loss with the
mask held fixed; the expectation over seeds; single-head slices against the full
problem).
"""
from __future__ import annotations

import numpy as np

from .attention import _f64, _softmax_rows, attn_scores_ref

__all__ = [
    "philox4x32_10",
    "keep_threshold",
    "dropout_keep_mask",
    "attn_dropout_fwd_ref",
    "attn_dropout_bwd_ref",
]

_M32 = np.uint64(0xFFFFFFFF)
# Philox4x32 multipliers and Weyl key increments (the SC 2011 paper, section on Philox).
_MUL0, _MUL1 = np.uint64(0xD2511F53), np.uint64(0xCD9E8D57)
_WEYL0, _WEYL1 = np.uint64(0x9E3779B9), np.uint64(0xBB67AE85)


def philox4x32_10(ctr, key):
    """Philox4x32 with 10 rounds, element-wise over arrays.

    ctr: four arrays (or ints) of 32-bit counter words; key: two 32-bit key words.
    Each round multiplies counter words 0 and 2 by the two multipliers (full 64-bit
    products split into high and low halves) and mixes the high halves with words 1
    and 3 and the round key; the key advances by the Weyl increments between rounds.
    Returns the four output words as uint64 arrays holding 32-bit values.
    """
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & _M32 for c in ctr)
    k0, k1 = (np.asarray(k, dtype=np.uint64) & _M32 for k in key)
    for r in range(10):
        if r > 0:
            k0 = (k0 + _WEYL0) & _M32
            k1 = (k1 + _WEYL1) & _M32
        p0 = _MUL0 * c0  # < 2^64: exact in uint64
        p1 = _MUL1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _M32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _M32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def keep_threshold(p: float) -> int:
    """Keep threshold t = round(256 (1 - p)) for drop probability p (0 <= p < 1);
    raises ValueError when t would be 0 (nothing kept) or p is out of range."""
    p = float(p)
    if not (0.0 <= p < 1.0):
        raise ValueError("dropout probability must be in [0, 1)")
    t = int(np.rint(256.0 * (1.0 - p)))
    if t < 1:
        raise ValueError("dropout probability too close to 1 (keep threshold 0)")
    return t


def dropout_keep_mask(B: int, H: int, n_q: int, n_k: int, p: float, seed: int, offset: int = 0,
                      rows=None, bh0: int = 0) -> np.ndarray:
    """Boolean keep mask [B, H, R, n_k] (R = n_q, or len(rows) for the given absolute
    query rows), following the block layout in the module docstring. bh0 is added to
    the head counter b * H + h: a single-head slice of a larger problem passes the
    head's own index b * H + h there."""
    t = keep_threshold(p)
    qi = np.arange(n_q, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    kj = np.arange(n_k, dtype=np.int64)
    bh = int(bh0) + np.arange(B * H, dtype=np.int64).reshape(B, H, 1, 1)
    shape = (B, H, qi.shape[0], n_k)
    c0 = np.broadcast_to((kj // 4)[None, None, None, :], shape)
    c1 = np.broadcast_to((qi // 4)[None, None, :, None], shape)
    c2 = np.broadcast_to(bh, shape)
    c3 = np.full(shape, int(offset) & 0xFFFFFFFF, dtype=np.int64)
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    words = philox4x32_10((c0, c1, c2, c3), (seed & 0xFFFFFFFF, seed >> 32))
    w_idx = np.broadcast_to((qi % 4)[None, None, :, None], shape)
    word = np.choose(w_idx, words)
    byte = (word >> (np.uint64(8) * np.broadcast_to((kj % 4)[None, None, None, :], shape).astype(np.uint64))) \
        & np.uint64(0xFF)
    return byte < np.uint64(t)


def attn_dropout_fwd_ref(q, k, v, p: float, seed: int, offset: int = 0, causal: bool = False,
                         scale: float | None = None, bh0: int = 0):
    """Forward with dropout for q [B, H, N_q, d], k, v [B, H, N_k, d]: (O, lse) in fp64.
    lse is that of the softmax before dropout (what the backward needs). bh0: as for
    ``dropout_keep_mask``."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    n_k = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    t = keep_threshold(p)
    keep = dropout_keep_mask(B, H, N, n_k, p, seed, offset, bh0=bh0)
    o = np.zeros((B, H, N, v.shape[-1]))
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            s = attn_scores_ref(q[b, h], k[b, h], scale, causal)
            pr, l = _softmax_rows(s)
            pd = np.where(keep[b, h], pr * (256.0 / t), 0.0)
            o[b, h] = pd @ v[b, h]
            lse[b, h] = l
    return o, lse


def attn_dropout_bwd_ref(q, k, v, do, p: float, seed: int, offset: int = 0, causal: bool = False,
                         scale: float | None = None, bh0: int = 0):
    """Gradients of L = sum(O * dO) with dropout (the mask fixed by seed and offset).
    Returns dq, dk, dv, the forward's o and lse, and D = sum_j P_ij dP_ij. bh0: as for
    ``dropout_keep_mask``. Also ``pv_abs`` = sum_j P~_ij |V_jc| (P~ the dropped, rescaled
    probabilities), the scale of the rounding error a bf16 P~ puts into O_ic, for the
    tests' element-wise error bounds."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    n_k = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    t = keep_threshold(p)
    keep = dropout_keep_mask(B, H, N, n_k, p, seed, offset, bh0=bh0)
    out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
           "o": np.zeros((B, H, N, v.shape[-1])), "lse": np.zeros((B, H, N)), "D": np.zeros((B, H, N)),
           "pv_abs": np.zeros((B, H, N, v.shape[-1]))}
    for b in range(B):
        for h in range(H):
            s = attn_scores_ref(q[b, h], k[b, h], scale, causal)
            pr, lse = _softmax_rows(s)
            m = np.where(keep[b, h], 256.0 / t, 0.0)
            pd = pr * m
            o = pd @ v[b, h]
            dpd = do[b, h] @ v[b, h].T
            dp = dpd * m
            D = np.sum(pr * dp, axis=1)
            ds = pr * (dp - D[:, None])
            out["dq"][b, h] = scale * (ds @ k[b, h])
            out["dk"][b, h] = scale * (ds.T @ q[b, h])
            out["dv"][b, h] = pd.T @ do[b, h]
            out["o"][b, h] = o
            out["pv_abs"][b, h] = pd @ np.abs(v[b, h])
            out["lse"][b, h] = lse
            out["D"][b, h] = D
    return out
