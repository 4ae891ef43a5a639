"""Helpers shared by the GPU parity tests: tolerances and oracle comparisons.

Tolerances (fixed by the workload definition): max|dO| <= 1e-2 on the bf16 output,
max|dlse| <= 1e-3 on the fp32 log-sum-exp, and for each gradient tensor
max|dg| <= 2e-2 * max|g_oracle|.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_O = 1e-2
TOL_LSE = 1e-3
TOL_GRAD_REL = 2e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def max_abs(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    both_ninf = np.isneginf(a) & np.isneginf(b)
    with np.errstate(invalid="ignore"):
        d = np.where(both_ninf, 0.0, np.abs(a - b))
    return float(np.max(d)) if d.size else 0.0


def tol_o_sharp(v) -> float:
    """O tolerance for stress cases: peaked softmaxes (scales far from 1/sqrt(d)) and
    tensors with many more rows than the workloads, where outputs near max|V| occur.

    O = sum_j P_j V_j / l with P rounded to bf16 and O itself rounded to bf16. bf16 keeps
    8 significant bits (unit roundoff 2^-8), so the P rounding moves O by at most
    2^-8 max|V| and the output rounding by at most 2^-8 |O| <= 2^-8 max|V|: the bound
    is 2^-7 max|V| (plus fp32 terms), and never below the workload tolerance 1e-2.
    """
    vmax = float(v.detach().float().abs().max()) if torch.is_tensor(v) else float(np.max(np.abs(v)))
    return max(TOL_O, 2.0 ** -7 * vmax)


def assert_fwd_close(o_gpu, lse_gpu, o_ref, lse_ref, what="", tol_o=None):
    tol_o = TOL_O if tol_o is None else tol_o
    eo = max_abs(f64(o_gpu) if torch.is_tensor(o_gpu) else o_gpu, o_ref)
    el = max_abs(f64(lse_gpu) if torch.is_tensor(lse_gpu) else lse_gpu, lse_ref)
    assert eo <= tol_o, f"{what}: max|dO| = {eo:.3e} > {tol_o}"
    assert el <= TOL_LSE, f"{what}: max|dlse| = {el:.3e} > {TOL_LSE}"
    return eo, el


def assert_grad_close(g_gpu, g_ref, name, what=""):
    g = f64(g_gpu) if torch.is_tensor(g_gpu) else g_gpu
    scale = float(np.max(np.abs(g_ref)))
    e = max_abs(g, g_ref)
    assert e <= TOL_GRAD_REL * max(scale, 1e-30), f"{what}: max|d{name}| = {e:.3e} > {TOL_GRAD_REL} * {scale:.3e}"
    return e / max(scale, 1e-30)


def sample_rows(N: int, n_random: int = 24, seed: int = 0) -> np.ndarray:
    """Rows at tile boundaries plus random rows (sorted, unique)."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 129, 255, N // 2, N - 129, N - 128, N - 1]
    rows = set(r for r in fixed if 0 <= r < N)
    rows.update(rng.integers(0, N, size=n_random).tolist())
    return np.array(sorted(rows))


def sampled_fwd_check(q, k, v, o, lse, causal, scale, heads, rows, mask=None, what=""):
    """Compare GPU outputs with the oracle on selected (b, h) and rows."""
    mk = None if mask is None else mask.cpu().numpy()
    worst = (0.0, 0.0)
    idx = torch.as_tensor(rows, dtype=torch.long)
    for (b, h) in heads:
        qh = f64(q[b, h])
        o_ref, l_ref = oracle.attn_fwd_rows_ref(qh[rows], rows, f64(k[b, h]), f64(v[b, h]), causal, scale, mk, 128)
        eo, el = assert_fwd_close(o[b, h][idx], lse[b, h][idx], o_ref, l_ref, f"{what} (b={b}, h={h})")
        worst = (max(worst[0], eo), max(worst[1], el))
    return worst
