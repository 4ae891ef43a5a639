"""Pins of the fp64 oracle to facts outside itself.

Each ``pin_*`` takes an oracle module (the real one, or a deliberately broken copy
in the mutation test) and raises AssertionError when the module disagrees with a
closed form, an invariant, brute force or a library routine. None of them calls the
CUDA library.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _tiny_mask(n, block, seed=3, density=0.5, keep_diag=True):
    nt = (n + block - 1) // block
    m = (np.random.default_rng(seed).random((nt, nt)) < density).astype(np.uint8)
    if keep_diag:
        np.fill_diagonal(m, 1)
    return m


# ---------------------------------------------------------------- forward pins

def pin_probs_rows_sum_to_one(mod):
    """Rows of P are a probability distribution (softmax definition)."""
    q, k = _rand((23, 8), 1), _rand((23, 8), 2)
    for causal, mask in ((False, None), (True, None), (False, _tiny_mask(23, 4))):
        p = mod.attn_probs_ref(q, k, 0.37, causal, mask, 4)
        assert np.all(p >= 0)
        assert np.max(np.abs(p.sum(axis=1) - 1.0)) < 1e-12


def pin_equal_keys_mean_of_v(mod):
    """All keys equal: P is uniform over visible keys, so O is a (cumulative) mean of V
    and lse = scale q.k + ln(#visible)."""
    N, d, scale = 19, 6, 0.5
    q = _rand((1, 1, N, d), 4)
    k = np.tile(_rand((1, d), 5), (N, 1))[None, None]
    v = _rand((1, 1, N, d), 6)
    o, lse = mod.attn_fwd_ref(q, k, v, False, scale)
    assert np.allclose(o[0, 0], np.tile(v[0, 0].mean(axis=0), (N, 1)), atol=1e-12)
    assert np.allclose(lse[0, 0], scale * q[0, 0] @ k[0, 0, 0] + math.log(N), atol=1e-12)
    o, lse = mod.attn_fwd_ref(q, k, v, True, scale)
    cum = np.cumsum(v[0, 0], axis=0) / np.arange(1, N + 1)[:, None]
    assert np.allclose(o[0, 0], cum, atol=1e-12)
    assert np.allclose(lse[0, 0], scale * q[0, 0] @ k[0, 0, 0] + np.log(np.arange(1, N + 1)), atol=1e-12)


def pin_causal_row0(mod):
    """Causal: query 0 sees only key 0, so O_0 = V_0 and lse_0 = scale q_0.k_0."""
    q, k, v = _rand((1, 2, 9, 5), 7), _rand((1, 2, 9, 5), 8), _rand((1, 2, 9, 5), 9)
    o, lse = mod.attn_fwd_ref(q, k, v, True, 0.8)
    assert np.array_equal(o[:, :, 0], v[:, :, 0])
    assert np.allclose(lse[:, :, 0], 0.8 * np.sum(q[:, :, 0] * k[:, :, 0], axis=-1), atol=1e-14)


def pin_n_equals_one(mod):
    """A single token attends to itself only: O = V, lse = scale q.k."""
    q, k, v = _rand((2, 3, 1, 4), 10), _rand((2, 3, 1, 4), 11), _rand((2, 3, 1, 4), 12)
    for causal in (False, True):
        o, lse = mod.attn_fwd_ref(q, k, v, causal, 1.3)
        assert np.array_equal(o, v)
        assert np.allclose(lse, 1.3 * np.sum(q * k, axis=-1)[..., 0:1].reshape(lse.shape), atol=1e-14)


def pin_sparse_all_ones_is_dense(mod):
    """Block-sparse with every tile kept is dense attention, bit for bit."""
    q, k, v = (_rand((1, 2, 16, 4), s) for s in (13, 14, 15))
    ones = np.ones((4, 4), dtype=np.uint8)
    for causal in (False, True):
        o1, l1 = mod.attn_fwd_ref(q, k, v, causal, 0.5)
        o2, l2 = mod.attn_fwd_ref(q, k, v, causal, 0.5, ones, 4)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def pin_sparse_diagonal_is_block_diagonal(mod):
    """A mask keeping only diagonal tiles is independent attention inside each block."""
    T, nt, d = 4, 3, 5
    q, k, v = (_rand((1, 1, T * nt, d), s) for s in (16, 17, 18))
    eye = np.eye(nt, dtype=np.uint8)
    o, lse = mod.attn_fwd_ref(q, k, v, False, 0.6, eye, T)
    for t in range(nt):
        sl = slice(t * T, (t + 1) * T)
        ob, lb = mod.attn_fwd_ref(q[:, :, sl], k[:, :, sl], v[:, :, sl], False, 0.6)
        assert np.allclose(o[:, :, sl], ob, atol=1e-13) and np.allclose(lse[:, :, sl], lb, atol=1e-13)


def pin_sparse_tile_granularity(mod):
    """Brute force: each score is kept iff its tile is kept (checked entry by entry)."""
    T, N = 4, 10
    q, k = _rand((N, 3), 19), _rand((N, 3), 20)
    mask = _tiny_mask(N, T, seed=21)
    mask[1, 2] = 0
    mask[2, 1] = 1
    s = mod.attn_scores_ref(q, k, 1.0, False, mask, T)
    for i in range(N):
        for j in range(N):
            kept = mask[i // T][j // T] != 0
            assert np.isfinite(s[i, j]) == kept
            if kept:
                assert abs(s[i, j] - float(np.dot(q[i], k[j]))) < 1e-12


def pin_shift_invariance(mod):
    """Adding u to every key leaves O unchanged and shifts lse_i by scale q_i.u."""
    q, k, v = (_rand((1, 1, 12, 6), s) for s in (22, 23, 24))
    u = _rand((6,), 25)
    for causal in (False, True):
        o1, l1 = mod.attn_fwd_ref(q, k, v, causal, 0.7)
        o2, l2 = mod.attn_fwd_ref(q, k + u, v, causal, 0.7)
        assert np.allclose(o1, o2, atol=1e-12)
        assert np.allclose(l2 - l1, 0.7 * q[0, 0] @ u, atol=1e-12)


def pin_permutation_invariance(mod):
    """Non-causal attention does not depend on the order of the (key, value) pairs."""
    q, k, v = (_rand((1, 1, 11, 4), s) for s in (26, 27, 28))
    perm = np.random.default_rng(29).permutation(11)
    o1, l1 = mod.attn_fwd_ref(q, k, v, False, 0.9)
    o2, l2 = mod.attn_fwd_ref(q, k[:, :, perm], v[:, :, perm], False, 0.9)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)


def pin_rows_match_full(mod):
    """The sampled-row forward equals the corresponding rows of the full forward."""
    N, T = 16, 4
    q, k, v = (_rand((1, 1, N, 4), s) for s in (30, 31, 32))
    mask = _tiny_mask(N, T, seed=33)
    rows = np.array([0, 3, 4, 9, 15])
    for causal, m in ((False, None), (True, None), (False, mask), (True, mask)):
        o, lse = mod.attn_fwd_ref(q, k, v, causal, 0.4, m, T)
        orow, lrow = mod.attn_fwd_rows_ref(q[0, 0, rows], rows, k[0, 0], v[0, 0], causal, 0.4, m, T)
        assert np.allclose(orow, o[0, 0, rows], atol=1e-13)
        assert np.allclose(lrow, lse[0, 0, rows], atol=1e-13)


def pin_empty_row(mod):
    """A row with no visible key: O = 0, lse = -inf, and it contributes no gradient."""
    T, N = 2, 6
    mask = np.ones((3, 3), dtype=np.uint8)
    mask[1, :] = 0  # rows 2, 3 see nothing
    q, k, v, do = (_rand((1, 1, N, 3), s) for s in (34, 35, 36, 37))
    o, lse = mod.attn_fwd_ref(q, k, v, False, 1.0, mask, T)
    assert np.all(o[0, 0, 2:4] == 0) and np.all(np.isneginf(lse[0, 0, 2:4]))
    assert np.all(np.isfinite(lse[0, 0, [0, 1, 4, 5]]))
    g = mod.attn_bwd_ref(q, k, v, do, False, 1.0, mask, T)
    assert np.all(g["dq"][0, 0, 2:4] == 0)
    p = mod.attn_probs_ref(q[0, 0], k[0, 0], 1.0, False, mask, T)
    assert np.all(p[2:4] == 0)
    assert np.allclose(g["dv"][0, 0], p.T @ do[0, 0], atol=1e-12)


def pin_golden_hand_example(mod):
    """A 2-token example worked out by hand (tests/golden/hand_2x2.json)."""
    with open(os.path.join(GOLDEN, "hand_2x2.json")) as f:
        g = json.load(f)
    q = np.array(g["q"], dtype=np.float64)[None, None]
    k = np.array(g["k"], dtype=np.float64)[None, None]
    v = np.array(g["v"], dtype=np.float64)[None, None]
    for causal in (False, True):
        key = "causal" if causal else "full"
        o, lse = mod.attn_fwd_ref(q, k, v, causal, g["scale"])
        assert np.allclose(o[0, 0], np.array(g[key]["o"]), atol=1e-12), (key, o)
        assert np.allclose(lse[0, 0], np.array(g[key]["lse"]), atol=1e-12), (key, lse)


# ------------------------------------------------------------- library cross-check

def _torch_mask(N, causal, mask, T):
    vis = torch.ones((N, N), dtype=torch.bool)
    if causal:
        vis = torch.tril(vis)
    if mask is not None:
        tm = torch.as_tensor(np.asarray(mask) != 0)
        idx = torch.arange(N) // T
        vis = vis & tm[idx[:, None], idx[None, :]]
    return vis


def pin_sdpa_crosscheck(mod):
    """torch's scaled_dot_product_attention (CPU, float64) and autograd agree with the
    oracle's O, lse (via torch.logsumexp) and all three gradients."""
    B, H, N, d, T = 1, 2, 12, 5, 4
    mask = _tiny_mask(N, T, seed=38)
    for causal, m, scale in ((False, None, 0.45), (True, None, 0.3), (False, mask, 0.6), (True, mask, 1.1)):
        arrs = [_rand((B, H, N, d), s) for s in (39, 40, 41, 42)]
        tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in arrs[:3])
        tdo = torch.tensor(arrs[3], dtype=torch.float64)
        vis = _torch_mask(N, causal, m, T)
        out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=vis, scale=scale)
        (out * tdo).sum().backward()
        s = scale * (tq.detach() @ tk.detach().transpose(-1, -2))
        lse_t = torch.logsumexp(s.masked_fill(~vis, float("-inf")), dim=-1)
        o, lse = mod.attn_fwd_ref(*arrs[:3], causal, scale, m, T)
        g = mod.attn_bwd_ref(*arrs, causal, scale, m, T)
        assert np.allclose(o, out.detach().numpy(), atol=1e-12)
        assert np.allclose(lse, lse_t.numpy(), atol=1e-12)
        assert np.allclose(g["dq"], tq.grad.numpy(), atol=1e-11)
        assert np.allclose(g["dk"], tk.grad.numpy(), atol=1e-11)
        assert np.allclose(g["dv"], tv.grad.numpy(), atol=1e-11)


# ------------------------------------------------------------------ backward pins

def _loss(mod, q, k, v, do, causal, scale, mask, T):
    o, _ = mod.attn_fwd_ref(q, k, v, causal, scale, mask, T)
    return float(np.sum(o * do))


def pin_finite_differences(mod):
    """Central differences of L = sum(O * dO) (brute force over every input entry)."""
    h = 1e-6
    T = 4
    cases = (
        (4, False, None),
        (7, True, None),
        (8, False, np.array([[1, 0], [1, 1]], dtype=np.uint8)),
        (8, True, np.array([[1, 1], [0, 1]], dtype=np.uint8)),
    )
    for N, causal, mask in cases:
        masked = mask is not None
        q, k, v, do = (_rand((1, 1, N, 4), s) for s in (44, 45, 46, 47))
        scale = 0.55
        g = mod.attn_bwd_ref(q, k, v, do, causal, scale, mask, T)
        for name, x in (("dq", q), ("dk", k), ("dv", v)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp = x.copy()
                xm = x.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p = {"q": q, "k": k, "v": v}
                args_m = {"q": q, "k": k, "v": v}
                args_p[name[1]] = xp
                args_m[name[1]] = xm
                lp = _loss(mod, args_p["q"], args_p["k"], args_p["v"], do, causal, scale, mask, T)
                lm = _loss(mod, args_m["q"], args_m["k"], args_m["v"], do, causal, scale, mask, T)
                num[idx] = (lp - lm) / (2 * h)
            err = np.max(np.abs(num - g[name])) / max(1e-12, np.max(np.abs(num)))
            assert err < 1e-6, (name, N, causal, masked, err)


def pin_D_two_ways(mod):
    """D_i = sum_j P_ij dP_ij equals sum_c dO_ic O_ic (gradient identity)."""
    q, k, v, do = (_rand((2, 2, 10, 4), s) for s in (48, 49, 50, 51))
    for causal in (False, True):
        g = mod.attn_bwd_ref(q, k, v, do, causal, 0.5)
        assert np.allclose(g["D"], np.sum(g["o"] * do, axis=-1), atol=1e-12)


def pin_gradient_invariants(mod):
    """Rows of dS sum to zero, so sum_j dK_j = 0; rows of P sum to one, so
    sum_j dV_j = sum_i dO_i (causal or not, any visible set)."""
    q, k, v, do = (_rand((1, 2, 13, 5), s) for s in (52, 53, 54, 55))
    mask = _tiny_mask(13, 4, seed=56)
    for causal, m in ((False, None), (True, None), (False, mask)):
        g = mod.attn_bwd_ref(q, k, v, do, causal, 0.8, m, 4)
        assert np.allclose(g["dk"].sum(axis=2), 0.0, atol=1e-11)
        assert np.allclose(g["dv"].sum(axis=2), do.sum(axis=2), atol=1e-11)


def pin_dq_rows_match_full(mod):
    """The sampled-row dQ equals the corresponding rows of the full backward."""
    N, T = 16, 4
    q, k, v, do = (_rand((1, 1, N, 4), s) for s in (57, 58, 59, 60))
    mask = _tiny_mask(N, T, seed=61)
    rows = np.array([0, 2, 5, 8, 15])
    for causal, m in ((False, None), (True, None), (False, mask)):
        g = mod.attn_bwd_ref(q, k, v, do, causal, 0.7, m, T)
        dq = mod.attn_dq_rows_ref(q[0, 0, rows], rows, k[0, 0], v[0, 0], do[0, 0, rows], causal, 0.7, m, T)
        assert np.allclose(dq, g["dq"][0, 0, rows], atol=1e-12)


def pin_dkdv_cols_match_full(mod):
    """The sampled-key dK, dV equal the corresponding rows of the full backward: square
    problems (dense, causal, block mask with an empty tile row, so some rows see nothing)
    and N_q != N_k with the causal mask (more keys than queries, and more queries than
    keys, where the leading rows see nothing); row statistics taken in blocks of 3 rows
    and in one block give the same result."""
    T = 4
    cases = []
    N = 16
    q, k, v, do = (_rand((N, 4), s) for s in (62, 63, 64, 65))
    mask = _tiny_mask(N, T, seed=66)
    mask[1, :] = 0  # query tile 1 sees no key
    cases += [(q, k, v, do, False, None), (q, k, v, do, True, None), (q, k, v, do, False, mask)]
    for nq, nk in ((6, 11), (11, 6)):
        qx, dox = _rand((nq, 4), 67 + nq), _rand((nq, 4), 68 + nq)
        kx, vx = _rand((nk, 4), 69 + nk), _rand((nk, 4), 70 + nk)
        cases.append((qx, kx, vx, dox, True, None))
    for (qq, kk, vv, dd, causal, m) in cases:
        g = mod.attn_bwd_ref(qq[None, None], kk[None, None], vv[None, None], dd[None, None], causal, 0.7, m, T)
        nk = kk.shape[0]
        cols = np.array(sorted({0, 1, nk // 2, nk - 2, nk - 1}))
        for rb in (3, 1024):
            dk, dv = mod.attn_dkdv_cols_ref(qq, kk, vv, dd, cols, causal, 0.7, m, T, row_block=rb)
            assert np.allclose(dk, g["dk"][0, 0, cols], atol=1e-12), (causal, rb)
            assert np.allclose(dv, g["dv"][0, 0, cols], atol=1e-12), (causal, rb)
        dk_all, dv_all = mod.attn_dkdv_cols_ref(qq, kk, vv, dd, np.arange(nk), causal, 0.7, m, T, row_block=5)
        assert np.allclose(dk_all, g["dk"][0, 0], atol=1e-12) and np.allclose(dv_all, g["dv"][0, 0], atol=1e-12)


# ---------------------------------------------------------------- N_q != N_k (bottom-right causal)

def pin_cross_decode_sees_every_key(mod):
    """One query against N_k keys with the causal mask: the last (only) query sees every
    key, so the result is the unmasked one."""
    q, k, v, do = _rand((1, 2, 1, 6), 40), _rand((1, 2, 9, 6), 41), _rand((1, 2, 9, 6), 42), _rand((1, 2, 1, 6), 43)
    oc, lc = mod.attn_fwd_ref(q, k, v, True, 0.6)
    on, ln = mod.attn_fwd_ref(q, k, v, False, 0.6)
    assert np.array_equal(oc, on) and np.array_equal(lc, ln)
    gc, gn = mod.attn_bwd_ref(q, k, v, do, True, 0.6), mod.attn_bwd_ref(q, k, v, do, False, 0.6)
    for name in ("dq", "dk", "dv"):
        assert gc[name].shape == (q.shape if name == "dq" else k.shape)
        assert np.array_equal(gc[name], gn[name])


def pin_cross_is_suffix_of_square(mod):
    """N_q < N_k, causal: the queries are the last N_q rows of a square causal problem
    whose first N_k - N_q query rows are arbitrary. O, lse and dQ are those rows of the
    square problem; dK and dV are the square problem's when the extra rows' dO is 0."""
    nq, nk = 5, 9
    q, k, v = _rand((1, 2, nq, 4), 44), _rand((1, 2, nk, 4), 45), _rand((1, 2, nk, 4), 46)
    do = _rand((1, 2, nq, 4), 47)
    extra = _rand((1, 2, nk - nq, 4), 48)
    qs = np.concatenate([extra, q], axis=2)
    dos = np.concatenate([np.zeros_like(extra), do], axis=2)
    o, lse = mod.attn_fwd_ref(q, k, v, True, 0.9)
    osq, lsq = mod.attn_fwd_ref(qs, k, v, True, 0.9)
    assert np.allclose(o, osq[:, :, nk - nq:], atol=1e-13) and np.allclose(lse, lsq[:, :, nk - nq:], atol=1e-13)
    g, gs = mod.attn_bwd_ref(q, k, v, do, True, 0.9), mod.attn_bwd_ref(qs, k, v, dos, True, 0.9)
    assert np.allclose(g["dq"], gs["dq"][:, :, nk - nq:], atol=1e-12)
    assert np.allclose(g["dk"], gs["dk"], atol=1e-12) and np.allclose(g["dv"], gs["dv"], atol=1e-12)


def pin_cross_more_queries_than_keys(mod):
    """N_q > N_k, causal: query i sees keys j <= i - (N_q - N_k); the first N_q - N_k
    queries see none (O = 0, lse = -inf, dQ = 0) and the rest form the square causal
    problem of the last N_k queries."""
    nq, nk = 9, 4
    q, k, v, do = _rand((1, 1, nq, 3), 49), _rand((1, 1, nk, 3), 50), _rand((1, 1, nk, 3), 51), _rand((1, 1, nq, 3), 52)
    o, lse = mod.attn_fwd_ref(q, k, v, True, 1.1)
    assert np.all(o[:, :, :nq - nk] == 0) and np.all(np.isneginf(lse[:, :, :nq - nk]))
    osq, lsq = mod.attn_fwd_ref(q[:, :, nq - nk:], k, v, True, 1.1)
    assert np.allclose(o[:, :, nq - nk:], osq, atol=1e-13) and np.allclose(lse[:, :, nq - nk:], lsq, atol=1e-13)
    g = mod.attn_bwd_ref(q, k, v, do, True, 1.1)
    gs = mod.attn_bwd_ref(q[:, :, nq - nk:], k, v, do[:, :, nq - nk:], True, 1.1)
    assert np.all(g["dq"][:, :, :nq - nk] == 0) and np.allclose(g["dq"][:, :, nq - nk:], gs["dq"], atol=1e-12)
    assert np.allclose(g["dk"], gs["dk"], atol=1e-12) and np.allclose(g["dv"], gs["dv"], atol=1e-12)


def pin_cross_brute_force(mod):
    """N_q = 3, N_k = 5, causal, written out element by element: key j counts for query
    i when j - i <= N_k - N_q; O_i = sum exp(s_ij) v_j / sum exp(s_ij), lse_i = ln sum."""
    q, k, v = _rand((3, 2), 53), _rand((5, 2), 54), _rand((5, 2), 55)
    sc = 0.7
    o_ref, lse_ref = np.zeros((3, 2)), np.zeros(3)
    for i in range(3):
        num, den = np.zeros(2), 0.0
        for j in range(5):
            if j - i <= 5 - 3:
                e = math.exp(sc * float(q[i] @ k[j]))
                num += e * v[j]
                den += e
        o_ref[i], lse_ref[i] = num / den, math.log(den)
    o, lse = mod.attn_fwd_ref(q[None, None], k[None, None], v[None, None], True, sc)
    assert np.allclose(o[0, 0], o_ref, atol=1e-13) and np.allclose(lse[0, 0], lse_ref, atol=1e-13)


def pin_cross_rows_match_full(mod):
    """Sampled-row forward and dQ of an N_q != N_k causal problem (n_q given) equal the
    full computation's rows."""
    nq, nk = 6, 11
    q, k, v, do = _rand((nq, 4), 56), _rand((nk, 4), 57), _rand((nk, 4), 58), _rand((nq, 4), 59)
    rows = np.array([0, 2, 5])
    o, lse = mod.attn_fwd_ref(q[None, None], k[None, None], v[None, None], True, 0.5)
    orow, lrow = mod.attn_fwd_rows_ref(q[rows], rows, k, v, True, 0.5, n_q=nq)
    assert np.allclose(orow, o[0, 0][rows], atol=1e-13) and np.allclose(lrow, lse[0, 0][rows], atol=1e-13)
    g = mod.attn_bwd_ref(q[None, None], k[None, None], v[None, None], do[None, None], True, 0.5)
    dqr = mod.attn_dq_rows_ref(q[rows], rows, k, v, do[rows], True, 0.5, n_q=nq)
    assert np.allclose(dqr, g["dq"][0, 0][rows], atol=1e-12)


# ---------------------------------------------------------------- key-block pins

def _split(n, sizes):
    out, o = [], 0
    for c in sizes:
        out.append((o, o + c))
        o += c
    assert o == n
    return out


def pin_blocks_merge_to_full(mod):
    """Partial results over a partition of the keys, merged by the textbook log-sum-exp
    rule (weights e^(lse_b - lse)), give the full attention (causal and not)."""
    N, d, scale = 11, 4, 0.6
    q, k, v = (_rand((N, d), s) for s in (81, 82, 83))
    for causal in (False, True):
        o_ref, lse_ref = mod.attn_fwd_ref(q[None, None], k[None, None], v[None, None], causal, scale)
        for q0, q1 in _split(N, (5, 6)):
            parts = [mod.attn_fwd_block_ref(q[q0:q1], k[k0:k1], v[k0:k1], scale, causal, q0, k0)
                     for (k0, k1) in _split(N, (4, 4, 3))]
            lse = np.logaddexp.reduce(np.stack([l for _, l in parts]), axis=0)
            w = [np.where(np.isfinite(l), np.exp(l - lse), 0.0)[:, None] for _, l in parts]
            o = sum(wi * oi for wi, (oi, _) in zip(w, parts))
            assert np.max(np.abs(lse - lse_ref[0, 0, q0:q1])) < 1e-12
            assert np.max(np.abs(o - o_ref[0, 0, q0:q1])) < 1e-12


def pin_block_grads_sum_to_full(mod):
    """Block gradients with the whole row's lse and D: the dQ shares sum to dQ, and each
    block's dK, dV shares summed over the query blocks are that block's rows of dK, dV."""
    N, d, scale = 10, 3, 0.8
    q, k, v, do = (_rand((N, d), s) for s in (84, 85, 86, 87))
    for causal in (False, True):
        full = mod.attn_bwd_ref(q[None, None], k[None, None], v[None, None], do[None, None], causal, scale)
        lse, D = full["lse"][0, 0], full["D"][0, 0]
        dq = np.zeros_like(q)
        dk = np.zeros_like(k)
        dv = np.zeros_like(v)
        for q0, q1 in _split(N, (3, 7)):
            for k0, k1 in _split(N, (6, 4)):
                a, b, c = mod.attn_bwd_block_ref(q[q0:q1], k[k0:k1], v[k0:k1], do[q0:q1], lse[q0:q1], D[q0:q1],
                                                 scale, causal, q0, k0)
                dq[q0:q1] += a
                dk[k0:k1] += b
                dv[k0:k1] += c
        for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
            assert np.max(np.abs(g - full[name][0, 0])) < 1e-12, (name, causal)


def pin_block_above_diagonal_is_empty(mod):
    """With the causal mask a key block entirely after the query block contributes
    nothing: lse -inf, O = 0, zero gradients."""
    q, k, v, do = (_rand((4, 3), s) for s in (88, 89, 90, 91))
    o, lse = mod.attn_fwd_block_ref(q, k, v, 0.5, True, 0, 4)
    assert np.all(np.isneginf(lse)) and np.all(o == 0)
    g = mod.attn_bwd_block_ref(q, k, v, do, np.zeros(4), np.zeros(4), 0.5, True, 0, 4)
    assert all(np.all(x == 0) for x in g)


BLOCK_PINS = [
    pin_blocks_merge_to_full,
    pin_block_grads_sum_to_full,
    pin_block_above_diagonal_is_empty,
]


FORWARD_PINS = [
    pin_probs_rows_sum_to_one,
    pin_equal_keys_mean_of_v,
    pin_causal_row0,
    pin_n_equals_one,
    pin_sparse_all_ones_is_dense,
    pin_sparse_diagonal_is_block_diagonal,
    pin_sparse_tile_granularity,
    pin_shift_invariance,
    pin_permutation_invariance,
    pin_rows_match_full,
    pin_empty_row,
    pin_golden_hand_example,
]
BACKWARD_PINS = [
    pin_sdpa_crosscheck,
    pin_finite_differences,
    pin_D_two_ways,
    pin_gradient_invariants,
    pin_dq_rows_match_full,
    pin_dkdv_cols_match_full,
]
CROSS_PINS = [
    pin_cross_decode_sees_every_key,
    pin_cross_is_suffix_of_square,
    pin_cross_more_queries_than_keys,
    pin_cross_brute_force,
    pin_cross_rows_match_full,
]
ALL_PINS = FORWARD_PINS + BACKWARD_PINS + CROSS_PINS + BLOCK_PINS
