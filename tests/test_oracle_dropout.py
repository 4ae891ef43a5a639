"""Pins of the dropout oracle to facts outside itself, and planted mistakes that the
pins must catch. CPU only: nothing here calls the CUDA library."""
from __future__ import annotations

import json
import math
import os
import types

import numpy as np
import pytest

import oracle
import oracle.dropout as oracle_dropout

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- pins

def pin_philox_known_answers(mod):
    """The generator reproduces the published Philox4x32-10 known-answer vectors."""
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.json")) as f:
        kat = json.load(f)["vectors"]
    for v in kat:
        ctr = [int(x, 16) for x in v["ctr"]]
        key = [int(x, 16) for x in v["key"]]
        out = [int(w) for w in mod.philox4x32_10(ctr, key)]
        assert out == [int(x, 16) for x in v["out"]], (v, [hex(w) for w in out])


def pin_golden_4x4(mod):
    """Hand-worked example: the 4 x 4 block of counter 0 (keep mask read off the first
    known-answer vector), uniform scores and V = I, so O = (256 / t) P * mask."""
    with open(os.path.join(GOLDEN, "dropout_4x4.json")) as f:
        g = json.load(f)
    keep = np.array(g["keep"], dtype=bool)
    got = mod.dropout_keep_mask(1, 1, 4, 4, g["p"], g["seed"], g["offset"])[0, 0]
    assert np.array_equal(got, keep)
    z = np.zeros((1, 1, 4, 4))
    v = np.eye(4).reshape(1, 1, 4, 4)
    o, lse = mod.attn_dropout_fwd_ref(z, z, v, g["p"], g["seed"], g["offset"])
    assert np.max(np.abs(o[0, 0] - keep * (g["o_scale_num"] / g["o_scale_den"]))) < 1e-15
    assert np.max(np.abs(lse - math.log(4.0))) < 1e-15


def _philox_scalar(c, k):
    """Independent scalar Philox4x32-10 on Python integers (SC 2011 paper's round)."""
    c = list(c)
    k0, k1 = k
    for r in range(10):
        if r:
            k0, k1 = (k0 + 0x9E3779B9) & 0xFFFFFFFF, (k1 + 0xBB67AE85) & 0xFFFFFFFF
        p0, p1 = 0xD2511F53 * c[0], 0xCD9E8D57 * c[2]
        c = [((p1 >> 32) ^ c[1] ^ k0) & 0xFFFFFFFF, p1 & 0xFFFFFFFF,
             ((p0 >> 32) ^ c[3] ^ k1) & 0xFFFFFFFF, p0 & 0xFFFFFFFF]
    return c


def pin_mask_layout(mod):
    """Every element of the mask is the stated byte of the stated Philox call:
    counter (j // 4, i // 4, b H + h, offset), word i % 4, byte j % 4."""
    B, H, N, Nk, p, seed, off = 2, 3, 9, 7, 0.4, 0x1234_5678_9ABC_DEF1, 77
    t = round(256 * (1 - p))
    m = mod.dropout_keep_mask(B, H, N, Nk, p, seed, off)
    assert m.shape == (B, H, N, Nk)
    for b in range(B):
        for h in range(H):
            for i in range(N):
                for j in range(Nk):
                    w = _philox_scalar((j // 4, i // 4, b * H + h, off), (seed & 0xFFFFFFFF, seed >> 32))
                    byte = (w[i % 4] >> (8 * (j % 4))) & 0xFF
                    assert bool(m[b, h, i, j]) == (byte < t), (b, h, i, j)
    # sampled rows give the same mask rows
    rows = np.array([8, 0, 5])
    assert np.array_equal(mod.dropout_keep_mask(B, H, N, Nk, p, seed, off, rows=rows), m[:, :, rows])
    # a single-head slice with its head index gives that head's mask
    for b in range(B):
        for h in range(H):
            one = mod.dropout_keep_mask(1, 1, N, Nk, p, seed, off, bh0=b * H + h)
            assert np.array_equal(one[0, 0], m[b, h])


def pin_p_zero_is_plain_attention(mod):
    """p = 0 keeps everything with scale 1: the result is plain attention."""
    q, k, v, do = (_rand((2, 2, 11, 5), s) for s in (1, 2, 3, 4))
    for causal in (False, True):
        o, lse = mod.attn_dropout_fwd_ref(q, k, v, 0.0, 99, 3, causal, 0.4)
        o_ref, lse_ref = oracle.attn_fwd_ref(q, k, v, causal, 0.4)
        assert np.max(np.abs(o - o_ref)) < 1e-13 and np.max(np.abs(lse - lse_ref)) < 1e-13
        g = mod.attn_dropout_bwd_ref(q, k, v, do, 0.0, 99, 3, causal, 0.4)
        r = oracle.attn_bwd_ref(q, k, v, do, causal, 0.4)
        for name in ("dq", "dk", "dv", "o", "lse", "D"):
            assert np.max(np.abs(g[name] - r[name])) < 1e-12, name


def pin_keep_rate(mod):
    """Bytes of a good generator are uniform: the kept fraction is t / 256 (within
    4.5 standard deviations), masks for different seeds or offsets are independent,
    and a block's 16 bytes are not correlated with its neighbours'."""
    B, H, N = 2, 3, 256
    n = B * H * N * N
    for p in (0.1, 0.5, 0.9):
        t = round(256 * (1 - p))
        qk = t / 256
        m = mod.dropout_keep_mask(B, H, N, N, p, 2024, 0)
        sd = math.sqrt(qk * (1 - qk) / n)
        assert abs(m.mean() - qk) < 4.5 * sd, (p, m.mean(), qk)
        m2 = mod.dropout_keep_mask(B, H, N, N, p, 2025, 0)
        m3 = mod.dropout_keep_mask(B, H, N, N, p, 2024, 1)
        agree = qk * qk + (1 - qk) * (1 - qk)
        sd2 = math.sqrt(agree * (1 - agree) / n)
        for other in (m2, m3):
            assert abs((m == other).mean() - agree) < 4.5 * sd2, p
        # rows and columns of every 4 x 4 block keep at the same rate
        for r in range(4):
            assert abs(m[:, :, r::4].mean() - qk) < 4.5 * sd * 2
            assert abs(m[:, :, :, r::4].mean() - qk) < 4.5 * sd * 2


def _loss(mod, q, k, v, do, p, seed, causal, scale):
    o, _ = mod.attn_dropout_fwd_ref(q, k, v, p, seed, 5, causal, scale)
    return float(np.sum(o * do))


def pin_dropout_finite_differences(mod):
    """Central differences of L = sum(O * dO) with the mask held fixed (brute force
    over every input entry) equal the oracle's gradients."""
    h = 1e-6
    for N, causal in ((6, False), (7, True)):
        q, k, v, do = (_rand((1, 2, N, 3), s) for s in (11, 12, 13, 14))
        p, seed, scale = 0.35, 31337, 0.6
        g = mod.attn_dropout_bwd_ref(q, k, v, do, p, seed, 5, causal, scale)
        o, _ = mod.attn_dropout_fwd_ref(q, k, v, p, seed, 5, causal, scale)
        assert np.max(np.abs(g["o"] - o)) < 1e-14
        assert np.allclose(g["D"], np.sum(o * do, axis=-1), atol=1e-12)  # D two ways
        for name, x in (("dq", q), ("dk", k), ("dv", v)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                args_p = {"q": q, "k": k, "v": v}
                args_m = {"q": q, "k": k, "v": v}
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p[name[1]], args_m[name[1]] = xp, xm
                num[idx] = (_loss(mod, args_p["q"], args_p["k"], args_p["v"], do, p, seed, causal, scale)
                            - _loss(mod, args_m["q"], args_m["k"], args_m["v"], do, p, seed, causal, scale)) / (2 * h)
            err = np.max(np.abs(num - g[name])) / max(1e-12, np.max(np.abs(num)))
            assert err < 1e-6, (name, N, causal, err)


def pin_head_slices_match_full(mod):
    """Forward and backward of one (b, h) slice with its head index equal the full
    problem's (b, h) results."""
    q, k, v, do = (_rand((2, 3, 9, 4), s) for s in (61, 62, 63, 64))
    full = mod.attn_dropout_bwd_ref(q, k, v, do, 0.4, 555, 2, True, 0.7)
    for b, h in ((0, 0), (1, 2), (0, 2)):
        sl = lambda x: x[b:b + 1, h:h + 1]
        one = mod.attn_dropout_bwd_ref(sl(q), sl(k), sl(v), sl(do), 0.4, 555, 2, True, 0.7, bh0=b * 3 + h)
        for name in ("dq", "dk", "dv", "o", "lse"):
            assert np.max(np.abs(one[name][0, 0] - full[name][b, h])) < 1e-13, (name, b, h)
        o, _ = mod.attn_dropout_fwd_ref(sl(q), sl(k), sl(v), 0.4, 555, 2, True, 0.7, bh0=b * 3 + h)
        assert np.max(np.abs(o[0, 0] - full["o"][b, h])) < 1e-13


def pin_expectation_over_seeds(mod):
    """Dropout is unbiased: the mean of O over seeds tends to plain attention's O
    (within 5 standard errors of the sample)."""
    q, k, v = (_rand((1, 1, 8, 4), s) for s in (21, 22, 23))
    o_ref, _ = oracle.attn_fwd_ref(q, k, v, False, 0.5)
    samples = np.stack([mod.attn_dropout_fwd_ref(q, k, v, 0.5, s, 0, False, 0.5)[0] for s in range(1500)])
    mean, se = samples.mean(axis=0), samples.std(axis=0) / math.sqrt(samples.shape[0])
    assert np.all(np.abs(mean - o_ref) < 5 * se + 1e-12)


def pin_threshold_rule(mod):
    """t = round(256 (1 - p)); p outside [0, 1) or t = 0 is rejected."""
    assert mod.keep_threshold(0.0) == 256 and mod.keep_threshold(0.5) == 128
    assert mod.keep_threshold(0.3) == 179 and mod.keep_threshold(0.1) == 230
    for bad in (-0.1, 1.0, 0.999, float("nan")):
        with pytest.raises(ValueError):
            mod.keep_threshold(bad)


def pin_pv_abs_bounds_o(mod):
    """sum_j P~_ij |V_jc| bounds |O_ic| (triangle inequality) and equals O_ic when V >= 0;
    with p = 0 it is plain attention's output on |V|."""
    q, k, v, do = (_rand((1, 2, 7, 4), s) for s in (71, 72, 73, 74))
    r = mod.attn_dropout_bwd_ref(q, k, v, do, 0.3, 99, 1, True, 0.6)
    assert np.all(r["pv_abs"] >= np.abs(r["o"]) - 1e-14)
    r_pos = mod.attn_dropout_bwd_ref(q, k, np.abs(v), do, 0.3, 99, 1, True, 0.6)
    assert np.max(np.abs(r_pos["pv_abs"] - r_pos["o"])) < 1e-14
    r0 = mod.attn_dropout_bwd_ref(q, k, v, do, 0.0, 99, 1, False, 0.6)
    o_abs, _ = oracle.attn_fwd_ref(q, k, np.abs(v), False, 0.6)
    assert np.max(np.abs(r0["pv_abs"] - o_abs)) < 1e-12


DROPOUT_PINS = [
    pin_philox_known_answers,
    pin_golden_4x4,
    pin_mask_layout,
    pin_p_zero_is_plain_attention,
    pin_keep_rate,
    pin_dropout_finite_differences,
    pin_expectation_over_seeds,
    pin_threshold_rule,
    pin_head_slices_match_full,
    pin_pv_abs_bounds_o,
]


@pytest.mark.parametrize("pin", DROPOUT_PINS, ids=lambda f: f.__name__)
def test_dropout_oracle_pin(pin):
    pin(oracle_dropout)


# ---------------------------------------------------------------- planted mistakes

MUTATIONS = {
    "philox_mul_swapped": ("p0 = _MUL0 * c0", "p0 = _MUL1 * c0"),
    "philox_no_key_bump": ("k0 = (k0 + _WEYL0) & _M32", "k0 = k0"),
    "philox_words_swapped": ("c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0",
                             "c0, c1, c2, c3 = hi0 ^ c1 ^ k0, lo1, hi1 ^ c3 ^ k1, lo0"),
    "scale_one_minus_p": ("pd = np.where(keep[b, h], pr * (256.0 / t), 0.0)",
                          "pd = np.where(keep[b, h], pr / (1.0 - p), 0.0)"),
    "word_by_column": ("w_idx = np.broadcast_to((qi % 4)[None, None, :, None], shape)",
                       "w_idx = np.broadcast_to((kj % 4)[None, None, None, :], shape)"),
    "counters_swapped": ("c0 = np.broadcast_to((kj // 4)[None, None, None, :], shape)\n"
                         "    c1 = np.broadcast_to((qi // 4)[None, None, :, None], shape)",
                         "c1 = np.broadcast_to((kj // 4)[None, None, None, :], shape)\n"
                         "    c0 = np.broadcast_to((qi // 4)[None, None, :, None], shape)"),
    "head_offset_ignored": ("bh = int(bh0) + np.arange(B * H", "bh = 0 * int(bh0) + np.arange(B * H"),
    "offset_ignored": ("c3 = np.full(shape, int(offset) & 0xFFFFFFFF, dtype=np.int64)",
                       "c3 = np.full(shape, 0, dtype=np.int64)"),
    "keep_le": ("return byte < np.uint64(t)", "return byte <= np.uint64(t)"),
    "threshold_floor": ("t = int(np.rint(256.0 * (1.0 - p)))", "t = int(256.0 * (1.0 - p))"),
    "ds_from_dropped": ("ds = pr * (dp - D[:, None])", "ds = pd * (dpd - D[:, None])"),
    "dp_unmasked": ("dp = dpd * m", "dp = dpd"),
    "dv_undropped": ('out["dv"][b, h] = pd.T @ do[b, h]', 'out["dv"][b, h] = pr.T @ do[b, h]'),
    "D_from_dropped": ("D = np.sum(pr * dp, axis=1)", "D = np.sum(pd * dpd * m, axis=1)"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src = open(oracle_dropout.__file__).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mod = types.ModuleType(f"oracle.dropout_mutant_{name}")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_dropout_mistake_is_caught(name):
    mod = _mutant(name)
    caught = []
    for pin in DROPOUT_PINS:
        try:
            pin(mod)
        except AssertionError:
            caught.append(pin.__name__)
        except Exception:  # a crash is also a detection
            caught.append(pin.__name__ + "(error)")
    assert caught, f"mutation {name} was not detected by any pin"
