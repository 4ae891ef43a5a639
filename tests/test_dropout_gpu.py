"""Dropout on the attention probabilities: GPU forward and backward (through the C
ABI) against the fp64 dropout oracle, the keep mask read back exactly from the
kernels, p = 0 against the plain kernels, and the autograd wrapper."""
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_34_b200 as fa
import oracle
from exact_tiled_attention_34_b200.inputs import make_qkv
from tests.parity import TOL_O, assert_fwd_close, assert_grad_close

pytestmark = pytest.mark.gpu

SEED = 0x5EED_0F_D20F_0A7


def _tol_o(v, p):
    """O = sum_j P~_j V_j with P~ = P * 256 / t rounded to bf16, then O rounded to bf16:
    each rounding moves O by at most 2^-8 (256 / t) max|V|."""
    rs = 256.0 / oracle.keep_threshold(p)
    return max(TOL_O, 2.0 ** -7 * rs * float(v.float().abs().max()))


def _assert_o_within_rounding(o, ref, what):
    """Element-wise bound, tighter than the worst case above wherever |O| or the row's
    spread is small: the kernels round each P~_ij (relative error <= 2^-8) before P~ V
    and round O once more (<= 2^-8 |O|), so |dO_ic| <= 2^-8 (sum_j P~_ij |V_jc| + |O_ic|);
    5% is left for the exponentials' own error (<= 1.02e-4 relative) and fp32 sums."""
    o = np.asarray(o.float().numpy(), dtype=np.float64)
    o_ref = np.asarray(ref["o"], dtype=np.float64).reshape(o.shape)
    bound = 2.0 ** -8 * 1.05 * (np.asarray(ref["pv_abs"]).reshape(o.shape) + np.abs(o_ref)) + 1e-5
    excess = np.abs(o - o_ref) - bound
    assert excess.max() <= 0, f"{what}: |dO| above its rounding bound by {excess.max():.3g}"
    assert np.median(bound) < TOL_O, what  # the bound is tighter than 1e-2 for most elements


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,p", [(256, 0.1), (300, 0.3), (640, 0.5)])
def test_dropout_parity(cuda_device, d, causal, N, p):
    B, H = 2, 2
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=700 + N + d).items()}
    sc = 1.0 / math.sqrt(d)
    off = 3 + N
    o, lse = fa.forward_dropout(t["q"], t["k"], t["v"], p, SEED, off, causal=causal, scale=sc)
    dq, dk, dv = fa.backward_dropout(t["q"], t["k"], t["v"], o, lse, t["do"], p, SEED, off, causal=causal,
                                     scale=sc)
    assert fa.device_status() == (0, 0)
    ref = oracle.attn_dropout_bwd_ref(t["q"].cpu(), t["k"].cpu(), t["v"].cpu(), t["do"].cpu(), p, SEED, off,
                                      causal, sc)
    what = f"N{N} d{d} causal={causal} p={p}"
    assert_fwd_close(o.cpu(), lse.cpu(), ref["o"], ref["lse"], what, tol_o=_tol_o(t["v"], p))
    _assert_o_within_rounding(o.cpu(), ref, what)
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert_grad_close(g.cpu(), ref[name], name, what)


@pytest.mark.parametrize("B,H,N,d,causal,heads", [
    (8, 16, 2048, 64, False, [(0, 0), (7, 15)]),
    (8, 16, 2048, 64, True, [(3, 9)]),
    (2, 16, 8192, 128, True, [(1, 15)]),
])
def test_dropout_full_size(cuda_device, B, H, N, d, causal, heads):
    """The bench table's dropout workloads (p = 0.1, seed 1234, offset 0, same inputs):
    every output of the listed heads against the oracle on that head alone."""
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=0).items()}
    sc, p = 1.0 / math.sqrt(d), 0.1
    o, lse = fa.forward_dropout(t["q"], t["k"], t["v"], p, 1234, 0, causal=causal, scale=sc)
    dq, dk, dv = fa.backward_dropout(t["q"], t["k"], t["v"], o, lse, t["do"], p, 1234, 0, causal=causal, scale=sc)
    assert fa.device_status() == (0, 0)
    for (b, h) in heads:
        sl = lambda x: x[b:b + 1, h:h + 1].cpu()
        ref = oracle.attn_dropout_bwd_ref(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["do"]), p, 1234, 0, causal, sc,
                                          bh0=b * H + h)
        what = f"B{B} H{H} N{N} d{d} causal={causal} (b={b}, h={h})"
        assert_fwd_close(sl(o), sl(lse), ref["o"], ref["lse"], what, tol_o=_tol_o(t["v"], p))
        _assert_o_within_rounding(sl(o), ref, what)
        for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
            assert_grad_close(sl(g), ref[name], name, what)


@pytest.mark.parametrize("causal", [False, True])
def test_dropout_mask_read_back(cuda_device, causal):
    """With q = k = 0 the probabilities of a row are equal, so O = P~ V with V the
    identity on one half of the keys exposes P~ for those keys: nonzero exactly where
    the mask keeps. dV = P~^T dO with dO the identity on one half of the queries
    exposes the mask as the dK/dV kernel draws it (its own layout, key-major)."""
    B, H, N, d, p = 1, 3, 256, 128, 0.3
    dev = cuda_device
    z = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device=dev)
    keep = oracle.dropout_keep_mask(B, H, N, N, p, SEED, 7)
    vis = np.tril(np.ones((N, N), dtype=bool)) if causal else np.ones((N, N), dtype=bool)
    want = keep & vis[None, None]
    eye = torch.eye(128, dtype=torch.bfloat16, device=dev)
    for half in range(2):
        v = torch.zeros_like(z)
        v[:, :, 128 * half:128 * half + 128, :] = eye
        o, lse = fa.forward_dropout(z, z, v, p, SEED, 7, causal=causal, scale=1.0)
        got = (o != 0).cpu().numpy()
        assert np.array_equal(got, want[:, :, :, 128 * half:128 * half + 128]), f"forward mask, keys half {half}"
        do = torch.zeros_like(z)
        do[:, :, 128 * half:128 * half + 128, :] = eye
        _, _, dv = fa.backward_dropout(z, z, v, o, lse, do, p, SEED, 7, causal=causal, scale=1.0)
        got_t = (dv != 0).cpu().numpy()  # dV[j, c] = P~[128 half + c, j]
        assert np.array_equal(got_t, np.swapaxes(want[:, :, 128 * half:128 * half + 128, :], 2, 3)), \
            f"dK/dV mask, queries half {half}"
    assert fa.device_status() == (0, 0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_p_zero_matches_plain_kernels(cuda_device, d, causal):
    """p = 0 keeps everything with scale 1: bit for bit the results of the plain kernels."""
    t = {k: x.to(cuda_device) for k, x in make_qkv(2, 3, 384, d, seed=91).items()}
    o0, l0 = fa.forward(t["q"], t["k"], t["v"], causal=causal)
    o1, l1 = fa.forward_dropout(t["q"], t["k"], t["v"], 0.0, 123, 0, causal=causal)
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
    g0 = fa.backward(t["q"], t["k"], t["v"], o0, l0, t["do"], causal=causal)
    g1 = fa.backward_dropout(t["q"], t["k"], t["v"], o0, l0, t["do"], 0.0, 123, 0, causal=causal)
    for a, b in zip(g0, g1):
        assert torch.equal(a, b)


def test_seed_and_offset_change_the_mask(cuda_device):
    t = {k: x.to(cuda_device) for k, x in make_qkv(1, 2, 256, 64, seed=5, with_do=False).items()}
    a, _ = fa.forward_dropout(t["q"], t["k"], t["v"], 0.5, 1, 0)
    b, _ = fa.forward_dropout(t["q"], t["k"], t["v"], 0.5, 2, 0)
    c, _ = fa.forward_dropout(t["q"], t["k"], t["v"], 0.5, 1, 1)
    a2, _ = fa.forward_dropout(t["q"], t["k"], t["v"], 0.5, 1, 0)
    assert torch.equal(a, a2)  # deterministic
    assert not torch.equal(a, b) and not torch.equal(a, c)


def test_autograd_dropout(cuda_device):
    t = {k: x.to(cuda_device) for k, x in make_qkv(1, 2, 256, 64, seed=8).items()}
    q, k, v = (t[n].clone().requires_grad_(True) for n in ("q", "k", "v"))
    o = fa.attention(q, k, v, causal=True, dropout_p=0.2, seed=77, offset=4)
    o.backward(t["do"])
    o_ref, lse = fa.forward_dropout(t["q"], t["k"], t["v"], 0.2, 77, 4, causal=True)
    g_ref = fa.backward_dropout(t["q"], t["k"], t["v"], o_ref, lse, t["do"], 0.2, 77, 4, causal=True)
    assert torch.equal(o.detach(), o_ref)
    for x, g in zip((q, k, v), g_ref):
        assert torch.equal(x.grad, g)


def test_dropout_rejects_unsupported(cuda_device):
    t = {k: x.to(cuda_device) for k, x in make_qkv(1, 1, 128, 64, seed=1, with_do=False).items()}
    with pytest.raises(ValueError):
        fa.forward_dropout(t["q"], t["k"], t["v"], 1.0, 0)
    with pytest.raises(fa.FAError):
        fa.forward_dropout(t["q"], t["k"], t["v"], 0.999, 0)  # keep threshold 0
    q96 = torch.zeros((1, 1, 128, 96), dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(fa.FAError):
        fa.forward_dropout(q96, q96, q96, 0.1, 0)
