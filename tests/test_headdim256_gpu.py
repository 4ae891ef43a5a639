"""Head dim 256 (its own forward kernel: one Q tile per work item, double-buffered scores):
forward against the fp64 oracle for square, ragged, N_q != N_k, block-sparse and
[B, N, H, d] inputs, with outputs as prefixes of NaN-filled buffers so that a write past
the last row is caught."""
import math

import pytest
import torch

import exact_tiled_attention_34_b200 as fa
import oracle
from exact_tiled_attention_34_b200.inputs import make_qkv, make_tile_mask
from tests.parity import assert_fwd_close, sample_rows, sampled_fwd_check, tol_o_sharp
from tests.test_ragged_gpu import _padded, _tail_untouched

pytestmark = pytest.mark.gpu

D = 256


def _check(B, H, Nq, Nk, causal, dev, seed, mask=None, scale=None):
    a = make_qkv(B, H, Nq, D, seed=seed, with_do=False)
    kv = a if Nk == Nq else make_qkv(B, H, Nk, D, seed=seed + 1000, with_do=False)
    t = {"q": a["q"].to(dev), "k": kv["k"].to(dev), "v": kv["v"].to(dev)}
    sc = 1.0 / math.sqrt(D) if scale is None else scale
    ob, o = _padded((B, H, Nq, D), torch.bfloat16, dev, float("nan"))
    lb, lse = _padded((B, H, Nq), torch.float32, dev, float("nan"))
    if mask is None:
        fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc, out=o, lse=lse)
    else:
        fa.forward_blocksparse(t["q"], t["k"], t["v"], mask.to(dev), scale=sc, out=o, lse=lse)
    torch.cuda.synchronize()
    assert fa.device_status() == (0, 0)
    assert _tail_untouched(ob, B * H * Nq * D, float("nan")) and _tail_untouched(lb, B * H * Nq, float("nan"))
    o_ref, l_ref = oracle.attn_fwd_ref(t["q"], t["k"], t["v"], causal, sc, None if mask is None else mask.numpy(),
                                       128)
    assert_fwd_close(o, lse, o_ref, l_ref, f"d256 B{B} H{H} Nq{Nq} Nk{Nk} causal={causal}",
                     tol_o=tol_o_sharp(t["v"]))
    return t, o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 300, 1000])
def test_lengths(cuda_device, N, causal):
    _check(2, 2, N, N, causal, cuda_device, seed=2560 + N)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(1, 700), (77, 300), (300, 77), (256, 640)])
def test_cross_lengths(cuda_device, nq, nk, causal):
    _, o, lse = _check(1, 2, nq, nk, causal, cuda_device, seed=2570 + nq)
    if causal and nq > nk:
        assert torch.all(o[:, :, : nq - nk] == 0) and torch.all(torch.isneginf(lse[:, :, : nq - nk]))


def test_causal_row0_exact(cuda_device):
    t, o, _ = _check(1, 2, 256, 256, True, cuda_device, seed=2580)
    assert torch.equal(o[:, :, 0], t["v"][:, :, 0])


@pytest.mark.parametrize("scale", [0.3, -0.2])
def test_scales(cuda_device, scale):
    """Peaked softmaxes (the running max is raised often, so O is rescaled in place)."""
    _check(1, 2, 512, 512, True, cuda_device, seed=2590, scale=scale)


def test_blocksparse(cuda_device):
    mask = make_tile_mask(6, seed=21, density=0.4)
    mask[2, :] = 0  # a query tile that keeps nothing: O = 0, lse = -inf
    _, o, lse = _check(1, 2, 700, 700, False, cuda_device, seed=2600, mask=mask)
    assert torch.all(o[:, :, 256:384] == 0) and torch.all(torch.isneginf(lse[:, :, 256:384]))


@pytest.mark.parametrize("causal", [False, True])
def test_many_items(cuda_device, causal):
    """More (query tile, head) items than SMs: each persistent CTA runs several."""
    _check(2, 64, 384, 384, causal, cuda_device, seed=2610)


def test_bnhd_layout(cuda_device):
    B, H, N = 2, 3, 300
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, D, seed=2620, with_do=False).items()}
    ref = fa.forward(t["q"], t["k"], t["v"], causal=True)
    tt = {k: x.transpose(1, 2).contiguous() for k, x in t.items()}
    o, lse = fa.forward(tt["q"], tt["k"], tt["v"], causal=True, layout="bnhd")
    torch.cuda.synchronize()
    assert torch.equal(o.transpose(1, 2), ref[0]) and torch.equal(lse, ref[1])


@pytest.mark.parametrize("causal", [False, True])
def test_long_sequence_sampled(cuda_device, causal):
    """B=1, H=8, N=8192: sampled rows of every head against the oracle."""
    B, H, N = 1, 8, 8192
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, D, seed=0, with_do=False).items()}
    sc = 1.0 / math.sqrt(D)
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc)
    torch.cuda.synchronize()
    assert fa.device_status() == (0, 0)
    c = {k: x.cpu() for k, x in t.items()}
    sampled_fwd_check(c["q"], c["k"], c["v"], o.cpu(), lse.cpu(), causal, sc, [(0, h) for h in range(H)],
                      sample_rows(N, n_random=32), what=f"d256 N{N} causal={causal}")


def test_backward_not_built_for_256(cuda_device):
    t = {k: x.to(cuda_device) for k, x in make_qkv(1, 1, 128, D, seed=2630).items()}
    o, lse = fa.forward(t["q"], t["k"], t["v"])
    with pytest.raises(fa.FAError) as e:
        fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"])
    assert e.value.status == 2
