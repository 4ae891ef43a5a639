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
from tests.parity import assert_fwd_close, assert_grad_close, sample_rows, sampled_fwd_check, tol_o_sharp
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


# ------------------------------------------------------------------ backward (fused kernel)

def _bwd_check(B, H, Nq, Nk, causal, dev, seed, mask=None, scale=None, heads=None):
    a = make_qkv(B, H, Nq, D, seed=seed)
    kv = a if Nk == Nq else make_qkv(B, H, Nk, D, seed=seed + 1000)
    t = {"q": a["q"].to(dev), "do": a["do"].to(dev), "k": kv["k"].to(dev), "v": kv["v"].to(dev)}
    sc = 1.0 / math.sqrt(D) if scale is None else scale
    m = None if mask is None else mask.to(dev)
    if m is None:
        o, lse = fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc)
    else:
        o, lse = fa.forward_blocksparse(t["q"], t["k"], t["v"], m, scale=sc)
    bufs = [_padded(shape, torch.bfloat16, dev, float("nan")) for shape in
            ((B, H, Nq, D), (B, H, Nk, D), (B, H, Nk, D))]
    grads = tuple(b[1] for b in bufs)
    if m is None:
        dq, dk, dv = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal=causal, scale=sc, grads=grads)
    else:
        dq, dk, dv = fa.backward_blocksparse(t["q"], t["k"], t["v"], o, lse, t["do"], m, scale=sc, grads=grads)
    torch.cuda.synchronize()
    assert fa.device_status() == (0, 0)
    for (big, g) in bufs:
        assert _tail_untouched(big, g.numel(), float("nan")), "gradient written past its end"
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for (b, h) in heads:
        sl = lambda x: x[b:b + 1, h:h + 1].cpu()
        ref = oracle.attn_bwd_ref(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["do"]), causal, sc,
                                  None if mask is None else mask.numpy(), 128)
        for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
            assert_grad_close(sl(g), ref[name], name, f"d256 bwd B{B} H{H} Nq{Nq} Nk{Nk} causal={causal} (b={b}, h={h})")
    return t, (dq, dk, dv)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 300, 1000])
def test_backward_lengths(cuda_device, N, causal):
    _bwd_check(2, 2, N, N, causal, cuda_device, seed=2640 + N)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(1, 700), (77, 300), (300, 77), (256, 640)])
def test_backward_cross_lengths(cuda_device, nq, nk, causal):
    _, (dq, _, _) = _bwd_check(1, 2, nq, nk, causal, cuda_device, seed=2650 + nq)
    if causal and nq > nk:
        assert torch.all(dq[:, :, : nq - nk] == 0)


@pytest.mark.parametrize("scale", [0.05, -0.2])
def test_backward_scales(cuda_device, scale):
    _bwd_check(1, 2, 384, 384, True, cuda_device, seed=2660, scale=scale)


def test_backward_blocksparse(cuda_device):
    mask = make_tile_mask(6, seed=23, density=0.4)
    mask[2, :] = 0
    mask[:, 4] = 0
    mask[4, 4] = 0
    _, (dq, dk, dv) = _bwd_check(1, 2, 768, 768, False, cuda_device, seed=2670, mask=mask)
    assert torch.all(dq[:, :, 256:384] == 0)
    assert torch.all(dk[:, :, 512:640] == 0) and torch.all(dv[:, :, 512:640] == 0)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_many_items(cuda_device, causal):
    """More (key tile, column half, head) items than SMs."""
    _bwd_check(2, 48, 384, 384, causal, cuda_device, seed=2680)


def test_backward_2048_full_heads(cuda_device):
    _bwd_check(1, 4, 2048, 2048, True, cuda_device, seed=0, heads=[(0, 0), (0, 3)])


def test_backward_bnhd_layout(cuda_device):
    B, H, N = 1, 3, 300
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, D, seed=2690).items()}
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal=True)
    ref = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal=True)
    tt = {k: x.transpose(1, 2).contiguous() for k, x in t.items()}
    g = fa.backward(tt["q"], tt["k"], tt["v"], o.transpose(1, 2).contiguous(), lse, tt["do"], causal=True,
                    layout="bnhd")
    torch.cuda.synchronize()
    for x, y in zip(g, ref):
        assert float((x.transpose(1, 2).float() - y.float()).abs().max()) <= 2e-2 * float(y.float().abs().max())


def test_backward_deterministic_path_is_not_offered(cuda_device):
    """Head dim 256 has only the fused backward: asking for the deterministic one raises,
    and the C entry point of the deterministic backward refuses the size."""
    t = {k: x.to(cuda_device) for k, x in make_qkv(1, 1, 128, D, seed=2700).items()}
    o, lse = fa.forward(t["q"], t["k"], t["v"])
    with pytest.raises(ValueError):
        fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], deterministic=True)
    ws = torch.empty(fa.bwd_workspace_bytes(1, 1, 128, D), dtype=torch.uint8, device=cuda_device)
    g = [torch.empty_like(t["q"]) for _ in range(3)]
    st = fa.lib().fa_bwd(t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), o.data_ptr(), lse.data_ptr(),
                         t["do"].data_ptr(), g[0].data_ptr(), g[1].data_ptr(), g[2].data_ptr(), ws.data_ptr(),
                         ws.numel(), 1, 1, 128, D, 0, 0.0625, fa._stream_ptr(cuda_device))
    assert st == 2
