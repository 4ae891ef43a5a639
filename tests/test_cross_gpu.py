"""Different query and key lengths (fa_fwd_qk / fa_bwd_qk through the binding): GPU
results against the fp64 oracle, with the causal mask aligned bottom-right (query i
sees key j iff j <= i + N_k - N_q), and sentinels that catch writes past the outputs."""
import math

import pytest
import torch

import exact_tiled_attention_34_b200 as fa
import oracle
from exact_tiled_attention_34_b200.inputs import make_qkv
from tests.parity import assert_fwd_close, assert_grad_close, tol_o_sharp
from tests.test_ragged_gpu import _padded, _tail_untouched

pytestmark = pytest.mark.gpu


def _inputs(B, H, Nq, Nk, d, seed, dev):
    a = make_qkv(B, H, Nq, d, seed=seed)          # q and dO from here
    b = make_qkv(B, H, Nk, d, seed=seed + 1000)   # k and v from here
    return {"q": a["q"].to(dev), "do": a["do"].to(dev), "k": b["k"].to(dev), "v": b["v"].to(dev)}


def _check(B, H, Nq, Nk, d, causal, dev, seed=0):
    t = _inputs(B, H, Nq, Nk, d, seed, dev)
    sc = 1.0 / math.sqrt(d)
    qs, ks = (B, H, Nq, d), (B, H, Nk, d)
    ob, o = _padded(qs, torch.bfloat16, dev, float("nan"))
    lb, lse = _padded((B, H, Nq), torch.float32, dev, float("nan"))
    fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc, out=o, lse=lse)
    gq = _padded(qs, torch.bfloat16, dev, float("nan"))
    gk = _padded(ks, torch.bfloat16, dev, float("nan"))
    gv = _padded(ks, torch.bfloat16, dev, float("nan"))
    dq, dk, dv = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal=causal, scale=sc,
                             grads=(gq[1], gk[1], gv[1]))
    torch.cuda.synchronize()
    assert fa.device_status() == (0, 0)
    assert _tail_untouched(ob, math.prod(qs), float("nan")) and _tail_untouched(lb, B * H * Nq, float("nan"))
    for (big, _), n in ((gq, math.prod(qs)), (gk, math.prod(ks)), (gv, math.prod(ks))):
        assert _tail_untouched(big, n, float("nan")), "gradient written past its end"
    what = f"B{B} H{H} Nq{Nq} Nk{Nk} d{d} causal={causal}"
    if causal and Nq > Nk:
        # the first Nq - Nk queries see no key: lse -inf, O and dQ exactly 0 (finite)
        blind = slice(0, Nq - Nk)
        assert torch.all(torch.isneginf(lse[:, :, blind]))
        assert torch.all(torch.isfinite(dq[:, :, blind])) and torch.all(dq[:, :, blind] == 0)
        assert torch.all(o[:, :, blind] == 0)
    for b in range(B):
        for h in range(H):
            sl = lambda x: x[b:b + 1, h:h + 1].cpu()
            ref = oracle.attn_bwd_ref(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["do"]), causal, sc)
            assert_fwd_close(sl(o), sl(lse), ref["o"], ref["lse"], f"{what} (b={b}, h={h})",
                             tol_o=tol_o_sharp(sl(t["v"])))
            for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
                assert_grad_close(sl(g), ref[name], name, f"{what} (b={b}, h={h})")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(1, 1000), (77, 300), (300, 77), (256, 640), (130, 200), (640, 256),
                                   (200, 130)])
def test_cross_lengths(cuda_device, nq, nk, causal, d):
    _check(2, 2, nq, nk, d, causal, cuda_device, seed=500 + nq + nk + d)


@pytest.mark.parametrize("causal", [False, True])
def test_cross_many_items(cuda_device, causal):
    """More work items than SMs on both sides (query and key tiles differ in number)."""
    _check(2, 64, 384, 1000, 64, causal, cuda_device, seed=61)


def test_cross_equal_lengths_match_square_call(cuda_device):
    """fa_fwd_qk / fa_bwd_qk with Nq = Nk give exactly what fa_fwd / fa_bwd give."""
    L = fa.lib()
    B, H, N, d = 1, 2, 333, 128
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=7).items()}
    o1, l1 = fa.forward(t["q"], t["k"], t["v"], causal=True)
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    st = L.fa_fwd_qk(t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), o2.data_ptr(), l2.data_ptr(),
                     B, H, N, N, d, 1, d ** -0.5, fa._stream_ptr(cuda_device))
    assert st == 0
    g1 = fa.backward(t["q"], t["k"], t["v"], o1, l1, t["do"], causal=True)
    ws = torch.empty(fa.bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=cuda_device)
    g2 = tuple(torch.empty_like(t["q"]) for _ in range(3))
    st = L.fa_bwd_qk(t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), o1.data_ptr(), l1.data_ptr(),
                     t["do"].data_ptr(), g2[0].data_ptr(), g2[1].data_ptr(), g2[2].data_ptr(), ws.data_ptr(),
                     ws.numel(), B, H, N, N, d, 1, d ** -0.5, fa._stream_ptr(cuda_device))
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for x, y in zip(g1, g2):
        assert torch.equal(x, y)
