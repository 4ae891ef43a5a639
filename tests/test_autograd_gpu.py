"""The torch.autograd wrapper: gradients through the library match the fp64 oracle and
are exactly what the C-ABI backward returns."""
import math

import pytest
import torch

import exact_tiled_attention_34_b200 as fa
import oracle
from exact_tiled_attention_34_b200.inputs import make_qkv, make_tile_mask
from tests.parity import assert_fwd_close, assert_grad_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_autograd_matches_oracle_and_c_abi(cuda_device, causal, d):
    B, H, N = 1, 2, 300
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=71 + d).items()}
    q, k, v = (t[n].clone().requires_grad_(True) for n in ("q", "k", "v"))
    o = fa.attention(q, k, v, causal=causal)
    (o.float() * t["do"].float()).sum().backward()
    torch.cuda.synchronize()
    sc = 1.0 / math.sqrt(d)
    o2, lse2 = fa.forward(t["q"], t["k"], t["v"], causal=causal)
    g2 = fa.backward(t["q"], t["k"], t["v"], o2, lse2, t["do"], causal=causal)
    assert torch.equal(o.detach(), o2)
    for a, b in zip((q.grad, k.grad, v.grad), g2):
        assert torch.equal(a, b)
    for b in range(B):
        for h in range(H):
            sl = lambda x: x[b:b + 1, h:h + 1].detach().cpu()
            ref = oracle.attn_bwd_ref(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["do"]), causal, sc)
            assert_fwd_close(sl(o), sl(lse2), ref["o"], ref["lse"], f"d{d} causal={causal}")
            for name, g in (("dq", q.grad), ("dk", k.grad), ("dv", v.grad)):
                assert_grad_close(sl(g), ref[name], name, f"autograd d{d} causal={causal}")


def test_autograd_blocksparse_and_cross(cuda_device):
    N, d = 384, 64
    t = {k: x.to(cuda_device) for k, x in make_qkv(1, 2, N, d, seed=73).items()}
    mask = make_tile_mask(3, seed=4, density=0.5).to(cuda_device)
    q, k, v = (t[n].clone().requires_grad_(True) for n in ("q", "k", "v"))
    o = fa.attention_blocksparse(q, k, v, mask)
    (o.float() * t["do"].float()).sum().backward()
    o2, lse2 = fa.forward_blocksparse(t["q"], t["k"], t["v"], mask)
    g2 = fa.backward_blocksparse(t["q"], t["k"], t["v"], o2, lse2, t["do"], mask)
    torch.cuda.synchronize()
    for a, b in zip((q.grad, k.grad, v.grad), g2):
        assert torch.equal(a, b)
    # different query and key lengths through autograd
    kv = {kk: x.to(cuda_device) for kk, x in make_qkv(1, 2, 640, d, seed=74, with_do=False).items()}
    q2 = t["q"].clone().requires_grad_(True)
    k2, v2 = kv["k"].clone().requires_grad_(True), kv["v"].clone().requires_grad_(True)
    o3 = fa.attention(q2, k2, v2, causal=True)
    (o3.float() * t["do"].float()).sum().backward()
    torch.cuda.synchronize()
    ref = oracle.attn_bwd_ref(t["q"].cpu(), kv["k"].cpu(), kv["v"].cpu(), t["do"].cpu(), True, d ** -0.5)
    for name, g in (("dq", q2.grad), ("dk", k2.grad), ("dv", v2.grad)):
        assert_grad_close(g.cpu(), ref[name], name, "autograd cross")
