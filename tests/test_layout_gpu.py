"""[B, N, H, d] tensors (layout="bnhd" through fa_fwd_ex / fa_bwd_ex): the results equal
those of the [B, H, N, d] path bit for bit (the same tiles in the same order), match the
fp64 oracle, and nothing is written past the outputs."""
import math

import pytest
import torch

import exact_tiled_attention_34_b200 as fa
import oracle
from exact_tiled_attention_34_b200.inputs import make_qkv
from tests.parity import assert_fwd_close, assert_grad_close
from tests.test_ragged_gpu import _padded, _tail_untouched

pytestmark = pytest.mark.gpu


def _bnhd(x):
    return x.transpose(1, 2).contiguous()


@pytest.mark.parametrize("case", [
    dict(B=2, H=3, Nq=384, Nk=384, d=64, causal=False),
    dict(B=2, H=3, Nq=384, Nk=384, d=128, causal=True),
    dict(B=1, H=4, Nq=300, Nk=300, d=96, causal=True),
    dict(B=2, H=2, Nq=200, Nk=777, d=64, causal=True),
    dict(B=1, H=5, Nq=650, Nk=130, d=128, causal=False),
])
def test_bnhd_equals_bhnd(cuda_device, case):
    B, H, Nq, Nk, d, causal = (case[x] for x in ("B", "H", "Nq", "Nk", "d", "causal"))
    a = make_qkv(B, H, Nq, d, seed=Nq + d)
    b = make_qkv(B, H, Nk, d, seed=Nk + d + 1, with_do=False)
    q, do = a["q"].to(cuda_device), a["do"].to(cuda_device)
    k, v = b["k"].to(cuda_device), b["v"].to(cuda_device)
    o1, l1 = fa.forward(q, k, v, causal=causal)
    g1 = fa.backward(q, k, v, o1, l1, do, causal=causal)
    qt, kt, vt, dot = _bnhd(q), _bnhd(k), _bnhd(v), _bnhd(do)
    ob, o2 = _padded(qt.shape, torch.bfloat16, cuda_device, float("nan"))
    lb, l2 = _padded((B, H, Nq), torch.float32, cuda_device, float("nan"))
    fa.forward(qt, kt, vt, causal=causal, out=o2, lse=l2, layout="bnhd")
    bufs = [_padded(qt.shape, torch.bfloat16, cuda_device, float("nan")),
            _padded(kt.shape, torch.bfloat16, cuda_device, float("nan")),
            _padded(kt.shape, torch.bfloat16, cuda_device, float("nan"))]
    g2 = fa.backward(qt, kt, vt, o2, l2, dot, causal=causal, grads=tuple(x[1] for x in bufs), layout="bnhd")
    torch.cuda.synchronize()
    assert fa.device_status() == (0, 0)
    assert _tail_untouched(ob, o2.numel(), float("nan")) and _tail_untouched(lb, l2.numel(), float("nan"))
    for (big, t) in bufs:
        assert _tail_untouched(big, t.numel(), float("nan"))
    assert torch.equal(_bnhd(o2), o1) and torch.equal(l2, l1)
    for x, y in zip(g2, g1):
        assert torch.equal(_bnhd(x), y)
    # and against the oracle for one head
    sc = 1.0 / math.sqrt(d)
    sl = lambda x: x[0:1, 0:1].cpu()
    ref = oracle.attn_bwd_ref(sl(q), sl(k), sl(v), sl(do), causal, sc)
    assert_fwd_close(sl(_bnhd(o2)), sl(l2), ref["o"], ref["lse"], f"bnhd {case}", tol_o=2.0 ** -7 * 4.5)
    for name, g in zip(("dq", "dk", "dv"), g2):
        assert_grad_close(sl(_bnhd(g)), ref[name], name, f"bnhd {case}")


def test_bnhd_autograd(cuda_device):
    t = {k: x.to(cuda_device) for k, x in make_qkv(2, 3, 256, 64, seed=5).items()}
    qt, kt, vt = (_bnhd(t[n]).requires_grad_(True) for n in ("q", "k", "v"))
    o = fa.attention(qt, kt, vt, causal=True, layout="bnhd")
    (o.float() * _bnhd(t["do"]).float()).sum().backward()
    o1, l1 = fa.forward(t["q"], t["k"], t["v"], causal=True)
    g1 = fa.backward(t["q"], t["k"], t["v"], o1, l1, t["do"], causal=True)
    torch.cuda.synchronize()
    assert torch.equal(_bnhd(o.detach()), o1)
    for x, y in zip((qt.grad, kt.grad, vt.grad), g1):
        assert torch.equal(_bnhd(x), y)
