"""Sequence lengths that are not a multiple of the 128-row tile: the last query and
key tiles are partial. GPU results against the fp64 oracle, plus checks that nothing
is written past the N rows of the last (batch, head)."""
import math

import pytest
import torch

import exact_tiled_attention_34_b200 as fa
import oracle
from exact_tiled_attention_34_b200.inputs import make_qkv, make_tile_mask
from tests.parity import assert_fwd_close, assert_grad_close, tol_o_sharp

pytestmark = pytest.mark.gpu

PAD = 4096  # sentinel elements after each output


def _padded(shape, dtype, dev, fill):
    """A contiguous tensor of `shape` that is a prefix view of a larger buffer filled
    with `fill`, so that writes past its end are visible."""
    n = math.prod(shape)
    big = torch.full((n + PAD,), fill, dtype=dtype, device=dev)
    return big, big[:n].view(shape)


def _tail_untouched(big, n, fill):
    tail = big[n:]
    if isinstance(fill, float) and math.isnan(fill):
        return bool(torch.isnan(tail.float()).all())
    return bool((tail == fill).all())


def _run(B, H, N, d, causal, dev, mask=None, seed=0, scale=None):
    t = {k: x.to(dev) for k, x in make_qkv(B, H, N, d, seed=seed).items()}
    sc = 1.0 / math.sqrt(d) if scale is None else scale
    shape = (B, H, N, d)
    ob, o = _padded(shape, torch.bfloat16, dev, float("nan"))
    lb, lse = _padded((B, H, N), torch.float32, dev, float("nan"))
    if mask is None:
        fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc, out=o, lse=lse)
    else:
        fa.forward_blocksparse(t["q"], t["k"], t["v"], mask.to(dev), scale=sc, out=o, lse=lse)
    grads = [_padded(shape, torch.bfloat16, dev, float("nan")) for _ in range(3)]
    ws = torch.empty(fa.bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
    dq, dk, dv = (g[1] for g in grads)
    fa.bwd_preprocess(o, t["do"], lse, ws)
    m = None if mask is None else mask.to(dev)
    fa.bwd_dkdv(t["q"], t["k"], t["v"], t["do"], dk, dv, ws, causal=causal, scale=sc, tile_mask=m)
    fa.bwd_dq(t["q"], t["k"], t["v"], t["do"], dq, ws, causal=causal, scale=sc, tile_mask=m)
    torch.cuda.synchronize()
    assert fa.device_status() == (0, 0)
    n = math.prod(shape)
    assert _tail_untouched(ob, n, float("nan")), "O written past the last row"
    assert _tail_untouched(lb, B * H * N, float("nan")), "lse written past the last row"
    for name, (big, _) in zip(("dq", "dk", "dv"), grads):
        assert _tail_untouched(big, n, float("nan")), f"{name} written past the last row"
    return t, sc, o, lse, (dq, dk, dv)


def _zero_grad_bound(sl, t, o, sc, other):
    """Bound on a gradient whose exact value is identically zero (every row sees one
    key, e.g. N = 1: softmax is constant, so dS = P (dP - D) = 0). The kernels form D
    from the stored bf16 O, which differs from the exact O by at most 2^-8 |O| per
    element, so |D - D_exact| <= 2^-8 max_i sum_c |dO_ic O_ic|, and the gradient
    dq = scale dS K (dk = scale dS^T Q) is at most scale |D - D_exact| max|K| (max|Q|)."""
    dd = (sl(t["do"]).double().abs() * sl(o).double().abs()).sum(-1).max().item()
    return abs(sc) * 2.0 ** -8 * dd * sl(t[other]).double().abs().max().item()


def _check(B, H, N, d, causal, dev, mask=None, seed=0, scale=None):
    t, sc, o, lse, (dq, dk, dv) = _run(B, H, N, d, causal, dev, mask, seed, scale)
    mk = None if mask is None else mask.numpy()
    what = f"B{B} H{H} N{N} d{d} causal={causal} sparse={mask is not None}"
    for b in range(B):
        for h in range(H):
            sl = lambda x: x[b:b + 1, h:h + 1].cpu()
            ref = oracle.attn_bwd_ref(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["do"]), causal, sc, mk, 128)
            assert_fwd_close(sl(o), sl(lse), ref["o"], ref["lse"], f"{what} (b={b}, h={h})",
                             tol_o=tol_o_sharp(sl(t["v"])))
            for name, g, other in (("dq", dq, "k"), ("dk", dk, "q"), ("dv", dv, None)):
                if other is not None and float(abs(ref[name]).max()) == 0.0:
                    err = sl(g).double().abs().max().item()
                    bound = _zero_grad_bound(sl, t, o, sc, other)
                    assert err <= bound, f"{what} (b={b}, h={h}): exact {name} is 0, got {err:.3e} > {bound:.3e}"
                else:
                    assert_grad_close(sl(g), ref[name], name, f"{what} (b={b}, h={h})")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 77, 129, 300, 1000])
def test_ragged_lengths(cuda_device, N, causal, d):
    _check(2, 2, N, d, causal, cuda_device, seed=300 + N + d)


@pytest.mark.parametrize("d", [64, 128])
def test_ragged_blocksparse(cuda_device, d):
    N = 650  # 6 tiles, the last with 10 rows
    nt = -(-N // 128)
    mask = make_tile_mask(nt, seed=17, density=0.4)
    mask[nt - 1, :] = 0          # the partial query tile sees nothing: O = 0, lse = -inf
    mask[nt - 1, nt - 1] = 0
    mask[2, nt - 1] = 1          # a full query tile that sees the partial key tile
    _check(1, 2, N, d, False, cuda_device, mask=mask, seed=31)


@pytest.mark.parametrize("d", [64, 128])
def test_ragged_many_items(cuda_device, d):
    """More work items than SMs with a partial last tile in every (batch, head)."""
    _check(2, 96, 200, d, True, cuda_device, seed=41)


def test_ragged_fa_bwd_matches_staged(cuda_device):
    """fa_bwd on a ragged length equals the three staged calls, bit for bit."""
    B, H, N, d = 1, 3, 333, 64
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=9).items()}
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal=True)
    a = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal=True)
    _, _, _, _, b = _run(B, H, N, d, True, cuda_device, seed=9)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
