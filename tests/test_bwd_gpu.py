"""GPU parity of the backward path (pre-processing, dK/dV kernel, dQ kernel),
called through the C ABI, against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_34_b200 as fa
import oracle
from exact_tiled_attention_34_b200.inputs import make_qkv, make_tile_mask, sweep_shape
from tests.parity import TOL_GRAD_REL, assert_grad_close, f64, sample_rows

pytestmark = pytest.mark.gpu


def _run(t, causal, scale, mask=None):
    if mask is None:
        o, lse = fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=scale)
        g = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal=causal, scale=scale)
    else:
        o, lse = fa.forward_blocksparse(t["q"], t["k"], t["v"], mask, scale=scale)
        g = fa.backward_blocksparse(t["q"], t["k"], t["v"], o, lse, t["do"], mask, scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == (0, 0)
    return o, lse, g


def _full_check(B, H, N, d, causal, dev, scale=None, seed=0, mask=None, heads=None, do_scale=1.0):
    t = {k: x.to(dev) for k, x in make_qkv(B, H, N, d, seed=seed, do_scale=do_scale).items()}
    sc = 1.0 / math.sqrt(d) if scale is None else scale
    m = None if mask is None else mask.to(dev)
    o, lse, (dq, dk, dv) = _run(t, causal, sc, m)
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    mk = None if mask is None else mask.cpu().numpy()
    worst = 0.0
    for (b, h) in heads:
        sl = lambda x: x[b:b + 1, h:h + 1].cpu()
        ref = oracle.attn_bwd_ref(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["do"]), causal, sc, mk, 128)
        what = f"B{B} H{H} N{N} d{d} causal={causal} (b={b}, h={h})"
        for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
            worst = max(worst, assert_grad_close(sl(g), ref[name], name, what))
    return t, (dq, dk, dv), worst


def test_smallest(cuda_device):
    _full_check(1, 2, 128, 64, False, cuda_device)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 384, 640])
def test_small_shapes(cuda_device, N, causal, d):
    _full_check(2, 2, N, d, causal, cuda_device, seed=100 + N + d)


@pytest.mark.parametrize("scale", [0.05, -0.2])
def test_scales(cuda_device, scale):
    _full_check(1, 2, 256, 64, True, cuda_device, scale=scale, seed=21)
    _full_check(1, 1, 256, 128, False, cuda_device, scale=scale, seed=22)


@pytest.mark.parametrize("d", [64, 128])
def test_blocksparse_small(cuda_device, d):
    N = 768
    mask = make_tile_mask(N // 128, seed=5, density=0.4)
    mask[3, :] = 0  # query tile with nothing kept
    mask[:, 4] = 0  # key tile nobody sees: dK = dV = 0 there
    mask[4, 4] = 0
    t, (dq, dk, dv), _ = _full_check(1, 2, N, d, False, cuda_device, seed=31, mask=mask)
    assert torch.all(dq[:, :, 384:512] == 0)
    assert torch.all(dk[:, :, 512:640] == 0) and torch.all(dv[:, :, 512:640] == 0)


def test_blocksparse_all_ones_equals_dense(cuda_device):
    t = {k: x.to(cuda_device) for k, x in make_qkv(1, 2, 512, 128, seed=41).items()}
    ones = torch.ones((4, 4), dtype=torch.uint8, device=cuda_device)
    _, _, a = _run(t, False, 0.1)
    _, _, b = _run(t, False, 0.1, ones)
    for x, y in zip(a, b):  # same tiles in the same order: bit-identical
        assert torch.equal(x, y)


@pytest.mark.parametrize("d", [64, 128])
def test_gradients_deterministic(cuda_device, d):
    """No atomics anywhere: two runs give bit-identical dQ, dK and dV."""
    t = {k: x.to(cuda_device) for k, x in make_qkv(2, 2, 1024, d, seed=42).items()}
    _, _, a = _run(t, True, d ** -0.5)
    _, _, b = _run(t, True, d ** -0.5)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_staged_calls_equal_fa_bwd(cuda_device):
    """fa_bwd_preprocess + fa_bwd_dkdv + fa_bwd_dq is exactly fa_bwd."""
    t = {k: x.to(cuda_device) for k, x in make_qkv(1, 3, 640, 128, seed=44).items()}
    o, lse, ref = _run(t, True, 0.09)
    ws = torch.empty(fa.bwd_workspace_bytes(1, 3, 640, 128), dtype=torch.uint8, device=cuda_device)
    dq, dk, dv = (torch.empty_like(t["q"]) for _ in range(3))
    fa.bwd_preprocess(o, t["do"], lse, ws)
    fa.bwd_dq(t["q"], t["k"], t["v"], t["do"], dq, ws, causal=True, scale=0.09)
    fa.bwd_dkdv(t["q"], t["k"], t["v"], t["do"], dk, dv, ws, causal=True, scale=0.09)
    torch.cuda.synchronize()
    for x, y in zip((dq, dk, dv), ref):
        assert torch.equal(x, y)


def test_workspace_too_small_is_rejected(cuda_device):
    t = {k: x.to(cuda_device) for k, x in make_qkv(1, 1, 128, 64, seed=43).items()}
    o, lse = fa.forward(t["q"], t["k"], t["v"])
    need = fa.bwd_workspace_bytes(1, 1, 128, 64)
    ws = torch.empty(need - 256, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(fa.FAError) as e:
        fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], workspace=ws)
    assert e.value.status == 4


def _sampled_bwd_check(t, grads, causal, sc, heads, rows, cols, mask=None, what=""):
    """Element-wise comparison with the oracle on sampled query rows (dQ) and sampled key
    rows (dK, dV) of the given heads; each tensor's bound is 2e-2 times the largest
    oracle value among its samples."""
    dq, dk, dv = grads
    mk = None if mask is None else mask.cpu().numpy()
    ridx, cidx = torch.as_tensor(rows), torch.as_tensor(cols)
    for (b, h) in heads:
        c = {k: x[b, h].cpu() for k, x in t.items()}
        w = f"{what} (b={b}, h={h})"
        ref_dq = oracle.attn_dq_rows_ref(f64(c["q"])[rows], rows, c["k"], c["v"], f64(c["do"])[rows], causal, sc,
                                         mk, 128)
        assert_grad_close(dq[b, h].cpu()[ridx], ref_dq, "dq", w)
        ref_dk, ref_dv = oracle.attn_dkdv_cols_ref(c["q"], c["k"], c["v"], c["do"], cols, causal, sc, mk, 128)
        assert_grad_close(dk[b, h].cpu()[cidx], ref_dk, "dk", w)
        assert_grad_close(dv[b, h].cpu()[cidx], ref_dv, "dv", w)


def _invariants(t, dk, dv):
    """sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i for every head (any size)."""
    dk64 = dk.double()
    s = dk64.sum(dim=2).abs().max().item()
    assert s <= 1e-2 * dk64.abs().sum(dim=2).max().item()
    sv = (dv.double().sum(dim=2) - t["do"].double().sum(dim=2)).abs().max().item()
    assert sv <= 1e-2 * dv.double().abs().sum(dim=2).max().item()


# ------------------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("causal", [False, True])
def test_b8h16n2048d64(cuda_device, causal):
    t, (dq, dk, dv), _ = _full_check(8, 16, 2048, 64, causal, cuda_device,
                                      heads=[(0, 0), (3, 7), (7, 15)])
    _invariants(t, dk, dv)


def test_b2h16n8192d128_causal(cuda_device):
    t, (dq, dk, dv), _ = _full_check(2, 16, 8192, 128, True, cuda_device, heads=[(0, 0), (1, 15)])
    _invariants(t, dk, dv)


def test_b1h16n16384d64_sparse(cuda_device):
    """Full size with the 128 x 128 tile mask: element-wise oracle comparison of sampled
    dQ rows and sampled dK, dV key rows (tile boundaries, keys of tiles that few query
    tiles keep, random keys) on three heads, gradient invariants on every head, and the
    full oracle on a 2048-token case with the same mask density."""
    B, H, N, d = 1, 16, 16384, 64
    mask = make_tile_mask(N // 128, seed=0, density=0.25)
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=0).items()}
    sc = 1.0 / math.sqrt(d)
    o, lse, grads = _run(t, False, sc, mask.to(cuda_device))
    _invariants(t, grads[1], grads[2])
    rows = sample_rows(N, n_random=24)
    # key tiles kept by the fewest and by the most query tiles, plus boundaries and random keys
    kept = mask.sum(dim=0).numpy()
    extra = [int(np.argmin(kept)) * 128 + 5, int(np.argmax(kept)) * 128 + 64]
    cols = np.array(sorted(set(sample_rows(N, n_random=24, seed=1).tolist()) | set(extra)))
    _sampled_bwd_check(t, grads, False, sc, [(0, 0), (0, 9), (0, 15)], rows, cols, mask, "B1 H16 N16384 d64 sparse")
    small = make_tile_mask(16, seed=0, density=0.25)
    _full_check(1, 2, 2048, 64, False, cuda_device, mask=small)


@pytest.mark.parametrize("N", [512, 4096])
@pytest.mark.parametrize("d", [64, 128])
def test_sweep_points(cuda_device, N, d):
    B, H = sweep_shape(N, d)
    for causal in (False, True):
        t, (dq, dk, dv), _ = _full_check(B, H, N, d, causal, cuda_device, do_scale=0.5,
                                          heads=[(0, 0), (B - 1, H - 1)])
        _invariants(t, dk, dv)


@pytest.mark.parametrize("N", [1024, 2048, 8192, 16384])
@pytest.mark.parametrize("d", [64, 128])
def test_sweep_points_sampled(cuda_device, N, d):
    """The other sweep lengths at full size (B N = 16384 tokens, H = 2048 / d), causal and
    not: sampled dQ rows and dK, dV key rows of two heads against the oracle, and the
    gradient invariants on every head."""
    B, H = sweep_shape(N, d)
    sc = 1.0 / math.sqrt(d)
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=0, do_scale=0.5).items()}
    rows = sample_rows(N, n_random=16)
    cols = sample_rows(N, n_random=16, seed=1)
    for causal in (False, True):
        _, _, grads = _run(t, causal, sc)
        _invariants(t, grads[1], grads[2])
        _sampled_bwd_check(t, grads, causal, sc, [(0, 0), (B - 1, H - 1)], rows, cols, None,
                           f"B{B} H{H} N{N} d{d} causal={causal}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_many_items_per_cta(cuda_device, causal, d):
    """More (tile, head) items than SMs: each persistent CTA of both backward
    kernels runs several, with an odd tile count."""
    _full_check(2, 80, 640, d, causal, cuda_device, seed=51 + d)


def test_many_items_blocksparse(cuda_device):
    N = 768
    mask = make_tile_mask(N // 128, seed=11, density=0.4)
    mask[2, :] = 0
    mask[:, 3] = 0
    t, (dq, dk, dv), _ = _full_check(1, 160, N, 64, False, cuda_device, seed=53, mask=mask)
    assert torch.all(dq[:, :, 256:384] == 0)
    assert torch.all(dk[:, :, 384:512] == 0) and torch.all(dv[:, :, 384:512] == 0)
