"""GPU parity of the fused backward (one kernel for dK, dV and dQ, dQ reduced in fp32
in the workspace), called through the C ABI, against the fp64 oracle: the same shapes,
masks, lengths, layouts and full-size workloads as the deterministic path, with the
same tolerances (max|dg| <= 2e-2 max|g_oracle| per gradient tensor)."""
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_34_b200 as fa
import oracle
from exact_tiled_attention_34_b200.inputs import make_qkv, make_tile_mask, sweep_shape
from tests.parity import assert_grad_close, f64, sample_rows
from tests.test_ragged_gpu import _padded, _tail_untouched

pytestmark = pytest.mark.gpu


def _fwd(t, causal, sc, mask=None):
    if mask is None:
        return fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc)
    return fa.forward_blocksparse(t["q"], t["k"], t["v"], mask, scale=sc)


def _fused(t, o, lse, causal, sc, mask=None, grads=None):
    if mask is None:
        g = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal=causal, scale=sc, grads=grads,
                        deterministic=False)
    else:
        g = fa.backward_blocksparse(t["q"], t["k"], t["v"], o, lse, t["do"], mask, scale=sc, grads=grads,
                                    deterministic=False)
    torch.cuda.synchronize()
    assert fa.device_status() == (0, 0)
    return g


def _full_check(B, H, N, d, causal, dev, scale=None, seed=0, mask=None, heads=None, do_scale=1.0):
    t = {k: x.to(dev) for k, x in make_qkv(B, H, N, d, seed=seed, do_scale=do_scale).items()}
    sc = 1.0 / math.sqrt(d) if scale is None else scale
    m = None if mask is None else mask.to(dev)
    o, lse = _fwd(t, causal, sc, m)
    dq, dk, dv = _fused(t, o, lse, causal, sc, m)
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    mk = None if mask is None else mask.cpu().numpy()
    for (b, h) in heads:
        sl = lambda x: x[b:b + 1, h:h + 1].cpu()
        ref = oracle.attn_bwd_ref(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["do"]), causal, sc, mk, 128)
        what = f"fused B{B} H{H} N{N} d{d} causal={causal} (b={b}, h={h})"
        for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
            assert_grad_close(sl(g), ref[name], name, what)
    return t, (o, lse), (dq, dk, dv)


def test_smallest(cuda_device):
    _full_check(1, 2, 128, 64, False, cuda_device)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 384, 640])
def test_small_shapes(cuda_device, N, causal, d):
    _full_check(2, 2, N, d, causal, cuda_device, seed=300 + N + d)


@pytest.mark.parametrize("scale", [0.05, -0.2])
def test_scales(cuda_device, scale):
    _full_check(1, 2, 256, 64, True, cuda_device, scale=scale, seed=321)
    _full_check(1, 1, 256, 128, False, cuda_device, scale=scale, seed=322)


@pytest.mark.parametrize("d", [64, 128])
def test_blocksparse_small(cuda_device, d):
    N = 768
    mask = make_tile_mask(N // 128, seed=5, density=0.4)
    mask[3, :] = 0  # query tile with nothing kept: dQ = 0 there
    mask[:, 4] = 0  # key tile nobody sees: dK = dV = 0 there
    mask[4, 4] = 0
    t, _, (dq, dk, dv) = _full_check(1, 2, N, d, False, cuda_device, seed=331, mask=mask)
    assert torch.all(dq[:, :, 384:512] == 0)
    assert torch.all(dk[:, :, 512:640] == 0) and torch.all(dv[:, :, 512:640] == 0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_many_items_per_cta(cuda_device, causal, d):
    """More (key tile, head) items than SMs: every persistent CTA runs several, and the
    dQ rows of one query tile receive reduce-adds from many CTAs."""
    _full_check(2, 80, 640, d, causal, cuda_device, seed=351 + d)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [300, 1000])
def test_paired_causal_items(cuda_device, N, d):
    """Causal items dealt as pairs of key tiles (j, n - 1 - j): with one head per SM the
    pairs fill every CTA round, so the launcher pairs them; N = 300 has a middle tile
    (3 key tiles) that forms a pair of its own."""
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    _full_check(1, sms, N, d, True, cuda_device, seed=371 + d, heads=[(0, 0), (0, sms // 2), (0, sms - 1)])


def test_head_dim_96(cuda_device):
    _full_check(1, 3, 384, 96, True, cuda_device, seed=361)
    _full_check(1, 2, 256, 96, False, cuda_device, seed=362)


@pytest.mark.parametrize("N", [1, 77, 129, 300, 1000])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_lengths(cuda_device, N, d, causal):
    """Partial last tiles, outputs as prefixes of NaN-filled buffers: nothing is written
    past N rows, and key rows past N contribute nothing to dQ."""
    B, H = 2, 3
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=370 + N + d).items()}
    sc = 1.0 / math.sqrt(d)
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc)
    shape = (B, H, N, d)
    bufs = [_padded(shape, torch.bfloat16, cuda_device, float("nan")) for _ in range(3)]
    dq, dk, dv = _fused(t, o, lse, causal, sc, grads=tuple(b[1] for b in bufs))
    for big, _ in bufs:
        assert _tail_untouched(big, math.prod(shape), float("nan")), "gradient written past its end"
    for b in range(B):
        for h in range(H):
            sl = lambda x: x[b:b + 1, h:h + 1].cpu()
            ref = oracle.attn_bwd_ref(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["do"]), causal, sc)
            for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
                g64 = f64(sl(g))
                if N == 1 and name in ("dq", "dk"):
                    # one visible key: the exact value is 0; the GPU value is bounded by the
                    # effect of forming D from the bf16-rounded O (scale 2^-8 |dO.O| |K|)
                    bound = sc * 2.0 ** -8 * float(np.abs(f64(sl(t["do"])) * f64(sl(o))).sum()) * \
                        float(np.abs(f64(sl(t["k"] if name == "dq" else t["q"]))).max())
                    assert float(np.abs(g64).max()) <= max(bound, 1e-6), (name, N)
                else:
                    assert_grad_close(sl(g), ref[name], name, f"fused ragged N{N} d{d} causal={causal}")


@pytest.mark.parametrize("nq,nk", [(1, 1000), (77, 300), (300, 77), (256, 640), (640, 256)])
@pytest.mark.parametrize("causal", [False, True])
def test_cross_lengths(cuda_device, nq, nk, causal):
    """N_q != N_k (bottom-right causal): rows that see no key get dQ = 0."""
    d, B, H = 64 if nq % 2 else 128, 2, 2
    a = make_qkv(B, H, nq, d, seed=380 + nq)
    kv = make_qkv(B, H, nk, d, seed=381 + nk)
    t = {"q": a["q"].to(cuda_device), "do": a["do"].to(cuda_device), "k": kv["k"].to(cuda_device),
         "v": kv["v"].to(cuda_device)}
    sc = 1.0 / math.sqrt(d)
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc)
    dq, dk, dv = _fused(t, o, lse, causal, sc)
    if causal and nq > nk:
        assert torch.all(dq[:, :, : nq - nk] == 0)
    for b in range(B):
        for h in range(H):
            sl = lambda x: x[b:b + 1, h:h + 1].cpu()
            ref = oracle.attn_bwd_ref(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["do"]), causal, sc)
            for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
                assert_grad_close(sl(g), ref[name], name, f"fused Nq{nq} Nk{nk} causal={causal}")


def test_bnhd_layout(cuda_device):
    """[B, N, H, d] tensors give the transposed [B, H, N, d] result."""
    B, H, N, d = 2, 3, 300, 128
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=391).items()}
    sc = d ** -0.5
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal=True, scale=sc)
    ref = _fused(t, o, lse, True, sc)
    tt = {k: x.transpose(1, 2).contiguous() for k, x in t.items()}
    g = fa.backward(tt["q"], tt["k"], tt["v"], o.transpose(1, 2).contiguous(), lse, tt["do"], causal=True,
                    scale=sc, layout="bnhd", deterministic=False)
    torch.cuda.synchronize()
    for x, y in zip(g, ref):
        assert float((x.transpose(1, 2).float() - y.float()).abs().max()) <= 2e-2 * float(y.float().abs().max())


def test_matches_deterministic_path(cuda_device):
    """dK and dV follow the same tile order as the deterministic dK/dV kernel; dQ sums
    the same shares in another order: all three agree within the gradient tolerance
    of each other, and the fused dV is bit-identical (same products, same order)."""
    B, H, N, d = 2, 4, 1024, 128
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=392).items()}
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal=True)
    a = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal=True)
    b = _fused(t, o, lse, True, d ** -0.5)
    assert torch.equal(a[2], b[2])
    for x, y in zip(a, b):
        assert float((x.float() - y.float()).abs().max()) <= 2e-2 * float(x.float().abs().max())


def test_staged_calls(cuda_device):
    """fa_bwd_fused_preprocess + fa_bwd_fused_main + fa_bwd_fused_dq is fa_bwd_fused."""
    B, H, N, d = 1, 3, 640, 64
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=393).items()}
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal=True, scale=0.11)
    ref = _fused(t, o, lse, True, 0.11)
    ws = torch.empty(fa.bwd_workspace_bytes(B, H, N, d, deterministic=False), dtype=torch.uint8,
                     device=cuda_device)
    dq, dk, dv = (torch.empty_like(t["q"]) for _ in range(3))
    fa.bwd_fused_preprocess(o, t["do"], lse, ws)
    fa.bwd_fused_main(t["q"], t["k"], t["v"], t["do"], dk, dv, ws, causal=True, scale=0.11)
    fa.bwd_fused_dq(dq, ws, scale=0.11)
    torch.cuda.synchronize()
    assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
    assert float((dq.float() - ref[0].float()).abs().max()) <= 1e-2 * float(ref[0].float().abs().max())


def test_workspace_too_small_is_rejected(cuda_device):
    t = {k: x.to(cuda_device) for k, x in make_qkv(1, 1, 128, 64, seed=394).items()}
    o, lse = fa.forward(t["q"], t["k"], t["v"])
    small = torch.empty(fa.bwd_workspace_bytes(1, 1, 128, 64), dtype=torch.uint8, device=cuda_device)
    with pytest.raises(fa.FAError) as e:
        fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], workspace=small, deterministic=False)
    assert e.value.status == 4


# ------------------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("causal", [False, True])
def test_b8h16n2048d64(cuda_device, causal):
    _full_check(8, 16, 2048, 64, causal, cuda_device, heads=[(0, 0), (3, 7), (7, 15)])


def test_b2h16n8192d128_causal(cuda_device):
    _full_check(2, 16, 8192, 128, True, cuda_device, heads=[(0, 0), (1, 15)])


def test_b1h16n16384d64_sparse(cuda_device):
    B, H, N, d = 1, 16, 16384, 64
    mask = make_tile_mask(N // 128, seed=0, density=0.25)
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=0).items()}
    sc = 1.0 / math.sqrt(d)
    m = mask.to(cuda_device)
    o, lse = _fwd(t, False, sc, m)
    dq, dk, dv = _fused(t, o, lse, False, sc, m)
    rows = sample_rows(N, n_random=16)
    cols = sample_rows(N, n_random=16, seed=1)
    mk = mask.numpy()
    for hh in (0, 15):
        c = {k: x[0, hh].cpu() for k, x in t.items()}
        ref_dq = oracle.attn_dq_rows_ref(f64(c["q"])[rows], rows, c["k"], c["v"], f64(c["do"])[rows], False, sc,
                                         mk, 128)
        assert_grad_close(dq[0, hh].cpu()[torch.as_tensor(rows)], ref_dq, "dq", f"fused sparse h={hh}")
        ref_dk, ref_dv = oracle.attn_dkdv_cols_ref(c["q"], c["k"], c["v"], c["do"], cols, False, sc, mk, 128)
        assert_grad_close(dk[0, hh].cpu()[torch.as_tensor(cols)], ref_dk, "dk", f"fused sparse h={hh}")
        assert_grad_close(dv[0, hh].cpu()[torch.as_tensor(cols)], ref_dv, "dv", f"fused sparse h={hh}")


@pytest.mark.parametrize("N", [512, 2048, 8192, 16384])
@pytest.mark.parametrize("d", [64, 128])
def test_sweep_points(cuda_device, N, d):
    B, H = sweep_shape(N, d)
    sc = 1.0 / math.sqrt(d)
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=0, do_scale=0.5).items()}
    rows = sample_rows(N, n_random=12)
    cols = sample_rows(N, n_random=12, seed=1)
    for causal in (False, True):
        o, lse = _fwd(t, causal, sc)
        dq, dk, dv = _fused(t, o, lse, causal, sc)
        for (b, hh) in ((0, 0), (B - 1, H - 1)):
            c = {k: x[b, hh].cpu() for k, x in t.items()}
            w = f"fused B{B} H{H} N{N} d{d} causal={causal} (b={b}, h={hh})"
            ref_dq = oracle.attn_dq_rows_ref(f64(c["q"])[rows], rows, c["k"], c["v"], f64(c["do"])[rows], causal,
                                             sc)
            assert_grad_close(dq[b, hh].cpu()[torch.as_tensor(rows)], ref_dq, "dq", w)
            ref_dk, ref_dv = oracle.attn_dkdv_cols_ref(c["q"], c["k"], c["v"], c["do"], cols, causal, sc)
            assert_grad_close(dk[b, hh].cpu()[torch.as_tensor(cols)], ref_dk, "dk", w)
            assert_grad_close(dv[b, hh].cpu()[torch.as_tensor(cols)], ref_dv, "dv", w)
