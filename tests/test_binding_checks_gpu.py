"""Caller-supplied outputs, row arrays, gradients and workspaces reach the C entry points as
bare pointers, so the binding checks their shape, dtype, contiguity and device: each call
below passes valid CUDA inputs except for one argument and must raise ValueError before
anything is launched. Valid calls of the same entry points run in the parity tests."""
import pytest
import torch

import exact_tiled_attention_34_b200 as fa
from exact_tiled_attention_34_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

B, H, N, D = 1, 2, 256, 64


@pytest.fixture(scope="module")
def case(cuda_device):
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, D, seed=2900).items()}
    o, lse = fa.forward(t["q"], t["k"], t["v"])
    ws = torch.empty(fa.bwd_workspace_bytes(B, H, N, D), dtype=torch.uint8, device=cuda_device)
    wsf = torch.empty(fa.bwd_workspace_bytes(B, H, N, D, deterministic=False), dtype=torch.uint8,
                      device=cuda_device)
    torch.cuda.synchronize()
    return t, o, lse, ws, wsf


def _bad(shape=None, dtype=torch.bfloat16, device="cuda:0"):
    return torch.zeros(shape if shape is not None else (B, H, N, D), dtype=dtype, device=device)


def test_forward_outputs(case):
    t, *_ = case
    q, k, v = t["q"], t["k"], t["v"]
    for kwargs in ({"out": _bad((B, H, N - 1, D))}, {"out": _bad(dtype=torch.float32)},
                   {"out": _bad(device="cpu")}, {"lse": _bad((B, H, N // 2), torch.float32)},
                   {"lse": _bad((B, H, N), torch.bfloat16)}, {"lse": _bad((B, H, N), torch.float32, "cpu")}):
        with pytest.raises(ValueError):
            fa.forward(q, k, v, **kwargs)
        with pytest.raises(ValueError):
            fa.forward_dropout(q, k, v, 0.1, 7, **kwargs)
    mask = torch.ones((N // 128, N // 128), dtype=torch.uint8, device=q.device)
    with pytest.raises(ValueError):
        fa.forward_blocksparse(q, k, v, mask, out=_bad((B, H, N - 1, D)))


def test_block_sparse_needs_equal_lengths(case):
    t, o, lse, ws, _ = case
    q = t["q"]
    k2 = torch.cat([t["k"], t["k"]], dim=2)
    mask = torch.ones((N // 128, N // 128), dtype=torch.uint8, device=q.device)
    with pytest.raises(ValueError):
        fa.forward_blocksparse(q, k2, k2, mask)
    with pytest.raises(ValueError):
        fa.backward_blocksparse(q, k2, k2, o, lse, t["do"], mask, workspace=ws)


def test_backward_gradients_and_workspace(case):
    t, o, lse, ws, wsf = case
    args = (t["q"], t["k"], t["v"], o, lse, t["do"])
    good = tuple(torch.empty_like(t[n]) for n in ("q", "k", "v"))
    for det, w in ((True, ws), (False, wsf)):
        with pytest.raises(ValueError):  # workspace in host memory
            fa.backward(*args, workspace=w.cpu(), deterministic=det)
        with pytest.raises(ValueError):  # not bytes
            fa.backward(*args, workspace=torch.empty(w.numel() // 4, device=w.device), deterministic=det)
        with pytest.raises(ValueError):
            fa.backward(*args, workspace=w, grads=good[:2], deterministic=det)
        with pytest.raises(ValueError):  # dk one key row short
            fa.backward(*args, workspace=w, grads=(good[0], _bad((B, H, N - 1, D)), good[2]), deterministic=det)
        with pytest.raises(ValueError):
            fa.backward(*args, workspace=w, grads=(good[0].float(), good[1], good[2]), deterministic=det)
    with pytest.raises(ValueError):
        fa.backward_dropout(*args, 0.1, 7, workspace=ws, grads=(good[0], good[1], _bad(device="cpu")))


def test_staged_calls(case):
    t, o, lse, ws, wsf = case
    q, k, v, do = t["q"], t["k"], t["v"], t["do"]
    g = _bad()
    short = _bad((B, H, N - 128, D))
    with pytest.raises(ValueError):
        fa.bwd_preprocess(o, do, lse[:, :, :-1].contiguous(), ws)
    with pytest.raises(ValueError):
        fa.bwd_preprocess(o, do, lse, ws.cpu())
    with pytest.raises(ValueError):
        fa.bwd_fused_preprocess(o, short, lse, wsf)
    with pytest.raises(ValueError):
        fa.bwd_dkdv(q, k, v, do, short, g, ws)
    with pytest.raises(ValueError):
        fa.bwd_dkdv(q, short, short, do, g, g, ws)
    with pytest.raises(ValueError):
        fa.bwd_dq(q, k, v, do, g.float(), ws)
    with pytest.raises(ValueError):
        fa.bwd_dq(q, k, v, do, g, ws, tile_mask=torch.ones((1, 1), dtype=torch.uint8, device=q.device))
    with pytest.raises(ValueError):
        fa.bwd_fused_main(q, k, v, do, g, _bad(device="cpu"), wsf)
    with pytest.raises(ValueError):
        fa.bwd_fused_dq(short, torch.empty(wsf.numel() // 4, device=wsf.device))
    with pytest.raises(ValueError):
        fa.bwd_fused_main_f32(q, k, v, do, g.float(), g.float().cpu(), wsf)
    with pytest.raises(ValueError):
        fa.forward_merge(q, k, v, g.float().cpu(), lse.clone())
    with pytest.raises(ValueError):
        fa.forward_merge(q, k, v, g.float(), lse.cpu())


def test_nothing_ran_and_valid_calls_still_pass(case):
    """The rejected calls left no error behind, and the same entry points accept valid
    arguments (supplied outputs and workspace included)."""
    t, o, lse, ws, wsf = case
    out, l2 = torch.empty_like(o), torch.empty_like(lse)
    fa.forward(t["q"], t["k"], t["v"], out=out, lse=l2)
    grads = tuple(torch.empty_like(t[n]) for n in ("q", "k", "v"))
    fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], workspace=ws, grads=grads)
    torch.cuda.synchronize()
    assert torch.equal(out, o) and torch.equal(l2, lse)
    assert all(torch.isfinite(x.float()).all() for x in grads)
    assert fa.device_status()[0] == 0
