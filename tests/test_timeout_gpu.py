"""The bounded device waits behind FA_ERR_DEVICE_TIMEOUT, made to run out on the
GPU without a fault. A self-test kernel waits on barriers that nothing completes:
the timeout must be recorded with its site, the sibling wait must leave on the
abort flag, and the status word must clear on read. Then the attention kernels
themselves, launched with an idle TMA producer (nothing is ever in flight), must
end through their timeout path and teardown, and the context must stay usable:
the next launches are parity-green against the oracle."""
import contextlib
import math

import pytest
import torch

import exact_tiled_attention_34_b200 as fa
import oracle
from exact_tiled_attention_34_b200.inputs import make_qkv
from tests.parity import assert_fwd_close, assert_grad_close

pytestmark = pytest.mark.gpu

TIMEOUT = 6  # FA_ERR_DEVICE_TIMEOUT
SITE = 901
# Waits that an idle producer leaves hanging first: the MMA issuer's wait for Q
# (forward) or for the first K/V or Q tiles (backward), and the softmax / compute
# warps' wait for the first score tile or staged tile.
FWD_SITES = {101, 106}
DKDV_SITES = {201, 203}
DQ_SITES = {201, 206}


@contextlib.contextmanager
def _stalled(timeout_us):
    fa.debug_stall_producer(True, timeout_us)
    try:
        yield
    finally:
        fa.debug_stall_producer(False)


@pytest.mark.parametrize("timeout_us", [200, 5000])
def test_wait_gives_up_and_reports(cuda_device, timeout_us):
    assert fa.device_status() == (0, 0)
    status, detail, out = fa.debug_wait_timeout(timeout_us)
    assert (status, detail) == (TIMEOUT, SITE)
    gave_up, left_on_flag, waited_us = out
    assert gave_up == 1 and left_on_flag == 1
    # bounded: at least the limit, and not the sibling's 64x longer one
    assert timeout_us <= waited_us < 64 * timeout_us + 20000
    assert fa.device_status() == (0, 0)  # cleared by the read


def test_context_usable_after_timeout(cuda_device):
    status, _, _ = fa.debug_wait_timeout(1000)
    assert status == TIMEOUT
    B, H, N, d = 1, 2, 300, 64
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=11).items()}
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal=True)
    assert fa.device_status() == (0, 0)
    ref = oracle.attn_bwd_ref(t["q"].cpu(), t["k"].cpu(), t["v"].cpu(), t["do"].cpu(), True, d ** -0.5, None, 128)
    assert_fwd_close(o.cpu(), lse.cpu(), ref["o"], ref["lse"], "forward after a timeout")


def _inputs(B, H, N, d, dev, seed):
    return {k: x.to(dev) for k, x in make_qkv(B, H, N, d, seed=seed).items()}


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_attention_kernels_end_through_timeout(cuda_device, d, causal):
    B, H, N = 2, 4, 640
    t = _inputs(B, H, N, d, cuda_device, seed=5)
    sc = 1.0 / math.sqrt(d)
    assert fa.device_status() == (0, 0)
    ws = torch.empty(fa.bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=cuda_device)
    dq, dk, dv = (torch.empty_like(t["q"]) for _ in range(3))
    o = torch.empty_like(t["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device=cuda_device)
    with _stalled(2000):
        fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc, out=o, lse=lse)
        st_fwd = fa.device_status()
        fa.bwd_preprocess(o, t["do"], lse, ws)
        fa.bwd_dkdv(t["q"], t["k"], t["v"], t["do"], dk, dv, ws, causal=causal, scale=sc)
        st_dkdv = fa.device_status()
        fa.bwd_dq(t["q"], t["k"], t["v"], t["do"], dq, ws, causal=causal, scale=sc)
        st_dq = fa.device_status()
    assert st_fwd[0] == TIMEOUT and st_fwd[1] in FWD_SITES, st_fwd
    assert st_dkdv[0] == TIMEOUT and st_dkdv[1] in DKDV_SITES, st_dkdv
    assert st_dq[0] == TIMEOUT and st_dq[1] in DQ_SITES, st_dq
    # Normal launches again, in the same context: parity with the oracle.
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc)
    dq, dk, dv = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal=causal, scale=sc)
    assert fa.device_status() == (0, 0)
    for b, h in ((0, 0), (B - 1, H - 1)):
        sl = lambda x: x[b:b + 1, h:h + 1].cpu()
        ref = oracle.attn_bwd_ref(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["do"]), causal, sc, None, 128)
        assert_fwd_close(sl(o), sl(lse), ref["o"], ref["lse"], f"after timeout d={d} causal={causal}")
        for name, g in (("q", dq), ("k", dk), ("v", dv)):
            assert_grad_close(sl(g), ref["d" + name], name, f"after timeout d={d} causal={causal}")


def test_stall_hook_arguments():
    with pytest.raises(fa.FAError):
        fa.debug_stall_producer(True, 0)
    with pytest.raises(fa.FAError):
        fa.debug_stall_producer(True, 100001)
    fa.debug_stall_producer(False)


# The fused backward (head dims 64, 128) and the head-dim-256 kernels: which of their
# waits gives up first depends on timing, so any site of the kernel is accepted.
FUSED_SITES = set(range(301, 315))
FWD256_SITES = set(range(401, 413))
BWD256_SITES = set(range(501, 515))


@pytest.mark.parametrize("d,causal", [(64, True), (128, False), (256, True)])
def test_fused_kernels_end_through_timeout(cuda_device, d, causal):
    B, H, N = 2, 2, 640
    t = _inputs(B, H, N, d, cuda_device, seed=6)
    sc = 1.0 / math.sqrt(d)
    assert fa.device_status() == (0, 0)
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc)
    ws = torch.empty(fa.bwd_workspace_bytes(B, H, N, d, deterministic=False), dtype=torch.uint8, device=cuda_device)
    dk, dv = torch.empty_like(t["q"]), torch.empty_like(t["q"])
    with _stalled(2000):
        if d == 256:
            fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc, out=torch.empty_like(o),
                       lse=torch.empty_like(lse))
            st_fwd = fa.device_status()
        fa.bwd_fused_preprocess(o, t["do"], lse, ws)
        fa.bwd_fused_main(t["q"], t["k"], t["v"], t["do"], dk, dv, ws, causal=causal, scale=sc)
        st_bwd = fa.device_status()
    if d == 256:
        assert st_fwd[0] == TIMEOUT and st_fwd[1] in FWD256_SITES, st_fwd
    assert st_bwd[0] == TIMEOUT and st_bwd[1] in (BWD256_SITES if d == 256 else FUSED_SITES), st_bwd
    # Normal launches again, in the same context: parity with the oracle.
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=sc)
    dq, dk, dv = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal=causal, scale=sc, deterministic=False)
    assert fa.device_status() == (0, 0)
    for b, h in ((0, 0), (B - 1, H - 1)):
        sl = lambda x: x[b:b + 1, h:h + 1].cpu()
        ref = oracle.attn_bwd_ref(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["do"]), causal, sc, None, 128)
        assert_fwd_close(sl(o), sl(lse), ref["o"], ref["lse"], f"after timeout d={d} causal={causal}")
        for name, g in (("q", dq), ("k", dk), ("v", dv)):
            assert_grad_close(sl(g), ref["d" + name], name, f"after timeout d={d} causal={causal}")
