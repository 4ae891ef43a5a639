"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Such callers (a plugin whose host application owns all device memory and passes
it only inputs and outputs, or a latency-critical loop that must not pay for
cudaMalloc's implicit synchronisation) get the same gradients as fa_bwd, with the
scratch taken from an array compiled into the library. This file is collected
last so that a run stopping at its first failure has already run every other test.
"""
import ctypes

import pytest
import torch

import exact_tiled_attention_34_b200 as fa
from exact_tiled_attention_34_b200.inputs import make_qkv, make_tile_mask
from tests.parity import assert_grad_close, f64

SCRATCH_BYTES = 8 * 1024 * 1024  # FA_BWD_NOALLOC_SCRATCH_BYTES in include/fa.h


def _noalloc_fn():
    from exact_tiled_attention_34_b200 import build
    build.build()
    fn = fa.lib().fa_bwd_noalloc
    v, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [v] * 10 + [i] * 6 + [ctypes.c_float, v]
    fn.restype = i
    return fn


def _call(fn, t, o, lse, grads, mask, causal, scale):
    B, H, N, d = t["q"].shape
    dq, dk, dv = grads
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), o.data_ptr(), lse.data_ptr(),
              t["do"].data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
              None if mask is None else mask.data_ptr(), 128, B, H, N, d, int(causal), scale, stream)


def test_oversized_request_is_rejected_without_touching_the_gpu():
    fn = _noalloc_fn()
    a = 1 << 20  # aligned stand-in addresses; the size check comes first
    # B*H*N = 1,048,576 rows fit (any d); 1,048,704 do not.
    assert fa.lib().fa_bwd_workspace_bytes(1, 16, 65536, 64) <= SCRATCH_BYTES
    assert fa.lib().fa_bwd_workspace_bytes(1, 1, 1048704, 64) > SCRATCH_BYTES
    assert fn(a, a, a, a, a, a, a, a, a, None, 128, 1, 1, 1048704, 64, 0, 0.125, None) == 4
    assert fn(a, a, a, a, a, a, a, a, a, None, 128, 3, 1, 349568, 128, 1, 0.125, None) == 4
    assert fn(None, a, a, a, a, a, a, a, a, None, 128, 1, 1, 128, 64, 0, 0.125, None) == 1
    assert fn(a, a, a, a, a, a, a, a, a, a, 64, 1, 1, 128, 64, 0, 0.125, None) == 2


@pytest.mark.gpu
@pytest.mark.parametrize("case", [
    dict(B=2, H=4, N=1024, d=128, causal=True, sparse=False),
    dict(B=2, H=3, N=768, d=64, causal=False, sparse=False),
    dict(B=1, H=2, N=1024, d=64, causal=False, sparse=True),
])
def test_matches_fa_bwd_on_two_calls_in_a_row(cuda_device, case):
    fn = _noalloc_fn()
    B, H, N, d = case["B"], case["H"], case["N"], case["d"]
    causal, scale = case["causal"], d ** -0.5
    t = {k: x.to(cuda_device) for k, x in make_qkv(B, H, N, d, seed=77).items()}
    mask = make_tile_mask(N // 128, seed=2, density=0.4).to(cuda_device) if case["sparse"] else None
    if mask is None:
        o, lse = fa.forward(t["q"], t["k"], t["v"], causal=causal, scale=scale)
        ref = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal=causal, scale=scale)
    else:
        o, lse = fa.forward_blocksparse(t["q"], t["k"], t["v"], mask, scale=scale)
        ref = fa.backward_blocksparse(t["q"], t["k"], t["v"], o, lse, t["do"], mask, scale=scale)
    for call in range(2):  # the second call runs on whatever the first left in the scratch array
        grads = tuple(torch.full_like(t["q"], float("nan")) for _ in range(3))
        assert _call(fn, t, o, lse, grads, mask, causal, scale) == 0
        torch.cuda.synchronize()
        assert fa.device_status() == (0, 0)
        for name, g, r in zip(("dq", "dk", "dv"), grads, ref):
            assert_grad_close(g, f64(r), name, f"call {call + 1}, {case}")
