"""CPU tests of the Python binding's argument checks for the dropout, merge and ring
entry points: bad arguments raise before any CUDA call, and there is no CPU path."""
import pytest
import torch

import exact_tiled_attention_34_b200 as fa
from exact_tiled_attention_34_b200 import ring


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_dropout_rejects_cpu_tensors_and_bad_rates():
    q = _bf16(1, 1, 128, 64)
    with pytest.raises(ValueError):
        fa.forward_dropout(q, q, q, 0.1, 0)  # CPU tensors: no CPU path
    with pytest.raises(ValueError):
        fa._seed_args(1.0, 0, 0)
    with pytest.raises(ValueError):
        fa._seed_args(-0.01, 0, 0)
    assert fa._seed_args(0.25, -1, -1) == (0.25, 2 ** 64 - 1, 2 ** 32 - 1)  # seed, offset wrap


def test_dropout_needs_equal_lengths():
    q, k = _bf16(1, 1, 128, 64), _bf16(1, 1, 256, 64)
    with pytest.raises(ValueError):
        fa.forward_dropout(q, k, k, 0.1, 0)
    with pytest.raises(ValueError):
        fa.backward_dropout(q, k, k, q, torch.zeros(1, 1, 128), q, 0.1, 0)


def test_attention_dropout_only_in_bhnd_layout():
    q = _bf16(1, 128, 1, 64)
    with pytest.raises(ValueError):
        fa.attention(q, q, q, layout="bnhd", dropout_p=0.1, seed=1)


def test_merge_and_accumulate_check_dtypes_and_devices():
    acc = torch.zeros(1, 1, 128, 64)
    lse = torch.zeros(1, 1, 128)
    part = _bf16(1, 1, 128, 64)
    with pytest.raises(ValueError):
        fa.merge_partial(acc, lse, acc, lse)  # partial O must be bf16
    with pytest.raises(ValueError):
        fa.merge_partial(acc, lse.double(), part, lse)
    with pytest.raises(ValueError):
        fa.merge_partial(acc, lse, part, lse)  # CPU tensors
    with pytest.raises(ValueError):  # more lse rows than rows of O: the kernel would run past O
        fa.merge_partial(acc, torch.zeros(1, 1, 256), part, torch.zeros(1, 1, 256))
    with pytest.raises(ValueError):  # fewer lse rows than rows of O
        fa.merge_partial(acc, torch.zeros(1, 1, 64), part, torch.zeros(1, 1, 64))
    with pytest.raises(ValueError):
        fa.accumulate_bf16(acc, acc)
    with pytest.raises(ValueError):
        fa.accumulate_bf16(acc, part)  # CPU tensors
    with pytest.raises(ValueError):
        fa.to_bf16(acc)  # CPU tensor


def test_ring_visibility_rule():
    # chunks of one length at multiples of it: causal key chunk before the query chunk is
    # fully visible, the same chunk is the causal diagonal, a later one is invisible
    n = 64
    assert [ring._pair_kind(True, 2 * n, s * n) for s in range(4)] == ["full", "full", "diag", None]
    assert all(ring._pair_kind(False, 0, s * n) == "full" for s in range(4))
    assert ring.chunk_offsets(1, 4, 128, False) == [128]
    assert ring.chunk_offsets(1, 4, 128, True) == [64, 6 * 64]  # chunks 1 and 2R - 1 - 1 = 6


class _RingThatMustNotExchange:
    """A two-rank ring whose exchange fails the test if it is ever started."""
    rank, world = 0, 2

    def start(self, tensors):
        raise AssertionError("an exchange was posted before the arguments were checked")

    finish = exchange = start


def test_ring_rejects_head_dim_96_before_any_exchange():
    q = _bf16(1, 1, 128, 96)
    ops = ring.CudaBlockOps(0.1)
    with pytest.raises(ValueError):
        ring.ring_forward(q, q, q, ring=_RingThatMustNotExchange(), ops=ops)
    lse = torch.zeros(1, 1, 128)
    with pytest.raises(ValueError):
        ring.ring_backward(q, q, q, q, lse, q, ring=_RingThatMustNotExchange(), ops=ops)


def test_ring_rejects_blocks_of_different_shapes():
    q, k = _bf16(1, 1, 128, 64), _bf16(1, 1, 256, 64)
    with pytest.raises(ValueError):
        ring.ring_forward(q, k, k, ring=_RingThatMustNotExchange(), ops=ring.CudaBlockOps(0.1))


def test_caller_buffers_are_checked_before_any_call():
    """Outputs, row arrays and workspaces a caller supplies reach the C entry points as bare
    pointers: shape, dtype, contiguity and device are checked in the binding."""
    cpu = torch.device("cpu")
    good = _bf16(1, 2, 128, 64)
    fa._check_buffer(good, (1, 2, 128, 64), torch.bfloat16, cpu, "out")  # accepted
    fa._check_buffer(torch.zeros(100, dtype=torch.uint8), None, torch.uint8, cpu, "workspace")
    with pytest.raises(ValueError):  # one query row short: the kernel would write past it
        fa._check_buffer(_bf16(1, 2, 127, 64), (1, 2, 128, 64), torch.bfloat16, cpu, "out")
    with pytest.raises(ValueError):
        fa._check_buffer(good.float(), (1, 2, 128, 64), torch.bfloat16, cpu, "out")
    with pytest.raises(ValueError):
        fa._check_buffer(_bf16(1, 2, 64, 128).transpose(2, 3), (1, 2, 128, 64), torch.bfloat16, cpu, "out")
    with pytest.raises(ValueError):  # a workspace must be bytes (its size is counted in elements)
        fa._check_buffer(torch.zeros(100), None, torch.uint8, cpu, "workspace")
    with pytest.raises(ValueError):  # on another device than q
        fa._check_buffer(good, (1, 2, 128, 64), torch.bfloat16, torch.device("cuda", 0), "out")
    with pytest.raises(ValueError):
        fa._check_outputs(good, None, torch.zeros(1, 2, 64), (1, 2, 128))
    with pytest.raises(ValueError):
        fa._check_equal_lengths(good, _bf16(1, 2, 256, 64), "block-sparse attention")
    fa._check_equal_lengths(good, good, "block-sparse attention")


def test_staged_calls_reject_cpu_tensors():
    q = _bf16(1, 1, 128, 64)
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    lse = torch.zeros(1, 1, 128)
    with pytest.raises(ValueError):
        fa.bwd_preprocess(q, q, lse, ws)
    with pytest.raises(ValueError):
        fa.bwd_fused_preprocess(q, q, lse, ws)
    with pytest.raises(ValueError):
        fa.bwd_dkdv(q, q, q, q, q, q, ws)
    with pytest.raises(ValueError):
        fa.bwd_dq(q, q, q, q, q, ws)
    with pytest.raises(ValueError):
        fa.bwd_fused_main(q, q, q, q, q, q, ws)
    with pytest.raises(ValueError):
        fa.bwd_fused_dq(q, ws)
    with pytest.raises(ValueError):
        fa.bwd_fused_main_f32(q, q, q, q, q.float(), q.float(), ws)
