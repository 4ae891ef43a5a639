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
