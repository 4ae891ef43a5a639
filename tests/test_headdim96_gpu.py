"""Head dim 96 (run on the 128-wide kernels with the last 32 columns read as zeros):
forward and backward against the fp64 oracle, square, ragged, N_q != N_k and
block-sparse, with sentinels that catch writes past the 96 stored columns' rows."""
import pytest

from exact_tiled_attention_34_b200.inputs import make_tile_mask
from tests.test_cross_gpu import _check as _check_cross
from tests.test_ragged_gpu import _check as _check_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 300, 1000])
def test_d96_lengths(cuda_device, N, causal):
    _check_rows(2, 2, N, 96, causal, cuda_device, seed=900 + N)


@pytest.mark.parametrize("causal", [False, True])
def test_d96_cross(cuda_device, causal):
    _check_cross(1, 2, 200, 650, 96, causal, cuda_device, seed=911)


def test_d96_blocksparse(cuda_device):
    mask = make_tile_mask(6, seed=19, density=0.4)
    _check_rows(1, 2, 700, 96, False, cuda_device, mask=mask, seed=913)


def test_d96_many_items(cuda_device):
    _check_rows(2, 80, 384, 96, True, cuda_device, seed=917)
