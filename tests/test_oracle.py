"""CPU tests of the fp64 oracle against its pins, plus a mutation check showing that
plausible mistakes planted in a copy of the oracle are caught by at least one pin."""
import importlib.util
import os
import sys
import types

import numpy as np
import pytest

import oracle
from oracle import attention as oracle_attention
from tests import oracle_pins

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle_attention)


def test_package_exports():
    for name in ("attn_fwd_ref", "attn_bwd_ref", "attn_fwd_rows_ref", "attn_probs_ref", "attn_scores_ref"):
        assert callable(getattr(oracle, name))


def test_oracle_does_not_import_cuda_path():
    src = open(oracle_attention.__file__).read()
    assert "exact_tiled_attention_34_b200" not in src
    assert "ctypes" not in src


# Each mutation is a plausible slip: a dropped term, a wrong sign or index, a
# transposed operand, an off-by-one in a mask.
MUTATIONS = {
    "dropped_scale": ("s = float(scale) * (q @ k.T)", "s = (q @ k.T)"),
    "causal_off_by_one": ("cols[None, :] <= rows[:, None] + causal_offset", "cols[None, :] < rows[:, None] + causal_offset"),
    "causal_flipped": ("cols[None, :] <= rows[:, None] + causal_offset", "cols[None, :] >= rows[:, None] + causal_offset"),
    "causal_offset_sign": ("mask_block, n_k - n_q)", "mask_block, n_q - n_k)"),
    "causal_offset_dropped": ("mask_block, n_k - n_q)", "mask_block, 0)"),
    "dk_shaped_like_q": ('"dk": np.zeros_like(k)', '"dk": np.zeros_like(q)'),
    "block_mask_transposed": ("bm[rows[:, None] // mask_block, cols[None, :] // mask_block]",
                              "bm[cols[None, :] // mask_block, rows[:, None] // mask_block]"),
    "pv_transposed": ("o[b, h] = p @ v[b, h]", "o[b, h] = p.T @ v[b, h]"),
    "lse_dropped_max": ("m_safe + np.log(np.where(empty, 1.0, z))", "np.log(np.where(empty, 1.0, z))"),
    "softmax_no_normalise": ("e / np.where(empty, 1.0, z)", "e"),
    "dv_transposed": ("dv = p.T @ do[b, h]", "dv = p @ do[b, h]"),
    "ds_sign": ("ds = p * (dp - D[:, None])", "ds = p * (dp + D[:, None])"),
    "ds_dropped_D": ("ds = p * (dp - D[:, None])", "ds = p * dp"),
    "dq_dropped_scale": ('out["dq"][b, h] = scale * (ds @ k[b, h])', 'out["dq"][b, h] = (ds @ k[b, h])'),
    "dk_wrong_operand": ('out["dk"][b, h] = scale * (ds.T @ q[b, h])', 'out["dk"][b, h] = scale * (ds.T @ k[b, h])'),
    "dp_wrong_operand": ("dp = do[b, h] @ v[b, h].T", "dp = do[b, h] @ k[b, h].T"),
    "block_causal_strict": ("s = np.where(cols <= rows, s, -np.inf)", "s = np.where(cols < rows, s, -np.inf)"),
    "block_offsets_swapped": ("rows = q_off + np.arange(s.shape[0])[:, None]",
                              "rows = k_off + np.arange(s.shape[0])[:, None]"),
    "block_ds_dropped_D": ("ds = p * (dp - _f64(D)[:, None])", "ds = p * dp"),
    "cols_p_without_lse": ("np.exp(s_c - np.where(fin, lse[:, None], 0.0))", "np.exp(s_c)"),
    "cols_ds_dropped_D": ("ds_c = p_c * (dp_c - D[:, None])", "ds_c = p_c * dp_c"),
    "cols_dp_wrong_operand": ("dp_c = do @ v[cols].T", "dp_c = do @ k[cols].T"),
    "cols_dk_dropped_scale": ("return scale * (ds_c.T @ q), p_c.T @ do", "return (ds_c.T @ q), p_c.T @ do"),
    "cols_D_without_o": ("D[rows] = np.sum(do[rows] * (p @ v), axis=1)", "D[rows] = np.sum(do[rows] * v[rows], axis=1)"),
    "cols_causal_offset_dropped": ("mask_block, n_k - n_q, key_cols=cols)", "mask_block, 0, key_cols=cols)"),
    "cols_last_row_block_skipped": ("for r0 in range(0, n_q, row_block):", "for r0 in range(0, n_q - row_block, row_block):"),
    "block_dv_from_q": ("return scale * (ds @ k), scale * (ds.T @ q), p.T @ do",
                        "return scale * (ds @ k), scale * (ds.T @ q), p.T @ q"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src = open(oracle_attention.__file__).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    src = src.replace(old, new)
    mod = types.ModuleType(f"oracle_mutant_{name}")
    exec(compile(src, f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    mod = _mutant(name)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mod)
        except AssertionError:
            caught.append(pin.__name__)
        except Exception:  # a crash is also a detection
            caught.append(pin.__name__ + "(error)")
    assert caught, f"mutation {name} was not detected by any pin"
