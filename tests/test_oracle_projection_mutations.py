"""Plant plausible mistakes in copies of the two projection oracles (the QKV
projection and the output projection) and check that their pins catch each
one.  The mutants replace the oracle function for the duration of one check;
the real oracle is untouched."""
import numpy as np
import pytest
import torch

import oracle
from tests import test_oracle_pins as pins


def _f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


def _qkv_kv_swapped(x, w, n_head, n_kv_head, head_dim):
    y = _f64(x) @ _f64(w).T
    T = y.shape[0]
    hq, hk = n_head * head_dim, n_kv_head * head_dim
    return (y[:, :hq].reshape(T, n_head, head_dim), y[:, hq + hk:].reshape(T, n_kv_head, head_dim),
            y[:, hq:hq + hk].reshape(T, n_kv_head, head_dim))


def _qkv_head_dim_first(x, w, n_head, n_kv_head, head_dim):
    y = _f64(x) @ _f64(w).T
    T = y.shape[0]
    hq, hk = n_head * head_dim, n_kv_head * head_dim

    def split(a, heads):
        return a.reshape(T, head_dim, heads).transpose(0, 2, 1)

    return split(y[:, :hq], n_head), split(y[:, hq:hq + hk], n_kv_head), split(y[:, hq + hk:], n_kv_head)


def _out_head_dim_first_merge(o, w_o):
    os_ = _f64(o)
    merged = os_.transpose(0, 2, 1).reshape(os_.shape[0], -1)
    return merged @ _f64(w_o).T


def _out_weight_read_input_major(o, w_o):
    """W_o's storage read as [in][out] instead of one row per output feature."""
    os_ = _f64(o)
    merged = os_.reshape(os_.shape[0], -1)
    return merged @ _f64(w_o).reshape(merged.shape[1], -1)


QKV_PINS = [pins.test_qkv_projection_brute_force_tiny, pins.test_qkv_projection_one_hot_weights_select_features,
            pins.test_qkv_projection_matches_torch_linear_fp64]
OUT_PINS = [pins.test_out_projection_brute_force_tiny, pins.test_out_projection_head_block_selects_that_head]

MUTANTS = {
    "qkv_k_and_v_ranges_swapped": ("qkv_projection", _qkv_kv_swapped, QKV_PINS),
    "qkv_head_dim_first_split": ("qkv_projection", _qkv_head_dim_first, QKV_PINS),
    "out_head_dim_first_merge": ("out_projection", _out_head_dim_first_merge, OUT_PINS),
    "out_weight_read_input_major": ("out_projection", _out_weight_read_input_major, OUT_PINS),
}


def _caught(calls) -> bool:
    for call in calls:
        try:
            call()
        except Exception:  # an assertion, or a shape error from the planted mistake
            return True
    return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_projection_mutant_is_caught(name, monkeypatch):
    attr, fn, calls = MUTANTS[name]
    monkeypatch.setattr(oracle, attr, fn)
    assert _caught(calls), f"mutant {name} passed every pin"


def test_unmutated_projection_oracles_pass():
    assert not _caught(QKV_PINS + OUT_PINS)
