"""The FMA-pipe exponential of the attention kernel (exp2_fma2) against exp2.

The pipelined kernel takes one exponential in eight of an unmasked block's
softmax as a Cody-Waite reduction plus a fitted cubic on the FMA pipe instead
of the MUFU ex2 unit.  Its stated accuracy is a relative error below 1e-4 for
inputs in [-125, 127] (the polynomial's own error is 8.4e-5; the fp32 Horner
evaluation adds a few ulp); inputs below -125 give about 2^-125.  The bound is
checked here, through the C ABI test hook, against exp2 in fp64 on a dense grid
plus the points where the reduction changes branch (integers and half-integers,
where round(y) switches)."""
import numpy as np
import pytest
import torch

from causal_prefill_attention_b200 import _lib

pytestmark = pytest.mark.gpu


def _run(x: np.ndarray) -> np.ndarray:
    y = _lib.exp2_fma2(torch.from_numpy(x.astype(np.float32)).cuda())
    torch.cuda.synchronize()
    return y.cpu().numpy()


def test_relative_error_over_the_range():
    grid = np.linspace(-125.0, 127.0, 4_000_001, dtype=np.float64).astype(np.float32)
    k = np.arange(-125, 128, dtype=np.float64)
    edges = np.concatenate([k, k + 0.5, np.nextafter(k + 0.5, -np.inf), np.nextafter(k + 0.5, np.inf)])
    x = np.concatenate([grid, edges[(edges >= -125) & (edges <= 127)].astype(np.float32)])
    y = _run(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert np.isfinite(y).all()
    assert rel.max() < 1e-4, f"max relative error {rel.max():.3e} at x = {x[rel.argmax()]}"


def test_inputs_below_the_range_give_about_2_to_the_minus_125():
    x = np.array([-125.0, -126.0, -200.0, -1e6, -np.inf], dtype=np.float32)
    y = _run(x).astype(np.float64)
    assert np.all(np.abs(y / 2.0 ** -125 - 1.0) < 1e-4), y


def test_odd_count_and_empty():
    x = np.array([0.0, 1.0, -1.0], dtype=np.float32)
    y = _run(x)
    assert np.allclose(y, [1.0, 2.0, 0.5], rtol=1e-4)
    assert _lib.exp2_fma2(torch.empty(0, dtype=torch.float32, device="cuda")).numel() == 0
