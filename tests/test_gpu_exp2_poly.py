"""The attention softmax's FMA-pipe exponential (Cody-Waite reduction and a
degree-4 minimax polynomial; a build-time option of the attention kernel)
against 2^x in fp64.

Its bound is 3e-6 relative over the clamp range [-126, 127] -- looser than
CUDA's exp2f (2 ulp), but 1/1300 of the bf16 rounding (2^-9) that P gets
before the P.V product, so it cannot move the attention output beyond the
bf16 gates."""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_pool_b200 import ops

pytestmark = pytest.mark.gpu

BOUND = 3e-6


def _rel_err(x32: np.ndarray, y32: np.ndarray) -> np.ndarray:
    ref = np.exp2(np.clip(x32.astype(np.float64), -126.0, 127.0))
    return np.abs(y32.astype(np.float64) - ref) / ref


def test_exp2_poly_relative_error_over_the_range():
    g = np.random.default_rng(7)
    x = np.concatenate([
        np.linspace(-126.0, 127.0, 2_000_001, dtype=np.float32),
        g.uniform(-126.0, 127.0, 1_000_000).astype(np.float32),
        g.uniform(-1.0, 1.0, 1_000_000).astype(np.float32),        # the softmax's usual range
        np.arange(-126, 128, dtype=np.float32),                     # integers: r = 0
        np.arange(-126, 127, dtype=np.float32) + np.float32(0.5),   # ties of the rounding
        np.nextafter(np.arange(-126, 127, dtype=np.float32) + np.float32(0.5), np.float32(0)),
    ]).astype(np.float32)
    y = ops.selftest_exp2_poly(torch.from_numpy(x).cuda()).cpu().numpy()
    err = _rel_err(x, y)
    assert np.all(np.isfinite(y))
    assert err.max() < BOUND, (err.max(), x[err.argmax()])
    # the polynomial's own bound (2.6e-6) is what dominates, not the fp32 steps
    assert err.max() > 1e-7


def test_exp2_poly_clamps_outside_the_range():
    x = np.array([-1e30, -1000.0, -127.5, -126.0, 127.0, 128.0, 1000.0, 1e30], dtype=np.float32)
    y = ops.selftest_exp2_poly(torch.from_numpy(x).cuda()).cpu().numpy()
    lo, hi = 2.0 ** -126, 2.0 ** 127
    assert np.all(np.abs(y[:4] / lo - 1) < BOUND), y[:4]
    assert np.all(np.abs(y[4:] / hi - 1) < BOUND), y[4:]


def test_exp2_poly_odd_length_and_empty():
    x = torch.tensor([0.25, -3.0, 5.5], dtype=torch.float32, device="cuda")
    y = ops.selftest_exp2_poly(x).cpu().numpy()
    assert np.all(_rel_err(x.cpu().numpy(), y) < BOUND)
    assert ops.selftest_exp2_poly(torch.empty(0, device="cuda")).numel() == 0
