"""The exponential the attention's softmax runs on the FMA pipe for a share
of its weights, alone on the GPU (rf_debug_exp2_poly).

2^x = 2^round(x) (exponent field) times a degree-3 polynomial for 2^f on
|f| <= 1/2, with x clamped to [-125, 128].  Checked against 2^x in fp64
(numpy's exp2, the value itself) and against the device's own exp2f (torch's
exp2 on CUDA, below 128 where it is finite) over [-130, 130]:
  * relative error at most 7.5e-5 (the fit) plus 2^-21 (its fp32 steps) on
    [-125, 128];
  * above 128 (and at +inf) the result is at least 2^127: an overflowing
    softmax sum stays visible, which the attention's hand-over to its
    rescaling pass relies on;
  * below -125 (and at -inf) the result is 2^-125 up to that error.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

REL = 7.5e-5 + 2.0 ** -21


def _run(x: np.ndarray) -> np.ndarray:
    from block_sparse_video_rf_b200 import rfsa
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    y = rfsa.rf_debug_exp2_poly(xd)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def _sweep() -> np.ndarray:
    dense = np.linspace(-130.0, 130.0, 2_600_001)
    halves = np.arange(-260, 261) / 2.0                               # every rounding tie of round(x)
    near = np.concatenate([halves + d for d in (-1e-6, 1e-6)])
    edges = np.array([-125.0, -124.5, -125.5, 127.5, 127.75, 128.0, 128.5, 129.0, 1e30, -1e30])
    return np.concatenate([dense, halves, near, edges]).astype(np.float32)


def test_exp2_poly_accuracy_and_clamps():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    x = _sweep()
    y = _run(x).astype(np.float64)
    x64 = x.astype(np.float64)
    inside = (x64 >= -125) & (x64 <= 128)
    ref = np.exp2(x64[inside])
    rel = np.abs(y[inside] / ref - 1)
    assert rel.max() <= REL, (float(rel.max()), float(x64[inside][rel.argmax()]))
    # against the device's own exp2f (within its few ulp of the true value),
    # where that is finite: exp2f(128) overflows to inf in fp32
    fin = inside & (x64 < 128)
    dev = torch.exp2(torch.from_numpy(x[fin]).cuda()).cpu().numpy().astype(np.float64)
    rel_dev = np.abs(y[fin] / dev - 1)
    assert rel_dev.max() <= REL + 2.0 ** -21, float(rel_dev.max())
    above = x64 > 128
    assert (y[above] >= 2.0 ** 127).all()
    below = x64 < -125
    assert (np.abs(y[below] / 2.0 ** -125 - 1) <= REL).all()
    # 2^x is never negative, never NaN, finite on the clamped range
    assert (y > 0).all() and np.isfinite(y).all()


def test_exp2_poly_infinities_and_odd_length():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    x = np.array([np.inf, -np.inf, 0.0, 1.0, -1.0], dtype=np.float32)   # odd count: the last pair is half used
    y = _run(x).astype(np.float64)
    assert y[0] >= 2.0 ** 127
    assert abs(y[1] / 2.0 ** -125 - 1) <= REL
    np.testing.assert_allclose(y[2:], [1.0, 2.0, 0.5], rtol=REL)
