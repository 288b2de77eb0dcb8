"""Pins of the oracle's output epilogue (``oracle.output_epilogue``: per-head
RMSNorm with a shared weight, then the sigmoid output gate) against closed
forms, a worked example and PyTorch's own rms_norm."""
import numpy as np
import torch

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def test_worked_example():
    """o = [3, 4]: mean square 12.5, so with eps = 0, weight 1 and an open
    gate the row becomes [3, 4] / sqrt(12.5); a zero raw gate halves it."""
    o = np.array([[[3.0, 4.0]]])
    open_gate = np.full_like(o, 800.0)
    y = oracle.output_epilogue(o, open_gate, np.ones(2), eps=0.0)
    np.testing.assert_allclose(y[0, 0], [3 / 12.5 ** 0.5, 4 / 12.5 ** 0.5], rtol=1e-15)
    y0 = oracle.output_epilogue(o, np.zeros_like(o), np.ones(2), eps=0.0)
    np.testing.assert_allclose(y0, 0.5 * y, rtol=1e-15)


def test_unit_rms_and_scale_invariance():
    """With eps = 0, weight 1 and an open gate every row has RMS 1 and is
    unchanged by a positive scale of o (sign-flipped by a negative one);
    with eps > 0 the RMS is sqrt(m / (m + eps)), m the row's mean square."""
    r = _rng(30)
    o = r.standard_normal((6, 3, 8))
    g = np.full_like(o, 800.0)
    y = oracle.output_epilogue(o, g, np.ones(8), eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(oracle.output_epilogue(7.0 * o, g, np.ones(8), eps=0.0), y, rtol=1e-14)
    np.testing.assert_allclose(oracle.output_epilogue(-0.5 * o, g, np.ones(8), eps=0.0), -y,
                               rtol=1e-14)
    eps = 0.3
    ye = oracle.output_epilogue(o, g, np.ones(8), eps=eps)
    m = np.mean(o * o, axis=-1)
    np.testing.assert_allclose(np.sqrt(np.mean(ye * ye, axis=-1)), np.sqrt(m / (m + eps)),
                               rtol=1e-13)


def test_matches_torch_rms_norm_and_sigmoid():
    """Equal to torch.nn.functional.rms_norm over the last dimension (same
    weight and eps) times torch.sigmoid of the gate, in fp64."""
    r = _rng(31)
    o = r.standard_normal((9, 4, 16))
    g = r.standard_normal((9, 4, 16))
    w = r.standard_normal(16)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(o), (16,), torch.from_numpy(w), 1e-6) * \
        torch.sigmoid(torch.from_numpy(g))
    np.testing.assert_allclose(oracle.output_epilogue(o, g, w), ref.numpy(), rtol=1e-13,
                               atol=1e-15)


def test_weight_is_per_channel_and_shared_by_heads():
    r = _rng(32)
    o = r.standard_normal((2, 3, 4))
    g = r.standard_normal((2, 3, 4))
    w = np.array([1.0, 2.0, -1.0, 0.0])
    y = oracle.output_epilogue(o, g, w)
    y1 = oracle.output_epilogue(o, g, np.ones(4))
    np.testing.assert_allclose(y, y1 * w[None, None, :], rtol=1e-15, atol=0)
