"""Pins of the oracle's input activations (``oracle.preprocess``) against
what the page and the mathematics fix: the identity tap, the impulse
response of the width-4 conv and its restart at every sequence start,
agreement with numpy's own convolution, the gate functions at known points
(including the printed sigma(5) ~ 0.993 of the alpha-gate bias) and the unit
norm and scale invariance of the normalised q, k."""
import json
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _case(r, lengths, H, d, scalar=False):
    T = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    x = [r.standard_normal((T, H, d)) for _ in range(3)]
    w = [r.standard_normal((H * d, 4)) for _ in range(3)]
    braw = r.standard_normal((T, H))
    araw = r.standard_normal((T, H) if scalar else (T, H, d))
    bias = r.standard_normal((H,) if scalar else (H, d))
    return x, w, braw, araw, bias, cu


def test_identity_tap_passes_values_through():
    """"Идея и архитектура": the conv is initialised as an identity tap, so
    with w = [0, 0, 0, 1] v is the raw projection and q, k are its
    normalised rows."""
    r = _rng(20)
    x, _, braw, araw, bias, cu = _case(r, [5, 1, 9], 2, 6)
    ident = np.tile([0.0, 0.0, 0.0, 1.0], (2 * 6, 1))
    out = oracle.preprocess(*x, ident, ident, ident, braw, araw, bias, cu)
    np.testing.assert_array_equal(out["v"], x[2])
    for name, raw in (("q", x[0]), ("k", x[1])):
        np.testing.assert_allclose(out[name], raw / np.linalg.norm(raw, axis=-1, keepdims=True),
                                   rtol=1e-15, atol=1e-15)


def test_impulse_response_and_sequence_restart():
    """An impulse at token t0 of channel c gives y[t0 + m, c] = w[c, 3 - m]
    for m = 0..3 while t0 + m stays in the sequence, and nothing anywhere
    else: the conv is causal, depthwise and never reaches across sequences."""
    H, d = 2, 3
    lengths = [6, 2, 5]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = sum(lengths)
    w = _rng(21).standard_normal((H * d, 4))
    for t0, h, c in ((1, 0, 2), (4, 1, 0), (6, 1, 1), (7, 0, 0)):
        x = np.zeros((T, H, d))
        x[t0, h, c] = 1.0
        y = oracle.preprocess(x, x, x, w, w, w, np.zeros((T, H)), np.zeros((T, H, d)),
                              np.zeros((H, d)), cu)["v"]
        seq_end = int(cu[np.searchsorted(cu, t0, side="right")])
        want = np.zeros_like(x)
        for m in range(4):
            if t0 + m < seq_end:
                want[t0 + m, h, c] = w[h * d + c, 3 - m]
        np.testing.assert_array_equal(y, want)


def test_conv_matches_numpy_convolve():
    """Per sequence and channel, the conv equals numpy.convolve of the
    channel's values with the reversed taps, cut to the sequence's length."""
    r = _rng(22)
    x, w, braw, araw, bias, cu = _case(r, [7, 1, 3, 12], 2, 5)
    v = oracle.preprocess(*x, *w, braw, araw, bias, cu)["v"]
    for n in range(len(cu) - 1):
        s, e = int(cu[n]), int(cu[n + 1])
        for h in range(2):
            for c in range(5):
                ref = np.convolve(x[2][s:e, h, c], w[2][h * 5 + c, ::-1])[: e - s]
                np.testing.assert_allclose(v[s:e, h, c], ref, rtol=1e-13, atol=1e-13)


def test_gates_at_known_points():
    """beta = sigmoid: 1/2 at 0.  log a = log-sigmoid of the biased gate:
    -ln 2 at 0, ~ z for very negative z, ~ -exp(-z) for large z (no overflow
    either way); with the page's bias +5 and a zero raw gate,
    a = sigmoid(5) rounds to the printed 0.993."""
    g = json.load(open(os.path.join(GOLDEN, "decay_magnitude.json")))
    T, H, d = 5, 1, 2
    z = np.array([0.0, -40.0, 40.0, -800.0, 800.0])
    zeros = np.zeros((T, H, d))
    ident = np.tile([0.0, 0.0, 0.0, 1.0], (d, 1))
    one = np.ones((T, H, d))
    out = oracle.preprocess(one, one, one, ident, ident, ident, z[:, None],
                            np.repeat(z[:, None, None], d, 2), np.zeros((H, d)), [0, T])
    np.testing.assert_allclose(out["beta"][:, 0], [0.5, math.exp(-40) / (1 + math.exp(-40)),
                                                    1 / (1 + math.exp(-40)), 0.0, 1.0],
                               rtol=1e-15, atol=0)
    la = out["log_a"][:, 0, 0]
    assert la[0] == -math.log(2.0)
    np.testing.assert_allclose(la[1], -40.0 - math.log1p(math.exp(-40.0)), rtol=1e-15)
    np.testing.assert_allclose(la[2], -math.exp(-40.0), rtol=1e-12)
    assert la[3] == -800.0 and la[4] == 0.0 and np.all(np.isfinite(la))
    # the page's gate bias
    out5 = oracle.preprocess(one, one, one, ident, ident, ident, np.zeros((T, H)), zeros,
                             np.full((H, d), g["gate_bias"]), [0, T])
    a = np.exp(out5["log_a"])
    assert np.all(np.round(a, g["sigma_printed_digits"]) == g["sigma_printed"])
    # scalar gate: one bias per head
    out_s = oracle.preprocess(one, one, one, ident, ident, ident, np.zeros((T, H)),
                              np.zeros((T, H)), np.full((H,), g["gate_bias"]), [0, T],
                              scalar_decay=True)
    assert out_s["log_a"].shape == (T, H)
    np.testing.assert_allclose(out_s["log_a"], out5["log_a"][:, :, 0], rtol=0, atol=0)


def test_normalised_rows_unit_and_scale_invariant():
    r = _rng(23)
    x, w, braw, araw, bias, cu = _case(r, [4, 9], 3, 8)
    out = oracle.preprocess(*x, *w, braw, araw, bias, cu)
    for name in ("q", "k"):
        np.testing.assert_allclose(np.linalg.norm(out[name], axis=-1), 1.0, rtol=1e-14)
    x2 = [3.5 * x[0], 0.25 * x[1], x[2]]
    out2 = oracle.preprocess(*x2, *w, braw, araw, bias, cu)
    np.testing.assert_allclose(out2["q"], out["q"], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(out2["k"], out["k"], rtol=1e-13, atol=1e-14)
    # a zero row stays zero instead of dividing by zero
    xz = [np.zeros_like(x[0])] * 3
    oz = oracle.preprocess(*xz, *w, braw, araw, bias, cu)
    assert np.all(oz["q"] == 0) and np.all(oz["k"] == 0)
