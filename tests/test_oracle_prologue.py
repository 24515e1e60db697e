"""Pins for the prologue oracle (oracle/prologue.py), each against something
other than the oracle itself: numpy's convolution, scipy's logistic function,
delta filters (pure shifts), the unit norm of normalised rows, causality and
central finite differences.  Page citation: "Gated Delta Networks: Improving
Mamba2 with Delta Rule" (paper review), section "Method" (short convolution,
SiLU, L2 normalisation of q and k; v without the norm)."""
import numpy as np
import scipy.special

from oracle import prologue


def _inputs(rng, B=2, T=9, H=2, d=5, K=4):
    return rng.standard_normal((B, T, H, d)), 0.5 * rng.standard_normal((H, d, K))


def test_conv_is_numpys_causal_convolution():
    """With the norm off, y = SiLU(z), where z is np.convolve of each channel
    with its filter, truncated to the first T outputs."""
    rng = np.random.default_rng(41)
    x, w = _inputs(rng)
    y = prologue.forward(x, w, norm=False)
    B, T, H, d = x.shape
    for b in range(B):
        for h in range(H):
            for c in range(d):
                z = np.convolve(x[b, :, h, c], w[h, c])[:T]
                ref = z * scipy.special.expit(z)
                assert np.abs(y[b, :, h, c] - ref).max() < 1e-13


def test_delta_filters_shift_the_sequence():
    rng = np.random.default_rng(42)
    x, _ = _inputs(rng, K=4)
    for j in range(4):
        w = np.zeros((2, 5, 4))
        w[:, :, j] = 1.0
        y = prologue.forward(x, w, norm=False)
        shifted = np.zeros_like(x)
        shifted[:, j:] = x[:, :x.shape[1] - j]
        assert np.abs(y - shifted * scipy.special.expit(shifted)).max() < 1e-13


def test_normalised_rows_have_unit_norm_and_the_silu_direction():
    rng = np.random.default_rng(43)
    x, w = _inputs(rng, d=16)
    y = prologue.forward(x, w, norm=True)
    s = prologue.forward(x, w, norm=False)
    n2 = (s * s).sum(-1, keepdims=True)
    assert np.abs((y * y).sum(-1, keepdims=True) - n2 / (n2 + prologue.EPS)).max() < 1e-12
    cos = (y * s).sum(-1) / np.sqrt((y * y).sum(-1) * n2[..., 0])
    assert np.abs(cos - 1.0).max() < 1e-12


def test_causal():
    rng = np.random.default_rng(44)
    x, w = _inputs(rng, T=12)
    y = prologue.forward(x, w, norm=True)
    x2 = x.copy()
    x2[:, 7] += 3.0
    y2 = prologue.forward(x2, w, norm=True)
    assert np.array_equal(y[:, :7], y2[:, :7])
    assert np.abs(y2[:, 7:11] - y[:, 7:11]).max() > 1e-6  # taps 0..3 reach t = 7..10
    assert np.array_equal(y[:, 11:], y2[:, 11:])


def test_backward_finite_differences():
    rng = np.random.default_rng(45)
    for norm in (False, True):
        x, w = _inputs(rng, B=1, T=6, H=1, d=4, K=3)
        dy = rng.standard_normal(x.shape)
        g = prologue.backward(x, w, dy, norm)
        f = lambda xx, ww: float((prologue.forward(xx, ww, norm) * dy).sum())  # noqa: E731
        h = 1e-6
        for idx in [(0, 0, 0, 0), (0, 3, 0, 2), (0, 5, 0, 3)]:
            e = np.zeros_like(x)
            e[idx] = h
            num = (f(x + e, w) - f(x - e, w)) / (2 * h)
            assert abs(num - g["dx"][idx]) < 1e-7 * max(1.0, abs(num))
        for idx in [(0, 0, 0), (0, 2, 1), (0, 3, 2)]:
            e = np.zeros_like(w)
            e[idx] = h
            num = (f(x, w + e) - f(x, w - e)) / (2 * h)
            assert abs(num - g["dw"][idx]) < 1e-7 * max(1.0, abs(num))
