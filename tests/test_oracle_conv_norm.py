"""Pins of the short convolution and the gated output norm (oracle/conv_norm.py),
CPU only: SiLU at closed-form points, the convolution's identity and delay taps,
a hand-worked single channel, causality with a carried state, and the gated
RMSNorm at a constant row, a zero gate and a hand-worked row."""
import numpy as np
import pytest

from oracle.conv_norm import gated_rmsnorm, short_conv, silu

LN3 = np.log(3.0)


def test_silu_closed_forms():
    # sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4
    np.testing.assert_allclose(silu([0.0, LN3, -LN3]), [0.0, 0.75 * LN3, -0.25 * LN3], rtol=1e-15, atol=0)


def test_identity_and_delay_taps():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 9, 5))
    ident = np.tile([0.0, 0.0, 0.0, 1.0], (5, 1))
    y, _ = short_conv(x, ident)
    np.testing.assert_allclose(y, silu(x), rtol=1e-15)
    delay = np.tile([1.0, 0.0, 0.0, 0.0], (5, 1))
    y, _ = short_conv(x, delay)
    assert np.all(y[:, :3] == 0.0)
    np.testing.assert_allclose(y[:, 3:], silu(x[:, :-3]), rtol=1e-15)


def test_single_channel_by_hand():
    # w = (1, 2, 3, 4) (oldest token first), x = (1, 0, 0, 0, 0, 2): the window
    # of token t multiplies x_{t-3+j} by w_j, so the pre-activations are
    # (4, 3, 2, 1, 0, 8)
    x = np.array([1.0, 0.0, 0.0, 0.0, 0.0, 2.0]).reshape(1, 6, 1)
    w = np.array([[1.0, 2.0, 3.0, 4.0]])
    y, st = short_conv(x, w)
    np.testing.assert_allclose(y.ravel(), silu([4.0, 3.0, 2.0, 1.0, 0.0, 8.0]), rtol=1e-15)
    np.testing.assert_array_equal(st.ravel(), [0.0, 0.0, 2.0])


def test_carried_state_equals_one_call_and_causality():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((2, 20, 3))
    w = rng.standard_normal((3, 4))
    y_all, st_all = short_conv(x, w)
    y_a, st_a = short_conv(x[:, :7], w)
    y_b, st_b = short_conv(x[:, 7:], w, state=st_a)
    np.testing.assert_allclose(np.concatenate([y_a, y_b], axis=1), y_all, rtol=1e-14)
    np.testing.assert_array_equal(st_b, st_all)
    x2 = x.copy()
    x2[:, 15] += 10.0
    y2, _ = short_conv(x2, w)
    np.testing.assert_array_equal(y2[:, :15], y_all[:, :15])
    assert np.all(y2[:, 15] != y_all[:, 15])


def test_gated_rmsnorm_closed_forms():
    c = 0.37
    o = np.full((3, 8), c)
    gamma = np.linspace(0.5, 2.0, 8)
    g = np.full((3, 8), LN3)
    want = gamma * 0.75 * LN3 * c / np.sqrt(c * c + 1e-6)
    np.testing.assert_allclose(gated_rmsnorm(o, g, gamma), np.broadcast_to(want, (3, 8)), rtol=1e-14)
    assert np.all(gated_rmsnorm(o, np.zeros((3, 8)), gamma) == 0.0)
    # one row by hand: o = (3, 4), mean(o^2) = 12.5, gamma = (2, 1/2), g = (ln 3, 0)
    y = gated_rmsnorm(np.array([[3.0, 4.0]]), np.array([[LN3, 0.0]]), np.array([2.0, 0.5]))
    assert y[0, 0] == pytest.approx(3.0 / np.sqrt(12.5 + 1e-6) * 2.0 * 0.75 * LN3, rel=1e-14)
    assert y[0, 1] == 0.0
