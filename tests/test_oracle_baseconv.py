"""Pins of the short gated convolution (BaseConv) oracle against things other than itself.

BASED App. C "Extended Architecture Details" (Convolution): short convolution,
SiLU, Hadamard product with the projected input. The pins: SiLU against a
library logistic function and its odd-part identity; the causal filter against
numpy's full convolution; delta and shift filters; a zero input leaving only the
bias; hand-worked integer convolutions; pure-Python brute force; the prompt +
generation split against the whole-sequence form; and planted mistakes.
"""

import math

import numpy as np
import pytest
from scipy.special import expit

import oracle

RNG = np.random.default_rng(7)


def test_silu_against_logistic_function():
    x = np.concatenate([np.linspace(-30, 30, 601), RNG.standard_normal(200) * 5])
    np.testing.assert_allclose(oracle.silu(x), x * expit(x), rtol=1e-14, atol=1e-300)
    assert oracle.silu(0.0) == 0.0
    # x*sig(x) - (-x)*sig(-x) = x (sig(x) + sig(-x)) = x
    np.testing.assert_allclose(oracle.silu(x) - oracle.silu(-x), x, rtol=1e-13, atol=1e-13)
    # very negative inputs go to zero without overflow warnings turning into errors
    assert abs(oracle.silu(-1000.0)) == 0.0
    np.testing.assert_allclose(oracle.silu(50.0), 50.0, rtol=1e-15)


@pytest.mark.parametrize("taps", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("n", [1, 3, 17])
def test_short_conv_matches_numpy_convolution(taps, n):
    d = 5
    x = RNG.standard_normal((2, n, d))
    h = RNG.standard_normal((d, taps))
    c = oracle.short_conv(x, h)
    for b in range(2):
        for ch in range(d):
            # np.convolve(x, g)[t] = sum_m x[m] g[t-m]; the causal filter has g = h reversed
            ref = np.convolve(x[b, :, ch], h[ch, ::-1])[:n]
            np.testing.assert_allclose(c[b, :, ch], ref, rtol=1e-12, atol=1e-12)


def test_delta_and_shift_filters():
    taps, n, d = 4, 9, 3
    x = RNG.standard_normal((1, n, d))
    last = np.zeros((d, taps)); last[:, taps - 1] = 1.0
    np.testing.assert_array_equal(oracle.short_conv(x, last), x)
    first = np.zeros((d, taps)); first[:, 0] = 1.0
    shifted = np.zeros_like(x); shifted[:, taps - 1:, :] = x[:, : n - taps + 1, :]
    np.testing.assert_array_equal(oracle.short_conv(x, first), shifted)
    # with the delta at the current token the layer is the plain gated SiLU
    g = RNG.standard_normal((1, n, d))
    np.testing.assert_allclose(oracle.baseconv(g, x, last), g * x * expit(x), rtol=1e-13)


def test_zero_input_leaves_the_bias():
    n, d = 6, 4
    g = RNG.standard_normal((1, n, d))
    bias = np.array([0.5, -1.0, 0.0, 2.0])
    y = oracle.baseconv(g, np.zeros((1, n, d)), RNG.standard_normal((d, 3)), bias)
    np.testing.assert_allclose(y, g * (bias / (1.0 + np.exp(-bias))), rtol=1e-14)


def test_hand_worked_convolution():
    # one channel, taps h = [1, 2, 3] (tap 2 meets the current token), x = 1, 0, -1, 2
    # c_0 = 3*1 = 3; c_1 = 2*1 + 3*0 = 2; c_2 = 1*1 + 2*0 + 3*(-1) = -2;
    # c_3 = 1*0 + 2*(-1) + 3*2 = 4
    x = np.array([1.0, 0.0, -1.0, 2.0])[None, :, None]
    h = np.array([[1.0, 2.0, 3.0]])
    np.testing.assert_array_equal(oracle.short_conv(x, h)[0, :, 0], [3.0, 2.0, -2.0, 4.0])
    np.testing.assert_array_equal(oracle.short_conv(x, h, [0.5])[0, :, 0], [3.5, 2.5, -1.5, 4.5])
    # the state after the prompt holds its last two tokens, oldest first
    np.testing.assert_array_equal(oracle.baseconv_state(x, 3)[0, :, 0], [-1.0, 2.0])
    # a one-token prompt leaves a zero in front of it
    np.testing.assert_array_equal(oracle.baseconv_state(x[:, :1], 3)[0, :, 0], [0.0, 1.0])


def _brute(g, x, h, bias):
    """Scalar loops over (token, channel, tap) with math.exp."""
    n, d = len(x), len(x[0])
    taps = len(h[0])
    y = [[0.0] * d for _ in range(n)]
    for t in range(n):
        for ch in range(d):
            acc = bias[ch]
            for j in range(taps):
                s = t - (taps - 1) + j
                if s >= 0:
                    acc += h[ch][j] * x[s][ch]
            y[t][ch] = g[t][ch] * acc / (1.0 + math.exp(-acc))
    return y


@pytest.mark.parametrize("taps,n", [(1, 4), (2, 1), (3, 5), (4, 8)])
def test_brute_force_tiny(taps, n):
    d = 3
    g = RNG.standard_normal((n, d))
    x = RNG.standard_normal((n, d))
    h = RNG.standard_normal((d, taps))
    bias = RNG.standard_normal(d)
    ref = np.array(_brute(g.tolist(), x.tolist(), h.tolist(), bias.tolist()))
    np.testing.assert_allclose(oracle.baseconv(g[None], x[None], h, bias)[0], ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("taps,prompt", [(4, 10), (4, 2), (3, 1), (1, 5), (2, 7)])
def test_prompt_then_generation_matches_whole_sequence(taps, prompt):
    n, d = 16, 6
    g = RNG.standard_normal((2, n, d))
    x = RNG.standard_normal((2, n, d))
    h = RNG.standard_normal((d, taps))
    bias = RNG.standard_normal(d)
    full = oracle.baseconv(g, x, h, bias)
    np.testing.assert_allclose(oracle.baseconv(g[:, :prompt], x[:, :prompt], h, bias), full[:, :prompt],
                               rtol=1e-14)
    st = oracle.baseconv_state(x[:, :prompt], taps)
    for t in range(prompt, n):
        y, st = oracle.baseconv_decode_step(st, g[:, t], x[:, t], h, bias)
        np.testing.assert_allclose(y, full[:, t], rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(st, oracle.baseconv_state(x, taps))


# ---------------------------------------------------------------- planted mistakes


def test_mutant_reversed_taps_caught():
    x = np.array([1.0, 0.0, -1.0, 2.0])[None, :, None]
    h = np.array([[1.0, 2.0, 3.0]])
    wrong = oracle.short_conv(x, h[:, ::-1])
    assert not np.array_equal(wrong[0, :, 0], [3.0, 2.0, -2.0, 4.0])


def test_mutant_silu_on_the_gate_caught():
    n, d, taps = 8, 4, 3
    g = RNG.standard_normal((1, n, d))
    x = RNG.standard_normal((1, n, d))
    h = RNG.standard_normal((d, taps))
    wrong = oracle.silu(g) * oracle.short_conv(x, h)
    ref = np.array(_brute(g[0].tolist(), x[0].tolist(), h.tolist(), [0.0] * d))
    assert not np.allclose(wrong[0], ref)


def test_mutant_bias_dropped_caught():
    n, d = 6, 4
    g = RNG.standard_normal((1, n, d))
    bias = np.array([0.5, -1.0, 0.25, 2.0])
    wrong = oracle.baseconv(g, np.zeros((1, n, d)), RNG.standard_normal((d, 3)), None)
    assert not np.allclose(wrong, g * (bias / (1.0 + np.exp(-bias))))


def test_mutant_state_newest_first_caught():
    x = np.array([1.0, 0.0, -1.0, 2.0])[None, :, None]
    st = oracle.baseconv_state(x, 3)
    # a state stored newest first meets the filter reversed: the next token differs
    g1, x1 = np.ones((1, 1)), np.array([[0.5]])
    h = np.array([[1.0, 2.0, 3.0]])
    y_ok, _ = oracle.baseconv_decode_step(st, g1, x1, h)
    y_bad, _ = oracle.baseconv_decode_step(st[:, ::-1], g1, x1, h)
    # c = 1*(-1) + 2*2 + 3*0.5 = 4.5
    np.testing.assert_allclose(y_ok, 4.5 * expit(4.5), rtol=1e-14)
    assert not np.allclose(y_bad, y_ok)
