"""The sequence-mixing core of a BaseConv (short gated convolution) layer, float64.

Test infrastructure only (see the package docstring).

BASED ("Simple linear attention language models balance the recall-throughput
tradeoff") §4 "The BASED Architecture" (Additional mixers) adds short gated
convolutions beside the sliding-window layers; App. C "Extended Architecture Details" (Convolution)
describes the BaseConv layer: a short convolution, a SiLU nonlinearity, three
learned linear projections with biases and a Hadamard product of the projected
input with the filtered sequence before the projection back to model width.

Readings of points the pages leave open:
* the three projections are plain per-token affine maps (channel mixing only);
  the caller computes the two input projections, u_gate = u W_g + b_g and
  u_conv = u W_c + b_c, and the output projection of the result. What is left
  between them, and what this module computes, is the sequence mixing:
      c_t = bias + sum_{j=0}^{K-1} h[:, j] * u_conv[t - (K-1) + j]   (causal,
            depthwise, zero before the first token; tap K-1 meets token t)
      y_t = u_gate[t] * SiLU(c_t),   SiLU(x) = x / (1 + exp(-x));
* the SiLU sits on the convolution branch, after the filter and its bias;
* a generation step keeps the last K-1 values of u_conv of each sequence as its
  state (a shift register, oldest first), which is all the filter can see.

Layouts: u_gate, u_conv, y [B, N, d] (token-major, channels innermost);
h [d, K]; bias [d]; state [B, K-1, d].
"""

from __future__ import annotations

import numpy as np


def silu(x):
    """x * sigmoid(x), written as x / (1 + exp(-x)); exp(-x) overflowing to inf gives -0."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def short_conv(u_conv, h, bias=None) -> np.ndarray:
    """c_t = bias + sum_j h[:, j] u_conv[t - (K-1) + j], zero-padded before token 0.

    One shifted copy of the sequence per tap: tap j reads the token K-1-j places back.
    """
    x = np.asarray(u_conv, dtype=np.float64)
    h = np.asarray(h, dtype=np.float64)
    n = x.shape[-2]
    taps = h.shape[-1]
    c = np.zeros_like(x)
    for j in range(taps):
        back = taps - 1 - j
        if back >= n:
            continue
        c[..., back:, :] += h[:, j] * x[..., : n - back, :]
    if bias is not None:
        c += np.asarray(bias, dtype=np.float64)
    return c


def baseconv(u_gate, u_conv, h, bias=None) -> np.ndarray:
    """y_t = u_gate[t] * SiLU(c_t) over a whole sequence (prefill)."""
    return np.asarray(u_gate, dtype=np.float64) * silu(short_conv(u_conv, h, bias))


def baseconv_state(u_conv, taps: int) -> np.ndarray:
    """The generation state after a prompt: u_conv of tokens N-K+1 .. N-1, zeros before token 0.

    Returned as [..., K-1, d], oldest token first.
    """
    x = np.asarray(u_conv, dtype=np.float64)
    n, d = x.shape[-2], x.shape[-1]
    st = np.zeros(x.shape[:-2] + (taps - 1, d), dtype=np.float64)
    for j in range(taps - 1):
        t = n - (taps - 1) + j
        if t >= 0:
            st[..., j, :] = x[..., t, :]
    return st


def baseconv_decode_step(state, u_gate, u_conv, h, bias=None):
    """One generated token: returns (y, new state).

    The filter meets the K-1 stored values (oldest at tap 0) and the new value
    (tap K-1); the state then drops its oldest row and appends the new value.
    state [..., K-1, d]; u_gate, u_conv [..., d].
    """
    st = np.asarray(state, dtype=np.float64)
    g = np.asarray(u_gate, dtype=np.float64)
    x = np.asarray(u_conv, dtype=np.float64)
    h = np.asarray(h, dtype=np.float64)
    taps = h.shape[-1]
    c = h[:, taps - 1] * x
    for j in range(taps - 1):
        c = c + h[:, j] * st[..., j, :]
    if bias is not None:
        c = c + np.asarray(bias, dtype=np.float64)
    y = g * silu(c)
    new = np.concatenate([st[..., 1:, :], x[..., None, :]], axis=-2) if taps > 1 else st
    return y, new
