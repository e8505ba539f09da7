"""GPU parity: the short gated convolution (BaseConv) mixer against the oracle.

y = u_gate * SiLU(bias + causal depthwise K-tap filter of u_conv). Tolerance,
from the arithmetic: the kernel computes in fp32 and rounds y once to the
dtype, so |y - ref| <= 2^-8 |ref| + 1e-5 for bf16 (one rounding, at most half
an ulp, plus fp32 error) and 1e-5 (|ref| + 1) for fp32 (a few ulps of the
fast exponential, scaled by |c| <= ~10). The generation state holds copies of
input values and must match bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
import linear_attention_sequence_causal_b200 as based
from linear_attention_sequence_causal_b200 import synthetic
from parity_util import to64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def assert_close(got, ref, dtype, what="y", terms=None):
    """`terms`: |u_gate| times the filter's sum of absolute products, where the
    fp32 accumulation's own rounding (a few ulps of that sum) can exceed the
    bound relative to a small |c|."""
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    if dtype == "bf16":
        bound = 2.0 ** -8 * np.abs(ref) + 1e-5
    else:
        bound = 1e-5 * (np.abs(ref) + 1.0)
    if terms is not None:
        bound = bound + 1e-6 * terms
    excess = np.abs(got - ref) - bound
    worst = np.unravel_index(int(np.argmax(excess)), excess.shape)
    assert excess[worst] <= 0, f"{what}: |diff| {abs(got[worst] - ref[worst]):.3e} at {worst} (ref {ref[worst]:.4g})"


def _dev(inp, bias=True):
    return (inp.u_gate.to(DEV), inp.u_conv.to(DEV), inp.h.to(DEV), inp.bias.to(DEV) if bias else None)


def _prefill(inp, bias=True, state=True):
    g, x, h, b = _dev(inp, bias)
    y, st = based.baseconv_prefill(g, x, h, b, state=state)
    assert based.get_last_error() == 0
    return y, st


def _ref(inp, bias=True):
    return oracle.baseconv(inp.gate64, inp.conv64, inp.h64, inp.bias64 if bias else None)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("N", [1, 2, 37, 300])
def test_prefill_taps_and_lengths(dtype, K, N):
    bias = (K + N) % 2 == 0
    inp = synthetic.conv_inputs(2, N, 64, K, dtype, seed=100 * K + N)
    y, st = _prefill(inp, bias)
    assert_close(to64(y), _ref(inp, bias), dtype)
    if K > 1:
        assert np.array_equal(to64(st), oracle.baseconv_state(inp.conv64, K))


@pytest.mark.parametrize("B,N,d", [(1, 5, 4), (2, 33, 12), (3, 129, 1028), (5, 1000, 24)])
def test_ragged_channel_groups_and_runs(B, N, d):
    inp = synthetic.conv_inputs(B, N, d, 4, "bf16", seed=d)
    y, st = _prefill(inp)
    assert_close(to64(y), _ref(inp), "bf16")
    assert np.array_equal(to64(st), oracle.baseconv_state(inp.conv64, 4))


def test_prompt_shorter_than_the_filter():
    inp = synthetic.conv_inputs(3, 2, 32, 6, "f32", seed=3)
    y, st = _prefill(inp)
    assert_close(to64(y), _ref(inp), "f32")
    ref_st = oracle.baseconv_state(inp.conv64, 6)
    assert np.all(ref_st[:, :3] == 0)
    assert np.array_equal(to64(st), ref_st)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K,prompt", [(4, 50), (3, 1), (8, 5), (2, 64)])
def test_decode_continues_the_prompt(dtype, K, prompt):
    steps = 20
    inp = synthetic.conv_inputs(4, prompt + steps, 256, K, dtype, seed=K * 7 + prompt)
    g, x, h, b = _dev(inp)
    _, st = based.baseconv_prefill(g[:, :prompt].contiguous(), x[:, :prompt].contiguous(), h, b)
    full = _ref(inp)
    for t in range(prompt, prompt + steps):
        y = based.baseconv_decode(st, g[:, t].contiguous(), x[:, t].contiguous(), h, b)
        assert_close(to64(y), full[:, t], dtype, what=f"y[{t}]")
    assert based.get_last_error() == 0
    assert np.array_equal(to64(st), oracle.baseconv_state(inp.conv64, K))


def test_decode_resume_from_copied_state_is_bit_identical():
    """The shift-register state is the decode checkpoint: copied to the host and
    back, it resumes bit for bit like the state that never left."""
    K, prompt, steps = 4, 40, 12
    inp = synthetic.conv_inputs(3, prompt + steps, 128, K, "bf16", seed=17)
    g, x, h, b = _dev(inp)
    _, st = based.baseconv_prefill(g[:, :prompt].contiguous(), x[:, :prompt].contiguous(), h, b)
    saved = st.cpu().clone()
    runs = []
    for s in (st, saved.to(DEV), saved.to(DEV)):
        torch.cuda.synchronize()
        ys = torch.stack([based.baseconv_decode(s, g[:, t].contiguous(), x[:, t].contiguous(), h, b)
                          for t in range(prompt, prompt + steps)])
        runs.append((ys, s))
    assert based.get_last_error() == 0
    for ys, s in runs[1:]:
        assert torch.equal(ys, runs[0][0]) and torch.equal(s, runs[0][1])


def test_decode_single_tap_needs_no_state():
    inp = synthetic.conv_inputs(5, 1, 64, 1, "bf16", seed=11)
    g, x, h, b = _dev(inp)
    y = based.baseconv_decode(None, g[:, 0].contiguous(), x[:, 0].contiguous(), h, b)
    assert based.get_last_error() == 0
    assert_close(to64(y), _ref(inp)[:, 0], "bf16")


def test_large_decode_batch():
    B, d, K = 256, 1024, 4
    inp = synthetic.conv_inputs(B, K, d, K, "bf16", seed=5)
    g, x, h, b = _dev(inp)
    _, st = based.baseconv_prefill(g[:, :K - 1].contiguous(), x[:, :K - 1].contiguous(), h, b)
    y = based.baseconv_decode(st, g[:, K - 1].contiguous(), x[:, K - 1].contiguous(), h, b)
    assert based.get_last_error() == 0
    assert_close(to64(y), _ref(inp)[:, K - 1], "bf16")


def test_extreme_filter_outputs_stay_finite():
    # taps x 40: c reaches +-200, where exp(-c) overflows and SiLU(c) must be -0 or c
    inp = synthetic.conv_inputs(2, 200, 64, 4, "f32", seed=9)
    inp.h.mul_(40.0)
    inp.h64 *= 40.0
    y, _ = _prefill(inp)
    terms = np.abs(inp.gate64) * oracle.short_conv(np.abs(inp.conv64), np.abs(inp.h64), np.abs(inp.bias64))
    assert_close(to64(y), _ref(inp), "f32", terms=terms)


def test_full_size_360m_shape():
    """B=8, N=2048, d=1024 (the 360M model width), K=4, bf16: every output against the oracle."""
    inp = synthetic.conv_inputs(8, 2048, 1024, 4, "bf16", seed=0)
    y, st = _prefill(inp)
    assert_close(to64(y), _ref(inp), "bf16")
    assert np.array_equal(to64(st), oracle.baseconv_state(inp.conv64, 4))


def test_deterministic():
    inp = synthetic.conv_inputs(2, 500, 512, 4, "bf16", seed=2)
    y1, s1 = _prefill(inp)
    y2, s2 = _prefill(inp)
    assert torch.equal(y1, y2) and torch.equal(s1, s2)
