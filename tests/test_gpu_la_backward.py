"""GPU parity of the linear-attention backward (dq, dk, dv) against the oracle.

based_la_backward takes q, k, v, the forward's output y and an upstream dy
(bf16) and returns the gradients of the causal Taylor linear attention. The
oracle's la_backward (float64, written from the derivative of the quadratic
form) is pinned on the CPU against autograd and finite differences.

Tolerance: every operand of the tensor-core products (g = dy/den, the Taylor
weights a, ds, and the inputs) is rounded to bf16 (relative error <= 2^-9)
and accumulated in fp32; each gradient passes through two or three such
roundings, so its error is a few 1e-3 of the gradient's scale. The bound is
max|got - ref| <= 2e-2 * max|ref| per output tensor.
"""

import numpy as np
import pytest
import torch

import oracle
import linear_attention_sequence_causal_b200 as based
from linear_attention_sequence_causal_b200 import synthetic
from parity_util import max_abs, to64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
BWD_TOL = 2e-2


def _case(B, H, N, d_feat, d_v, seed):
    inp = synthetic.la_inputs(B, H, N, d_feat, d_v, "bf16", seed=seed)
    dy, dy64 = synthetic.upstream_grad((B, H, N, d_v), "bf16", seed=seed + 1000)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y, _, _ = based.la_prefill(q, k, v, want_state=False)
    dq, dk, dv = based.la_backward(q, k, v, y, dy.to(DEV))
    assert based.get_last_error() == 0
    return inp, dy64, (dq, dk, dv)


def _assert_grads(got, ref, what=""):
    errs = []
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = to64(g) if isinstance(g, torch.Tensor) else np.asarray(g, np.float64)
        assert np.all(np.isfinite(g)), f"{what}{name}: non-finite"
        rel = max_abs(g, r) / max(1e-30, float(np.max(np.abs(r))))
        assert rel <= BWD_TOL, f"{what}{name}: relative error {rel:.3e} > {BWD_TOL:.0e}"
        errs.append(rel)
    return errs


@pytest.mark.parametrize("d_feat,d_v", [(16, 64), (16, 128), (32, 64), (32, 128)])
def test_backward_ragged(d_feat, d_v):
    """Three 128-row tiles with a ragged tail (300 tokens), two heads."""
    inp, dy64, got = _case(1, 2, 300, d_feat, d_v, seed=d_feat + d_v)
    ref = oracle.la_backward(inp.q64, inp.k64, inp.v64, dy64)
    _assert_grads(got, ref)


@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 256])
def test_backward_tile_edges(N):
    inp, dy64, got = _case(1, 1, N, 16, 64, seed=N)
    ref = oracle.la_backward(inp.q64, inp.k64, inp.v64, dy64)
    _assert_grads(got, ref, f"N={N} ")


def test_backward_first_token():
    """One token: the exact output is y = v, so ds = 0 (dq = dk = 0 up to fp32
    accumulation order) and dv = a g = dy up to the bf16 rounding of g."""
    inp = synthetic.la_inputs(2, 3, 1, 32, 128, "bf16", seed=5)
    dy, dy64 = synthetic.upstream_grad((2, 3, 1, 128), "bf16", seed=6)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    dq, dk, dv = based.la_backward(q, k, v, v, dy.to(DEV))
    assert based.get_last_error() == 0
    assert float(dq.abs().max()) <= 1e-4 and float(dk.abs().max()) <= 1e-4
    assert max_abs(to64(dv), dy64) <= 2 ** -7 * float(np.max(np.abs(dy64)))


def test_backward_many_units():
    """More 128-row units (5 tiles x 64 heads) than SMs: each CTA walks several."""
    inp, dy64, got = _case(4, 16, 600, 16, 64, seed=11)
    ref = oracle.la_backward(inp.q64, inp.k64, inp.v64, dy64)
    _assert_grads(got, ref)


def test_backward_full_size_sampled_heads():
    """The 360M training shape (B=8, H=16, N=2048, d'=16, dv=64) through the C ABI;
    the oracle checks three whole heads (heads are independent)."""
    B, H, N = 8, 16, 2048
    inp, dy64, got = _case(B, H, N, 16, 64, seed=21)
    for b, h in ((0, 0), (3, 7), (7, 15)):
        ref = oracle.la_backward(inp.q64[b, h], inp.k64[b, h], inp.v64[b, h], dy64[b, h])
        _assert_grads(tuple(g[b, h] for g in got), ref, f"head ({b},{h}) ")


def test_backward_large_shape_sampled_heads():
    """d'=32, dv=128 at 8192 tokens (the large-state shape); two heads checked."""
    B, H, N = 1, 2, 8192
    inp, dy64, got = _case(B, H, N, 32, 128, seed=31)
    ref = oracle.la_backward(inp.q64[0, 1], inp.k64[0, 1], inp.v64[0, 1], dy64[0, 1])
    _assert_grads(tuple(g[0, 1] for g in got), ref)


def test_backward_deterministic_and_workspace_reuse():
    inp = synthetic.la_inputs(2, 4, 500, 32, 64, "bf16", seed=2)
    dy, _ = synthetic.upstream_grad((2, 4, 500, 64), "bf16", seed=3)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    dy = dy.to(DEV)
    y, _, _ = based.la_prefill(q, k, v, want_state=False)
    ws = torch.empty(based.la_backward_workspace(2, 4, 500, 32, 64), dtype=torch.uint8, device=DEV)
    first = based.la_backward(q, k, v, y, dy, workspace=ws)
    for _ in range(3):
        again = based.la_backward(q, k, v, y, dy, workspace=ws)
        assert all(torch.equal(a, b) for a, b in zip(first, again))
    assert based.get_last_error() == 0


def test_backward_rejects_fp32():
    inp = synthetic.la_inputs(1, 1, 64, 16, 64, "f32", seed=1)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    with pytest.raises(based.BasedError):
        based.la_backward(q, k, v, v.clone(), v.clone())
