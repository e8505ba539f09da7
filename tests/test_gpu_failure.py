"""Failure detection on the GPU without a fault: a kernel whose bounded waits
expire reports BASED_ERR_TIMEOUT through based_get_last_error, and the CUDA
context stays usable for the next call.

BASED_DEBUG_SKIP_MMA=1 makes the tensor-core kernels issue no MMA, so the
waits on their completion barriers run out (after about two seconds); the
kernels then free their tensor memory and return.
"""

import math

import numpy as np
import pytest

import oracle
import linear_attention_sequence_causal_b200 as based
from linear_attention_sequence_causal_b200 import synthetic
from parity_util import assert_y, to64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TIMEOUT = 4


def test_stalled_la_prefill_reports_timeout(monkeypatch):
    import torch
    inp = synthetic.la_inputs(1, 1, 300, 16, 64, "bf16", seed=3)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    monkeypatch.setenv("BASED_DEBUG_SKIP_MMA", "1")
    based.la_prefill(q, k, v)                       # the launch itself succeeds
    assert based.get_last_error() == TIMEOUT
    assert based.get_last_error() == 0              # the word was cleared
    monkeypatch.delenv("BASED_DEBUG_SKIP_MMA")
    y, S, z = based.la_prefill(q, k, v)
    assert based.get_last_error() == 0
    assert_y(to64(y), oracle.la_quadratic(inp.q64, inp.k64, inp.v64), torch.bfloat16)


def test_stalled_chunked_state_path_reports_timeout(monkeypatch):
    """d'=32, dv=128 in 128-token chunks: the chunk start-state sweep and the
    output kernel both stall and report; the next call is correct."""
    import torch
    inp = synthetic.la_inputs(1, 2, 300, 32, 128, "bf16", seed=9)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    monkeypatch.setenv("BASED_DEBUG_SKIP_MMA", "1")
    based.la_prefill(q, k, v, chunk=128)
    assert based.get_last_error() == TIMEOUT
    monkeypatch.delenv("BASED_DEBUG_SKIP_MMA")
    y, S, z = based.la_prefill(q, k, v, chunk=128)
    assert based.get_last_error() == 0
    assert_y(to64(y), oracle.la_quadratic(inp.q64, inp.k64, inp.v64), torch.bfloat16)


def test_stalled_swa_prefill_reports_timeout(monkeypatch):
    import torch
    inp = synthetic.swa_inputs(1, 2, 200, 64, "bf16", seed=4)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    monkeypatch.setenv("BASED_DEBUG_SKIP_MMA", "1")
    based.swa_prefill(q, k, v, w=64)
    assert based.get_last_error() == TIMEOUT
    monkeypatch.delenv("BASED_DEBUG_SKIP_MMA")
    y, _, _ = based.swa_prefill(q, k, v, w=64)
    assert based.get_last_error() == 0
    assert_y(to64(y), oracle.swa(inp.q64, inp.k64, inp.v64, 64, 1 / math.sqrt(64)), torch.bfloat16)


def test_stalled_la_backward_reports_timeout(monkeypatch):
    import torch
    inp = synthetic.la_inputs(1, 2, 300, 16, 64, "bf16", seed=5)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    dy, dy64 = synthetic.upstream_grad((1, 2, 300, 64), "bf16", seed=6)
    dy = dy.to(DEV)
    y, _, _ = based.la_prefill(q, k, v, want_state=False)
    monkeypatch.setenv("BASED_DEBUG_SKIP_MMA", "1")
    based.la_backward(q, k, v, y, dy)                 # both launches succeed; their waits expire
    assert based.get_last_error() == TIMEOUT
    monkeypatch.delenv("BASED_DEBUG_SKIP_MMA")
    dq, dk, dv = based.la_backward(q, k, v, y, dy)
    assert based.get_last_error() == 0
    ref = oracle.la_backward(inp.q64, inp.k64, inp.v64, dy64)
    for got, r in zip((dq, dk, dv), ref):
        assert float(np.abs(to64(got) - r).max() / np.abs(r).max()) < 2e-2
