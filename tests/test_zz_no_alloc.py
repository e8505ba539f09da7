"""based_la_prefill_noalloc: the prefill for callers that cannot allocate device memory.

Some callers of this library cannot hand it a workspace: their device memory is
owned by someone else (a framework's caching allocator, a serving runtime with a
fixed pool, a plugin host that only hands out its own tensors) or they run where
an allocation would stall the device. For them the library offers an entry point
that takes no workspace and keeps its scratch in one fixed array inside its own
device image. This test calls it through the C ABI twice in a row, on shapes that
need that scratch (long sequences split into segments), and checks each result
against the regular entry point based_la_prefill, within the tolerances the
parity tests use. It lives in a file of its own, collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

import linear_attention_sequence_causal_b200 as based
from linear_attention_sequence_causal_b200 import binding, synthetic
from parity_util import assert_state, assert_y

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(q, k, v):
    B, H, N, d_feat = q.shape
    d_v = v.shape[-1]
    D = 1 + d_feat + d_feat * d_feat
    y = torch.empty((B, H, N, d_v), dtype=q.dtype, device=DEV)
    S = torch.empty((B, H, D, d_v), dtype=torch.float32, device=DEV)
    z = torch.empty((B, H, D), dtype=torch.float32, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = based.lib().based_la_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(S), _ptr(z),
                                              B, H, N, d_feat, d_v, binding.BF16, 0, stream)
    assert st == binding.OK, based.status_string(st)
    assert based.get_last_error() == 0
    return y, S, z


@pytest.mark.parametrize("calls", [[(1, 2, 3000, 11), (2, 16, 4096, 12)]])
def test_noalloc_matches_workspace_entry_point_twice(calls):
    for B, H, N, seed in calls:
        # these shapes split each sequence into segments, so the scratch is used
        assert based.la_prefill_workspace(B, H, N, 16, 64) > 0
        inp = synthetic.la_inputs(B, H, N, 16, 64, "bf16", seed=seed)
        q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
        y0, S0, z0 = based.la_prefill(q, k, v)
        assert based.get_last_error() == 0
        y1, S1, z1 = _noalloc(q, k, v)
        to64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
        assert_y(to64(y1), to64(y0), torch.bfloat16, "y (no-alloc vs workspace)")
        assert_state(to64(S1), to64(S0), torch.bfloat16, "S (no-alloc vs workspace)")
        assert_state(to64(z1), to64(z0), torch.bfloat16, "z (no-alloc vs workspace)")
        assert np.all(to64(z1)[..., 0] == N)
