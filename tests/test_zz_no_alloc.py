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

import oracle
import linear_attention_sequence_causal_b200 as based
from linear_attention_sequence_causal_b200 import binding, synthetic
from parity_util import assert_state, assert_y

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(q, k, v, want_state=True, chunk=0):
    B, H, N, d_feat = q.shape
    d_v = v.shape[-1]
    D = 1 + d_feat + d_feat * d_feat
    y = torch.empty((B, H, N, d_v), dtype=q.dtype, device=DEV)
    S = torch.empty((B, H, D, d_v), dtype=torch.float32, device=DEV) if want_state else None
    z = torch.empty((B, H, D), dtype=torch.float32, device=DEV) if want_state else None
    dt = binding.BF16 if q.dtype == torch.bfloat16 else binding.F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = based.lib().based_la_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(S), _ptr(z),
                                              B, H, N, d_feat, d_v, dt, chunk, stream)
    assert st == binding.OK, based.status_string(st)
    assert based.get_last_error() == 0
    return y, S, z


def _to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


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


# Shapes that take the other paths: the chunked quadratic path (d'=32, dv=128;
# at these lengths its chunk start states fit the scratch), the CUDA-core fp32
# path, and the segmented bf16 chunked kernel again. Each with and without the
# final state, two calls in a row against based_la_prefill.
@pytest.mark.parametrize("d_feat,d_v,dtype,N", [(32, 128, "bf16", 1500), (32, 128, "bf16", 600),
                                               (16, 64, "f32", 300), (16, 64, "bf16", 3000)])
@pytest.mark.parametrize("want_state", [True, False])
def test_noalloc_other_paths_match_twice(d_feat, d_v, dtype, N, want_state):
    torch_dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    inp = synthetic.la_inputs(1, 3, N, d_feat, d_v, dtype, seed=N + d_feat)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y0, S0, z0 = based.la_prefill(q, k, v, want_state=want_state)
    assert based.get_last_error() == 0
    for _ in range(2):
        y1, S1, z1 = _noalloc(q, k, v, want_state=want_state)
        assert_y(_to64(y1), _to64(y0), torch_dt, "y (no-alloc vs workspace)")
        if want_state:
            assert_state(_to64(S1), _to64(S0), torch_dt, "S (no-alloc vs workspace)")
            assert_state(_to64(z1), _to64(z0), torch_dt, "z (no-alloc vs workspace)")


def test_noalloc_matches_oracle():
    """One case end to end against the float64 oracle (segmented bf16 prefill)."""
    inp = synthetic.la_inputs(1, 2, 2500, 16, 64, "bf16", seed=21)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y, S, z = _noalloc(q, k, v)
    assert_y(_to64(y), oracle.la_quadratic(inp.q64, inp.k64, inp.v64), torch.bfloat16)
    ref_S, ref_z = oracle.la_state(inp.k64, inp.v64)
    assert_state(_to64(S), ref_S, torch.bfloat16, "S")
    assert_state(_to64(z), ref_z, torch.bfloat16, "z")


def test_noalloc_refuses_a_chunk_whose_scratch_does_not_fit():
    """An explicit chunk whose chunk start states need more than the fixed
    scratch is refused with BASED_ERR_UNSUPPORTED (and nothing is launched);
    leaving the chunk to the library falls back to one chunk and succeeds."""
    B, H, N, d_feat, d_v = 2, 8, 8192, 32, 128
    assert based.la_prefill_workspace(B, H, N, d_feat, d_v, torch.bfloat16, 128) > 8 << 20
    inp = synthetic.la_inputs(B, H, N, d_feat, d_v, "bf16", seed=2)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y = torch.empty((B, H, N, d_v), dtype=q.dtype, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = based.lib().based_la_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(y), None, None,
                                              B, H, N, d_feat, d_v, binding.BF16, 128, stream)
    assert st == binding.ERR_UNSUPPORTED
    y1, _, _ = _noalloc(q, k, v, want_state=False)
    y0, _, _ = based.la_prefill(q, k, v, chunk=N, want_state=False)     # the same one-chunk form
    assert torch.equal(y1, y0)
