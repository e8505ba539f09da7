"""GPU parity of coarse decay (one gamma per 128-token tile) against the oracle.

based_la_prefill_decay weighs key j for query i >= j by the product of gamma
over the tiles after j's up to i's, in numerator and denominator alike, and
returns the decayed final state; based_la_decode_step_decay scales the state
by gamma before a token. The oracle's la_quadratic_decay, la_state_decay and
la_recurrent_decay are pinned on the CPU (closed form, gamma = 1, pairwise
weights against the step recurrence). Tolerances are the undecayed ones.
"""

import numpy as np
import pytest
import torch

import oracle
import linear_attention_sequence_causal_b200 as based
from linear_attention_sequence_causal_b200 import synthetic
from parity_util import assert_state, assert_y, to64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _gamma(B, H, N, seed, lo=0.5):
    rng = np.random.default_rng(seed)
    g = rng.uniform(lo, 1.0, (B, H, oracle.decay_chunks(N))).astype(np.float32)
    return torch.from_numpy(g), g.astype(np.float64)


@pytest.mark.parametrize("d_feat,d_v", [(16, 64), (16, 128), (32, 64), (32, 128)])
def test_prefill_decay(d_feat, d_v):
    B, H, N = 1, 2, 300
    inp = synthetic.la_inputs(B, H, N, d_feat, d_v, "bf16", seed=d_feat + d_v)
    g, g64 = _gamma(B, H, N, seed=5)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y, S, z = based.la_prefill_decay(q, k, v, g.to(DEV))
    assert based.get_last_error() == 0
    assert_y(to64(y), oracle.la_quadratic_decay(inp.q64, inp.k64, inp.v64, g64), torch.bfloat16)
    rS, rz = oracle.la_state_decay(inp.k64, inp.v64, g64)
    assert_state(to64(S), rS, torch.bfloat16, "S")
    assert_state(to64(z), rz, torch.bfloat16, "z")


def test_prefill_decay_of_one_is_the_undecayed_kernel():
    """gamma = 1 gives weights of exactly 1: the same bits as the undecayed
    quadratic form (one chunk of at least the sequence, which the decayed path
    of this shape always uses)."""
    inp = synthetic.la_inputs(2, 2, 700, 32, 128, "bf16", seed=9)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    ones = torch.ones((2, 2, oracle.decay_chunks(700)), dtype=torch.float32, device=DEV)
    y1, S1, z1 = based.la_prefill_decay(q, k, v, ones)
    y0, S0, z0 = based.la_prefill(q, k, v, chunk=768)
    assert based.get_last_error() == 0
    assert torch.equal(y1, y0) and torch.equal(S1, S0) and torch.equal(z1, z0)


@pytest.mark.parametrize("d_feat,d_v", [(16, 64), (32, 128)])
def test_decode_continues_decayed_prefill(d_feat, d_v):
    """Prefill 256 tokens (tiles 0, 1), then decode tokens 256..299: token 256 begins
    tile 2 and takes gamma_2, the rest take 1."""
    B, H, N0, N = 2, 3, 256, 300
    inp = synthetic.la_inputs(B, H, N, d_feat, d_v, "bf16", seed=3)
    g, g64 = _gamma(B, H, N, seed=4)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    _, S, z = based.la_prefill_decay(q[:, :, :N0].contiguous(), k[:, :, :N0].contiguous(),
                                     v[:, :, :N0].contiguous(), g[..., :2].contiguous().to(DEV))
    steps = oracle.decay_per_step(g64, N - N0, t0=N0)
    ys = []
    for t in range(N0, N):
        gs = torch.from_numpy(steps[..., t - N0].astype(np.float32)).contiguous().to(DEV)
        ys.append(based.la_decode_step_decay(S, z, q[:, :, t].contiguous(), k[:, :, t].contiguous(),
                                             v[:, :, t].contiguous(), gs))
    assert based.get_last_error() == 0
    ref = oracle.la_quadratic_decay(inp.q64, inp.k64, inp.v64, g64)
    assert_y(to64(torch.stack(ys, dim=2)), ref[..., N0:, :], torch.bfloat16, "decode y")
    rS, rz = oracle.la_state_decay(inp.k64, inp.v64, g64)
    assert_state(to64(S), rS, torch.bfloat16, "S")
    assert_state(to64(z), rz, torch.bfloat16, "z")


def test_decode_decay_packed_from_empty_state():
    """Symmetric layout, decaying every step from an empty state: the oracle's step
    recurrence with the same per-step gamma."""
    B, H, N, d_feat, d_v = 2, 2, 40, 16, 64
    inp = synthetic.la_inputs(B, H, N, d_feat, d_v, "bf16", seed=6)
    rng = np.random.default_rng(7)
    steps = rng.uniform(0.6, 1.0, (B, H, N))
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    Dp = based.packed_dim(d_feat)
    S = torch.zeros((B, H, Dp, d_v), dtype=torch.float32, device=DEV)
    z = torch.zeros((B, H, Dp), dtype=torch.float32, device=DEV)
    ys = []
    for t in range(N):
        gs = torch.from_numpy(steps[..., t].astype(np.float32)).contiguous().to(DEV)
        ys.append(based.la_decode_step_decay(S, z, q[:, :, t].contiguous(), k[:, :, t].contiguous(),
                                             v[:, :, t].contiguous(), gs, packed=True))
    assert based.get_last_error() == 0
    g32 = steps.astype(np.float32).astype(np.float64)
    ref, _, _ = oracle.la_recurrent_decay(inp.q64, inp.k64, inp.v64, g32)
    assert_y(to64(torch.stack(ys, dim=2)), ref, torch.bfloat16, "decode y")


@pytest.mark.parametrize("d_feat,d_v", [(16, 64), (32, 128)])
def test_prefill_decay_long_sampled_heads(d_feat, d_v):
    """4096 tokens (32 tiles), gamma near 1 as a trained decay would be: the chunked
    kernel (d'=16, dv=64) rescales its state 31 times, the quadratic form weighs
    tile pairs up to 31 tiles apart."""
    B, H, N = 1, 4, 4096
    inp = synthetic.la_inputs(B, H, N, d_feat, d_v, "bf16", seed=11)
    g, g64 = _gamma(B, H, N, seed=12, lo=0.9)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y, S, z = based.la_prefill_decay(q, k, v, g.to(DEV))
    assert based.get_last_error() == 0
    for h in (0, 3):
        ref = oracle.la_quadratic_decay(inp.q64[0, h], inp.k64[0, h], inp.v64[0, h], g64[0, h])
        assert_y(to64(y[0, h]), ref, torch.bfloat16, f"y head {h}")
        rS, rz = oracle.la_state_decay(inp.k64[0, h], inp.v64[0, h], g64[0, h])
        assert_state(to64(S[0, h]), rS, torch.bfloat16, f"S head {h}")


def test_prefill_decay_segments_of_many_tiles():
    """32 (b, h) pairs of 4096 tokens: each sequence is cut into four segments of
    eight 128-token tiles, so the totals CTA of a segment rescales its state
    tile by tile over eight tiles, more than its ring of input stages holds."""
    B, H, N = 2, 16, 4096
    inp = synthetic.la_inputs(B, H, N, 16, 64, "bf16", seed=21)
    g, g64 = _gamma(B, H, N, seed=22, lo=0.9)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y, S, z = based.la_prefill_decay(q, k, v, g.to(DEV))
    assert based.get_last_error() == 0
    for b, h in ((0, 0), (0, 15), (1, 6), (1, 15)):
        ref = oracle.la_quadratic_decay(inp.q64[b, h], inp.k64[b, h], inp.v64[b, h], g64[b, h])
        assert_y(to64(y[b, h]), ref, torch.bfloat16, f"y head ({b}, {h})")
        rS, rz = oracle.la_state_decay(inp.k64[b, h], inp.v64[b, h], g64[b, h])
        assert_state(to64(S[b, h]), rS, torch.bfloat16, f"S head ({b}, {h})")
        assert_state(to64(z[b, h]), rz, torch.bfloat16, f"z head ({b}, {h})")


@pytest.mark.parametrize("d_feat,d_v", [(16, 64), (32, 128)])
def test_prefill_decay_fp32_cuda_cores(d_feat, d_v):
    """fp32 inputs: the CUDA-core kernel scales its state at every 128-token tile."""
    B, H, N = 1, 2, 400
    inp = synthetic.la_inputs(B, H, N, d_feat, d_v, "f32", seed=d_feat)
    g, g64 = _gamma(B, H, N, seed=13)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y, S, z = based.la_prefill_decay(q, k, v, g.to(DEV))
    assert based.get_last_error() == 0
    assert_y(to64(y), oracle.la_quadratic_decay(inp.q64, inp.k64, inp.v64, g64), torch.float32)
    rS, rz = oracle.la_state_decay(inp.k64, inp.v64, g64)
    assert_state(to64(S), rS, torch.float32, "S")
    assert_state(to64(z), rz, torch.float32, "z")
