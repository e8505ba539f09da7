"""GPU parity: causal Taylor linear attention (prefill + decode) against the CPU oracle.

Every case runs the CUDA library through its C ABI (via the ctypes binding) on
seeded synthetic inputs and compares element by element with the float64
oracle evaluated on the same (bf16-rounded) inputs. Tolerances: y max-abs 1e-4
(fp32 inputs) / 2e-2 (bf16 inputs); S, z max|diff|/max|ref| 1e-5 / 1e-2; the
constant feature of z counts tokens and must equal N exactly.
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
DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _run_prefill(inp, chunk=0, want_state=True):
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y, S, z = based.la_prefill(q, k, v, chunk=chunk, want_state=want_state)
    assert based.get_last_error() == 0
    return y, S, z


def _check_full(inp, dtype, y, S, z):
    ref_y = oracle.la_quadratic(inp.q64, inp.k64, inp.v64)
    assert_y(to64(y), ref_y, dtype)
    if S is not None:
        ref_S, ref_z = oracle.la_state(inp.k64, inp.v64)
        assert_state(to64(S), ref_S, dtype, "S")
        assert_state(to64(z), ref_z, dtype, "z")
        assert np.all(to64(z)[..., 0] == inp.k64.shape[-2])


# ------------------------------------------------------------ small / ragged cases

@pytest.mark.parametrize("chunk", [0, 16, 32, 64])
def test_tiny_fp32(chunk):
    """B=1, H=1, N=256, d'=16, dv=64, fp32 inputs (the tiny workload)."""
    inp = synthetic.la_inputs(1, 1, 256, 16, 64, "f32", seed=0)
    y, S, z = _run_prefill(inp, chunk)
    _check_full(inp, torch.float32, y, S, z)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [1, 7, 64, 65, 127, 128, 129, 300])
def test_ragged_lengths(dtype, N):
    inp = synthetic.la_inputs(2, 3, N, 16, 64, dtype, seed=N)
    y, S, z = _run_prefill(inp)
    _check_full(inp, DT[dtype], y, S, z)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d_feat,d_v", [(16, 128), (32, 64), (32, 128)])
def test_other_shapes(dtype, d_feat, d_v):
    inp = synthetic.la_inputs(1, 2, 200, d_feat, d_v, dtype, seed=d_feat + d_v)
    y, S, z = _run_prefill(inp)
    _check_full(inp, DT[dtype], y, S, z)


def test_bf16_chunks_agree_with_oracle():
    inp = synthetic.la_inputs(1, 2, 777, 16, 64, "bf16", seed=5)
    for chunk in (0, 16, 32, 64, 128, 256):
        try:
            y, S, z = _run_prefill(inp, chunk)
        except based.BasedError as e:
            assert e.status == 2, (chunk, e)     # chunk not built for this dtype
            continue
        _check_full(inp, torch.bfloat16, y, S, z)


# Chunk lengths of the chunked tensor-core kernel (d'=16, dv=64, bf16): 128-token
# MMA tiles holding two 64-token chunks, one 128-token chunk, or half of a
# 256-token chunk.
TC_CHUNKS = [64, 128, 256]


@pytest.mark.parametrize("chunk", TC_CHUNKS)
@pytest.mark.parametrize("N", [1, 7, 63, 64, 65, 127, 128, 129, 191, 255, 256, 257, 300, 513])
def test_tc_chunks_ragged(chunk, N):
    """Every output and the final state, for lengths that end inside a chunk,
    on a chunk boundary, inside the second tile of a 256-token chunk and inside
    the second half of a tile holding two 64-token chunks."""
    inp = synthetic.la_inputs(2, 3, N, 16, 64, "bf16", seed=N + chunk)
    y, S, z = _run_prefill(inp, chunk)
    _check_full(inp, torch.bfloat16, y, S, z)


@pytest.mark.parametrize("chunk", TC_CHUNKS)
@pytest.mark.parametrize("B,H,N", [(1, 1, 300), (1, 2, 3000), (2, 3, 1000), (1, 1, 2500), (1, 1, 129)])
def test_tc_chunks_segmented(chunk, B, H, N):
    """Few (b, h) pairs, so sequences are split into segments of whole chunks
    (at 256 tokens, segments whose last one has an odd number of tiles)."""
    inp = synthetic.la_inputs(B, H, N, 16, 64, "bf16", seed=3 * N + chunk)
    y, S, z = _run_prefill(inp, chunk)
    _check_full(inp, torch.bfloat16, y, S, z)


@pytest.mark.parametrize("chunk", TC_CHUNKS)
def test_tc_chunks_repeated_calls_agree(chunk):
    """Repeated calls complete (no expired wait) and agree bit for bit."""
    inp = synthetic.la_inputs(3, 5, 1200, 16, 64, "bf16", seed=chunk)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y0, S0, z0 = based.la_prefill(q, k, v, chunk=chunk)
    assert based.get_last_error() == 0
    for _ in range(4):
        y, S, z = based.la_prefill(q, k, v, chunk=chunk)
        assert based.get_last_error() == 0
        assert torch.equal(y, y0) and torch.equal(S, S0) and torch.equal(z, z0)


def test_no_state_output():
    inp = synthetic.la_inputs(2, 2, 100, 16, 64, "bf16", seed=6)
    y, S, z = _run_prefill(inp, want_state=False)
    assert S is None and z is None
    assert_y(to64(y), oracle.la_quadratic(inp.q64, inp.k64, inp.v64), torch.bfloat16)


def test_zero_query_is_cumulative_mean():
    inp = synthetic.la_inputs(1, 2, 150, 16, 64, "f32", seed=7)
    q = torch.zeros_like(inp.q).to(DEV)
    y, _, _ = based.la_prefill(q, inp.k.to(DEV), inp.v.to(DEV))
    mean = np.cumsum(inp.v64, axis=-2) / np.arange(1, 151)[:, None]
    assert_y(to64(y), mean, torch.float32)


@pytest.mark.parametrize("d_feat,d_v", [(16, 128), (32, 64), (32, 128)])
@pytest.mark.parametrize("N", [1, 65, 129, 300])
def test_quadratic_path_ragged(d_feat, d_v, N):
    """bf16 shapes whose state exceeds one SM's tensor memory: quadratic-form tiles
    with a ragged last tile, single-step units, and the separate state contraction."""
    inp = synthetic.la_inputs(1, 3, N, d_feat, d_v, "bf16", seed=N + d_feat)
    y, S, z = _run_prefill(inp)
    _check_full(inp, torch.bfloat16, y, S, z)


@pytest.mark.parametrize("d_feat,d_v", [(16, 128), (32, 64)])
def test_quadratic_path_many_units(d_feat, d_v):
    """More (query tile, head) units than SMs: every CTA sweeps several units of
    different lengths, so S buffers, O accumulators and row sums change hands."""
    B, H, N = 2, 40, 1100
    inp = synthetic.la_inputs(B, H, N, d_feat, d_v, "bf16", seed=11)
    y, S, z = _run_prefill(inp)
    y2, _, _ = _run_prefill(inp, want_state=False)
    assert torch.equal(y, y2)
    rng = np.random.default_rng(3)
    heads = [(0, 0), (0, 17), (1, 39)]
    _sampled_check(inp, torch.bfloat16, y, S, z, heads, _rows(N, rng, 24), heads)


# Chunks of the chunked quadratic path (the shapes whose state does not fit one
# SM's tensor memory): chunk start states go through the workspace.
@pytest.mark.parametrize("d_feat,d_v", [(16, 128), (32, 64), (32, 128)])
@pytest.mark.parametrize("chunk", [128, 256, 512])
@pytest.mark.parametrize("N", [129, 300, 700, 1100])
def test_chunked_state_path(d_feat, d_v, chunk, N):
    """Every output and the final state; N from just past one chunk of 128 to
    several chunks with a ragged last tile."""
    inp = synthetic.la_inputs(1, 3, N, d_feat, d_v, "bf16", seed=N + chunk + d_feat)
    y, S, z = _run_prefill(inp, chunk)
    _check_full(inp, torch.bfloat16, y, S, z)


@pytest.mark.parametrize("d_feat,d_v", [(16, 128), (32, 64), (32, 128)])
def test_chunked_state_path_many_units(d_feat, d_v):
    """More (query tile, head) units than SMs in 256-token chunks: units with
    and without chunk start states, of different lengths, on every CTA; the
    result agrees with the one-chunk quadratic form and with the oracle."""
    B, H, N = 2, 40, 1100
    inp = synthetic.la_inputs(B, H, N, d_feat, d_v, "bf16", seed=13)
    y, S, z = _run_prefill(inp, 256)
    y1, S1, z1 = _run_prefill(inp, 1152)             # one chunk: no start states
    assert_y(to64(y), to64(y1), torch.bfloat16, "chunked vs one chunk")
    assert_state(to64(S), to64(S1), torch.bfloat16, "S")
    rng = np.random.default_rng(4)
    heads = [(0, 0), (0, 17), (1, 39), (1, 2)]
    _sampled_check(inp, torch.bfloat16, y, S, z, heads, _rows(N, rng, 24), heads)


def test_chunked_state_path_rejects_bad_chunks():
    inp = synthetic.la_inputs(1, 1, 300, 32, 128, "bf16", seed=1)
    for chunk in (100, 192 + 1, -128):
        with pytest.raises(based.BasedError) as e:
            _run_prefill(inp, chunk)
        assert e.value.status in (1, 2)


def test_quadratic_path_repeated_calls_agree():
    """Two O issuers (dv = 64) hand P buffers back and forth across many steps:
    repeated calls must all complete (no expired wait) and agree bit for bit."""
    B, H, N = 8, 16, 2048
    inp = synthetic.la_inputs(B, H, N, 32, 64, "bf16", seed=21)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y0, S0, z0 = based.la_prefill(q, k, v)
    assert based.get_last_error() == 0
    for _ in range(6):
        y, S, z = based.la_prefill(q, k, v)
        assert based.get_last_error() == 0
        assert torch.equal(y, y0) and torch.equal(S, S0) and torch.equal(z, z0)
    rng = np.random.default_rng(5)
    heads = [(0, 0), (7, 15)]
    _sampled_check(inp, torch.bfloat16, y0, S0, z0, heads, _rows(N, rng, 16), heads)


def test_outputs_stay_in_bounds_and_deterministic():
    inp = synthetic.la_inputs(1, 2, 130, 16, 64, "bf16", seed=8)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    canary = torch.full((2 * 130 * 64 + 4096,), 7.0, dtype=torch.bfloat16, device=DEV)
    y = canary[: 2 * 130 * 64].view(1, 2, 130, 64)
    based.la_prefill(q, k, v, y=y)
    torch.cuda.synchronize()
    assert torch.all(canary[2 * 130 * 64:] == 7.0)
    y2, _, _ = based.la_prefill(q, k, v)
    assert torch.equal(y, y2)


# ------------------------------------------------------------ full-size workloads (sampled)

def _sampled_check(inp, dtype, y, S, z, heads, rows, state_heads):
    """y of `heads` at `rows` (a list, or a function (b, h) -> rows) against the
    oracle row by row; the final S and z of `state_heads` in full."""
    y64, S64, z64 = to64(y), to64(S), to64(z)
    for (b, h) in heads:
        rr = rows(b, h) if callable(rows) else rows
        ref = oracle.la_rows(inp.q64[b, h], inp.k64[b, h], inp.v64[b, h], rr)
        assert_y(y64[b, h, rr], ref, dtype, f"y[{b},{h}]")
    for (b, h) in state_heads:                  # one head at a time: phi(K) of a long head is large
        ref_S, ref_z = oracle.la_state(inp.k64[b, h], inp.v64[b, h])
        assert_state(S64[b, h], ref_S, dtype, f"S[{b},{h}]")
        assert_state(z64[b, h], ref_z, dtype, f"z[{b},{h}]")
    assert np.all(z64[..., 0] == inp.k64.shape[-2])


def _rows(N, rng, n=48):
    fixed = [0, 1, 63, 64, 127, 128, 255, 256, N // 2, N - 2, N - 1]
    return sorted(set([r for r in fixed if r < N] + rng.integers(0, N, n).tolist()))


def _every_head(B, H):
    return [(b, h) for b in range(B) for h in range(H)]


def _head_rows(N, seed, n=16):
    """Rows for one head: chunk, tile and segment boundaries plus n random rows.
    Every head gets its own random rows (a boundary bug confined to some heads
    or segments still meets a checked row)."""
    edges = [0, 1, 63, 64, 65, 127, 128, 129, 255, 256, 257, N // 4, N // 2, 3 * N // 4, N - 2, N - 1]
    def rows(b, h):
        rng = np.random.default_rng(seed + 1000 * b + h)
        return sorted(set([r for r in edges if 0 <= r < N] + rng.integers(0, N, n).tolist()))
    return rows


@pytest.mark.parametrize("chunk", [0, 64, 128, 256])
def test_360m_prefill_sampled(chunk):
    """B=8, H=16, N=2048, d'=16, dv=64, bf16: every head at 16+ rows (chunk,
    tile and random rows of its own) and every head's final state."""
    inp = synthetic.la_inputs(8, 16, 2048, 16, 64, "bf16", seed=0)
    y, S, z = _run_prefill(inp, chunk)
    _sampled_check(inp, torch.bfloat16, y, S, z, _every_head(8, 16), _head_rows(2048, 0), _every_head(8, 16))
    # all outputs finite, in a sane range (y is a convex-ish average of v)
    assert torch.isfinite(y.float()).all()


@pytest.mark.parametrize("chunk", [0, 64, 128, 256])
def test_long_prefill_sampled(chunk):
    """B=2, H=16, N=16384, chunk length swept over 64/128/256 (each on the
    tensor cores; none may be refused): every head at 16+ rows including
    segment boundaries, every head's final S and z."""
    inp = synthetic.la_inputs(2, 16, 16384, 16, 64, "bf16", seed=0)
    y, S, z = _run_prefill(inp, chunk)
    _sampled_check(inp, torch.bfloat16, y, S, z, _every_head(2, 16), _head_rows(16384, 1, 24),
                   _every_head(2, 16))


def test_large_state_prefill_sampled():
    """d'=32 (D=1057), H=8, dv=128, B=4, N=8192, bf16: every head at 16+ rows,
    the final state of eight heads."""
    inp = synthetic.la_inputs(4, 8, 8192, 32, 128, "bf16", seed=0)
    y, S, z = _run_prefill(inp)
    _sampled_check(inp, torch.bfloat16, y, S, z, _every_head(4, 8), _head_rows(8192, 2),
                   [(0, 0), (0, 7), (1, 3), (1, 4), (2, 5), (2, 1), (3, 6), (3, 7)])


# ------------------------------------------------------------ decode

def _decode_run(B, H, d_feat, d_v, dtype, prompt, steps, seed, check_heads):
    """Prefill `prompt` tokens, then `steps` decode steps; compare with the oracle."""
    inp = synthetic.la_inputs(B, H, prompt + steps, d_feat, d_v, dtype, seed=seed)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    _, S, z = based.la_prefill(q[:, :, :prompt].contiguous(), k[:, :, :prompt].contiguous(),
                               v[:, :, :prompt].contiguous())
    ys = torch.empty((B, H, steps, d_v), dtype=q.dtype, device=DEV)
    # step-major copies so each step's q, k, v are contiguous [B, H, *] slices
    qd, kd, vd = (x[:, :, prompt:].permute(2, 0, 1, 3).contiguous() for x in (q, k, v))
    for t in range(steps):
        ys[:, :, t] = based.la_decode_step(S, z, qd[t], kd[t], vd[t])
    assert based.get_last_error() == 0
    dt = DT[dtype]
    ys64, S64, z64 = to64(ys), to64(S), to64(z)
    bs = [b for b, _ in check_heads]
    hs = [h for _, h in check_heads]
    ref = oracle.la_quadratic(inp.q64[bs, hs], inp.k64[bs, hs], inp.v64[bs, hs])
    assert_y(ys64[bs, hs], ref[..., prompt:, :], dt, "decode y")
    ref_S, ref_z = oracle.la_state(inp.k64[bs, hs], inp.v64[bs, hs])
    assert_state(S64[bs, hs], ref_S, dt, "S")
    assert_state(z64[bs, hs], ref_z, dt, "z")
    assert np.all(z64[..., 0] == prompt + steps)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_small(dtype):
    _decode_run(2, 3, 16, 64, dtype, prompt=37, steps=40, seed=11,
                check_heads=[(b, h) for b in range(2) for h in range(3)])


@pytest.mark.parametrize("batch", [1, 16, 64, 128, 256])
def test_decode_workload(batch):
    """H=16, d'=16, dv=64, 512-token prompt then 1024 decode steps, bf16 q/k/v, fp32 state."""
    rng = np.random.default_rng(batch)
    heads = [(int(rng.integers(batch)), int(rng.integers(16))) for _ in range(4)] + [(batch - 1, 15)]
    _decode_run(batch, 16, 16, 64, "bf16", prompt=512, steps=1024, seed=batch, check_heads=heads)


def test_decode_large_state():
    """d'=32, dv=128, H=8, batch 64, 256 decode steps after a 512-token prompt."""
    _decode_run(64, 8, 32, 128, "bf16", prompt=512, steps=256, seed=3,
                check_heads=[(0, 0), (31, 4), (63, 7)])


def test_decode_resume_from_copied_state_is_bit_identical():
    """The state (S, z) is the checkpoint: copying it out and back resumes exactly."""
    inp = synthetic.la_inputs(2, 4, 80, 16, 64, "bf16", seed=12)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    _, S, z = based.la_prefill(q[:, :, :60].contiguous(), k[:, :, :60].contiguous(), v[:, :, :60].contiguous())
    S_saved, z_saved = S.cpu().clone(), z.cpu().clone()
    outs = []
    for _ in range(2):
        S2, z2 = S_saved.to(DEV), z_saved.to(DEV)
        ys = [based.la_decode_step(S2, z2, q[:, :, t].contiguous(), k[:, :, t].contiguous(),
                                   v[:, :, t].contiguous()) for t in range(60, 80)]
        outs.append((torch.stack(ys), S2, z2))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_decode_rejects_unsupported():
    S = torch.zeros(1, 1, 1 + 24 + 576, 64, device=DEV)
    z = torch.zeros(1, 1, 1 + 24 + 576, device=DEV)
    x = torch.zeros(1, 1, 24, device=DEV)
    with pytest.raises(based.BasedError) as e:
        based.la_decode_step(S, z, x, x, torch.zeros(1, 1, 64, device=DEV))
    assert e.value.status == 2


# ------------------------------------------------------------ segments (few heads, long sequences)

@pytest.mark.parametrize("B,H,N", [(1, 1, 300), (1, 2, 3000), (2, 3, 1000), (1, 1, 129)])
def test_segmented_prefill_full(B, H, N):
    """Few (b, h) pairs: each sequence is split into segments whose start states come
    from a totals pass through the workspace; every output and the final state checked."""
    inp = synthetic.la_inputs(B, H, N, 16, 64, "bf16", seed=N + H)
    assert based.la_prefill_workspace(B, H, N, 16, 64) > 0 or N <= 128
    y, S, z = _run_prefill(inp)
    _check_full(inp, torch.bfloat16, y, S, z)


def test_workspace_too_small_is_rejected():
    import ctypes
    from linear_attention_sequence_causal_b200 import binding
    inp = synthetic.la_inputs(1, 2, 3000, 16, 64, "bf16", seed=1)
    need = based.la_prefill_workspace(1, 2, 3000, 16, 64)
    assert need > 0
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y = torch.empty(1, 2, 3000, 64, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    st = based.lib().based_la_prefill(P(q), P(k), P(v), P(y), None, None, 1, 2, 3000, 16, 64, binding.BF16, 0,
                                      P(ws), need - 16, None)
    assert st == binding.ERR_INVALID_ARG
    st = based.lib().based_la_prefill(P(q), P(k), P(v), P(y), None, None, 1, 2, 3000, 16, 64, binding.BF16, 0,
                                      None, 0, None)
    assert st == binding.ERR_INVALID_ARG
