"""Out-of-bounds writes, checked two ways without a sanitizer.

1. Canary-padded outputs: every entry point writes into views of larger
   buffers whose tails hold a sentinel; after the call the tails must be
   unchanged and the outputs equal to those of a call on ordinary buffers.
2. The debug library (libbased_debug.so, built with BASED_DEBUG_BOUNDS): its
   kernels check the index of every hand-indexed global store against the
   buffer's extent and report a miss as BASED_ERR_BOUNDS instead of writing.
   The same calls through its C ABI must report nothing and give the same
   bits as the regular library.
"""

import ctypes
import math
import os

import pytest
import torch

import linear_attention_sequence_causal_b200 as based
from linear_attention_sequence_causal_b200 import binding, synthetic

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
PAD = 4096                       # elements of sentinel after every output
SENT = {torch.float32: 12345.0, torch.bfloat16: 777.0, torch.uint8: 0xA5}


def padded(shape, dtype, init=None):
    """(view of the buffer's head with `shape`, the whole buffer) with a sentinel tail."""
    n = math.prod(shape)
    buf = torch.full((n + PAD,), SENT[dtype], dtype=dtype, device=DEV)
    view = buf[:n].view(shape)
    if init is not None:
        view.copy_(init)
    return view, buf


def tail_intact(buf, n):
    return bool(torch.all(buf[n:] == SENT[buf.dtype]).item())


def check(pairs):
    torch.cuda.synchronize()
    for view, buf in pairs:
        assert tail_intact(buf, view.numel()), "a kernel wrote past the end of its output"


# ---------------------------------------------------------------- canaries (regular library)

@pytest.mark.parametrize("d_feat,d_v,N,chunk", [(16, 64, 3000, 0), (16, 64, 700, 256), (16, 64, 300, 64),
                                                (32, 128, 1100, 256), (16, 128, 700, 0)])
def test_la_prefill_canaries(d_feat, d_v, N, chunk):
    B, H = 1, 3
    inp = synthetic.la_inputs(B, H, N, d_feat, d_v, "bf16", seed=N)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    D = based.feature_dim(d_feat)
    y0, S0, z0 = based.la_prefill(q, k, v, chunk=chunk)
    y, yb = padded((B, H, N, d_v), torch.bfloat16)
    S, Sb = padded((B, H, D, d_v), torch.float32)
    z, zb = padded((B, H, D), torch.float32)
    ws_bytes = based.la_prefill_workspace(B, H, N, d_feat, d_v, torch.bfloat16, chunk)
    ws, wsb = padded((max(ws_bytes, 16),), torch.uint8)
    based.la_prefill(q, k, v, chunk=chunk, y=y, S=S, z=z, workspace=ws)
    assert based.get_last_error() == 0
    check([(y, yb), (S, Sb), (z, zb), (ws, wsb)])
    assert torch.equal(y, y0) and torch.equal(S, S0) and torch.equal(z, z0)


@pytest.mark.parametrize("d_feat,d_v,packed", [(16, 64, False), (32, 128, False), (16, 64, True)])
def test_la_decode_canaries(d_feat, d_v, packed):
    B, H = 5, 3
    inp = synthetic.la_inputs(B, H, 41, d_feat, d_v, "bf16", seed=d_feat)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    _, S_init, z_init = based.la_prefill(q[:, :, :40].contiguous(), k[:, :, :40].contiguous(),
                                         v[:, :, :40].contiguous(), packed=packed)
    q1, k1, v1 = (x[:, :, 40].contiguous() for x in (q, k, v))
    S0, z0 = S_init.clone(), z_init.clone()
    y0 = based.la_decode_step(S0, z0, q1, k1, v1, packed=packed)
    S, Sb = padded(tuple(S_init.shape), torch.float32, S_init)
    z, zb = padded(tuple(z_init.shape), torch.float32, z_init)
    y, yb = padded((B, H, d_v), torch.bfloat16)
    based.la_decode_step(S, z, q1, k1, v1, y=y, packed=packed)
    assert based.get_last_error() == 0
    check([(S, Sb), (z, zb), (y, yb)])
    assert torch.equal(y, y0) and torch.equal(S, S0) and torch.equal(z, z0)


@pytest.mark.parametrize("N,w", [(200, 64), (40, 64), (130, 17)])
def test_swa_canaries(N, w):
    B, H, d = 3, 4, 64
    inp = synthetic.swa_inputs(B, H, N + 1, d, "bf16", seed=N + w)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    qp, kp, vp = (x[:, :, :N].contiguous() for x in (q, k, v))
    q1, k1, v1 = (x[:, :, N].contiguous() for x in (q, k, v))
    y0, kc0, vc0 = based.swa_prefill(qp, kp, vp, w=w)
    yd0 = based.swa_decode(kc0, vc0, N, q1, k1, v1, w=w)
    y, yb = padded((B, H, N, d), torch.bfloat16)
    kc, kcb = padded((B, H, w, d), torch.bfloat16)
    vc, vcb = padded((B, H, w, d), torch.bfloat16)
    based.swa_prefill(qp, kp, vp, w=w, y=y, k_cache=kc, v_cache=vc)
    yd, ydb = padded((B, H, d), torch.bfloat16)
    based.swa_decode(kc, vc, N, q1, k1, v1, w=w, y=yd)
    assert based.get_last_error() == 0
    check([(y, yb), (kc, kcb), (vc, vcb), (yd, ydb)])
    assert torch.equal(y, y0) and torch.equal(yd, yd0) and torch.equal(kc, kc0) and torch.equal(vc, vc0)


def test_la_backward_canaries():
    B, H, N = 1, 3, 300
    inp = synthetic.la_inputs(B, H, N, 16, 64, "bf16", seed=3)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    dy = synthetic.upstream_grad((B, H, N, 64), "bf16", seed=4)[0].to(DEV)
    y, _, _ = based.la_prefill(q, k, v, want_state=False)
    g0 = based.la_backward(q, k, v, y, dy)
    dq, dqb = padded(tuple(q.shape), torch.bfloat16)
    dk, dkb = padded(tuple(k.shape), torch.bfloat16)
    dv, dvb = padded(tuple(v.shape), torch.bfloat16)
    ws_bytes = based.la_backward_workspace(B, H, N, 16, 64)
    # the workspace must start 256-byte aligned: a fresh allocation is
    ws, wsb = padded((ws_bytes,), torch.uint8)
    based.la_backward(q, k, v, y, dy, dq, dk, dv, workspace=ws)
    assert based.get_last_error() == 0
    check([(dq, dqb), (dk, dkb), (dv, dvb), (ws, wsb)])
    for a, b in zip((dq, dk, dv), g0):
        assert torch.equal(a, b)


@pytest.mark.parametrize("K,d", [(4, 64), (3, 12), (1, 8)])
def test_baseconv_canaries(K, d):
    B, N = 3, 50
    c = synthetic.conv_inputs(B, N + 1, d, K, "bf16", seed=K + d)
    g, x, h, bias = (t.to(DEV) for t in (c.u_gate, c.u_conv, c.h, c.bias))
    gp, xp = g[:, :N].contiguous(), x[:, :N].contiguous()
    g1, x1 = g[:, N].contiguous(), x[:, N].contiguous()
    y0, st0 = based.baseconv_prefill(gp, xp, h, bias)
    yd0 = based.baseconv_decode(st0, g1, x1, h, bias) if K > 1 else based.baseconv_decode(None, g1, x1, h, bias)
    y, yb = padded((B, N, d), torch.bfloat16)
    st, stb = padded((B, max(K - 1, 0), d), torch.bfloat16)
    based.baseconv_prefill(gp, xp, h, bias, state=st, y=y)
    yd, ydb = padded((B, d), torch.bfloat16)
    based.baseconv_decode(st if K > 1 else None, g1, x1, h, bias, y=yd)
    assert based.get_last_error() == 0
    check([(y, yb), (st, stb), (yd, ydb)])
    assert torch.equal(y, y0) and torch.equal(yd, yd0)
    if K > 1:
        assert torch.equal(st, st0)


# ---------------------------------------------------------------- the index-checking debug library

DEBUG_LIB = os.path.join(os.path.dirname(binding.library_path()), "libbased_debug.so")


@pytest.fixture(scope="module")
def dbg():
    if not os.path.exists(DEBUG_LIB):
        from linear_attention_sequence_causal_b200 import build
        build.build(debug_bounds=True)
    return binding._declare(ctypes.CDLL(DEBUG_LIB))


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ok(lib, st):
    assert st == binding.OK, lib.based_status_string(st)
    assert lib.based_get_last_error(_stream()) == binding.OK     # no index check failed


@pytest.mark.parametrize("d_feat,d_v,N,chunk", [(16, 64, 3000, 0), (16, 64, 700, 256), (16, 64, 300, 64),
                                                (32, 128, 1100, 256), (32, 64, 600, 0)])
def test_debug_library_la_prefill(dbg, d_feat, d_v, N, chunk):
    B, H = 1, 3
    inp = synthetic.la_inputs(B, H, N, d_feat, d_v, "bf16", seed=N + 7)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    y0, S0, z0 = based.la_prefill(q, k, v, chunk=chunk)
    D = based.feature_dim(d_feat)
    y = torch.empty_like(y0)
    S = torch.empty_like(S0)
    z = torch.empty_like(z0)
    ws_bytes = dbg.based_la_prefill_workspace(B, H, N, d_feat, d_v, binding.BF16, chunk)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=DEV)
    st = dbg.based_la_prefill(_p(q), _p(k), _p(v), _p(y), _p(S), _p(z), B, H, N, d_feat, d_v, binding.BF16, chunk,
                              _p(ws), ws.numel(), _stream())
    _ok(dbg, st)
    assert S.shape == (B, H, D, d_v)
    assert torch.equal(y, y0) and torch.equal(S, S0) and torch.equal(z, z0)


def test_debug_library_decode_swa_conv(dbg):
    B, H, d_feat, d_v = 4, 3, 16, 64
    inp = synthetic.la_inputs(B, H, 21, d_feat, d_v, "bf16", seed=9)
    q, k, v = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    _, S_init, z_init = based.la_prefill(q[:, :, :20].contiguous(), k[:, :, :20].contiguous(),
                                         v[:, :, :20].contiguous())
    q1, k1, v1 = (x[:, :, 20].contiguous() for x in (q, k, v))
    S0, z0 = S_init.clone(), z_init.clone()
    y0 = based.la_decode_step(S0, z0, q1, k1, v1)
    S, z, y = S_init.clone(), z_init.clone(), torch.empty_like(y0)
    _ok(dbg, dbg.based_la_decode_step(_p(S), _p(z), _p(q1), _p(k1), _p(v1), _p(y), B, H, d_feat, d_v,
                                      binding.BF16, _stream()))
    assert torch.equal(y, y0) and torch.equal(S, S0) and torch.equal(z, z0)

    w, N = 64, 100
    sw = synthetic.swa_inputs(B, H, N + 1, 64, "bf16", seed=10)
    sq, sk, sv = (t.to(DEV) for t in (sw.q, sw.k, sw.v))
    qp, kp, vp = (x[:, :, :N].contiguous() for x in (sq, sk, sv))
    sq1, sk1, sv1 = (x[:, :, N].contiguous() for x in (sq, sk, sv))
    ys0, kc0, vc0 = based.swa_prefill(qp, kp, vp, w=w)
    yd0 = based.swa_decode(kc0, vc0, N, sq1, sk1, sv1, w=w)
    ys, kc, vc = torch.empty_like(ys0), torch.empty_like(kc0), torch.empty_like(vc0)
    _ok(dbg, dbg.based_swa_prefill(_p(qp), _p(kp), _p(vp), _p(ys), _p(kc), _p(vc), B, H, N, 64, w, 0.125,
                                   binding.BF16, _stream()))
    yd = torch.empty_like(yd0)
    _ok(dbg, dbg.based_swa_decode(_p(kc), _p(vc), N, _p(sq1), _p(sk1), _p(sv1), _p(yd), B, H, 64, w, 0.125,
                                  binding.BF16, _stream()))
    assert torch.equal(ys, ys0) and torch.equal(yd, yd0) and torch.equal(kc, kc0) and torch.equal(vc, vc0)

    K, d, Nc = 4, 64, 50
    c = synthetic.conv_inputs(B, Nc + 1, d, K, "bf16", seed=11)
    g, x, h, bias = (t.to(DEV) for t in (c.u_gate, c.u_conv, c.h, c.bias))
    gp, xp = g[:, :Nc].contiguous(), x[:, :Nc].contiguous()
    g1, x1 = g[:, Nc].contiguous(), x[:, Nc].contiguous()
    yc0, st0 = based.baseconv_prefill(gp, xp, h, bias)
    ycd0 = based.baseconv_decode(st0, g1, x1, h, bias)
    yc, stt, ycd = torch.empty_like(yc0), torch.empty_like(st0), torch.empty_like(ycd0)
    _ok(dbg, dbg.based_baseconv_prefill(_p(gp), _p(xp), _p(h), _p(bias), _p(yc), _p(stt), B, Nc, d, K,
                                        binding.BF16, _stream()))
    _ok(dbg, dbg.based_baseconv_decode(_p(stt), _p(g1), _p(x1), _p(h), _p(bias), _p(ycd), B, d, K,
                                       binding.BF16, _stream()))
    assert torch.equal(yc, yc0) and torch.equal(ycd, ycd0) and torch.equal(stt, st0)


def test_debug_library_reports_bounds_status_name(dbg):
    assert dbg.based_status_string(5) == b"BASED_ERR_BOUNDS"
