"""The C ABI library loads and exports every symbol include/*.h declares (CPU only).

Also checks the synchronous argument validation, which returns before any CUDA
call and so runs without a GPU (no kernel is launched: every case here fails
validation first).
"""

import ctypes
import glob
import os
import re

import pytest

import linear_attention_sequence_causal_b200 as based
from linear_attention_sequence_causal_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names |= set(re.findall(r"BASED_API\s+[\w\s\*]+?\b(based_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(binding.library_path()):
        from linear_attention_sequence_causal_b200 import build
        build.build()
    return based.lib()


def test_header_declares_the_boundary():
    names = _declared_symbols()
    for n in ("based_la_prefill", "based_la_decode_step", "based_swa_prefill", "based_swa_decode",
              "based_get_last_error", "based_la_prefill_workspace"):
        assert n in names
    assert set(binding.SYMBOLS) <= names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(binding.library_path())
    for name in sorted(_declared_symbols()):
        assert hasattr(raw, name), name


def test_version_and_status_strings(lib):
    assert lib.based_version() >= 100
    assert based.status_string(0) == "BASED_OK"
    assert based.status_string(4) == "BASED_ERR_TIMEOUT"
    assert based.status_string(99) == "BASED_ERR_UNKNOWN"


FAKE = ctypes.c_void_p(1 << 20)        # aligned, never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)


@pytest.mark.parametrize("entry", ["based_la_prefill", "based_la_prefill_packed"])
def test_la_prefill_rejects_bad_arguments(lib, entry):
    f = getattr(lib, entry)
    ok = dict(B=1, H=1, N=16, df=16, dv=64, dt=1, chunk=0)

    def call(q=FAKE, S=FAKE, z=FAKE, **kw):
        a = dict(ok, **kw)
        return f(q, FAKE, FAKE, FAKE, S, z, a["B"], a["H"], a["N"], a["df"], a["dv"], a["dt"],
                 a["chunk"], None, 0, None)

    assert call(q=None) == binding.ERR_INVALID_ARG
    assert call(q=MISALIGNED) == binding.ERR_INVALID_ARG
    assert call(S=None) == binding.ERR_INVALID_ARG          # S without z
    assert call(N=0) == binding.ERR_INVALID_ARG
    assert call(B=-1) == binding.ERR_INVALID_ARG
    assert call(dt=7) == binding.ERR_INVALID_ARG
    assert call(chunk=-1) == binding.ERR_INVALID_ARG
    assert call(df=8) == binding.ERR_UNSUPPORTED
    assert call(dv=96) == binding.ERR_UNSUPPORTED


def test_decode_and_swa_reject_bad_arguments(lib):
    assert lib.based_la_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 1, 16, 64, 1, None) \
        == binding.ERR_INVALID_ARG
    assert lib.based_la_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 24, 64, 1, None) \
        == binding.ERR_UNSUPPORTED
    assert lib.based_la_decode_step_packed(FAKE, None, FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 64, 1, None) \
        == binding.ERR_INVALID_ARG
    assert lib.based_la_decode_step_packed(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 96, 1, None) \
        == binding.ERR_UNSUPPORTED
    sp = lib.based_swa_prefill
    assert sp(FAKE, FAKE, FAKE, FAKE, None, None, 1, 1, 8, 64, 0, 0.125, 1, None) == binding.ERR_INVALID_ARG
    assert sp(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 1, 8, 64, 64, 0.125, 1, None) == binding.ERR_INVALID_ARG
    assert sp(FAKE, FAKE, FAKE, FAKE, None, None, 1, 1, 8, 64, 64, float("nan"), 1, None) \
        == binding.ERR_INVALID_ARG
    assert sp(FAKE, FAKE, FAKE, FAKE, None, None, 1, 1, 8, 128, 64, 0.1, 1, None) == binding.ERR_UNSUPPORTED
    assert sp(FAKE, FAKE, FAKE, FAKE, None, None, 1, 1, 8, 64, 65, 0.1, 1, None) == binding.ERR_UNSUPPORTED
    sd = lib.based_swa_decode
    assert sd(FAKE, FAKE, -1, FAKE, FAKE, FAKE, FAKE, 1, 1, 64, 64, 0.125, 1, None) == binding.ERR_INVALID_ARG
    assert sd(FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, 1, 1, 64, 80, 0.125, 1, None) == binding.ERR_UNSUPPORTED


def test_la_backward_rejects_bad_arguments(lib):
    f = lib.based_la_backward
    ok = dict(B=1, H=1, N=16, df=16, dv=64, dt=1, ws=FAKE, nbytes=1 << 20)

    def call(q=FAKE, dq=FAKE, **kw):
        a = dict(ok, **kw)
        return f(q, FAKE, FAKE, FAKE, FAKE, dq, FAKE, FAKE, a["B"], a["H"], a["N"], a["df"], a["dv"],
                 a["dt"], a["ws"], a["nbytes"], None)

    assert call(q=None) == binding.ERR_INVALID_ARG
    assert call(dq=MISALIGNED) == binding.ERR_INVALID_ARG
    assert call(N=0) == binding.ERR_INVALID_ARG
    assert call(dt=7) == binding.ERR_INVALID_ARG
    assert call(dt=0) == binding.ERR_UNSUPPORTED             # fp32: bf16 tensor cores only
    assert call(df=8) == binding.ERR_UNSUPPORTED
    assert call(dv=96) == binding.ERR_UNSUPPORTED
    assert call(ws=None) == binding.ERR_INVALID_ARG
    assert call(ws=MISALIGNED) == binding.ERR_INVALID_ARG    # 256-byte alignment
    assert call(nbytes=16) == binding.ERR_INVALID_ARG        # smaller than the query


def test_decay_entries_reject_bad_arguments(lib):
    pd = lib.based_la_prefill_decay
    # d'=32, dv=128: the quadratic-form path, whose workspace need is known without a device
    ok = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 300, 32, 128, 1, FAKE, 1 << 20, None)

    def call(**kw):
        a = list(ok)
        names = ["q", "k", "v", "y", "S", "z", "gamma", "B", "H", "N", "df", "dv", "dt", "ws", "nbytes", "st"]
        for key, val in kw.items():
            a[names.index(key)] = val
        return pd(*a)

    assert call(gamma=None) == binding.ERR_INVALID_ARG
    assert call(S=None) == binding.ERR_INVALID_ARG            # S without z
    assert call(ws=None) == binding.ERR_INVALID_ARG
    assert call(nbytes=8) == binding.ERR_INVALID_ARG          # smaller than the query (3 tiles x 4 bytes)
    assert call(df=24) == binding.ERR_UNSUPPORTED
    assert call(dt=7) == binding.ERR_INVALID_ARG
    assert lib.based_la_prefill_decay_workspace(2, 3, 300, 32, 128) == 2 * 3 * 3 * 4
    assert lib.based_la_prefill_decay_workspace(1, 1, 0, 32, 128) == 0
    assert lib.based_la_prefill_decay_workspace(1, 1, 64, 24, 128) == 0
    dd = lib.based_la_decode_step_decay
    assert dd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 1, 16, 64, 1, 0, None) == binding.ERR_INVALID_ARG
    assert dd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 24, 64, 1, 0, None) == binding.ERR_UNSUPPORTED


def test_baseconv_entries_reject_bad_arguments(lib):
    pf = lib.based_baseconv_prefill
    names = ["g", "x", "h", "bias", "y", "state", "B", "N", "d", "K", "dt", "st"]
    ok = [FAKE, FAKE, FAKE, None, FAKE, FAKE, 2, 100, 64, 4, 1, None]

    def call(f, okv, nm, **kw):
        a = list(okv)
        for key, val in kw.items():
            a[nm.index(key)] = val
        return f(*a)

    p = lambda **kw: call(pf, ok, names, **kw)
    assert p(g=None) == binding.ERR_INVALID_ARG
    assert p(x=MISALIGNED) == binding.ERR_INVALID_ARG
    assert p(h=None) == binding.ERR_INVALID_ARG
    assert p(h=ctypes.c_void_p((1 << 20) + 4)) == binding.ERR_INVALID_ARG     # taps read 16 bytes at a time
    assert p(bias=ctypes.c_void_p((1 << 20) + 4)) == binding.ERR_INVALID_ARG
    assert p(state=MISALIGNED) == binding.ERR_INVALID_ARG
    assert p(N=0) == binding.ERR_INVALID_ARG
    assert p(K=0) == binding.ERR_INVALID_ARG
    assert p(dt=5) == binding.ERR_INVALID_ARG
    assert p(d=62) == binding.ERR_UNSUPPORTED                               # channels in groups of 4
    assert p(K=9) == binding.ERR_UNSUPPORTED
    dn = ["state", "g", "x", "h", "bias", "y", "B", "d", "K", "dt", "st"]
    dok = [FAKE, FAKE, FAKE, FAKE, None, FAKE, 2, 64, 4, 0, None]
    q = lambda **kw: call(lib.based_baseconv_decode, dok, dn, **kw)
    assert q(state=None) == binding.ERR_INVALID_ARG                         # K > 1 needs a state
    assert q(y=MISALIGNED) == binding.ERR_INVALID_ARG
    assert q(B=0) == binding.ERR_INVALID_ARG
    assert q(d=10) == binding.ERR_UNSUPPORTED
    assert q(K=9) == binding.ERR_UNSUPPORTED
    assert q(K=1, d=10, state=None) == binding.ERR_UNSUPPORTED               # K = 1 needs no state


def test_la_backward_workspace_query(lib):
    # g (bf16) and c (fp32) per token, rows padded to a multiple of 128.
    assert lib.based_la_backward_workspace(2, 3, 300, 16, 64, 1) == 2 * 3 * 384 * (64 * 2 + 4)
    assert lib.based_la_backward_workspace(1, 1, 128, 32, 128, 1) == 128 * (128 * 2 + 4)
    assert lib.based_la_backward_workspace(1, 1, 128, 32, 128, 0) == 0
    assert lib.based_la_backward_workspace(1, 1, 0, 32, 128, 1) == 0
    assert lib.based_la_backward_workspace(1, 1, 8, 24, 128, 1) == 0


def test_workspace_query_rejects_bad_arguments(lib):
    assert lib.based_la_prefill_workspace(0, 1, 1, 16, 64, 1, 0) == 0
    assert lib.based_la_prefill_workspace(1, 1, 1, 8, 64, 1, 0) == 0


def test_python_binding_requires_cuda_tensors():
    import torch
    x = torch.zeros(1, 1, 4, 16)
    with pytest.raises(based.BasedError):
        based.la_prefill(x, x, torch.zeros(1, 1, 4, 64))
    u = torch.zeros(1, 4, 8)
    with pytest.raises(based.BasedError):
        based.baseconv_prefill(u, u, torch.zeros(8, 4))
    with pytest.raises(based.BasedError):
        based.baseconv_decode(torch.zeros(1, 3, 8), u[:, 0], u[:, 0], torch.zeros(8, 4))


def test_noalloc_binding_rejects_wrong_state_shapes():
    """The kernels write exactly [B,H,D,dv] and [B,H,D] floats: a caller's S or z
    of another shape is refused before any tensor reaches the library."""
    import torch
    q = torch.zeros(1, 2, 8, 16)
    v = torch.zeros(1, 2, 8, 64)
    D = 1 + 16 + 16 * 16
    good_S, good_z = torch.zeros(1, 2, D, 64), torch.zeros(1, 2, D)
    for S, z in ((torch.zeros(1, 2, D - 1, 64), good_z), (good_S, torch.zeros(1, 2, D + 1)),
                 (torch.zeros(1, 1, D, 64), good_z), (good_S.double(), good_z)):
        with pytest.raises(based.BasedError) as e:
            based.la_prefill_noalloc(q, q, v, S=S, z=z)
        assert e.value.status == binding.ERR_INVALID_ARG
        assert "S, z must be" in str(e.value) or "contiguous float32" in str(e.value)
