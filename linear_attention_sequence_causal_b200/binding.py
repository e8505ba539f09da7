"""Thin ctypes binding over libbased.so (argument marshalling only).

Every function takes CUDA torch tensors, allocates outputs with torch on the
inputs' device, and passes raw device pointers plus the current torch stream to
the C ABI declared in include/based.h. All arithmetic runs in the library's CUDA
kernels; there is no CPU path. If libbased.so is missing or cannot be loaded,
every call raises BasedError.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbased.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = 0, 1, 2, 3, 4
F32, BF16 = 0, 1
_DTYPES = {torch.float32: F32, torch.bfloat16: BF16}

SYMBOLS = (
    "based_la_prefill",
    "based_la_prefill_workspace",
    "based_la_prefill_noalloc",
    "based_la_decode_step",
    "based_la_prefill_packed",
    "based_la_decode_step_packed",
    "based_la_prefill_decay_workspace",
    "based_la_prefill_decay",
    "based_la_decode_step_decay",
    "based_la_backward_workspace",
    "based_la_backward",
    "based_swa_prefill",
    "based_swa_decode",
    "based_baseconv_prefill",
    "based_baseconv_decode",
    "based_get_last_error",
    "based_status_string",
    "based_version",
)


class BasedError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status) if _lib_or_none() else status}")


_LIB = None


def _declare(lib):
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.based_la_prefill.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
    lib.based_la_prefill.restype = i
    lib.based_la_prefill_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
    lib.based_la_prefill_noalloc.restype = i
    lib.based_la_prefill_workspace.argtypes = [i, i, i, i, i, i, i]
    lib.based_la_prefill_workspace.restype = sz
    lib.based_la_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
    lib.based_la_decode_step.restype = i
    lib.based_la_prefill_packed.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
    lib.based_la_prefill_packed.restype = i
    lib.based_la_decode_step_packed.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
    lib.based_la_decode_step_packed.restype = i
    lib.based_la_prefill_decay_workspace.argtypes = [i, i, i, i, i]
    lib.based_la_prefill_decay_workspace.restype = sz
    lib.based_la_prefill_decay.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, sz, vp]
    lib.based_la_prefill_decay.restype = i
    lib.based_la_decode_step_decay.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    lib.based_la_decode_step_decay.restype = i
    lib.based_la_backward_workspace.argtypes = [i, i, i, i, i, i]
    lib.based_la_backward_workspace.restype = sz
    lib.based_la_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, sz, vp]
    lib.based_la_backward.restype = i
    lib.based_swa_prefill.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    lib.based_swa_prefill.restype = i
    lib.based_swa_decode.argtypes = [vp, vp, ctypes.c_int64, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.based_swa_decode.restype = i
    lib.based_baseconv_prefill.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
    lib.based_baseconv_prefill.restype = i
    lib.based_baseconv_decode.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, vp]
    lib.based_baseconv_decode.restype = i
    lib.based_get_last_error.argtypes = [vp]
    lib.based_get_last_error.restype = i
    lib.based_status_string.argtypes = [i]
    lib.based_status_string.restype = ctypes.c_char_p
    lib.based_version.argtypes = []
    lib.based_version.restype = i
    return lib


def _lib_or_none():
    global _LIB
    if _LIB is None and os.path.exists(_LIB_PATH):
        try:
            _LIB = _declare(ctypes.CDLL(_LIB_PATH))
        except OSError:
            _LIB = None
    return _LIB


def lib():
    """The loaded libbased.so (ctypes.CDLL); raises BasedError when it is missing."""
    L = _lib_or_none()
    if L is None:
        raise BasedError(ERR_CUDA, f"libbased.so not loadable at {_LIB_PATH}; build it with "
                                   "python -m linear_attention_sequence_causal_b200.build")
    return L


def library_path() -> str:
    return _LIB_PATH


def status_string(status: int) -> str:
    return lib().based_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != OK:
        raise BasedError(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(*ts: torch.Tensor) -> int:
    dt = ts[0].dtype
    for t in ts:
        if not t.is_cuda:
            raise BasedError(ERR_INVALID_ARG, "tensors must be on a CUDA device")
        if t.dtype != dt:
            raise BasedError(ERR_INVALID_ARG, "q, k, v must share one dtype")
        if not t.is_contiguous():
            raise BasedError(ERR_INVALID_ARG, "tensors must be contiguous")
    if dt not in _DTYPES:
        raise BasedError(ERR_UNSUPPORTED, f"dtype {dt} (float32 or bfloat16 only)")
    return _DTYPES[dt]


def feature_dim(d_feat: int) -> int:
    return 1 + d_feat + d_feat * d_feat


def packed_dim(d_feat: int) -> int:
    """Rows of the symmetric (packed) state: 1 + d' + d'(d'+1)/2."""
    return 1 + d_feat + d_feat * (d_feat + 1) // 2


def _check_state_shape(S, z, B, H, D, d_v):
    """S [B,H,D,dv] and z [B,H,D] float32, contiguous (either may be None: not given):
    the kernels write exactly that much."""
    for name, t, shape in (("S", S, (B, H, D, d_v)), ("z", z, (B, H, D))):
        if t is None:
            continue
        if tuple(t.shape) != shape:
            raise BasedError(ERR_INVALID_ARG, f"S, z must be [{B},{H},{D},{d_v}] and [{B},{H},{D}]")
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise BasedError(ERR_INVALID_ARG, f"{name} must be contiguous float32")


def la_prefill_workspace(B, H, N, d_feat, d_v, dtype=torch.bfloat16, chunk=0) -> int:
    return int(lib().based_la_prefill_workspace(B, H, N, d_feat, d_v, _DTYPES[dtype], chunk))


def la_prefill(q, k, v, chunk: int = 0, want_state: bool = True, y=None, S=None, z=None,
               workspace=None, packed: bool = False) -> Tuple[torch.Tensor, Optional[torch.Tensor], Optional[torch.Tensor]]:
    """Causal Taylor linear attention over [B,H,N,*] inputs; returns (y, S, z).

    S [B,H,D,dv] and z [B,H,D] (float32) hold the final state when want_state;
    D = 1 + d' + d'^2, or 1 + d' + d'(d'+1)/2 with packed (symmetric layout).
    """
    dt = _dtype_code(q, k, v)
    B, H, N, d_feat = q.shape
    d_v = v.shape[-1]
    D = packed_dim(d_feat) if packed else feature_dim(d_feat)
    dev = q.device
    with torch.cuda.device(dev):
        if y is None:
            y = torch.empty((B, H, N, d_v), dtype=q.dtype, device=dev)
        if want_state:
            S = torch.empty((B, H, D, d_v), dtype=torch.float32, device=dev) if S is None else S
            z = torch.empty((B, H, D), dtype=torch.float32, device=dev) if z is None else z
        else:
            S = z = None
        _check_state_shape(S, z, B, H, D, d_v)
        ws_bytes = int(lib().based_la_prefill_workspace(B, H, N, d_feat, d_v, dt, chunk))
        if ws_bytes and (workspace is None or workspace.numel() < ws_bytes):
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        fn = lib().based_la_prefill_packed if packed else lib().based_la_prefill
        st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(S), _ptr(z), B, H, N, d_feat, d_v, dt, chunk,
                _ptr(workspace) if ws_bytes else None, ws_bytes, _stream(dev))
    _check(st, "based_la_prefill_packed" if packed else "based_la_prefill")
    return y, S, z


def la_prefill_noalloc(q, k, v, chunk: int = 0, want_state: bool = True, y=None, S=None, z=None):
    """la_prefill without a workspace: the library's fixed device scratch is used
    instead (for callers that must not allocate; calls must not overlap on the GPU)."""
    B, H, N, d_feat = q.shape
    d_v = v.shape[-1]
    D = feature_dim(d_feat)
    if want_state:
        _check_state_shape(S, z, B, H, D, d_v)     # caller-supplied S, z (None: allocated below)
    dt = _dtype_code(q, k, v)
    dev = q.device
    with torch.cuda.device(dev):
        if y is None:
            y = torch.empty((B, H, N, d_v), dtype=q.dtype, device=dev)
        if want_state:
            S = torch.empty((B, H, D, d_v), dtype=torch.float32, device=dev) if S is None else S
            z = torch.empty((B, H, D), dtype=torch.float32, device=dev) if z is None else z
        else:
            S = z = None
        st = lib().based_la_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(S), _ptr(z),
                                            B, H, N, d_feat, d_v, dt, chunk, _stream(dev))
    _check(st, "based_la_prefill_noalloc")
    return y, S, z


DECAY_TILE = 128


def la_prefill_decay(q, k, v, gamma, want_state: bool = True, y=None, S=None, z=None, workspace=None):
    """Causal Taylor linear attention with coarse decay: gamma [B,H,ceil(N/128)] float32,
    one value per 128-token tile (bf16 q, k, v). Returns (y, S, z)."""
    dt = _dtype_code(q, k, v)
    B, H, N, d_feat = q.shape
    d_v = v.shape[-1]
    D = feature_dim(d_feat)
    nt = (N + DECAY_TILE - 1) // DECAY_TILE
    if tuple(gamma.shape) != (B, H, nt) or gamma.dtype != torch.float32 or not gamma.is_contiguous() \
            or gamma.device != q.device:
        raise BasedError(ERR_INVALID_ARG, f"gamma must be a contiguous float32 [{B},{H},{nt}] on q's device")
    dev = q.device
    with torch.cuda.device(dev):
        if y is None:
            y = torch.empty((B, H, N, d_v), dtype=q.dtype, device=dev)
        if want_state:
            S = torch.empty((B, H, D, d_v), dtype=torch.float32, device=dev) if S is None else S
            z = torch.empty((B, H, D), dtype=torch.float32, device=dev) if z is None else z
        else:
            S = z = None
        ws_bytes = int(lib().based_la_prefill_decay_workspace(B, H, N, d_feat, d_v))
        if workspace is None or workspace.numel() < ws_bytes:
            workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        st = lib().based_la_prefill_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(S), _ptr(z), _ptr(gamma),
                                          B, H, N, d_feat, d_v, dt, _ptr(workspace), workspace.numel(),
                                          _stream(dev))
    _check(st, "based_la_prefill_decay")
    return y, S, z


def la_decode_step_decay(S, z, q, k, v, gamma, y=None, packed: bool = False) -> torch.Tensor:
    """One recurrent step after scaling the state by gamma [B,H] float32 (S, z in place)."""
    dt = _dtype_code(q, k, v)
    B, H, d_feat = q.shape
    d_v = v.shape[-1]
    if tuple(gamma.shape) != (B, H) or gamma.dtype != torch.float32 or not gamma.is_contiguous():
        raise BasedError(ERR_INVALID_ARG, f"gamma must be a contiguous float32 [{B},{H}]")
    dev = q.device
    with torch.cuda.device(dev):
        if y is None:
            y = torch.empty((B, H, d_v), dtype=q.dtype, device=dev)
        st = lib().based_la_decode_step_decay(_ptr(S), _ptr(z), _ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(gamma),
                                              B, H, d_feat, d_v, dt, 1 if packed else 0, _stream(dev))
    _check(st, "based_la_decode_step_decay")
    return y


def la_backward_workspace(B, H, N, d_feat, d_v, dtype=torch.bfloat16) -> int:
    return int(lib().based_la_backward_workspace(B, H, N, d_feat, d_v, _DTYPES[dtype]))


def la_backward(q, k, v, y, dy, dq=None, dk=None, dv=None, workspace=None):
    """Gradients (dq, dk, dv) of the causal Taylor linear attention for the
    upstream gradient dy; y is the forward output for q, k, v. bf16 [B,H,N,*]."""
    dt = _dtype_code(q, k, v, y, dy)
    B, H, N, d_feat = q.shape
    d_v = v.shape[-1]
    if tuple(k.shape) != (B, H, N, d_feat) or tuple(v.shape[:3]) != (B, H, N) or \
            tuple(y.shape) != (B, H, N, d_v) or tuple(dy.shape) != (B, H, N, d_v):
        raise BasedError(ERR_INVALID_ARG, "q, k [B,H,N,d'] and v, y, dy [B,H,N,dv] expected")
    dev = q.device
    with torch.cuda.device(dev):
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        for name, t, ref in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
            if t.shape != ref.shape or t.dtype != ref.dtype or not t.is_contiguous() or t.device != dev:
                raise BasedError(ERR_INVALID_ARG, f"{name} must match its input's shape, dtype and device")
        ws_bytes = int(lib().based_la_backward_workspace(B, H, N, d_feat, d_v, dt))
        if ws_bytes and (workspace is None or workspace.numel() < ws_bytes):
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        st = lib().based_la_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv),
                                     B, H, N, d_feat, d_v, dt, _ptr(workspace) if ws_bytes else None,
                                     ws_bytes, _stream(dev))
    _check(st, "based_la_backward")
    return dq, dk, dv


def la_decode_step(S, z, q, k, v, y=None, packed: bool = False) -> torch.Tensor:
    """One recurrent step, S and z updated in place; q, k [B,H,d'], v [B,H,dv].

    packed: S, z are in the symmetric layout (1 + d' + d'(d'+1)/2 rows)."""
    dt = _dtype_code(q, k, v)
    B, H, d_feat = q.shape
    d_v = v.shape[-1]
    D = packed_dim(d_feat) if packed else feature_dim(d_feat)
    if tuple(S.shape) != (B, H, D, d_v) or tuple(z.shape) != (B, H, D):
        raise BasedError(ERR_INVALID_ARG, f"S, z must be [{B},{H},{D},{d_v}] and [{B},{H},{D}]")
    if S.dtype != torch.float32 or z.dtype != torch.float32 or not (S.is_contiguous() and z.is_contiguous()):
        raise BasedError(ERR_INVALID_ARG, "S and z must be contiguous float32")
    dev = q.device
    with torch.cuda.device(dev):
        if y is None:
            y = torch.empty((B, H, d_v), dtype=q.dtype, device=dev)
        fn = lib().based_la_decode_step_packed if packed else lib().based_la_decode_step
        st = fn(_ptr(S), _ptr(z), _ptr(q), _ptr(k), _ptr(v), _ptr(y), B, H, d_feat, d_v, dt, _stream(dev))
    _check(st, "based_la_decode_step_packed" if packed else "based_la_decode_step")
    return y


def swa_prefill(q, k, v, w: int = 64, scale: Optional[float] = None, want_cache: bool = True,
                y=None, k_cache=None, v_cache=None):
    """Sliding-window softmax attention over [B,H,N,d]; returns (y, k_cache, v_cache)."""
    dt = _dtype_code(q, k, v)
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dev = q.device
    with torch.cuda.device(dev):
        if y is None:
            y = torch.empty_like(q)
        if want_cache:
            k_cache = torch.empty((B, H, w, d), dtype=q.dtype, device=dev) if k_cache is None else k_cache
            v_cache = torch.empty((B, H, w, d), dtype=q.dtype, device=dev) if v_cache is None else v_cache
        else:
            k_cache = v_cache = None
        st = lib().based_swa_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(k_cache), _ptr(v_cache),
                                     B, H, N, d, w, scale, dt, _stream(dev))
    _check(st, "based_swa_prefill")
    return y, k_cache, v_cache


def swa_decode(k_cache, v_cache, t: int, q, k, v, w: int = 64, scale: Optional[float] = None,
               y=None) -> torch.Tensor:
    """One step over the ring cache (updated in place); q, k, v [B,H,d]."""
    dt = _dtype_code(q, k, v)
    B, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dev = q.device
    with torch.cuda.device(dev):
        if y is None:
            y = torch.empty_like(q)
        st = lib().based_swa_decode(_ptr(k_cache), _ptr(v_cache), int(t), _ptr(q), _ptr(k), _ptr(v),
                                    _ptr(y), B, H, d, w, scale, dt, _stream(dev))
    _check(st, "based_swa_decode")
    return y


def _conv_filter(h, bias, d: int):
    if h.dtype != torch.float32 or not h.is_cuda or not h.is_contiguous() or h.dim() != 2 or h.shape[0] != d:
        raise BasedError(ERR_INVALID_ARG, "h must be a contiguous CUDA float32 tensor [d, K]")
    if bias is not None and (bias.dtype != torch.float32 or not bias.is_cuda or not bias.is_contiguous()
                             or tuple(bias.shape) != (d,)):
        raise BasedError(ERR_INVALID_ARG, "bias must be a contiguous CUDA float32 tensor [d]")
    return int(h.shape[1])


def baseconv_prefill(u_gate, u_conv, h, bias=None, state=True, y=None):
    """Short gated convolution over [B, N, d] streams: y = u_gate * SiLU(bias + causal h * u_conv).

    h [d, K] float32 (tap K-1 meets the current token); bias [d] float32 or None.
    Returns (y, state): state [B, K-1, d] holds u_conv of the last K-1 tokens
    (zeros before token 0); `state` may be False (not written) or a tensor to write.
    """
    dt = _dtype_code(u_gate, u_conv)
    B, N, d = u_gate.shape
    if tuple(u_conv.shape) != (B, N, d):
        raise BasedError(ERR_INVALID_ARG, "u_gate and u_conv must have one shape [B, N, d]")
    K = _conv_filter(h, bias, d)
    dev = u_gate.device
    with torch.cuda.device(dev):
        if y is None:
            y = torch.empty_like(u_gate)
        if isinstance(state, torch.Tensor):
            _dtype_code(state, u_gate)
            if tuple(state.shape) != (B, max(K - 1, 0), d):
                raise BasedError(ERR_INVALID_ARG, "state must be [B, K-1, d]")
            st_t = state
        else:
            st_t = torch.empty((B, max(K - 1, 0), d), dtype=u_gate.dtype, device=dev) if state else None
        st = lib().based_baseconv_prefill(_ptr(u_gate), _ptr(u_conv), _ptr(h), _ptr(bias), _ptr(y),
                                          _ptr(st_t) if (st_t is not None and K > 1) else None,
                                          B, N, d, K, dt, _stream(dev))
    _check(st, "based_baseconv_prefill")
    return y, st_t


def baseconv_decode(state, u_gate, u_conv, h, bias=None, y=None) -> torch.Tensor:
    """One token per sequence through the filter; state [B, K-1, d] is updated in place."""
    dt = _dtype_code(u_gate, u_conv)
    B, d = u_gate.shape
    K = _conv_filter(h, bias, d)
    if K > 1:
        if state is None:
            raise BasedError(ERR_INVALID_ARG, "a filter of K > 1 taps needs its state [B, K-1, d]")
        _dtype_code(state, u_gate)
        if tuple(state.shape) != (B, K - 1, d):
            raise BasedError(ERR_INVALID_ARG, "state must be [B, K-1, d]")
    dev = u_gate.device
    with torch.cuda.device(dev):
        if y is None:
            y = torch.empty_like(u_gate)
        st = lib().based_baseconv_decode(_ptr(state) if K > 1 else None, _ptr(u_gate), _ptr(u_conv), _ptr(h),
                                         _ptr(bias), _ptr(y), B, d, K, dt, _stream(dev))
    _check(st, "based_baseconv_decode")
    return y


def get_last_error(device=None) -> int:
    """Synchronise the current stream and return the device status (0 = OK)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(lib().based_get_last_error(_stream(dev)))
