"""Seeded synthetic inputs shared by the tests, the smoke check and bench.py.

This module holds none of the method's arithmetic: it draws N(0, 1) samples
with numpy's PCG64 generator, applies the input scaling of the workloads
(q and k multiplied by d'^(-1/4), so that q.k carries 1/sqrt(d') as in
exp(q.k/sqrt(d'))), rounds to the compute dtype and returns both the device-
ready tensors and float64 copies of the exact rounded values.

Workload shapes (B batch, H heads, N tokens, d' feature dim, dv value dim):
  tiny       B=1,  H=1,  N=256,   d'=16, dv=64,  fp32
  360M       B=8,  H=16, N=2048,  d'=16, dv=64,  bf16
  long       B=2,  H=16, N=16384, d'=16, dv=64,  bf16
  decode     H=16, d'=16, dv=64, batch 1..256, 512-token prompt + 1024 steps
  large      B=4,  H=8,  N=8192,  d'=32, dv=128, bf16
Sliding-window inputs use head dim 64 with q, k drawn like the linear-attention
ones (N(0,1) * 16^(-1/4)) and v ~ N(0, 1).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

_TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass
class Triple:
    """q, k, v as torch CPU tensors of the compute dtype plus exact float64 copies."""

    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    q64: np.ndarray
    k64: np.ndarray
    v64: np.ndarray


def _round(x: np.ndarray, dtype: str):
    t = torch.from_numpy(np.ascontiguousarray(x)).to(_TORCH_DTYPES[dtype])
    return t, t.to(torch.float64).numpy()


def qkv(shape_qk, shape_v, qk_scale: float, dtype: str = "bf16", seed: int = 0) -> Triple:
    """Draw q, k ~ N(0,1)*qk_scale of shape_qk and v ~ N(0,1) of shape_v."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal(shape_qk, dtype=np.float32) * np.float32(qk_scale)
    k = rng.standard_normal(shape_qk, dtype=np.float32) * np.float32(qk_scale)
    v = rng.standard_normal(shape_v, dtype=np.float32)
    tq, q64 = _round(q, dtype)
    tk, k64 = _round(k, dtype)
    tv, v64 = _round(v, dtype)
    return Triple(tq, tk, tv, q64, k64, v64)


def la_inputs(B, H, N, d_feat, d_v, dtype="bf16", seed=0) -> Triple:
    """Linear-attention inputs: q, k [B,H,N,d'] scaled by d'^(-1/4); v [B,H,N,dv]."""
    return qkv((B, H, N, d_feat), (B, H, N, d_v), d_feat ** -0.25, dtype, seed)


def swa_inputs(B, H, N, d, dtype="bf16", seed=0, qk_scale=16 ** -0.25) -> Triple:
    """Sliding-window inputs: q, k, v [B,H,N,d]; q, k scaled like the d'=16 inputs."""
    return qkv((B, H, N, d), (B, H, N, d), qk_scale, dtype, seed)


def device_qkv(shape_qk, shape_v, qk_scale: float, device, seed: int = 0):
    """The same distribution as qkv (q, k ~ N(0,1)*qk_scale, v ~ N(0,1), bf16),
    drawn on the device by a seeded torch generator: for timing-only workloads
    too large to draw on the host in seconds. No float64 copies (not a parity case)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = (torch.randn(shape_qk, generator=g, device=device) * qk_scale).to(torch.bfloat16)
    k = (torch.randn(shape_qk, generator=g, device=device) * qk_scale).to(torch.bfloat16)
    v = torch.randn(shape_v, generator=g, device=device).to(torch.bfloat16)
    return q, k, v


def device_la_inputs(B, H, N, d_feat, d_v, device, seed=0):
    return device_qkv((B, H, N, d_feat), (B, H, N, d_v), d_feat ** -0.25, device, seed)


def device_swa_inputs(B, H, N, d, device, seed=0):
    return device_qkv((B, H, N, d), (B, H, N, d), 16 ** -0.25, device, seed)


WORKLOADS = {
    "tiny": dict(B=1, H=1, N=256, d_feat=16, d_v=64, dtype="f32", swa_heads=1),
    "360M": dict(B=8, H=16, N=2048, d_feat=16, d_v=64, dtype="bf16", swa_heads=16),
    "long": dict(B=2, H=16, N=16384, d_feat=16, d_v=64, dtype="bf16", swa_heads=16),
    "large": dict(B=4, H=8, N=8192, d_feat=32, d_v=128, dtype="bf16", swa_heads=8),
}
SWA_WINDOW = 64
SWA_HEAD_DIM = 64


def upstream_grad(shape, dtype: str = "bf16", seed: int = 0):
    """An upstream gradient dy ~ N(0, 1) of `shape`: (tensor of the dtype, float64 copy)."""
    rng = np.random.default_rng(seed)
    return _round(rng.standard_normal(shape, dtype=np.float32), dtype)


@dataclass
class ConvInputs:
    """Inputs of the short gated convolution: the two projected streams and the filter.

    u_gate, u_conv [B, N, d] torch CPU tensors of the compute dtype (plus float64
    copies of the rounded values); h [d, K] and bias [d] float32 (plus float64 copies).
    """

    u_gate: torch.Tensor
    u_conv: torch.Tensor
    h: torch.Tensor
    bias: torch.Tensor
    gate64: np.ndarray
    conv64: np.ndarray
    h64: np.ndarray
    bias64: np.ndarray


def conv_inputs(B, N, d, taps, dtype="bf16", seed=0) -> ConvInputs:
    """u_gate, u_conv ~ N(0, 1); filter taps ~ N(0, 1/K); bias ~ N(0, 0.1^2)."""
    rng = np.random.default_rng(seed)
    g = rng.standard_normal((B, N, d), dtype=np.float32)
    x = rng.standard_normal((B, N, d), dtype=np.float32)
    h = rng.standard_normal((d, taps), dtype=np.float32) * np.float32(taps ** -0.5)
    b = rng.standard_normal((d,), dtype=np.float32) * np.float32(0.1)
    tg, g64 = _round(g, dtype)
    tx, x64 = _round(x, dtype)
    th, h64 = _round(h, "f32")
    tb, b64 = _round(b, "f32")
    return ConvInputs(tg, tx, th, tb, g64, x64, h64, b64)
