"""GPU parity of the symmetric (packed) state layout against the CPU oracle.

The packed entry points write and update S [B,H,D_s,dv], z [B,H,D_s] with
D_s = 1 + d' + d'(d'+1)/2 rows, one per unordered feature pair. The oracle's
packed feature map and state (oracle.feature_map_packed, la_state_packed,
la_recurrent_packed) are pinned on the CPU against the Taylor closed form and
against the full-layout state. Tolerances are those of the full layout.
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


def _dev(inp):
    return tuple(t.to(DEV) for t in (inp.q, inp.k, inp.v))


# (d', dv, dtype, chunk): every prefill path -- chunked tensor cores (16, 64,
# bf16, 0), CUDA cores (explicit chunks, fp32), quadratic tensor cores (the rest).
PATHS = [(16, 64, "bf16", 0), (16, 64, "bf16", 64), (16, 64, "bf16", 256), (16, 64, "f32", 0), (16, 128, "bf16", 0),
         (32, 64, "bf16", 0), (32, 128, "bf16", 0), (32, 128, "bf16", 128), (32, 128, "f32", 32)]


@pytest.mark.parametrize("d_feat,d_v,dtype,chunk", PATHS)
def test_packed_prefill_state(d_feat, d_v, dtype, chunk):
    inp = synthetic.la_inputs(1, 2, 200, d_feat, d_v, dtype, seed=d_feat + d_v + chunk)
    q, k, v = _dev(inp)
    y_full, _, _ = based.la_prefill(q, k, v, chunk=chunk)
    y, S, z = based.la_prefill(q, k, v, chunk=chunk, packed=True)
    assert based.get_last_error() == 0
    Ds = oracle.packed_dim(d_feat)
    assert tuple(S.shape) == (1, 2, Ds, d_v) and tuple(z.shape) == (1, 2, Ds)
    assert torch.equal(y, y_full)                       # the layout only changes the state write
    assert_y(to64(y), oracle.la_quadratic(inp.q64, inp.k64, inp.v64), DT[dtype])
    ref_S, ref_z = oracle.la_state_packed(inp.k64, inp.v64)
    assert_state(to64(S), ref_S, DT[dtype], "S packed")
    assert_state(to64(z), ref_z, DT[dtype], "z packed")
    assert np.all(to64(z)[..., 0] == 200)


@pytest.mark.parametrize("chunk", [0, 64, 256])
def test_packed_prefill_segmented(chunk):
    """Few long sequences: the chunked tensor-core path splits them into segments."""
    inp = synthetic.la_inputs(1, 2, 3000, 16, 64, "bf16", seed=4)
    q, k, v = _dev(inp)
    _, S, z = based.la_prefill(q, k, v, chunk=chunk, packed=True)
    assert based.get_last_error() == 0
    ref_S, ref_z = oracle.la_state_packed(inp.k64, inp.v64)
    assert_state(to64(S), ref_S, torch.bfloat16, "S packed")
    assert_state(to64(z), ref_z, torch.bfloat16, "z packed")


@pytest.mark.parametrize("d_feat,d_v", [(16, 64), (32, 128)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_packed_decode_continues_prefill(d_feat, d_v, dtype):
    B, H, prompt, steps = 2, 3, 130, 24
    inp = synthetic.la_inputs(B, H, prompt + steps, d_feat, d_v, dtype, seed=7 + d_feat)
    q, k, v = _dev(inp)
    _, S, z = based.la_prefill(q[:, :, :prompt].contiguous(), k[:, :, :prompt].contiguous(),
                               v[:, :, :prompt].contiguous(), packed=True)
    ys = torch.empty((B, H, steps, d_v), dtype=q.dtype, device=DEV)
    for t in range(steps):
        ys[:, :, t] = based.la_decode_step(S, z, q[:, :, prompt + t].contiguous(), k[:, :, prompt + t].contiguous(),
                                           v[:, :, prompt + t].contiguous(), packed=True)
    assert based.get_last_error() == 0
    ref = oracle.la_quadratic(inp.q64, inp.k64, inp.v64)[..., prompt:, :]
    assert_y(to64(ys), ref, DT[dtype], "packed decode y")
    ref_S, ref_z = oracle.la_state_packed(inp.k64, inp.v64)
    assert_state(to64(S), ref_S, DT[dtype], "S packed")
    assert_state(to64(z), ref_z, DT[dtype], "z packed")
    assert np.all(to64(z)[..., 0] == prompt + steps)


@pytest.mark.parametrize("batch", [1, 64, 256])
def test_packed_decode_agrees_with_full_decode(batch):
    """Same step in both layouts from one prompt: outputs within rounding, and the
    packed state equals the full one folded (mirrored rows summed, times 1/sqrt2)."""
    H, d_feat, d_v = 16, 16, 64
    inp = synthetic.la_inputs(batch, H, 65, d_feat, d_v, "bf16", seed=batch)
    q, k, v = _dev(inp)
    p = (q[:, :, :64].contiguous(), k[:, :, :64].contiguous(), v[:, :, :64].contiguous())
    _, Sf, zf = based.la_prefill(*p)
    _, Sp, zp = based.la_prefill(*p, packed=True)
    x = (q[:, :, 64].contiguous(), k[:, :, 64].contiguous(), v[:, :, 64].contiguous())
    yf = based.la_decode_step(Sf, zf, *x)
    yp = based.la_decode_step(Sp, zp, *x, packed=True)
    assert based.get_last_error() == 0
    assert (yf.double() - yp.double()).abs().max().item() <= 2e-2
    Sf64, zf64 = to64(Sf), to64(zf)
    r = np.sqrt(0.5)
    rows, zrows = [Sf64[..., : 1 + d_feat, :]], [zf64[..., : 1 + d_feat]]
    for a, b in oracle.packed_pairs(d_feat):
        fa, fb = 1 + d_feat + a * d_feat + b, 1 + d_feat + b * d_feat + a
        rows.append(Sf64[..., fa:fa + 1, :] if a == b else (Sf64[..., fa:fa + 1, :] + Sf64[..., fb:fb + 1, :]) * r)
        zrows.append(zf64[..., fa:fa + 1] if a == b else (zf64[..., fa:fa + 1] + zf64[..., fb:fb + 1]) * r)
    folded, zfolded = np.concatenate(rows, axis=-2), np.concatenate(zrows, axis=-1)
    assert np.abs(to64(Sp) - folded).max() <= 1e-4 * max(1.0, np.abs(folded).max())
    assert np.abs(to64(zp) - zfolded).max() <= 1e-4 * max(1.0, np.abs(zfolded).max())


def test_packed_shapes_are_checked():
    x = torch.zeros(1, 1, 16, device=DEV, dtype=torch.bfloat16)
    S = torch.zeros(1, 1, 273, 64, device=DEV)
    z = torch.zeros(1, 1, 273, device=DEV)
    with pytest.raises(based.BasedError) as e:
        based.la_decode_step(S, z, x, x, torch.zeros(1, 1, 64, device=DEV, dtype=torch.bfloat16), packed=True)
    assert e.value.status == 1
