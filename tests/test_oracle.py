"""Pins for the CPU oracle (CPU only, no GPU).

The oracle is checked against things other than itself: hand-derived golden
values, a mathematical identity of the feature map, a library softmax-attention
routine (torch scaled_dot_product_attention in float64), textbook special cases,
the O(eps^3) convergence of the Taylor weights to exp, equivalence of
independently written formulations, and pure-Python brute force on N <= 8.
The mutation tests at the end plant plausible mistakes in copies of the oracle
and check that at least one pin rejects each of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute

RNG = np.random.default_rng(1234)


def _qkv(B, H, N, d, dv, scale=None, seed=0):
    rng = np.random.default_rng(seed)
    s = d ** -0.25 if scale is None else scale
    q = rng.standard_normal((B, H, N, d)) * s
    k = rng.standard_normal((B, H, N, d)) * s
    v = rng.standard_normal((B, H, N, dv))
    return q, k, v


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- feature map

@pytest.mark.parametrize("d", [1, 2, 3, 16, 32])
def test_phi_product_is_taylor_polynomial(d):
    # phi(q).phi(k) must equal 1 + s + s^2/2 with s = q.k for every q, k.
    q = RNG.standard_normal((50, d))
    k = RNG.standard_normal((50, d))
    lhs = np.einsum("nf,nf->n", oracle.feature_map(q), oracle.feature_map(k))
    s = np.einsum("nd,nd->n", q, k)
    np.testing.assert_allclose(lhs, 1 + s + s * s / 2, rtol=1e-12, atol=1e-12)


def test_phi_width():
    assert oracle.feature_dim(16) == 273 and oracle.feature_dim(32) == 1057
    assert oracle.feature_map(np.zeros((4, 16))).shape == (4, 273)


def test_phi_golden_order(golden_dir):
    g = _golden(golden_dir, "phi_d2.json")
    np.testing.assert_allclose(oracle.feature_map(np.array(g["x"])), g["phi"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(brute.phi(g["x"]), g["phi"], rtol=0, atol=1e-15)


def test_taylor_weight_minimum():
    # 1 + s + s^2/2 = ((s+1)^2 + 1)/2 has its minimum 1/2 at s = -1.
    s = np.linspace(-5, 5, 100001)
    w = 1 + s + s * s / 2
    assert abs(w.min() - 0.5) < 1e-9 and abs(s[w.argmin()] + 1) < 1e-4


# ---------------------------------------------------------------- linear attention

def test_la_hand_example(golden_dir):
    g = _golden(golden_dir, "la_hand_d1.json")
    q = np.array(g["q"])[None, None, :, None]
    k = np.array(g["k"])[None, None, :, None]
    v = np.array(g["v"])[None, None, :, None]
    np.testing.assert_allclose(oracle.la_quadratic(q, k, v)[0, 0, :, 0], g["y"], rtol=1e-14)
    y, S, z = oracle.la_recurrent(q, k, v)
    np.testing.assert_allclose(y[0, 0, :, 0], g["y"], rtol=1e-14)
    S2, z2 = oracle.la_state(k, v)
    np.testing.assert_allclose(S2[0, 0, :, 0], g["S"], rtol=1e-14)
    np.testing.assert_allclose(z2[0, 0], g["z"], rtol=1e-14)
    np.testing.assert_allclose(S[0, 0, :, 0], g["S"], rtol=1e-14)


@pytest.mark.parametrize("d,dv,N", [(1, 1, 5), (2, 3, 7), (3, 2, 8)])
def test_la_brute_force(d, dv, N):
    q, k, v = _qkv(1, 1, N, d, dv, scale=0.8, seed=d * 10 + N)
    yb, Sb, zb = brute.la(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist())
    np.testing.assert_allclose(oracle.la_quadratic(q, k, v)[0, 0], yb, rtol=1e-12, atol=1e-13)
    S, z = oracle.la_state(k, v)
    np.testing.assert_allclose(S[0, 0], Sb, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(z[0, 0], zb, rtol=1e-12, atol=1e-13)


def test_la_quadratic_equals_recurrent():
    q, k, v = _qkv(2, 3, 97, 16, 8, seed=1)
    yq = oracle.la_quadratic(q, k, v, row_block=32)
    yr, Sr, zr = oracle.la_recurrent(q, k, v)
    np.testing.assert_allclose(yq, yr, rtol=1e-10, atol=1e-12)
    S, z = oracle.la_state(k, v)
    np.testing.assert_allclose(S, Sr, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(z, zr, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("chunk", [1, 5, 16, 64, 200])
def test_la_chunked_equals_quadratic(chunk):
    q, k, v = _qkv(1, 2, 131, 16, 16, seed=2)
    y, S, z = oracle.la_chunked(q, k, v, chunk)
    np.testing.assert_allclose(y, oracle.la_quadratic(q, k, v), rtol=1e-10, atol=1e-12)
    S2, z2 = oracle.la_state(k, v)
    np.testing.assert_allclose(S, S2, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(z, z2, rtol=1e-10, atol=1e-10)


def test_la_taylor_terms_compose():
    q, k, v = _qkv(1, 1, 40, 4, 3, seed=3)
    (t0, t1, t2), (d0, d1, d2) = oracle.la_taylor_terms(q, k, v)
    y = (t0 + t1 + t2) / (d0 + d1 + d2)[..., None]
    np.testing.assert_allclose(y, oracle.la_quadratic(q, k, v), rtol=1e-12, atol=1e-13)
    # order 0 alone is the cumulative sum of v, order-0 denominator the count
    np.testing.assert_allclose(t0, np.cumsum(v, axis=-2), rtol=1e-12)
    np.testing.assert_allclose(d0[0, 0], np.arange(1, 41))


def test_la_decode_continues_prefill():
    q, k, v = _qkv(1, 2, 60, 16, 8, seed=4)
    n0 = 45
    S0, z0 = oracle.la_state(k[..., :n0, :], v[..., :n0, :])
    y, S, z = oracle.la_recurrent(q[..., n0:, :], k[..., n0:, :], v[..., n0:, :], S0, z0)
    np.testing.assert_allclose(y, oracle.la_quadratic(q, k, v)[..., n0:, :], rtol=1e-10, atol=1e-12)
    S2, z2 = oracle.la_state(k, v)
    np.testing.assert_allclose(S, S2, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(z, z2, rtol=1e-10)


def test_la_rows_matches_quadratic():
    q, k, v = _qkv(1, 1, 300, 16, 8, seed=5)
    rows = [0, 1, 63, 64, 127, 128, 299]
    np.testing.assert_allclose(oracle.la_rows(q[0, 0], k[0, 0], v[0, 0], rows),
                               oracle.la_quadratic(q, k, v)[0, 0, rows], rtol=1e-12, atol=1e-13)


def test_la_zero_query_is_cumulative_mean():
    # q = 0 makes every weight 1: y_i = mean(v_0..v_i).
    _, k, v = _qkv(1, 2, 50, 16, 5, seed=6)
    q = np.zeros_like(k)
    mean = np.cumsum(v, axis=-2) / np.arange(1, 51)[:, None]
    np.testing.assert_allclose(oracle.la_quadratic(q, k, v), mean, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(oracle.la_recurrent(q, k, v)[0], mean, rtol=1e-12, atol=1e-13)


def test_la_single_token_is_identity():
    q, k, v = _qkv(3, 2, 1, 16, 7, seed=7)
    np.testing.assert_allclose(oracle.la_quadratic(q, k, v), v, rtol=1e-14)


def test_la_denominator_bound_attained():
    # s = q.k = -1 for every pair gives weight 1/2: den_i = (i+1)/2 exactly.
    n = 20
    q = np.zeros((1, 1, n, 3)); q[..., 0] = 1.0
    k = np.zeros((1, 1, n, 3)); k[..., 0] = -1.0
    v = RNG.standard_normal((1, 1, n, 2))
    _, den = oracle.la_quadratic_parts(q, k, v)
    np.testing.assert_allclose(den[0, 0], 0.5 * np.arange(1, n + 1), rtol=1e-15)


def test_la_denominator_bound_random():
    q, k, v = _qkv(2, 2, 200, 16, 4, scale=1.5, seed=8)
    _, den = oracle.la_quadratic_parts(q, k, v)
    assert np.all(den >= 0.5 * np.arange(1, 201))


def _softmax_causal_torch(q, k, v):
    # library routine: causal softmax attention with unit scale
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), is_causal=True, scale=1.0).numpy()


def _taylor_error_ratio(la_fn):
    q, k, v = _qkv(1, 2, 64, 16, 8, seed=9)
    errs = []
    for eps in (0.2, 0.1, 0.05):
        y = la_fn(eps * q, k, v)
        errs.append(np.abs(y - _softmax_causal_torch(eps * q, k, v)).max())
    return errs[0] / errs[1], errs[1] / errs[2]


def test_la_converges_to_softmax_at_third_order():
    # 1 + s + s^2/2 = exp(s) - s^3/6 + ...: the gap to softmax attention is O(eps^3).
    r1, r2 = _taylor_error_ratio(oracle.la_quadratic)
    assert 6.5 < r1 < 9.5 and 7.0 < r2 < 9.0, (r1, r2)


# ---------------------------------------------------------------- packed (symmetric) state

def test_packed_width_and_pair_order():
    assert oracle.packed_dim(16) == 153 and oracle.packed_dim(32) == 561
    assert oracle.packed_pairs(3) == [(0, 0), (0, 1), (0, 2), (1, 1), (1, 2), (2, 2)]
    assert len(oracle.packed_pairs(32)) == 32 * 33 // 2


def test_packed_feature_map_hand_example():
    # d' = 2, x = (3, -2): [1, x0, x1, x0^2/sqrt2, x0 x1, x1^2/sqrt2], written out by hand.
    r = math.sqrt(0.5)
    want = [1.0, 3.0, -2.0, 9.0 * r, -6.0, 4.0 * r]
    got = oracle.feature_map_packed(np.array([3.0, -2.0]))
    assert np.allclose(got, want, rtol=0, atol=1e-15)


@pytest.mark.parametrize("d", [1, 2, 16, 32])
def test_packed_product_is_taylor_polynomial(d):
    q = RNG.standard_normal((40, d))
    k = RNG.standard_normal((40, d))
    s = np.sum(q * k, axis=-1)
    got = np.sum(oracle.feature_map_packed(q) * oracle.feature_map_packed(k), axis=-1)
    assert np.allclose(got, 1.0 + s + 0.5 * s * s, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("d,dv", [(16, 64), (32, 8)])
def test_packed_state_folds_the_full_state(d, dv):
    # Independent constructions: the full state from phi, the packed one from
    # phi_s. Entry (a, b), a < b, of the packed state is the two mirrored full
    # entries (each x_a x_b / sqrt2) added and scaled by 1/sqrt2.
    _, k, v = _qkv(1, 2, 37, d, dv, seed=5)
    S, z = oracle.la_state(k, v)
    Ss, zs = oracle.la_state_packed(k, v)
    assert np.allclose(Ss[..., : 1 + d, :], S[..., : 1 + d, :], rtol=1e-12, atol=1e-12)
    assert np.allclose(zs[..., : 1 + d], z[..., : 1 + d], rtol=1e-12, atol=1e-12)
    r = math.sqrt(0.5)
    for idx, (a, b) in enumerate(oracle.packed_pairs(d)):
        f_ab, f_ba = 1 + d + a * d + b, 1 + d + b * d + a
        want_S = S[..., f_ab, :] if a == b else (S[..., f_ab, :] + S[..., f_ba, :]) * r
        want_z = z[..., f_ab] if a == b else (z[..., f_ab] + z[..., f_ba]) * r
        assert np.allclose(Ss[..., 1 + d + idx, :], want_S, rtol=1e-12, atol=1e-12)
        assert np.allclose(zs[..., 1 + d + idx], want_z, rtol=1e-12, atol=1e-12)


def test_packed_recurrent_matches_quadratic_form():
    q, k, v = _qkv(2, 2, 50, 16, 8, seed=9)
    y, Ss, zs = oracle.la_recurrent_packed(q, k, v)
    assert np.allclose(y, oracle.la_quadratic(q, k, v), rtol=1e-10, atol=1e-12)
    Ss_ref, zs_ref = oracle.la_state_packed(k, v)
    assert np.allclose(Ss, Ss_ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(zs, zs_ref, rtol=1e-12, atol=1e-12)
    assert np.all(zs[..., 0] == 50.0)


def test_packed_decode_continues_packed_prefill():
    q, k, v = _qkv(1, 3, 40, 32, 4, seed=11)
    S0, z0 = oracle.la_state_packed(k[..., :25, :], v[..., :25, :])
    y, _, _ = oracle.la_recurrent_packed(q[..., 25:, :], k[..., 25:, :], v[..., 25:, :], S0, z0)
    assert np.allclose(y, oracle.la_quadratic(q, k, v)[..., 25:, :], rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- sliding window

def test_swa_hand_example(golden_dir):
    g = _golden(golden_dir, "swa_hand_w2.json")
    a = lambda key: np.array(g[key])[None, None, :, None]
    y = oracle.swa(a("q"), a("k"), a("v"), g["w"], g["scale"])
    np.testing.assert_allclose(y[0, 0, :, 0], g["y"], rtol=1e-14)


@pytest.mark.parametrize("w", [1, 2, 3, 8])
def test_swa_brute_force(w):
    q, k, v = _qkv(1, 1, 8, 4, 3, scale=1.0, seed=10 + w)
    yb = brute.swa(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), w, 0.7)
    np.testing.assert_allclose(oracle.swa(q, k, v, w, 0.7)[0, 0], yb, rtol=1e-12, atol=1e-13)


def test_swa_full_window_is_causal_softmax_library():
    q, k, v = _qkv(2, 2, 50, 64, 64, scale=0.6, seed=11)
    scale = 1 / 8
    ref = _softmax_causal_torch(q * scale, k, v)
    np.testing.assert_allclose(oracle.swa(q, k, v, 64, scale, row_block=16), ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(oracle.swa(q, k, v, 50, scale), ref, rtol=1e-12, atol=1e-13)


def test_swa_window_one_is_identity():
    q, k, v = _qkv(1, 3, 30, 8, 8, seed=12)
    np.testing.assert_allclose(oracle.swa(q, k, v, 1, 0.3), v, rtol=1e-14)


def test_swa_rows_before_window_are_causal_prefix():
    q, k, v = _qkv(1, 1, 200, 64, 64, scale=0.6, seed=13)
    y = oracle.swa(q, k, v, 64, 0.125, row_block=37)
    ref = _softmax_causal_torch(q[..., :64, :] * 0.125, k[..., :64, :], v[..., :64, :])
    np.testing.assert_allclose(y[..., :64, :], ref, rtol=1e-12, atol=1e-13)
    # row 150 sees exactly keys 87..150: one query, 64 keys, no mask
    i = 150
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    ref_i = torch.nn.functional.scaled_dot_product_attention(
        t(q[..., i:i + 1, :]), t(k[..., i - 63:i + 1, :]), t(v[..., i - 63:i + 1, :]),
        scale=0.125).numpy()
    np.testing.assert_allclose(y[..., i:i + 1, :], ref_i, rtol=1e-12, atol=1e-13)
    rows = [0, 5, 63, 64, 65, 150, 199]
    np.testing.assert_allclose(oracle.swa_rows(q[0, 0], k[0, 0], v[0, 0], 64, 0.125, rows),
                               y[0, 0, rows], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("n0", [0, 1, 30, 64, 100])
def test_swa_ring_decode_continues_prefill(n0):
    w, scale = 16, 0.25
    q, k, v = _qkv(2, 2, n0 + 40, 8, 8, scale=0.7, seed=14 + n0)
    full = oracle.swa(q, k, v, w, scale)
    kc, vc = oracle.swa_ring_after_prefill(k[..., :n0, :], v[..., :n0, :], w)
    for t in range(n0, n0 + 40):
        y, kc, vc = oracle.swa_decode_step(kc, vc, t, q[..., t, :], k[..., t, :], v[..., t, :], w, scale)
        np.testing.assert_allclose(y, full[..., t, :], rtol=1e-12, atol=1e-13)


def test_swa_ring_contents():
    k = np.arange(10, dtype=np.float64).reshape(1, 1, 10, 1)
    kc, _ = oracle.swa_ring_after_prefill(k, k, 4)
    # tokens 6..9 at slots 6%4=2, 7%4=3, 8%4=0, 9%4=1
    np.testing.assert_array_equal(kc[0, 0, :, 0], [8, 9, 6, 7])
    kc, _ = oracle.swa_ring_after_prefill(k[..., :2, :], k[..., :2, :], 4)
    np.testing.assert_array_equal(kc[0, 0, :, 0], [0, 1, 0, 0])


# ---------------------------------------------------------------- planted mistakes

def _mut_phi_no_sqrt(x):
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    outer = (x[..., :, None] * x[..., None, :]).reshape(*x.shape[:-1], d * d)
    return np.concatenate([np.ones(x.shape[:-1] + (1,)), x, outer], axis=-1)


def _mut_la(coef1=1.0, coef2=0.5, strict=False):
    def la(q, k, v):
        s = q @ np.swapaxes(k, -1, -2)
        a = 1.0 + coef1 * s + coef2 * s * s
        n = s.shape[-1]
        m = np.tril(np.ones((n, n), dtype=bool), k=-1 if strict else 0)
        a = np.where(m, a, 0.0)
        den = a.sum(-1)
        den = np.where(den == 0, 1.0, den)
        return (a @ v) / den[..., None]
    return la


def test_mutant_phi_without_sqrt_half_is_caught(golden_dir):
    q = RNG.standard_normal((10, 16))
    k = RNG.standard_normal((10, 16))
    lhs = np.einsum("nf,nf->n", _mut_phi_no_sqrt(q), _mut_phi_no_sqrt(k))
    s = np.einsum("nd,nd->n", q, k)
    assert not np.allclose(lhs, 1 + s + s * s / 2)
    g = _golden(golden_dir, "phi_d2.json")
    assert not np.allclose(_mut_phi_no_sqrt(np.array(g["x"])), g["phi"])


@pytest.mark.parametrize("mutant", [
    _mut_la(coef2=1.0),          # wrong second-order coefficient
    _mut_la(coef1=-1.0),         # wrong sign of the first-order term
])
def test_mutant_coefficients_caught_by_convergence(mutant):
    r1, r2 = _taylor_error_ratio(mutant)
    assert not (6.5 < r1 < 9.5 and 7.0 < r2 < 9.0)


def test_mutant_exclusive_mask_caught(golden_dir):
    g = _golden(golden_dir, "la_hand_d1.json")
    a = lambda key: np.array(g[key])[None, None, :, None]
    y = _mut_la(strict=True)(a("q"), a("k"), a("v"))
    assert not np.allclose(y[0, 0, :, 0], g["y"])
    np.testing.assert_allclose(_mut_la()(a("q"), a("k"), a("v"))[0, 0, :, 0], g["y"], rtol=1e-14)


def test_mutant_window_off_by_one_caught(golden_dir):
    g = _golden(golden_dir, "swa_hand_w2.json")
    a = lambda key: np.array(g[key])[None, None, :, None]
    # a window of w+1 keys (reading "preceding w keys" as excluding self)
    y = oracle.swa(a("q"), a("k"), a("v"), g["w"] + 1, g["scale"])
    assert not np.allclose(y[0, 0, :, 0], g["y"])


def _mut_phi_packed(x, diag_scale, off_scale):
    """A copy of the packed feature map with the pair coefficients replaced."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    cols = [x[..., a] * x[..., b] * (diag_scale if a == b else off_scale) for a, b in oracle.packed_pairs(d)]
    return np.concatenate([np.ones(x.shape[:-1] + (1,)), x, np.stack(cols, axis=-1)], axis=-1)


@pytest.mark.parametrize("diag_scale,off_scale", [
    (1.0, 1.0),                  # 1/sqrt2 dropped on the diagonal
    (math.sqrt(0.5), math.sqrt(0.5)),   # off-diagonal pairs scaled as in the unfolded map
])
def test_mutant_packed_coefficients_caught(diag_scale, off_scale):
    q = RNG.standard_normal((10, 16))
    k = RNG.standard_normal((10, 16))
    s = np.einsum("nd,nd->n", q, k)
    lhs = np.einsum("nf,nf->n", _mut_phi_packed(q, diag_scale, off_scale), _mut_phi_packed(k, diag_scale, off_scale))
    assert not np.allclose(lhs, 1 + s + s * s / 2)
    r = math.sqrt(0.5)
    assert not np.allclose(_mut_phi_packed(np.array([3.0, -2.0]), diag_scale, off_scale),
                           [1.0, 3.0, -2.0, 9.0 * r, -6.0, 4.0 * r])


# ---------------------------------------------------------------- backward (training)

def _torch_forward(q, k, v):
    """The masked quadratic form written directly in torch float64 (for autograd)."""
    n = q.shape[-2]
    s = q @ k.transpose(-1, -2)
    a = torch.tril(1.0 + s + 0.5 * s * s)
    return (a @ v) / a.sum(dim=-1, keepdim=True)


@pytest.mark.parametrize("d,dv,N", [(16, 8, 40), (32, 16, 23), (2, 3, 7)])
def test_backward_matches_autograd(d, dv, N):
    q, k, v = _qkv(2, 2, N, d, dv, seed=N)
    dy = np.random.default_rng(N + 1).standard_normal((2, 2, N, dv))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    _torch_forward(tq, tk, tv).backward(torch.tensor(dy))
    dq, dk, dvv = oracle.la_backward(q, k, v, dy)
    for got, want in ((dq, tq.grad), (dk, tk.grad), (dvv, tv.grad)):
        assert np.allclose(got, want.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_matches_finite_differences():
    q, k, v = _qkv(1, 1, 6, 3, 2, seed=3)
    dy = np.random.default_rng(4).standard_normal((1, 1, 6, 2))
    loss = lambda q_, k_, v_: float(np.sum(oracle.la_quadratic(q_, k_, v_) * dy))
    dq, dk, dvv = oracle.la_backward(q, k, v, dy)
    h = 1e-6
    for x, grad, which in ((q, dq, 0), (k, dk, 1), (v, dvv, 2)):
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (which, idx, fd, grad[idx])


def test_backward_of_first_token_only_touches_itself():
    # y_0 = v_0 (one causal key): dy on token 0 alone gives dv_0 = dy_0 and no q, k gradient.
    q, k, v = _qkv(1, 1, 5, 4, 3, seed=8)
    dy = np.zeros((1, 1, 5, 3))
    dy[..., 0, :] = [1.0, -2.0, 0.5]
    dq, dk, dvv = oracle.la_backward(q, k, v, dy)
    assert np.allclose(dq, 0) and np.allclose(dk, 0)
    assert np.allclose(dvv[..., 0, :], dy[..., 0, :]) and np.allclose(dvv[..., 1:, :], 0)


def test_feature_map_vjp_matches_finite_differences():
    rng = np.random.default_rng(31)
    for d in (1, 3, 16):
        x = rng.standard_normal(d)
        u = rng.standard_normal(oracle.feature_dim(d))
        h = 1e-6
        fd = np.array([(u @ oracle.feature_map(x + h * e) - u @ oracle.feature_map(x - h * e)) / (2 * h)
                       for e in np.eye(d)])
        assert np.allclose(oracle.feature_map_vjp(x, u), fd, rtol=1e-7, atol=1e-8)


@pytest.mark.parametrize("chunk", [1, 4, 16, 23, 64])
def test_backward_by_chunks_matches_autograd(chunk):
    """The state form (forward state at a chunk's start, backward state at its
    end) gives autograd's gradients at every chunk length, ragged last chunks
    and a single chunk (64 > N) included."""
    N, d, dv = 23, 5, 4
    q, k, v = _qkv(2, 1, N, d, dv, seed=chunk)
    dy = np.random.default_rng(chunk + 7).standard_normal((2, 1, N, dv))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    _torch_forward(tq, tk, tv).backward(torch.tensor(dy))
    dq, dk, dvv = oracle.la_backward_chunked(q, k, v, dy, chunk)
    for got, want in ((dq, tq.grad), (dk, tk.grad), (dvv, tv.grad)):
        assert np.allclose(got, want.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_by_chunks_matches_the_quadratic_form_at_d16():
    q, k, v = _qkv(1, 2, 150, 16, 8, seed=5)
    dy = np.random.default_rng(6).standard_normal((1, 2, 150, 8))
    ref = oracle.la_backward(q, k, v, dy)
    for chunk in (7, 64, 128):
        for got, want in zip(oracle.la_backward_chunked(q, k, v, dy, chunk), ref):
            assert np.max(np.abs(got - want)) <= 1e-12 * np.max(np.abs(want))


# ---------------------------------------------------------------- coarse decay (reading: one gamma per 128-token chunk)

def _decay_case(B, H, N, d, dv, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, N, d)) * d ** -0.25
    k = rng.standard_normal((B, H, N, d)) * d ** -0.25
    v = rng.standard_normal((B, H, N, dv))
    gamma = rng.uniform(0.5, 1.0, (B, H, oracle.decay_chunks(N)))
    return q, k, v, gamma


def test_decay_closed_form_with_constant_scores():
    """q = 0 makes every a_ij = 1, so y_i is the w-weighted mean of v_j: for query i in
    chunk 1, keys of chunk 0 weigh gamma_1 and keys of chunk 1 weigh 1."""
    N, dv = 300, 3
    rng = np.random.default_rng(7)
    q = np.zeros((1, N, 4))
    k = rng.standard_normal((1, N, 4))
    v = rng.standard_normal((1, N, dv))
    g = np.array([[0.9, 0.5, 0.25]])
    y = oracle.la_quadratic_decay(q, k, v, g)[0]
    for i in (0, 127, 128, 200, 255):
        if i < 128:
            ref = v[0, : i + 1].mean(axis=0)
        else:
            ref = (0.5 * v[0, :128].sum(axis=0) + v[0, 128 : i + 1].sum(axis=0)) / (0.5 * 128 + (i - 127))
        assert np.allclose(y[i], ref, rtol=1e-13, atol=1e-13)
    # chunk 2: chunk 0 weighs gamma_1 gamma_2, chunk 1 weighs gamma_2
    i = 299
    num = 0.5 * 0.25 * v[0, :128].sum(axis=0) + 0.25 * v[0, 128:256].sum(axis=0) + v[0, 256:300].sum(axis=0)
    den = 0.5 * 0.25 * 128 + 0.25 * 128 + 44
    assert np.allclose(y[i], num / den, rtol=1e-13, atol=1e-13)


def test_decay_of_one_is_the_undecayed_attention():
    q, k, v, g = _decay_case(1, 2, 260, 8, 5, 1)
    y = oracle.la_quadratic_decay(q, k, v, np.ones_like(g))
    assert np.allclose(y, oracle.la_quadratic(q, k, v), rtol=1e-12, atol=1e-12)
    S, z = oracle.la_state_decay(k, v, np.ones_like(g))
    S0, z0 = oracle.la_state(k, v)
    assert np.allclose(S, S0, rtol=1e-12) and np.allclose(z, z0, rtol=1e-12)


def test_decay_quadratic_matches_recurrence_and_state():
    """Two independent formulations: pairwise weights against the per-step state
    recurrence (decay where a chunk begins), outputs and final state."""
    q, k, v, g = _decay_case(2, 1, 290, 4, 3, 2)
    y_quad = oracle.la_quadratic_decay(q, k, v, g)
    y_rec, S, z = oracle.la_recurrent_decay(q, k, v, oracle.decay_per_step(g, 290))
    assert np.allclose(y_quad, y_rec, rtol=1e-10, atol=1e-12)
    S2, z2 = oracle.la_state_decay(k, v, g)
    assert np.allclose(S, S2, rtol=1e-10, atol=1e-10) and np.allclose(z, z2, rtol=1e-10)


def test_decay_recurrence_continues_across_a_split():
    """Prefill state of the first 256 tokens, then steps from t0 = 256: the first of
    them begins chunk 2 and takes gamma_2."""
    q, k, v, g = _decay_case(1, 1, 300, 4, 3, 3)
    S0, z0 = oracle.la_state_decay(k[..., :256, :], v[..., :256, :], g[..., :2])
    y2, S2, z2 = oracle.la_recurrent_decay(q[..., 256:, :], k[..., 256:, :], v[..., 256:, :],
                                           oracle.decay_per_step(g, 44, t0=256), S0, z0)
    y_all = oracle.la_quadratic_decay(q, k, v, g)
    assert np.allclose(y2, y_all[..., 256:, :], rtol=1e-10, atol=1e-12)
    S, z = oracle.la_state_decay(k, v, g)
    assert np.allclose(S2, S, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("mutant", ["own_chunk_decayed", "no_decay_in_den"])
def test_decay_mutants_caught(mutant):
    """A plausible slip -- decaying a chunk's own keys, or leaving the denominator
    undecayed -- breaks the closed form."""
    N = 300
    rng = np.random.default_rng(8)
    q = np.zeros((1, N, 4))
    k = rng.standard_normal((1, N, 4))
    v = rng.standard_normal((1, N, 2))
    g = np.array([[0.9, 0.5, 0.25]])
    w = oracle.decay_weights(g, N)[0]
    if mutant == "own_chunk_decayed":
        w = w * g[0, np.arange(N) // 128][None, :]          # the key's own chunk decayed too
        y = (w @ v[0]) / w.sum(axis=-1)[:, None]
    else:
        y = (w @ v[0]) / np.tril(np.ones((N, N))).sum(axis=-1)[:, None]
    assert not np.allclose(y, oracle.la_quadratic_decay(q, k, v, g)[0], rtol=1e-6, atol=1e-6)
