"""Causal Taylor linear attention, float64, written from its definition.

Test infrastructure only (see the package docstring).

Notation follows "Simple linear attention language models balance the
recall-throughput tradeoff" (BASED): q, k in R^{d'} (the projected feature
dimension of §4 "Taylor Linear Attention"), v in R^{dv}, feature map phi,
state S = sum_j phi(k_j) v_j^T, normaliser z = sum_j phi(k_j) (the "K-state" of
App. D.4 "State size").

Layouts: q, k are [B, H, N, d'], v is [B, H, N, dv]; S is [B, H, D, dv] and z
is [B, H, D] with D = 1 + d' + d'^2. Feature order: index 0 is the constant 1,
indices 1..d' are x_a, index 1 + d' + a*d' + b is x_a*x_b/sqrt(2) (row-major
vec of the outer product).

Readings of points the pages leave open:
* the quadratic block is the full d'^2 outer product (widths 273 / 1057);
* phi carries no extra scale: callers pre-scale q and k;
* the output is normalised by the K-state, with no epsilon: every causal term
  is 1 + s + s^2/2 = ((s+1)^2 + 1)/2 >= 1/2, so row i's denominator is at
  least (i+1)/2 (asserted below);
* causality is inclusive: token i attends to keys j <= i.
"""

from __future__ import annotations

import numpy as np

_SQRT_HALF = np.sqrt(0.5)


def feature_dim(d_feat: int) -> int:
    """Width D = 1 + d' + d'^2 of the Taylor feature map."""
    return 1 + d_feat + d_feat * d_feat


def feature_map(x: np.ndarray) -> np.ndarray:
    """phi(x) = [1, x, vec(x (x) x)/sqrt(2)] along the last axis, float64.

    BASED §4 "Taylor Linear Attention": the 2nd-order Taylor approximation of
    exp(q.k) written as a feature map; phi(q).phi(k) = 1 + q.k + (q.k)^2/2.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    outer = x[..., :, None] * x[..., None, :]             # [..., d', d'], (a, b)
    second = outer.reshape(*x.shape[:-1], d * d) * _SQRT_HALF
    ones = np.ones(x.shape[:-1] + (1,), dtype=np.float64)
    return np.concatenate([ones, x, second], axis=-1)


def _check_den(den: np.ndarray, n_keys: np.ndarray) -> None:
    # Each causal weight is ((s+1)^2 + 1)/2 >= 1/2, so den >= (#keys)/2.
    if not np.all(den >= 0.5 * n_keys * (1.0 - 1e-12)):
        raise AssertionError("denominator below its lower bound (#keys)/2")


def la_quadratic_parts(q, k, v, row_block: int = 1024):
    """Numerator and denominator of the masked quadratic form.

    num_i = sum_{j<=i} a_ij v_j, den_i = sum_{j<=i} a_ij, a_ij = 1 + s_ij + s_ij^2/2,
    s_ij = q_i . k_j (BASED §2 "Efficient attentions": linear attention replaces
    exp(q^T k) by phi(q)^T phi(k); §4 fixes phi to the 2nd-order Taylor map, whose
    product is this polynomial). Computed in blocks of query rows; each block is
    a dense matmul followed by the causal mask -- no reordering of the sum.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    *lead, n, _ = q.shape
    dv = v.shape[-1]
    num = np.empty(tuple(lead) + (n, dv), dtype=np.float64)
    den = np.empty(tuple(lead) + (n,), dtype=np.float64)
    for r0 in range(0, n, row_block):
        r1 = min(n, r0 + row_block)
        s = q[..., r0:r1, :] @ np.swapaxes(k[..., :r1, :], -1, -2)   # [..., rows, r1]
        a = 1.0 + s + 0.5 * s * s
        rows = np.arange(r0, r1)[:, None]
        cols = np.arange(r1)[None, :]
        a = np.where(cols <= rows, a, 0.0)
        num[..., r0:r1, :] = a @ v[..., :r1, :]
        den[..., r0:r1] = a.sum(axis=-1)
    _check_den(den, np.arange(1, n + 1, dtype=np.float64))
    return num, den


def la_quadratic(q, k, v, row_block: int = 1024) -> np.ndarray:
    """y_i = num_i / den_i of the causal Taylor linear attention (quadratic form)."""
    num, den = la_quadratic_parts(q, k, v, row_block)
    return num / den[..., None]


def la_rows(q, k, v, rows) -> np.ndarray:
    """y at selected query rows of one head: q [N, d'], k [N, d'], v [N, dv].

    Same definition as la_quadratic, evaluated row by row (cost O(i) per row), for
    checking sampled outputs of large problems.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    out = np.empty((len(rows), v.shape[-1]), dtype=np.float64)
    for r, i in enumerate(rows):
        s = k[: i + 1] @ q[i]
        a = 1.0 + s + 0.5 * s * s
        den = a.sum()
        _check_den(np.array([den]), np.array([i + 1.0]))
        out[r] = (a @ v[: i + 1]) / den
    return out


def la_state(k, v):
    """S = sum_j phi(k_j) v_j^T and z = sum_j phi(k_j) over all tokens.

    The recurrent state of linear attention ("Gated Slot Attention", App. A: an
    additive matrix-valued state of key-value outer products) together with the
    K-state for the denominator (BASED App. D.4). phi is built explicitly, so the
    feature order and the 1/sqrt(2) are part of what this pins.
    """
    fk = feature_map(k)                                            # [..., N, D]
    v = np.asarray(v, dtype=np.float64)
    S = np.swapaxes(fk, -1, -2) @ v                                # [..., D, dv]
    z = fk.sum(axis=-2)                                            # [..., D]
    return S, z


def la_recurrent(q, k, v, S0=None, z0=None):
    """Token-by-token recurrent form (BASED §2: recurrent generation).

    For t = 0..N-1: S += phi(k_t) v_t^T; z += phi(k_t);
    y_t = phi(q_t)^T S / phi(q_t)^T z   (the output includes token t itself).
    Starts from S0, z0 (zeros when omitted). Returns (y, S, z).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    *lead, n, d_feat = q.shape
    dv = v.shape[-1]
    D = feature_dim(d_feat)
    S = np.zeros(tuple(lead) + (D, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    z = np.zeros(tuple(lead) + (D,)) if z0 is None else np.array(z0, dtype=np.float64)
    y = np.empty(tuple(lead) + (n, dv), dtype=np.float64)
    fq = feature_map(q)
    fk = feature_map(k)
    for t in range(n):
        S += fk[..., t, :, None] * v[..., t, None, :]
        z += fk[..., t, :]
        num = np.einsum("...f,...fe->...e", fq[..., t, :], S)
        den = np.einsum("...f,...f->...", fq[..., t, :], z)
        y[..., t, :] = num / den[..., None]
    return y, S, z


def la_chunked(q, k, v, chunk: int):
    """Chunkwise form: on-diagonal masked quadratic part + off-diagonal state part.

    For chunk c holding tokens [cC, (c+1)C):
      y_c = (A_c V_c + phi(Q_c) S_{c-1}) / (rowsum(A_c) + phi(Q_c) z_{c-1}),
      A_c = (1 + Q_c K_c^T + (Q_c K_c^T)^2/2) with the causal mask inside the chunk,
      S_c = S_{c-1} + phi(K_c)^T V_c,  z_c = z_{c-1} + colsum(phi(K_c)).
    BASED App. B (Algorithm 1: quadratic on-diagonal tiles with local causal
    masking plus linear off-diagonal cumulative state) and "Gated Slot
    Attention" App. A.1 (inter-chunk and intra-chunk terms). Returns (y, S, z).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    *lead, n, d_feat = q.shape
    dv = v.shape[-1]
    D = feature_dim(d_feat)
    S = np.zeros(tuple(lead) + (D, dv))
    z = np.zeros(tuple(lead) + (D,))
    y = np.empty(tuple(lead) + (n, dv))
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        qc, kc, vc = q[..., c0:c1, :], k[..., c0:c1, :], v[..., c0:c1, :]
        s = qc @ np.swapaxes(kc, -1, -2)
        a = 1.0 + s + 0.5 * s * s
        m = np.tril(np.ones((c1 - c0, c1 - c0), dtype=bool))
        a = np.where(m, a, 0.0)
        fq = feature_map(qc)
        fk = feature_map(kc)
        num = a @ vc + fq @ S
        den = a.sum(axis=-1) + np.einsum("...tf,...f->...t", fq, z)
        y[..., c0:c1, :] = num / den[..., None]
        S = S + np.swapaxes(fk, -1, -2) @ vc
        z = z + fk.sum(axis=-2)
    return y, S, z


def la_taylor_terms(q, k, v):
    """Order-0, order-1 and order-2 Taylor terms of the causal numerator and denominator.

    BASED App. B (Algorithm 1) writes the output as y = T0 + T1 + T2, one term
    per Taylor order. With the K-state normalisation each order contributes to
    both the numerator and the denominator:
      T0_i = sum_{j<=i} v_j,              d0_i = i + 1,
      T1_i = sum_{j<=i} (q_i.k_j) v_j,    d1_i = sum_{j<=i} q_i.k_j,
      T2_i = sum_{j<=i} (q_i.k_j)^2/2 v_j, d2_i = sum_{j<=i} (q_i.k_j)^2/2,
    and y_i = (T0 + T1 + T2)_i / (d0 + d1 + d2)_i. Returns ((T0, T1, T2), (d0, d1, d2)).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n = q.shape[-2]
    mask = np.tril(np.ones((n, n), dtype=bool))
    s = q @ np.swapaxes(k, -1, -2)
    w0 = np.where(mask, 1.0, 0.0) * np.ones_like(s)
    w1 = np.where(mask, s, 0.0)
    w2 = np.where(mask, 0.5 * s * s, 0.0)
    terms = tuple(w @ v for w in (w0, w1, w2))
    dens = tuple(w.sum(axis=-1) for w in (w0, w1, w2))
    return terms, dens


# ---------------------------------------------------------------- symmetric (packed) state
#
# The order-2 block of phi is the outer product x (x) x, which is symmetric:
# entries (a, b) and (b, a) are equal. Folding each pair gives an equivalent
# feature map of width 1 + d' + d'(d'+1)/2 (153 at d' = 16, 561 at d' = 32):
#     phi_s(x) = [1, x, (x_a x_b * c_ab)_{a <= b, a-major}],  c_aa = 1/sqrt(2), c_ab = 1,
# for which phi_s(q).phi_s(k) = 1 + q.k + sum_a q_a^2 k_a^2 / 2 + sum_{a<b} q_a q_b k_a k_b
#                             = 1 + q.k + (q.k)^2/2 = phi(q).phi(k).
# This is a derivation from BASED §4's feature map, not a form the pages print.
# The packed state S_s = sum_j phi_s(k_j) v_j^T, z_s = sum_j phi_s(k_j) carries
# the same information in about half the rows.


def packed_dim(d_feat: int) -> int:
    """Width 1 + d' + d'(d'+1)/2 of the symmetric (packed) feature map."""
    return 1 + d_feat + d_feat * (d_feat + 1) // 2


def packed_pairs(d_feat: int):
    """The (a, b) pairs of the packed order-2 features, a <= b, a-major."""
    return [(a, b) for a in range(d_feat) for b in range(a, d_feat)]


def feature_map_packed(x: np.ndarray) -> np.ndarray:
    """phi_s(x) = [1, x, x_a x_b (a <= b, a-major; x_a^2 / sqrt(2) on the diagonal)], float64."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    cols = []
    for a, b in packed_pairs(d):
        p = x[..., a] * x[..., b]
        cols.append(p * _SQRT_HALF if a == b else p)
    second = np.stack(cols, axis=-1)
    ones = np.ones(x.shape[:-1] + (1,), dtype=np.float64)
    return np.concatenate([ones, x, second], axis=-1)


def la_state_packed(k, v):
    """Packed S_s = sum_j phi_s(k_j) v_j^T and z_s = sum_j phi_s(k_j), phi_s built explicitly."""
    fk = feature_map_packed(k)
    v = np.asarray(v, dtype=np.float64)
    return np.swapaxes(fk, -1, -2) @ v, fk.sum(axis=-2)


def la_recurrent_packed(q, k, v, S0=None, z0=None):
    """The recurrent form of la_recurrent with the packed feature map and state."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    *lead, n, d_feat = q.shape
    dv = v.shape[-1]
    Ds = packed_dim(d_feat)
    S = np.zeros(tuple(lead) + (Ds, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    z = np.zeros(tuple(lead) + (Ds,)) if z0 is None else np.array(z0, dtype=np.float64)
    y = np.empty(tuple(lead) + (n, dv), dtype=np.float64)
    fq = feature_map_packed(q)
    fk = feature_map_packed(k)
    for t in range(n):
        S += fk[..., t, :, None] * v[..., t, None, :]
        z += fk[..., t, :]
        num = np.einsum("...f,...fe->...e", fq[..., t, :], S)
        den = np.einsum("...f,...f->...", fq[..., t, :], z)
        y[..., t, :] = num / den[..., None]
    return y, S, z


# ---------------------------------------------------------------- backward (training)
#
# Gradients of the causal Taylor linear attention of la_quadratic (the pages'
# prefill "during training", BASED §5 "Execution stages"). With s_ij = q_i.k_j,
# a_ij = 1 + s_ij + s_ij^2/2 (j <= i), den_i = sum_j a_ij, y_i = sum_j a_ij v_j / den_i
# and an upstream gradient dy:
#     g_i   = dy_i / den_i,          c_i = g_i . y_i,
#     da_ij = g_i . v_j - c_i        (the quotient rule: num_i / den_i),
#     ds_ij = da_ij (1 + s_ij)       (d a / d s = 1 + s),
#     dq_i  = sum_{j<=i} ds_ij k_j,  dk_j = sum_{i>=j} ds_ij q_i,
#     dv_j  = sum_{i>=j} a_ij g_i.


def la_backward(q, k, v, dy):
    """(dq, dk, dv) of la_quadratic for the upstream gradient dy, float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    n = q.shape[-2]
    mask = np.tril(np.ones((n, n), dtype=bool))
    s = q @ np.swapaxes(k, -1, -2)
    a = np.where(mask, 1.0 + s + 0.5 * s * s, 0.0)
    den = a.sum(axis=-1)
    _check_den(den, np.arange(1, n + 1, dtype=np.float64))
    y = (a @ v) / den[..., None]
    g = dy / den[..., None]
    c = np.sum(g * y, axis=-1)
    da = np.where(mask, g @ np.swapaxes(v, -1, -2) - c[..., None], 0.0)
    ds = da * (1.0 + s)
    dq = ds @ k
    dk = np.swapaxes(ds, -1, -2) @ q
    dv = np.swapaxes(a, -1, -2) @ g
    return dq, dk, dv


def feature_map_vjp(x, u):
    """u^T dphi/dx for phi(x) = [1, x, vec(x x^T)/sqrt2]: with u = [u_0, u_1, U_2]
    (U_2 the d' x d' block, row-major), it is u_1 + (U_2 + U_2^T) x / sqrt2."""
    x = np.asarray(x, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    d = x.shape[-1]
    u2 = u[..., 1 + d:].reshape(u.shape[:-1] + (d, d))
    sym = u2 + np.swapaxes(u2, -1, -2)
    return u[..., 1:1 + d] + _SQRT_HALF * np.einsum("...ab,...b->...a", sym, x)


def la_backward_chunked(q, k, v, dy, chunk: int):
    """(dq, dk, dv) of the forward by chunks, with states instead of the full
    causal square: the gradient of la_backward in the form a state-based
    (reverse-scan) backward evaluates.

    With a_ij = phi(q_i).phi(k_j), den_i = phi(q_i).z_i, g_i = dy_i / den_i,
    c_i = g_i.y_i and da_ij = g_i.v_j - c_i (j <= i):
      dphi(q_i) = sum_{j<=i} da_ij phi(k_j) = S_i g_i - c_i z_i,
      dphi(k_j) = sum_{i>=j} da_ij phi(q_i) = R_j v_j - r_j,
      dv_j      = sum_{i>=j} a_ij g_i       = R_j^T phi(k_j),
    where S_i, z_i sum phi(k) v^T and phi(k) over keys up to i (the forward
    state), and R_j = sum_{i>=j} phi(q_i) g_i^T, r_j = sum_{i>=j} c_i phi(q_i)
    sum over queries from j on (a state carried backwards). Within a chunk the
    pairs are taken directly; the earlier chunks enter through the forward
    state at the chunk's start, the later ones through the backward state at
    its end (BASED App. B: quadratic on-diagonal tiles plus cumulative state,
    here for the derivative of that forward). dq, dk follow by the chain rule
    through phi (feature_map_vjp).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    *lead, n, d_feat = q.shape
    dv_dim = v.shape[-1]
    D = feature_dim(d_feat)
    fq, fk = feature_map(q), feature_map(k)
    bounds = [(c0, min(n, c0 + chunk)) for c0 in range(0, n, chunk)]
    masks = {c1 - c0: np.tril(np.ones((c1 - c0, c1 - c0), dtype=bool)) for c0, c1 in bounds}

    # Forward pass over the chunks: y, den, and the state entering each chunk.
    S = np.zeros(tuple(lead) + (D, dv_dim))
    z = np.zeros(tuple(lead) + (D,))
    S_in, z_in, a_in = [], [], []
    g = np.empty(tuple(lead) + (n, dv_dim))
    cc = np.empty(tuple(lead) + (n,))
    for c0, c1 in bounds:
        a = np.where(masks[c1 - c0], fq[..., c0:c1, :] @ np.swapaxes(fk[..., c0:c1, :], -1, -2), 0.0)
        num = a @ v[..., c0:c1, :] + fq[..., c0:c1, :] @ S
        den = a.sum(axis=-1) + np.einsum("...tf,...f->...t", fq[..., c0:c1, :], z)
        _check_den(den, np.arange(c0 + 1, c1 + 1, dtype=np.float64))
        y = num / den[..., None]
        g[..., c0:c1, :] = dy[..., c0:c1, :] / den[..., None]
        cc[..., c0:c1] = np.sum(g[..., c0:c1, :] * y, axis=-1)
        S_in.append(S)
        z_in.append(z)
        a_in.append(a)
        S = S + np.swapaxes(fk[..., c0:c1, :], -1, -2) @ v[..., c0:c1, :]
        z = z + fk[..., c0:c1, :].sum(axis=-2)

    # Backward pass over the chunks, last first, carrying R and r.
    R = np.zeros(tuple(lead) + (D, dv_dim))
    r = np.zeros(tuple(lead) + (D,))
    dfq = np.empty_like(fq)
    dfk = np.empty_like(fk)
    dv = np.empty_like(v)
    for idx in range(len(bounds) - 1, -1, -1):
        c0, c1 = bounds[idx]
        m = masks[c1 - c0]
        gc, ccc, vc = g[..., c0:c1, :], cc[..., c0:c1], v[..., c0:c1, :]
        fqc, fkc = fq[..., c0:c1, :], fk[..., c0:c1, :]
        da = np.where(m, gc @ np.swapaxes(vc, -1, -2) - ccc[..., None], 0.0)
        dfq[..., c0:c1, :] = (da @ fkc + np.swapaxes(S_in[idx] @ np.swapaxes(gc, -1, -2), -1, -2)
                              - ccc[..., None] * z_in[idx][..., None, :])
        dfk[..., c0:c1, :] = np.swapaxes(da, -1, -2) @ fqc + vc @ np.swapaxes(R, -1, -2) - r[..., None, :]
        dv[..., c0:c1, :] = np.swapaxes(a_in[idx], -1, -2) @ gc + fkc @ R
        R = R + np.swapaxes(fqc, -1, -2) @ gc
        r = r + np.einsum("...t,...tf->...f", ccc, fqc)
    return feature_map_vjp(q, dfq), feature_map_vjp(k, dfk), dv


# ---------------------------------------------------------------------------
# Coarse input-dependent decay.
#
# BASED App. C "Extended Architecture Details" (Decay) and App. D.4 "BASED
# Quality Ablations" (Input-dependent decay) describe a coarser input-dependent
# decay of the state that avoids a parallel scan, and print no formula. Reading taken (one scalar per chunk of DECAY_CHUNK tokens, applied to
# the state where a chunk begins; the chunk's own tokens are not decayed among
# themselves):
#     S_c = gamma_c S_{c-1} + sum_{t in chunk c} phi(k_t) v_t^T,   z likewise;
# token i of chunk c reads gamma_c S_{c-1} + (its chunk's keys j <= i). Pairwise,
# key j contributes to query i >= j with the weight
#     w_ij = prod_{c = chunk(j)+1 .. chunk(i)} gamma_c   (1 inside one chunk),
# in the numerator and the denominator alike. gamma is [..., n_chunks], caller
# supplied (the projection that makes it input-dependent is outside this path).

DECAY_CHUNK = 128


def decay_chunks(n: int) -> int:
    """Number of decay chunks covering n tokens."""
    return (n + DECAY_CHUNK - 1) // DECAY_CHUNK


def decay_weights(gamma, n: int) -> np.ndarray:
    """w [..., n, n]: w_ij = product of gamma over the chunks after chunk(j) up to
    chunk(i), for j <= i; 0 above the diagonal. Built with explicit loops over
    the chunk pairs."""
    gamma = np.asarray(gamma, dtype=np.float64)
    nc = decay_chunks(n)
    assert gamma.shape[-1] == nc, (gamma.shape, nc)
    lead = gamma.shape[:-1]
    pair = np.ones(lead + (nc, nc), dtype=np.float64)    # pair[ci, cj]
    for ci in range(nc):
        for cj in range(ci):
            w = np.ones(lead, dtype=np.float64)
            for c in range(cj + 1, ci + 1):
                w = w * gamma[..., c]
            pair[..., ci, cj] = w
    chunk = np.arange(n) // DECAY_CHUNK
    w = pair[..., chunk[:, None], chunk[None, :]]
    return np.where(np.tril(np.ones((n, n), dtype=bool)), w, 0.0)


def la_quadratic_decay(q, k, v, gamma) -> np.ndarray:
    """y_i = sum_{j<=i} w_ij a_ij v_j / sum_{j<=i} w_ij a_ij with a_ij = 1 + s + s^2/2."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n = q.shape[-2]
    s = q @ np.swapaxes(k, -1, -2)
    a = (1.0 + s + 0.5 * s * s) * decay_weights(gamma, n)
    return (a @ v) / a.sum(axis=-1)[..., None]


def la_state_decay(k, v, gamma):
    """Final S, z: sum_j u_j phi(k_j) v_j^T and sum_j u_j phi(k_j), with u_j the
    product of gamma over the chunks after chunk(j)."""
    fk = feature_map(k)
    v = np.asarray(v, dtype=np.float64)
    gamma = np.asarray(gamma, dtype=np.float64)
    n = fk.shape[-2]
    nc = decay_chunks(n)
    u = np.ones(gamma.shape[:-1] + (n,), dtype=np.float64)
    for j in range(n):
        for c in range(j // DECAY_CHUNK + 1, nc):
            u[..., j] = u[..., j] * gamma[..., c]
    fku = fk * u[..., None]
    return np.swapaxes(fku, -1, -2) @ v, fku.sum(axis=-2)


def la_recurrent_decay(q, k, v, gamma_step, S0=None, z0=None):
    """Token by token with a decay per step: S <- gamma_t S, z <- gamma_t z, then
    S += phi(k_t) v_t^T, z += phi(k_t), y_t = phi(q_t) S / phi(q_t) z.

    gamma_step is [..., n] (1 except where a chunk begins); this is the decode
    step's form. Returns (y, S, z)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(gamma_step, dtype=np.float64)
    *lead, n, d_feat = q.shape
    dv = v.shape[-1]
    D = feature_dim(d_feat)
    S = np.zeros(tuple(lead) + (D, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    z = np.zeros(tuple(lead) + (D,)) if z0 is None else np.array(z0, dtype=np.float64)
    y = np.empty(tuple(lead) + (n, dv), dtype=np.float64)
    fq = feature_map(q)
    fk = feature_map(k)
    for t in range(n):
        S = S * g[..., t, None, None] + fk[..., t, :, None] * v[..., t, None, :]
        z = z * g[..., t, None] + fk[..., t, :]
        num = np.einsum("...f,...fe->...e", fq[..., t, :], S)
        den = np.einsum("...f,...f->...", fq[..., t, :], z)
        y[..., t, :] = num / den[..., None]
    return y, S, z


def decay_per_step(gamma, n: int, t0: int = 0) -> np.ndarray:
    """gamma_step [..., n] for tokens t0 .. t0+n-1: gamma_c on the first token of
    chunk c (c >= 1), 1 elsewhere. gamma holds one value per chunk from chunk 0."""
    gamma = np.asarray(gamma, dtype=np.float64)
    out = np.ones(gamma.shape[:-1] + (n,), dtype=np.float64)
    for t in range(n):
        tok = t0 + t
        if tok > 0 and tok % DECAY_CHUNK == 0:
            out[..., t] = gamma[..., tok // DECAY_CHUNK]
    return out
