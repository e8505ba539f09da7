"""Causal sliding-window softmax attention, float64, written from its definition.

Test infrastructure only (see the package docstring).

BASED ("Simple linear attention language models balance the recall-throughput
tradeoff") §4 "Local Exact Attention": each query attends with exact softmax
to a window of preceding keys, at O(Nw) time and space and a w-sized KV cache
during generation; App. A.1 gives the O(Nw) cost.

Readings of points the pages leave open:
* the window holds w keys including the query's own position: token i sees keys
  j with i - w < j <= i, which is exactly what a w-slot ring cache holds;
* the score scale is an explicit argument (1/sqrt(head dim) in the workloads);
* the ring slot of token t is t mod w; slots that have never held a token are 0.
"""

from __future__ import annotations

import numpy as np


def swa(q, k, v, w: int, scale: float, row_block: int = 512) -> np.ndarray:
    """y_i = sum_j p_ij v_j, p_ij = softmax_j(scale * q_i.k_j) over i - w < j <= i.

    Plain masked softmax with the row maximum subtracted before exponentiation;
    blocks of query rows, each a dense matmul then the band mask.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    *lead, n, _ = q.shape
    y = np.empty(tuple(lead) + (n, v.shape[-1]), dtype=np.float64)
    for r0 in range(0, n, row_block):
        r1 = min(n, r0 + row_block)
        c0 = max(0, r0 - w + 1)
        s = scale * (q[..., r0:r1, :] @ np.swapaxes(k[..., c0:r1, :], -1, -2))
        rows = np.arange(r0, r1)[:, None]
        cols = np.arange(c0, r1)[None, :]
        band = (cols <= rows) & (cols > rows - w)
        s = np.where(band, s, -np.inf)
        s = s - s.max(axis=-1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=-1, keepdims=True)
        y[..., r0:r1, :] = p @ v[..., c0:r1, :]
    return y


def swa_rows(q, k, v, w: int, scale: float, rows) -> np.ndarray:
    """swa() at selected rows of one head (q, k [N, d], v [N, dv])."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    out = np.empty((len(rows), v.shape[-1]), dtype=np.float64)
    for r, i in enumerate(rows):
        j0 = max(0, i - w + 1)
        s = scale * (k[j0 : i + 1] @ q[i])
        p = np.exp(s - s.max())
        out[r] = (p / p.sum()) @ v[j0 : i + 1]
    return out


def swa_ring_after_prefill(k, v, w: int):
    """Ring KV cache after a prefill of N tokens: slot t mod w holds token t.

    Slots hold tokens max(0, N - w) .. N - 1; slots never written are zero.
    Returns (k_cache, v_cache) shaped [..., w, d] and [..., w, dv].
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n = k.shape[-2]
    kc = np.zeros(k.shape[:-2] + (w, k.shape[-1]))
    vc = np.zeros(v.shape[:-2] + (w, v.shape[-1]))
    for t in range(max(0, n - w), n):
        kc[..., t % w, :] = k[..., t, :]
        vc[..., t % w, :] = v[..., t, :]
    return kc, vc


def swa_decode_step(k_cache, v_cache, t: int, q, k, v, w: int, scale: float):
    """One generation step over the w-slot ring (§4 "Local Exact Attention").

    t is the number of tokens seen before this one. The new (k, v) goes to slot
    t mod w, then the query attends to the min(t + 1, w) slots holding tokens
    max(0, t - w + 1) .. t. q, k: [..., d], v: [..., dv]; caches [..., w, d|dv].
    Returns (y, k_cache', v_cache') without modifying the inputs.
    """
    kc = np.array(k_cache, dtype=np.float64)
    vc = np.array(v_cache, dtype=np.float64)
    kc[..., t % w, :] = np.asarray(k, dtype=np.float64)
    vc[..., t % w, :] = np.asarray(v, dtype=np.float64)
    slots = [u % w for u in range(max(0, t - w + 1), t + 1)]
    ks = kc[..., slots, :]                                   # [..., n_valid, d]
    vs = vc[..., slots, :]
    s = scale * np.einsum("...d,...jd->...j", np.asarray(q, dtype=np.float64), ks)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=-1, keepdims=True)
    y = np.einsum("...j,...jd->...d", p, vs)
    return y, kc, vc
