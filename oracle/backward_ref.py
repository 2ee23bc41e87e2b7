"""Float64 oracle for the gradients of the attention forward (test
infrastructure only, like the rest of this package).

Page 1, "CANN ops-transformer FlashAttentionScore", section
反向传播的重算策略及其合理性: training needs dQ, dK and dV; the forward keeps only
its row statistics, and the backward recomputes the attention weights tile by
tile from them, then forms the gradient pieces per tile.

``attention_backward`` is the definition (the chain rule through the softmax,
written out); ``attention_backward_tiled`` follows the page's recompute scheme
with arbitrary tile sizes and only the forward's LSE, and is pinned against the
definition.  Both take the forward's inputs and the output gradient dO (and an
optional dLSE).  With S = scale * Q K^T (masked keys removed), P = softmax(S),
O = P V:

    dV = P^T dO,   dP = dO V^T,   D_i = sum_j P_ij dP_ij (= dO_i . O_i),
    dS = P * (dP - D) (+ P * dLSE),   dQ = scale * dS K,   dK = scale * dS^T Q.
"""

from __future__ import annotations

import numpy as np

from .attention_ref import _as_f64, allowed_keys, resolve_scale


def _probs(q, k, scale, causal, rows):
    """P for the given query rows (visible keys only, exact softmax)."""
    s = scale * (q[rows] @ k.T)
    if causal:
        nkv = k.shape[0]
        for a, i in enumerate(rows):
            vis = allowed_keys(int(i), nkv, True)
            mask = np.ones(nkv, dtype=bool)
            mask[vis] = False
            s[a, mask] = -np.inf
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=1, keepdims=True)


def attention_backward(q, k, v, do, scale=None, causal: bool = False, dlse=None):
    """(dQ, dK, dV) of O = softmax(scale Q K^T [+causal]) V for one head:
    q [Nq, d], k, v [Nkv, d], do [Nq, d]; dlse [Nq] optional (the gradient
    reaching the LSE output)."""
    q, k, v, do = (_as_f64(x) for x in (q, k, v, do))
    nq, d = q.shape
    sc = resolve_scale(scale, d)
    rows = np.arange(nq)
    p = _probs(q, k, sc, causal, rows)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    dd = np.sum(do * o, axis=1, keepdims=True)
    ds = p * (dp - dd)
    if dlse is not None:
        ds = ds + p * _as_f64(dlse).reshape(-1, 1)
    dq = sc * (ds @ k)
    dk = sc * (ds.T @ q)
    return dq, dk, dv


def attention_backward_tiled(q, k, v, do, lse, block_r: int, block_c: int, scale=None, causal: bool = False):
    """The page's recompute scheme: for every (query tile i, key tile j), rebuild
    P_ij = exp(S_ij - LSE_i) from the forward's LSE alone, then accumulate
    dV_j += P_ij^T dO_i, dP_ij = dO_i V_j^T, dS_ij = P_ij (dP_ij - D_i) with
    D_i = rowsum(dO_i * O_i) formed once per query tile, dQ_i += scale dS_ij K_j,
    dK_j += scale dS_ij^T Q_i.  Any tile sizes; the result equals the definition."""
    q, k, v, do, lse = (_as_f64(x) for x in (q, k, v, do, lse))
    nq, d = q.shape
    nkv = k.shape[0]
    sc = resolve_scale(scale, d)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    # O is recomputed from the same statistics (the page keeps O from the forward)
    for i0 in range(0, nq, block_r):
        i1 = min(nq, i0 + block_r)
        o_i = np.zeros((i1 - i0, v.shape[1]))
        for j0 in range(0, nkv, block_c):
            j1 = min(nkv, j0 + block_c)
            o_i += _tile_p(q, k, lse, sc, causal, i0, i1, j0, j1) @ v[j0:j1]
        d_i = np.sum(do[i0:i1] * o_i, axis=1, keepdims=True)
        for j0 in range(0, nkv, block_c):
            j1 = min(nkv, j0 + block_c)
            p_ij = _tile_p(q, k, lse, sc, causal, i0, i1, j0, j1)
            dv[j0:j1] += p_ij.T @ do[i0:i1]
            dp_ij = do[i0:i1] @ v[j0:j1].T
            ds_ij = p_ij * (dp_ij - d_i)
            dq[i0:i1] += sc * (ds_ij @ k[j0:j1])
            dk[j0:j1] += sc * (ds_ij.T @ q[i0:i1])
    return dq, dk, dv


def _tile_p(q, k, lse, sc, causal, i0, i1, j0, j1):
    s = sc * (q[i0:i1] @ k[j0:j1].T)
    if causal:
        rows = np.arange(i0, i1).reshape(-1, 1)
        cols = np.arange(j0, j1).reshape(1, -1)
        s = np.where(cols <= rows, s, -np.inf)
    return np.exp(s - lse[i0:i1].reshape(-1, 1))


def attention_backward_batched(q, k, v, do, scale=None, causal: bool = False, layout: str = "BHND"):
    """``attention_backward`` for every (b, h), the layouts and K/V head
    grouping of ``attention_batched`` (query head h uses K/V head
    h // (H // Hkv)); a K/V head's gradient is the sum over its group."""
    q, k, v, do = (_as_f64(x) for x in (q, k, v, do))
    if layout == "BSND":
        q, k, v, do = (x.transpose(0, 2, 1, 3) for x in (q, k, v, do))
    elif layout != "BHND":
        raise ValueError(f"unknown layout {layout!r}")
    B, H = q.shape[:2]
    hkv = k.shape[1]
    if hkv < 1 or H % hkv:
        raise ValueError(f"K/V heads ({hkv}) must divide the query heads ({H})")
    g = H // hkv
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            a, bb, c = attention_backward(q[b, h], k[b, h // g], v[b, h // g], do[b, h], scale, causal)
            dq[b, h] = a
            dk[b, h // g] += bb
            dv[b, h // g] += c
    if layout == "BSND":
        dq, dk, dv = (x.transpose(0, 2, 1, 3) for x in (dq, dk, dv))
    return dq, dk, dv
