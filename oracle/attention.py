"""Oracle: decode attention over the compressed cache (iS-KV reading notes, Algorithm 3 steps 7-9).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Step 9 runs the model's original dense attention over the cache that steps 7-8 rebuild: every
cached position holds either a compressed row (``U[i] diag(sigma) B^T`` at ``pos[i]``) or an exact
row, keys are rotated by their own position, values are not. Section 5.2 names the factor-aware
form of this step (scores and value mixing computed from the factors, never writing the dense
cache) as the route to a speed-up; whatever the route, it computes this definition.

Readings (the pages give no attention formula): single-query decode with scaled dot-product
scores ``scale * q_j . k_p`` over every key position p, softmax over those positions, output
``sum_p softmax_j(p) v_p``; grouped-query attention maps query head j to KV head
``j // (n_q_heads // n_kv_heads)``; the query arrives already rotated for its own position (as
the model produces it); the K and V caches must cover the same set of positions.
"""

from __future__ import annotations

import math

import numpy as np

from .reconstruct import reconstruct


def decode_attention(k_factors, v_factors, k_exact, k_exact_pos, v_exact, v_exact_pos,
                     n_total: int, q, n_kv_heads: int, head_dim: int, theta: float = 500000.0,
                     scale: float | None = None):
    """Outputs ``[n_q_heads][head_dim]`` of one decode query over one layer's cache.

    k_factors, v_factors: ``(U, sigma, B, pos)`` of the K and V histories. Exact rows are
    pre-RoPE keys and values at their positions.
    """
    q = np.asarray(q, dtype=np.float64)
    n_q = q.shape[0]
    if n_q % n_kv_heads:
        raise ValueError("query heads must be a multiple of KV heads")
    group = n_q // n_kv_heads
    scale = 1.0 / math.sqrt(head_dim) if scale is None else float(scale)
    Uk, sk, Bk, pk = k_factors
    Uv, sv, Bv, pv = v_factors
    nan = float("nan")
    K = reconstruct(Uk, sk, Bk, pk, k_exact, k_exact_pos, n_total, n_kv_heads, head_dim, True,
                    theta, fill=nan)
    V = reconstruct(Uv, sv, Bv, pv, v_exact, v_exact_pos, n_total, n_kv_heads, head_dim, False,
                    theta, fill=nan)
    kpos = np.flatnonzero(~np.isnan(K[:, 0]))
    vpos = np.flatnonzero(~np.isnan(V[:, 0]))
    if not np.array_equal(kpos, vpos):
        raise ValueError("K and V caches cover different positions")
    out = np.empty((n_q, head_dim))
    for j in range(n_q):
        h = j // group
        cols = slice(h * head_dim, (h + 1) * head_dim)
        s = scale * (K[kpos, cols] @ q[j])
        w = np.exp(s - s.max())
        w /= w.sum()
        out[j] = w @ V[kpos, cols]
    return out


def decode_attention_loops(K, V, q, n_kv_heads: int, head_dim: int, scale: float):
    """The same attention written as scalar loops over an already rebuilt dense cache (rows of K
    post-RoPE): an independent restatement used to pin the vectorised oracle on tiny inputs."""
    n_q = len(q)
    group = n_q // n_kv_heads
    out = []
    for j in range(n_q):
        h = j // group
        scores = []
        for p in range(len(K)):
            dot = 0.0
            for f in range(head_dim):
                dot += float(q[j][f]) * float(K[p][h * head_dim + f])
            scores.append(scale * dot)
        top = max(scores)
        ex = [math.exp(v - top) for v in scores]
        tot = sum(ex)
        row = []
        for f in range(head_dim):
            acc = 0.0
            for p in range(len(V)):
                acc += ex[p] / tot * float(V[p][h * head_dim + f])
            row.append(acc)
        out.append(row)
    return np.array(out)
