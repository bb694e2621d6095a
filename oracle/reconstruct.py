"""Oracle: per-step reconstruction of the cache (iS-KV reading notes, Algorithm 3 steps 7-8).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Compressed row ``i`` of a history is ``U[i] diag(sigma) B^T`` and belongs at its original token
position ``pos[i]`` (Section 2.2; Section 3.2 warns that the K and V histories index different
tokens, so rows are scattered by position, never paired by array index). Exact rows (protected,
recent, pending) are copied to their own positions. Keys are then rotated per position with RoPE
(step 8); values are not.
"""

from __future__ import annotations

import numpy as np

from .rope import apply_rope


def reconstruct(U, sigma, B, pos, exact_rows, exact_pos, n_total: int, n_heads: int,
                head_dim: int, rope: bool, theta: float = 500000.0, fill: float = 0.0):
    """Dense ``n_total x d`` cache rebuilt from the factors and the exact rows.

    Positions covered by neither set keep ``fill``. A position covered twice is an input error.
    """
    U = np.asarray(U, dtype=np.float64)
    sigma = np.asarray(sigma, dtype=np.float64).reshape(-1)
    B = np.asarray(B, dtype=np.float64)
    d = B.shape[0]
    pos = np.asarray(pos, dtype=np.int64).reshape(-1)
    exact_pos = np.asarray(exact_pos, dtype=np.int64).reshape(-1)
    exact_rows = np.asarray(exact_rows, dtype=np.float64).reshape(exact_pos.shape[0], d)
    allpos = np.concatenate([pos, exact_pos])
    if allpos.size and (allpos.min() < 0 or allpos.max() >= n_total):
        raise ValueError("position out of range")
    if np.unique(allpos).size != allpos.size:
        raise ValueError("a position is covered twice")
    out = np.full((n_total, d), float(fill))
    comp = (U * sigma[None, :]) @ B.T
    if rope:
        comp = apply_rope(comp, pos, n_heads, head_dim, theta)
        ex = apply_rope(exact_rows, exact_pos, n_heads, head_dim, theta)
    else:
        ex = exact_rows
    out[pos] = comp
    out[exact_pos] = ex
    return out
