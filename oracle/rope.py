"""Oracle: rotary position embedding applied to reconstructed keys.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

iS-KV compresses keys *before* RoPE and gives every reconstructed key its own position's rotation
(iS-KV reading notes, Section 3.1 and Algorithm 3 step 8; Section 5.2 explains why a shared basis
cannot be rotated once for all positions). The pages do not print the RoPE variant. Reading adopted:
the rotate-half form used by Llama-family checkpoints -- within each head of size ``hd`` the pairs are
``(j, j + hd/2)``, angle ``pos * theta**(-2j/hd)`` for ``j = 0 .. hd/2 - 1``, no frequency scaling.
"""

from __future__ import annotations

import numpy as np


def inv_freq(head_dim: int, theta: float) -> np.ndarray:
    """``theta ** (-2 j / head_dim)`` for ``j = 0 .. head_dim/2 - 1`` (float64)."""
    if head_dim % 2:
        raise ValueError("head_dim must be even")
    j = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * j / head_dim)


def apply_rope(x, pos, n_heads: int, head_dim: int, theta: float):
    """Rotate each row ``x[i]`` (``n_heads * head_dim`` wide) by position ``pos[i]``.

    ``out[h, j]      = x[h, j] cos(a_j) - x[h, j + hd/2] sin(a_j)``
    ``out[h, j+hd/2] = x[h, j + hd/2] cos(a_j) + x[h, j] sin(a_j)``, ``a_j = pos * inv_freq[j]``.
    """
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[0]
    if x.shape[1] != n_heads * head_dim:
        raise ValueError("row width must equal n_heads * head_dim")
    pos = np.asarray(pos, dtype=np.float64).reshape(n)
    half = head_dim // 2
    ang = pos[:, None] * inv_freq(head_dim, theta)[None, :]          # n x half
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    xh = x.reshape(n, n_heads, head_dim)
    lo, hi = xh[..., :half], xh[..., half:]
    out = np.empty_like(xh)
    out[..., :half] = lo * c - hi * s
    out[..., half:] = hi * c + lo * s
    return out.reshape(n, n_heads * head_dim)
