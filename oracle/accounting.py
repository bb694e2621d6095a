"""Oracle: persistent-storage arithmetic (iS-KV reading notes, Section 5.1, eq. 12 and Fig. 5).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Eq. (12) [formula rebuilt from the prose; the printed one was lost]: per layer and per path X in
{K, V}, with ``n_c`` compressed rows at rank ``k``, feature width ``d`` and ``n_e`` exact rows,

    bytes = s_f * (n_c * k + d * k + k) + s_e * n_e * d

The first term is U, the shared basis B and the diagonal of Sigma; the second term holds every exact
row (protected, recent, pending). Position indices, reserved capacity, the reconstructed dense cache
and workspace are not counted.
"""

from __future__ import annotations

import math


def persistent_bytes(n_c: int, k: int, d: int, n_e: int, s_f: int = 2, s_e: int = 2) -> int:
    """Eq. (12) for one path of one layer."""
    return s_f * (n_c * k + d * k + k) + s_e * n_e * d


def dense_bytes(n: int, d: int, s: int = 2) -> int:
    """Uncompressed bytes of one path of one layer."""
    return s * n * d


def break_even_rows(k: int, d: int) -> int:
    """Smallest ``n_c`` with ``n_c * d >= n_c * k + d * k + k`` (exact-row terms cancel), i.e.
    ``n_c >= k (d + 1) / (d - k)``."""
    if k >= d:
        raise ValueError("no break-even when k >= d")
    return math.ceil(k * (d + 1) / (d - k))


def asymptotic_ratio(d: int, k: int) -> float:
    """Limit of dense / persistent bytes for a long history with fixed exact rows: ``d / k``."""
    return d / k


def compression_ratio(n_c: int, k: int, d: int, n_e: int, s_f: int = 2, s_e: int = 2,
                      s_dense: int = 2) -> float:
    """Dense bytes of all ``n_c + n_e`` rows divided by eq. (12)."""
    return dense_bytes(n_c + n_e, d, s_dense) / persistent_bytes(n_c, k, d, n_e, s_f, s_e)
