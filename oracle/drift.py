"""Oracle: coordinate drift and factor drift.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

* Section 2.3 of the iS-KV reading notes: if the basis is rotated within its own subspace,
  ``B' = B Q`` with ``Q`` orthogonal, the coordinates must become ``U Q`` (eq. 3) for the rows to be
  unchanged. Keeping the old coordinates reconstructs ``U Sigma B'^T`` instead -- the drift. Fig. 3's
  2-D example: a unit vector whose full orthonormal basis turns by ``theta`` while its coordinates are
  kept is off by ``2 sin(theta/2)``.
* Section 7.3 (appendix measure, eq. 14) [formula rebuilt from the prose]: factor drift is the
  relative reconstruction error of the incremental factors minus that of a fresh rank-r SVD of the
  same reference matrix: ``||X - X_inc||/||X|| - ||X - X_svd,r||/||X||``.
"""

from __future__ import annotations

import numpy as np

from .fold import low_rank_product, truncated_svd


def rotate_basis(U, sigma, B, Q, rotate_coordinates: bool):
    """Apply an in-subspace basis rotation ``B <- B Q``; rotate ``U <- U Q`` too when asked."""
    U = np.asarray(U, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    Q = np.asarray(Q, dtype=np.float64)
    B2 = B @ Q
    U2 = U @ Q if rotate_coordinates else U.copy()
    return U2, np.asarray(sigma, dtype=np.float64).copy(), B2


def represented_drift(before, after) -> float:
    """Relative change of the already-represented rows: ``||X_after - X_before|| / ||X_before||``
    (the quantity of the drift probe in Section 2.3, measured against the history as it was
    represented before the update, not against the uncompressed cache)."""
    Xb = low_rank_product(*before)
    Xa = low_rank_product(*after)
    return float(np.linalg.norm(Xa - Xb) / np.linalg.norm(Xb))


def factor_drift(X, X_inc, r: int) -> float:
    """Eq. (14): excess relative error of the incremental approximation over a fresh rank-r SVD."""
    X = np.asarray(X, dtype=np.float64)
    nx = np.linalg.norm(X)
    Uf, s, Bf = truncated_svd(X, r)
    e_inc = np.linalg.norm(X - np.asarray(X_inc, dtype=np.float64)) / nx
    e_svd = np.linalg.norm(X - low_rank_product(Uf, s, Bf)) / nx
    return float(e_inc - e_svd)
