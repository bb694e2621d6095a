"""Oracle: periodic re-orthogonalisation (iS-KV reading notes, Section 4.4).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Repeated low-precision folds let the columns of ``U`` and ``B`` drift away from orthonormality.
Section 4.4 takes thin QR factorisations ``U = Q_U R_U`` and ``B = Q_B R_B``, decomposes the small
matrix ``R_U diag(sigma) R_B^T = X diag(sigma') Y^T`` and replaces the factors by ``Q_U X``,
``sigma'`` and ``Q_B Y``. In exact arithmetic the product ``U diag(sigma) B^T`` is unchanged; no
discarded information comes back.
"""

from __future__ import annotations

import numpy as np


def reorth(U, sigma, B):
    """Section 4.4, step by step. Returns ``(U', sigma', B')`` with the same rank k."""
    U = np.asarray(U, dtype=np.float64)
    sigma = np.asarray(sigma, dtype=np.float64).reshape(-1)
    B = np.asarray(B, dtype=np.float64)
    k = sigma.shape[0]
    if k == 0:
        return U.copy(), sigma.copy(), B.copy()
    Q_U, R_U = np.linalg.qr(U, mode="reduced")          # n x k, k x k
    Q_B, R_B = np.linalg.qr(B, mode="reduced")          # d x k, k x k
    M = (R_U * sigma[None, :]) @ R_B.T                  # R_U diag(sigma) R_B^T
    X, s, Yt = np.linalg.svd(M)
    return Q_U @ X, s, Q_B @ Yt.T


def orthogonality_error(A) -> float:
    """``||A^T A - I||_F``: the orthogonality diagnostic reported before and after Section 4.4."""
    A = np.asarray(A, dtype=np.float64)
    return float(np.linalg.norm(A.T @ A - np.eye(A.shape[1])))
