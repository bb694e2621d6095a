"""Oracle: the block-incremental SVD fold (iS-KV reading notes, Section 4, Algorithm 2).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Notation follows the pages. A compressed history of ``n`` rows is kept as ``U diag(sigma) B^T``
with ``U`` (n x k), ``sigma`` (k,) descending, ``B`` (d x k), ``k <= r`` (Section 2.2). A pending
block ``F`` (b x d) of exact rows is merged in by Algorithm 2. Algorithm 2 calls the projection
``Q = F B``; it is called ``C`` here so that it does not clash with the ``Q`` of a QR factorisation.

Every floating-point step is float64. Library primitives used as steps: ``np.linalg.qr`` (Householder
QR, LAPACK geqrf/orgqr) and ``np.linalg.svd`` (LAPACK gesdd).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

#: Machine epsilon of the compute precision. Section 4.4 states that projection, residual handling,
#: core SVD, re-orthogonalisation and reconstruction run in FP32, and Section 4.1 sets the residual
#: floor from "the machine epsilon of the compute precision": so FP32's 2^-23.
EPS_FP32 = 2.0 ** -23


def residual_tolerance(sigma_1: float, rho_1: float, b: int, d: int,
                       tau_rel: float = 0.0, eps: float = EPS_FP32) -> float:
    """Residual-direction threshold of Section 4.1 [formula rebuilt; the printed one was lost].

    The surviving prose says the kept count is the number of residual singular values above a
    scale-dependent floor built from the machine epsilon. Reading adopted here:
    ``tol = max(tau_rel, eps * max(b, d)) * s_ref`` with ``s_ref = max(sigma_1, rho_1)`` (the largest
    singular value in play) and ``tau_rel = 0`` by default (pure numerical floor).
    """
    s_ref = max(float(sigma_1), float(rho_1))
    return max(float(tau_rel), float(eps) * max(int(b), int(d))) * s_ref


@dataclass
class FoldResult:
    """Output of one fold. ``U``, ``sigma``, ``B`` are the new factors (k' columns)."""

    U: np.ndarray
    sigma: np.ndarray
    B: np.ndarray
    p: int                  # kept residual directions
    k_new: int              # k' = min(r, k + p)
    rho: np.ndarray         # all residual singular values (descending)
    tol: float              # threshold applied to rho
    core_sigma: np.ndarray  # all singular values of the core Z (descending)
    C: np.ndarray           # projection F B (b x k)
    P: np.ndarray           # kept residual basis (d x p)


def fold_block(U, sigma, B, F, r: int, tau_rel: float = 0.0, eps: float = EPS_FP32) -> FoldResult:
    """Merge the pending block ``F`` into ``U diag(sigma) B^T`` (Algorithm 2, Section 4).

    Steps, in the order of Algorithm 2:

    1. Empty history (k = 0): the general steps below with ``k = 0`` reduce to a rank-r SVD of ``F``
       (C is empty, E = F, the core is ``Y_R diag(rho)``, already diagonal). Directions with
       ``rho <= tol`` are not added, as for any other fold.
    2. ``C = F B``, ``E = F - C B^T`` (Section 4.1).
    3. Subtract E's leftover component along B once more: ``E <- E - (E B) B^T``.
    4. Reduced QR of ``E^T = Q_R R_R``, SVD ``R_R = W_R diag(rho) Y_R^T``; keep
       ``p = #{rho_i > tol}`` directions, ``P = Q_R W_R[:, :p]``. No residual directions when the old
       basis already spans all d features (k = d).
    5. Core ``Z = [[diag(sigma), 0], [F B, F P]]`` of size (k+b) x (k+p) (Section 4.2).
    6. SVD ``Z = G diag(sigma+) H^T``; keep the top ``k' = min(r, k+p)`` components.
    7. Old positions: ``U <- U G[:k]`` (every history row is rotated with the basis).
    8. New positions: append ``G[k:]``; ``B+ = [B, P] H``.
    """
    U = np.asarray(U, dtype=np.float64)
    sigma = np.asarray(sigma, dtype=np.float64).reshape(-1)
    B = np.asarray(B, dtype=np.float64)
    F = np.asarray(F, dtype=np.float64)
    b, d = F.shape
    k = sigma.shape[0]
    if U.shape[1] != k or B.shape != (d, k):
        raise ValueError("shape mismatch between U, sigma, B and F")
    if b > d:
        raise ValueError("block rows b must not exceed the feature width d")

    # Steps 2-3: projection and twice-subtracted residual.
    C = F @ B                                   # b x k
    E = F - C @ B.T
    E = E - (E @ B) @ B.T

    # Step 4: residual basis.
    if k >= d:
        rho = np.zeros(0)
        tol = 0.0
        p = 0
        P = np.zeros((d, 0))
    else:
        Q_R, R_R = np.linalg.qr(E.T, mode="reduced")     # d x b, b x b
        W_R, rho, _ = np.linalg.svd(R_R)                 # R_R = W_R diag(rho) Y_R^T
        sigma_1 = sigma[0] if k > 0 else 0.0
        tol = residual_tolerance(sigma_1, rho[0] if rho.size else 0.0, b, d, tau_rel, eps)
        p = int(np.count_nonzero(rho > tol))
        P = Q_R @ W_R[:, :p]                             # d x p

    # Step 5: the small core.
    Z = np.zeros((k + b, k + p))
    Z[:k, :k] = np.diag(sigma)
    Z[k:, :k] = C
    Z[k:, k:] = F @ P

    # Step 6: truncated SVD of the core.
    G, core_sigma, Ht = np.linalg.svd(Z, full_matrices=False)
    k_new = min(int(r), k + p)
    G = G[:, :k_new]
    H = Ht[:k_new].T

    # Steps 7-8: rotate history coordinates, append the new rows, rotate the basis.
    U_new = np.vstack([U @ G[:k], G[k:]])
    B_new = np.hstack([B, P]) @ H
    return FoldResult(U=U_new, sigma=core_sigma[:k_new].copy(), B=B_new, p=p, k_new=k_new,
                      rho=rho, tol=tol, core_sigma=core_sigma, C=C, P=P)


def empty_history(d: int):
    """An empty history: ``U`` 0 x 0, ``sigma`` empty, ``B`` d x 0."""
    return np.zeros((0, 0)), np.zeros(0), np.zeros((d, 0))


def fold_stream(X, b: int, r: int, tau_rel: float = 0.0, eps: float = EPS_FP32,
                n_blocks: int | None = None):
    """Fold the rows of ``X`` block by block, from an empty history (Algorithm 3 step 4 repeated).

    Returns ``(U, sigma, B, results)``. Rows beyond the last full block are not folded.
    """
    X = np.asarray(X, dtype=np.float64)
    n_rows, d = X.shape
    nb = n_rows // b if n_blocks is None else int(n_blocks)
    U, sigma, B = empty_history(d)
    results = []
    for i in range(nb):
        res = fold_block(U, sigma, B, X[i * b:(i + 1) * b], r, tau_rel, eps)
        U, sigma, B = res.U, res.sigma, res.B
        results.append(res)
    return U, sigma, B, results


def truncated_svd(X, r: int):
    """Plain definition the fold must reach: the best rank-r approximation of ``X`` in Frobenius
    norm (Section 2.2). Returns ``(U, s, B)`` with ``X ~= U diag(s) B^T``."""
    X = np.asarray(X, dtype=np.float64)
    Uf, s, Vt = np.linalg.svd(X, full_matrices=False)
    r = min(int(r), s.shape[0])
    return Uf[:, :r], s[:r].copy(), Vt[:r].T


def low_rank_product(U, sigma, B):
    """``U diag(sigma) B^T``: the rows the history represents (Section 2.2)."""
    U = np.asarray(U, dtype=np.float64)
    return (U * np.asarray(sigma, dtype=np.float64)[None, :]) @ np.asarray(B, dtype=np.float64).T


def rel_fro(A, Bm) -> float:
    """Relative Frobenius error ``||A - B||_F / ||B||_F`` (``||A||_F`` if ``B`` is zero)."""
    A = np.asarray(A, dtype=np.float64)
    Bm = np.asarray(Bm, dtype=np.float64)
    den = np.linalg.norm(Bm)
    if den == 0.0:
        return float(np.linalg.norm(A))
    return float(np.linalg.norm(A - Bm) / den)
