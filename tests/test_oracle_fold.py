"""Pins for the fold oracle: each checks it against something other than itself.

* batch SVD when the rank fits (Section 4.3: the fold is the exact SVD of its target);
* single-fold optimality and the dropped-residual error split (Section 4.3, after eq. 7);
* Eckart-Young on the truncated SVD, with a brute-force check on 2-column data (Section 2.2);
* the rank-1 counterexample's printed numbers (Section 4.3, Fig. 4; tests/golden);
* k = d (no residual directions) and k = 0 (rank-r SVD of F) special cases (Section 4.1-4.2).
"""

import json
import os

import numpy as np
import pytest

from conftest import GOLDEN
from oracle import fold as of
import synth


def _random_history(n, d, k, seed):
    g = synth.rng(seed)
    U = np.linalg.qr(g.standard_normal((n, k)))[0]
    B = np.linalg.qr(g.standard_normal((d, k)))[0]
    sigma = np.sort(g.uniform(1.0, 10.0, k))[::-1] * np.sqrt(n)
    return U, sigma, B


def test_fold_equals_batch_svd_when_rank_fits():
    # Config-1 shape, noiseless, spectrum cut at rank 12 <= r = 16.
    X = synth.lowrank_rows(512, 128, 1.0, 0.0, seed=0, rank=12)
    U, s, B, res = of.fold_stream(X[:480], 16, 16)
    Xf = X[:480]
    assert of.rel_fro(of.low_rank_product(U, s, B), Xf) < 1e-10
    _, s_ref, _ = of.truncated_svd(Xf, 16)
    assert s.shape[0] == 12                       # threshold removes the numerically-zero rest
    np.testing.assert_allclose(s, s_ref[:12], rtol=1e-10)
    assert s_ref[12] / s_ref[0] < 1e-12


def test_fold_full_width_rank_is_exact_and_skips_residual():
    # r = d: after d/b folds k = d, then no residual direction may be added (p = 0).
    X = synth.lowrank_rows(256, 32, 0.5, 0.05, seed=3)
    U, s, B, res = of.fold_stream(X, 8, 32)
    assert any(r.p == 0 and r.k_new == 32 for r in res[4:])
    assert all(r.p == 0 for r in res[4:])
    assert of.rel_fro(of.low_rank_product(U, s, B), X) < 1e-12


def test_single_fold_is_best_rank_r_of_target():
    n, d, k, b, r = 200, 48, 12, 8, 14
    U, sigma, B = _random_history(n, d, k, seed=11)
    F = synth.rng(12).standard_normal((b, d))
    res = of.fold_block(U, sigma, B, F, r)
    T = np.vstack([of.low_rank_product(U, sigma, B), F])
    sT = np.linalg.svd(T, compute_uv=False)
    assert res.p == b and res.k_new == r
    np.testing.assert_allclose(res.sigma, sT[:r], rtol=1e-10)
    err2 = np.linalg.norm(T - of.low_rank_product(res.U, res.sigma, res.B)) ** 2
    np.testing.assert_allclose(err2, np.sum(sT[r:] ** 2), rtol=1e-9)
    # New factors are orthonormal.
    np.testing.assert_allclose(res.U.T @ res.U, np.eye(r), atol=1e-10)
    np.testing.assert_allclose(res.B.T @ res.B, np.eye(r), atol=1e-10)


def test_dropped_residual_error_split():
    # A large tau_rel drops residual directions; error^2 = core tail^2 + dropped rho^2.
    n, d, k, b, r = 150, 40, 10, 8, 20
    U, sigma, B = _random_history(n, d, k, seed=21)
    g = synth.rng(22)
    F = g.standard_normal((b, k)) @ B.T * 5 + g.standard_normal((b, d)) * np.geomspace(1, 1e-3, d)
    tau = 0.02
    res = of.fold_block(U, sigma, B, F, r, tau_rel=tau)
    assert 0 < res.p < b
    T = np.vstack([of.low_rank_product(U, sigma, B), F])
    err2 = np.linalg.norm(T - of.low_rank_product(res.U, res.sigma, res.B)) ** 2
    dropped = res.rho[res.rho <= res.tol]
    expect = np.sum(res.core_sigma[res.k_new:] ** 2) + np.sum(dropped ** 2)
    np.testing.assert_allclose(err2, expect, rtol=1e-9)


def test_residual_is_orthogonal_to_basis():
    n, d, k, b = 100, 64, 16, 16
    U, sigma, B = _random_history(n, d, k, seed=31)
    F = synth.rng(32).standard_normal((b, d))
    res = of.fold_block(U, sigma, B, F, 64)
    np.testing.assert_allclose(B.T @ res.P, 0.0, atol=1e-12)
    np.testing.assert_allclose(res.P.T @ res.P, np.eye(res.p), atol=1e-12)
    np.testing.assert_allclose(res.C, F @ B, rtol=1e-12)


def test_empty_history_fold_is_rank_r_svd_of_block():
    F = synth.rng(41).standard_normal((16, 64))
    U0, s0, B0 = of.empty_history(64)
    res = of.fold_block(U0, s0, B0, F, 10)
    Ur, sr, Br = of.truncated_svd(F, 10)
    np.testing.assert_allclose(res.sigma, sr, rtol=1e-12)
    assert of.rel_fro(of.low_rank_product(res.U, res.sigma, res.B),
                      of.low_rank_product(Ur, sr, Br)) < 1e-12


def test_zero_block_adds_nothing_but_keeps_history():
    n, d, k, b = 60, 32, 6, 4
    U, sigma, B = _random_history(n, d, k, seed=51)
    res = of.fold_block(U, sigma, B, np.zeros((b, d)), 8)
    assert res.p == 0 and res.k_new == k
    np.testing.assert_allclose(res.sigma, sigma, rtol=1e-12)
    X0 = of.low_rank_product(U, sigma, B)
    X1 = of.low_rank_product(res.U, res.sigma, res.B)
    assert of.rel_fro(X1[:n], X0) < 1e-12
    np.testing.assert_allclose(X1[n:], 0.0, atol=1e-12)


def test_eckart_young_truncation_error():
    X = synth.rng(61).standard_normal((40, 12))
    s_all = np.linalg.svd(X, compute_uv=False)
    for r in (1, 3, 7, 12):
        Ur, sr, Br = of.truncated_svd(X, r)
        err2 = np.linalg.norm(X - of.low_rank_product(Ur, sr, Br)) ** 2
        np.testing.assert_allclose(err2, np.sum(s_all[r:] ** 2), rtol=1e-10, atol=1e-10)


def test_eckart_young_brute_force_two_columns():
    # Best rank-1 approximation of an n x 2 matrix: the unit direction v maximising |X v| --
    # found here by a dense scan over angles, independently of LAPACK.
    X = synth.rng(71).standard_normal((9, 2)) @ np.array([[3.0, 1.0], [0.5, 1.0]])
    th = np.linspace(0, np.pi, 200001)
    V = np.stack([np.cos(th), np.sin(th)])
    energy = np.sum((X @ V) ** 2, axis=0)
    best = energy.max()
    Ur, sr, Br = of.truncated_svd(X, 1)
    np.testing.assert_allclose(sr[0] ** 2, best, rtol=1e-9)
    err2 = np.linalg.norm(X - of.low_rank_product(Ur, sr, Br)) ** 2
    np.testing.assert_allclose(err2, np.sum(X ** 2) - best, rtol=1e-7)


def test_rank1_counterexample_printed_numbers():
    gd = json.load(open(os.path.join(GOLDEN, "rank1_example.json")))
    X1 = np.array(gd["first_batch"])
    X2 = np.array(gd["new_rows"])
    r = gd["r"]
    U0, s0, B0 = of.empty_history(2)
    a = of.fold_block(U0, s0, B0, X1, r)
    kept_first = np.abs(a.B[:, 0])
    b = of.fold_block(a.U, a.sigma, a.B, X2, r)
    pr = gd["printed"]
    np.testing.assert_allclose(b.core_sigma ** 2, pr["incremental_core_sigma_squared"], atol=1e-12)
    np.testing.assert_allclose(np.abs(b.B[:, 0]), kept_first, atol=1e-12)  # keeps the old direction
    full = np.vstack([X1, X2])
    Uf, sf, Bf = of.truncated_svd(full, r)
    fresh_err = np.linalg.norm(full - of.low_rank_product(Uf, sf, Bf))
    np.testing.assert_allclose(fresh_err, pr["fresh_svd_best_error"], atol=1e-12)
    other_energy = np.sum((full @ (np.array([1.0, 1.0]) - kept_first)) ** 2)
    assert other_energy > pr["fresh_keeps_other_direction_because_energy_exceeds"]
    inc_err = np.linalg.norm(full - of.low_rank_product(b.U, b.sigma, b.B))
    assert inc_err > fresh_err


def test_threshold_reading():
    # tol = max(tau, eps * max(b, d)) * max(sigma_1, rho_1)
    assert of.residual_tolerance(10.0, 2.0, 64, 1024) == pytest.approx(2.0 ** -23 * 1024 * 10.0)
    assert of.residual_tolerance(1.0, 3.0, 64, 32) == pytest.approx(2.0 ** -23 * 64 * 3.0)
    assert of.residual_tolerance(1.0, 1.0, 8, 8, tau_rel=0.5) == pytest.approx(0.5)
