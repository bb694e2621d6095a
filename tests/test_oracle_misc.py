"""Pins for the re-orthogonalisation, RoPE, reconstruction, accounting and drift oracles."""

import json
import math
import os

import numpy as np
import pytest

from conftest import GOLDEN
from oracle import accounting, drift, reconstruct, reorth, rope
from oracle import fold as of
import synth


# ---------------------------------------------------------------- re-orthogonalisation (Section 4.4)

def test_reorth_keeps_product_and_restores_orthogonality():
    g = synth.rng(5)
    n, d, k = 300, 64, 20
    U = np.linalg.qr(g.standard_normal((n, k)))[0] + 1e-3 * g.standard_normal((n, k))
    B = np.linalg.qr(g.standard_normal((d, k)))[0] + 1e-3 * g.standard_normal((d, k))
    sigma = np.geomspace(50, 0.5, k)
    X0 = of.low_rank_product(U, sigma, B)
    assert reorth.orthogonality_error(U) > 1e-3
    U2, s2, B2 = reorth.reorth(U, sigma, B)
    assert of.rel_fro(of.low_rank_product(U2, s2, B2), X0) < 1e-12
    assert reorth.orthogonality_error(U2) < 1e-12
    assert reorth.orthogonality_error(B2) < 1e-12
    assert np.all(np.diff(s2) <= 0)
    # New sigma are the singular values of the product (it is an SVD after reorth).
    np.testing.assert_allclose(s2, np.linalg.svd(X0, compute_uv=False)[:k], rtol=1e-10)


# ---------------------------------------------------------------- RoPE

def test_rope_closed_form_single_pair():
    hd, H = 128, 2
    x = np.zeros((1, H * hd))
    x[0, hd + 0] = 1.0            # head 1, j = 0 (frequency 1)
    x[0, 3] = 2.0                 # head 0, j = 3
    theta = 10000.0
    out = rope.apply_rope(x, [5], H, hd, theta)
    assert out[0, hd + 0] == pytest.approx(math.cos(5.0), abs=1e-15)
    assert out[0, hd + 64] == pytest.approx(math.sin(5.0), abs=1e-15)
    a = 5.0 * theta ** (-6.0 / 128)
    assert out[0, 3] == pytest.approx(2 * math.cos(a), abs=1e-14)
    assert out[0, 67] == pytest.approx(2 * math.sin(a), abs=1e-14)


def test_rope_invariants():
    g = synth.rng(7)
    x = g.standard_normal((6, 8 * 128))
    pos = np.array([0, 1, 17, 4095, 16383, 65535])
    y = rope.apply_rope(x, pos, 8, 128, 500000.0)
    np.testing.assert_allclose(y[0], x[0], atol=0)                    # position 0 is identity
    pair = lambda z: z.reshape(6, 8, 2, 64)
    np.testing.assert_allclose(np.hypot(pair(y)[:, :, 0], pair(y)[:, :, 1]),
                               np.hypot(pair(x)[:, :, 0], pair(x)[:, :, 1]), rtol=1e-12)
    back = rope.apply_rope(y, -pos, 8, 128, 500000.0)
    np.testing.assert_allclose(back, x, atol=1e-11)


# ---------------------------------------------------------------- reconstruction (Algorithm 3)

def test_reconstruct_scatters_by_position():
    g = synth.rng(9)
    n, d, k, H, hd = 10, 2 * 16, 4, 2, 16
    U = g.standard_normal((n, k))
    sigma = np.array([4.0, 3.0, 2.0, 1.0])
    B = np.linalg.qr(g.standard_normal((d, k)))[0]
    perm = g.permutation(16)
    pos, exact_pos = perm[:n], perm[n:]
    exact = g.standard_normal((16 - n, d))
    out = reconstruct.reconstruct(U, sigma, B, pos, exact, exact_pos, 16, H, hd, rope=False)
    for i in range(n):                                                   # row-by-row definition
        row = sum(U[i, j] * sigma[j] * B[:, j] for j in range(k))
        np.testing.assert_allclose(out[pos[i]], row, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out[exact_pos], exact)
    outk = reconstruct.reconstruct(U, sigma, B, pos, exact, exact_pos, 16, H, hd, rope=True,
                                   theta=100.0)
    np.testing.assert_allclose(outk[exact_pos[0]],
                               rope.apply_rope(exact[:1], [exact_pos[0]], H, hd, 100.0)[0])
    with pytest.raises(ValueError):
        reconstruct.reconstruct(U, sigma, B, pos, exact, np.r_[pos[:1], exact_pos[1:]], 16, H, hd,
                                rope=False)


# ---------------------------------------------------------------- accounting (Section 5.1, 7.2)

def test_accounting_printed_numbers():
    gd = json.load(open(os.path.join(GOLDEN, "accounting.json")))
    be = gd["break_even"]
    assert accounting.break_even_rows(be["k"], be["d"]) == be["rows"]
    n = be["rows"]
    assert accounting.dense_bytes(n, be["d"]) >= accounting.persistent_bytes(n, be["k"], be["d"], 0)
    assert accounting.dense_bytes(n - 1, be["d"]) < accounting.persistent_bytes(n - 1, be["k"],
                                                                                 be["d"], 0)
    a = gd["asymptote"]
    assert accounting.asymptotic_ratio(a["d"], a["k"]) == a["ratio"]
    # The ratio with 192 exact rows (Fig. 5) approaches, but stays below, d / k.
    r_long = accounting.compression_ratio(10 ** 8, a["k"], a["d"], 192)
    assert a["ratio"] - 0.01 < r_long < a["ratio"]
    ds = gd["dense_storage_gib"]
    for L, gib in zip(ds["prompt_tokens"], ds["printed_gib"]):
        total = ds["layers"] * ds["kv_paths"] * accounting.dense_bytes(
            L + ds["generated_tokens"], ds["d"], ds["bytes_per_scalar"])
        assert total / 2 ** 30 == pytest.approx(gib, abs=1e-9)


# ---------------------------------------------------------------- drift (Section 2.3, eq. 14)

def test_drift_2d_example():
    gd = json.load(open(os.path.join(GOLDEN, "drift_2d.json")))
    for th in gd["thetas"]:
        Q = np.array([[math.cos(th), -math.sin(th)], [math.sin(th), math.cos(th)]])
        U = np.array([[0.6, 0.8]])          # one unit vector's coordinates
        B = np.eye(2)
        kept = drift.represented_drift((U, [1.0, 1.0], B), drift.rotate_basis(U, [1, 1], B, Q, False))
        synced = drift.represented_drift((U, [1.0, 1.0], B), drift.rotate_basis(U, [1, 1], B, Q, True))
        assert kept == pytest.approx(2 * math.sin(th / 2), rel=1e-12)
        assert synced < 1e-15


def test_basis_only_drift_formula_and_fold_trend():
    g = synth.rng(13)
    n, d, k = 80, 24, 6
    U = np.linalg.qr(g.standard_normal((n, k)))[0]
    B = np.linalg.qr(g.standard_normal((d, k)))[0]
    s = np.geomspace(10, 1, k)
    Q = synth.random_orthogonal(k, g)
    kept = drift.represented_drift((U, s, B), drift.rotate_basis(U, s, B, Q, False))
    expect = np.linalg.norm((U * s) @ (Q.T - np.eye(k))) / np.linalg.norm(U * s)
    assert kept == pytest.approx(expect, rel=1e-12)
    # Fold-level trend of the Section 2.3 probe: after a fold, rotating the coordinates with the
    # basis keeps the represented history; keeping the old coordinates does not.
    X = synth.lowrank_rows(400, 32, 0.8, 0.05, seed=14)
    Uh, sh, Bh, _ = of.fold_stream(X[:384], 16, 8)
    res = of.fold_block(Uh, sh, Bh, X[384:400], 8)
    m = Uh.shape[0]
    synced = of.rel_fro(of.low_rank_product(res.U[:m], res.sigma, res.B),
                        of.low_rank_product(Uh, sh, Bh))
    basis_only = of.rel_fro(of.low_rank_product(Uh, res.sigma, res.B),
                            of.low_rank_product(Uh, sh, Bh))
    assert synced < 0.05 and basis_only > 10 * synced


def test_factor_drift_definition():
    X = synth.lowrank_rows(120, 16, 1.0, 0.01, seed=15)
    Ur, sr, Br = of.truncated_svd(X, 4)
    assert abs(drift.factor_drift(X, of.low_rank_product(Ur, sr, Br), 4)) < 1e-14
    e_svd = np.linalg.norm(X - of.low_rank_product(Ur, sr, Br)) / np.linalg.norm(X)
    assert drift.factor_drift(X, np.zeros_like(X), 4) == pytest.approx(1 - e_svd, rel=1e-12)
