"""GPU parity of whole fold trajectories at the one-layer shape: d = 1024 (8 KV heads x 128),
n = 8192 rows folded in blocks of b = 64 into rank r = 256, keys with spectrum i^-1.2 (seed 1) and
values with i^-0.6 (seed 2), plus 0.02 N(0, 1) noise; re-orthogonalisation every 4 folds (every
256 folded rows, the cadence of the iS-KV reading notes, Section 4.4).

float32 storage: the GPU trajectory must equal the oracle's (fold_stream with the same reorth
cadence) to 1e-4 in reconstruction and singular values.

bf16 storage: the trajectory is not fixed by the method. Every fold rewrites all n history rows
(the coordinate rotation of Algorithm 2 steps 7-8) and stores them again in bf16, so the
represented rows take a fresh rounding of relative size 2^-9 at every step; these add up like a
random walk, and near the truncation boundary, which at this workload lies inside the noise bulk,
they change which near-degenerate directions are kept. The same steps in exact arithmetic with only
the stored factors rounded to bf16 already end about 3 % (relative Frobenius) away from the exact
trajectory, with tail singular values up to 2 % apart. So, following "compare what is unique and
check that the rest is valid", the bf16 test checks
  * every step -- each of the 128 folds and 32 re-orthogonalisations -- against the oracle started
    from the GPU's stored state before that step (singular values 1e-4, reconstruction 2e-2 on the
    folded rows), and
  * the end state's quality against the exact oracle trajectory: its relative error to the folded
    rows and the eq. (14) factor drift (Section 7.3: excess error over a fresh rank-r SVD) agree
    with the oracle's to within 5e-3 absolute, the scale of the drift the pages report for 2-byte
    factors (K 0.0016-0.0071, V 0.0160-0.0207 in Table 5).
"""

import numpy as np
import pytest
import torch

from gpu_util import kv, np64, state, stored
from oracle import drift as odr
from oracle import fold as of
from oracle import reorth as oreo
import synth

pytestmark = pytest.mark.gpu

D, N, B, R, EVERY = 1024, 8192, 64, 256, 4
SIDES = {"K": (1.2, 1), "V": (0.6, 2)}


def _rows(side, storage):
    ex, seed = SIDES[side]
    return stored(synth.lowrank_rows(N, D, ex, 0.02, seed=seed), storage)


def _oracle_trajectory(X):
    U, s, Bm = of.empty_history(D)
    for i in range(N // B):
        res = of.fold_block(U, s, Bm, X[i * B:(i + 1) * B], R)
        U, s, Bm = res.U, res.sigma, res.B
        if (i + 1) % EVERY == 0:
            U, s, Bm = oreo.reorth(U, s, Bm)
    return U, s, Bm


def _sample_rel(U1, s1, B1, U0, s0, B0, rows):
    return of.rel_fro((U1[rows] * s1) @ B1.T, (U0[rows] * s0) @ B0.T)


@pytest.mark.parametrize("side", ["K", "V"])
def test_config2_trajectory_float32(side):
    m = kv()
    X = _rows(side, torch.float32)
    Xd = torch.as_tensor(X, dtype=torch.float32, device="cuda")
    h = m.LowRankHistory(D, R, N, storage=torch.float32)
    for i in range(N // B):
        m.fold_block(h, Xd[i * B:(i + 1) * B].contiguous(),
                     torch.arange(i * B, (i + 1) * B, dtype=torch.int32, device="cuda"))
        if (i + 1) % EVERY == 0:
            m.reorth(h)
    U, s, Bm, pos, (k, n, folds, st) = state(h)
    assert (k, n, folds, st) == (R, N, 0, 0)
    assert np.array_equal(pos, np.arange(N))
    Uo, so, Bo = _oracle_trajectory(X)
    np.testing.assert_allclose(s, so, rtol=1e-4)
    P, Po = of.low_rank_product(U, s, Bm), of.low_rank_product(Uo, so, Bo)
    assert of.rel_fro(P, Po) < 1e-4
    d_gpu, d_ora = odr.factor_drift(X, P, R), odr.factor_drift(X, Po, R)
    print(f"\n{side} float32: factor drift (eq. 14) GPU {d_gpu:.5f} oracle {d_ora:.5f}")
    assert abs(d_gpu - d_ora) < 1e-5


@pytest.mark.parametrize("side", ["K", "V"])
def test_config2_trajectory_bf16_stepwise(side):
    m = kv()
    X = _rows(side, torch.bfloat16)
    Xd = torch.as_tensor(X, dtype=torch.bfloat16, device="cuda")
    h = m.LowRankHistory(D, R, N, storage=torch.bfloat16)
    g = np.random.Generator(np.random.PCG64(11))
    U0, s0, B0 = of.empty_history(D)
    worst_fold = worst_reorth = worst_sig = 0.0
    for i in range(N // B):
        F = X[i * B:(i + 1) * B]
        m.fold_block(h, Xd[i * B:(i + 1) * B].contiguous(),
                     torch.arange(i * B, (i + 1) * B, dtype=torch.int32, device="cuda"))
        U1, s1, B1, pos, (k1, n1, _, st) = state(h)
        res = of.fold_block(U0, s0, B0, F, R)
        assert st == 0 and (k1, n1) == (res.k_new, (i + 1) * B)
        assert np.array_equal(pos, np.arange(n1))
        np.testing.assert_allclose(s1, res.sigma, rtol=1e-4)
        worst_sig = max(worst_sig, float(np.max(np.abs(s1 - res.sigma) / res.sigma)))
        rows = np.r_[g.choice(n1 - B, min(512, n1 - B), replace=False), np.arange(n1 - B, n1)] \
            if n1 > B else np.arange(n1)
        e = _sample_rel(U1, s1, B1, res.U, res.sigma, res.B, rows)
        assert e < 2e-2, (i, e)
        worst_fold = max(worst_fold, e)
        U0, s0, B0 = U1, s1, B1
        if (i + 1) % EVERY == 0:
            m.reorth(h)
            U2, s2, B2, _, (k2, n2, folds, st2) = state(h)
            assert st2 == 0 and (k2, n2, folds) == (k1, n1, 0)
            Ur, sr, Br = oreo.reorth(U0, s0, B0)
            np.testing.assert_allclose(s2, sr, rtol=1e-4)
            e = _sample_rel(U2, s2, B2, Ur, sr, Br, rows)
            assert e < 2e-2, (i, e)
            worst_reorth = max(worst_reorth, e)
            U0, s0, B0 = U2, s2, B2
    Uo, so, Bo = _oracle_trajectory(X)
    P, Po = of.low_rank_product(U0, s0, B0), of.low_rank_product(Uo, so, Bo)
    err_gpu, err_ora = of.rel_fro(P, X), of.rel_fro(Po, X)
    d_gpu, d_ora = odr.factor_drift(X, P, R), odr.factor_drift(X, Po, R)
    print(f"\n{side} bf16: steps: fold rec <= {worst_fold:.2e}, reorth rec <= {worst_reorth:.2e}, "
          f"sigma <= {worst_sig:.2e}; end state vs exact oracle trajectory: rec "
          f"{of.rel_fro(P, Po):.4f}, sigma max rel {np.max(np.abs(s0 - so) / so):.4f}; error to "
          f"rows GPU {err_gpu:.5f} oracle {err_ora:.5f}; factor drift (eq. 14) GPU {d_gpu:.5f} "
          f"oracle {d_ora:.5f}")
    assert abs(err_gpu - err_ora) < 5e-3
    assert abs(d_gpu - d_ora) < 5e-3
