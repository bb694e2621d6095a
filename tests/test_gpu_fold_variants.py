"""GPU parity of fold variants the iS-KV reading notes discuss, against the float64 oracle:

* a relative residual threshold tau_rel > 0 (Section 4.1): residual directions whose singular value
  is at or below tau_rel * max(sigma_1, rho_1) are not added, so p < b, down to p = 0;
* keys and values with different rank budgets in one workflow (the separate K / V ranks of the
  policy, Section 8);
* the long-prompt compression shape: rank r = 512 at d = 1024 with folds of b = 128.

float32 storage is held to 1e-4 (reconstruction, relative Frobenius) and 1e-4 (singular values);
bf16 storage to 2e-2 and 1e-4.
"""

import numpy as np
import pytest
import torch

from gpu_util import kv, state, stored
from oracle import fold as of
import synth

pytestmark = pytest.mark.gpu


def _fold_all(m, h, X, b, dtype, tau_rel=0.0, start=0, nblocks=None):
    Xd = torch.as_tensor(X, dtype=dtype, device="cuda")
    nblocks = X.shape[0] // b - start if nblocks is None else nblocks
    for i in range(start, start + nblocks):
        m.fold_block(h, Xd[i * b:(i + 1) * b].contiguous(),
                     torch.arange(i * b, (i + 1) * b, dtype=torch.int32, device="cuda"),
                     tau_rel=tau_rel)


@pytest.mark.parametrize("r,tau", [(16, 1e-2), (16, 3e-2), (32, 3e-2)])
def test_residual_threshold_trajectory(r, tau):
    """Config-1 rows (d = 128, spectrum i^-1, noise 0.01, b = 16, 480 rows) with tau_rel > 0."""
    m = kv()
    X = stored(synth.lowrank_rows(480, 128, 1.0, 0.01, seed=0), torch.float32)
    Uo, so, Bo, res = of.fold_stream(X, 16, r, tau_rel=tau)
    ps = [x.p for x in res]
    assert min(ps) < 16, ps                               # the threshold drops directions
    margin = min(float(np.min(np.abs(x.rho - x.tol)) / x.tol) for x in res)
    assert margin > 1e-4                                  # no rho sits at the threshold
    h = m.LowRankHistory(128, r, 480, storage=torch.float32)
    _fold_all(m, h, X, 16, torch.float32, tau_rel=tau)
    U, s, B, pos, (k, n, folds, st) = state(h)
    assert (k, n, folds, st) == (len(so), 480, 30, 0)
    np.testing.assert_allclose(s, so, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U, s, B), of.low_rank_product(Uo, so, Bo)) < 1e-4
    assert np.array_equal(pos, np.arange(480))


def test_single_fold_keeps_no_residual_direction():
    """p = 0: every residual singular value is below the threshold; the fold only rotates the old
    basis, and the new rows' coordinates are their projections."""
    m = kv()
    X = stored(synth.lowrank_rows(480, 128, 1.0, 0.01, seed=0), torch.float32)
    _, _, _, res = of.fold_stream(X, 16, 16, tau_rel=3e-2)
    i = next(j for j, x in enumerate(res) if x.p == 0)
    h = m.LowRankHistory(128, 16, 480, storage=torch.float32)
    _fold_all(m, h, X, 16, torch.float32, tau_rel=3e-2, nblocks=i)
    U0, s0, B0, _, _ = state(h)
    _fold_all(m, h, X, 16, torch.float32, tau_rel=3e-2, start=i, nblocks=1)
    U1, s1, B1, _, (k, n, _, st) = state(h)
    ref = of.fold_block(U0, s0, B0, X[i * 16:(i + 1) * 16], 16, tau_rel=3e-2)
    assert ref.p == 0 and st == 0 and (k, n) == (ref.k_new, (i + 1) * 16)
    np.testing.assert_allclose(s1, ref.sigma, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U1, s1, B1),
                      of.low_rank_product(ref.U, ref.sigma, ref.B)) < 1e-4
    # With no new direction the new rows are represented by their projection on the old basis.
    proj = X[i * 16:(i + 1) * 16] @ B0 @ B0.T
    assert of.rel_fro((U1[-16:] * s1) @ B1.T, proj) < 1e-4


def test_keys_and_values_with_different_ranks():
    """One sequence's K (spectrum i^-1.2, r = 16) and V (i^-0.6, r = 32) folded step by step in
    the same loop, each against its own oracle trajectory."""
    m = kv()
    XK = stored(synth.lowrank_rows(480, 128, 1.2, 0.01, seed=20), torch.float32)
    XV = stored(synth.lowrank_rows(480, 128, 0.6, 0.01, seed=21), torch.float32)
    hK = m.LowRankHistory(128, 16, 480, storage=torch.float32)
    hV = m.LowRankHistory(128, 32, 480, storage=torch.float32)
    XKd = torch.as_tensor(XK, dtype=torch.float32, device="cuda")
    XVd = torch.as_tensor(XV, dtype=torch.float32, device="cuda")
    for i in range(30):
        p = torch.arange(i * 16, (i + 1) * 16, dtype=torch.int32, device="cuda")
        m.fold_block(hK, XKd[i * 16:(i + 1) * 16].contiguous(), p)
        m.fold_block(hV, XVd[i * 16:(i + 1) * 16].contiguous(), p)
    for h, X, r in ((hK, XK, 16), (hV, XV, 32)):
        U, s, B, _, (k, n, _, st) = state(h)
        Uo, so, Bo, _ = of.fold_stream(X, 16, r)
        assert (k, n, st) == (r, 480, 0)
        np.testing.assert_allclose(s, so, rtol=1e-4)
        assert of.rel_fro(of.low_rank_product(U, s, B), of.low_rank_product(Uo, so, Bo)) < 1e-4


def test_rank512_block128_float32_trajectory():
    """Long-prompt compression shape: d = 1024, r = 512, b = 128 -- eight folds of value-like rows
    (spectrum i^-0.6, noise 0.02), the first four filling the rank budget without truncation."""
    m = kv()
    X = stored(synth.lowrank_rows(1024, 1024, 0.6, 0.02, seed=40), torch.float32)
    h = m.LowRankHistory(1024, 512, 1024, storage=torch.float32)
    _fold_all(m, h, X, 128, torch.float32)
    U, s, B, pos, (k, n, folds, st) = state(h)
    Uo, so, Bo, res = of.fold_stream(X, 128, 512)
    assert (k, n, folds, st) == (512, 1024, 8, 0)
    np.testing.assert_allclose(s, so, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U, s, B), of.low_rank_product(Uo, so, Bo)) < 1e-4
    assert np.array_equal(pos, np.arange(1024))
    # The first four folds add every direction: the history equals the rows (rank 512 fits).
    h2 = m.LowRankHistory(1024, 512, 512, storage=torch.float32)
    _fold_all(m, h2, X[:512], 128, torch.float32)
    U2, s2, B2, _, (k2, _, _, _) = state(h2)
    assert k2 == 512
    assert of.rel_fro(of.low_rank_product(U2, s2, B2), X[:512]) < 1e-4


def test_rank512_block128_bf16_single_fold():
    """One b = 128 fold into a GPU-built r = 512 bf16 history of 1024 rows; the oracle starts from
    the stored state."""
    m = kv()
    X = stored(synth.lowrank_rows(1152, 1024, 0.6, 0.02, seed=41), torch.bfloat16)
    h = m.LowRankHistory(1024, 512, 1152, storage=torch.bfloat16)
    _fold_all(m, h, X, 128, torch.bfloat16, nblocks=8)
    U0, s0, B0, _, (k0, n0, _, st0) = state(h)
    assert (k0, n0, st0) == (512, 1024, 0)
    _fold_all(m, h, X, 128, torch.bfloat16, start=8, nblocks=1)
    U1, s1, B1, pos, (k1, n1, _, st1) = state(h)
    ref = of.fold_block(U0, s0, B0, X[1024:], 512)
    assert (k1, n1, st1) == (ref.k_new, 1152, 0)
    np.testing.assert_allclose(s1, ref.sigma, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U1, s1, B1),
                      of.low_rank_product(ref.U, ref.sigma, ref.B)) < 2e-2
    assert np.array_equal(pos, np.arange(1152))
