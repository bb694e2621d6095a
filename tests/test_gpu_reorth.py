"""GPU parity of re-orthogonalisation (Section 4.4) against the float64 oracle."""

import numpy as np
import pytest
import torch

from gpu_util import kv, set_state, state, stored
from oracle import fold as of
from oracle import reorth as oreo

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("storage,tol", [(torch.float32, 1e-4), (torch.bfloat16, 2e-2)])
def test_reorth_parity(storage, tol):
    m = kv()
    n, d, r, k = 4096, 1024, 256, 256
    g = np.random.Generator(np.random.PCG64(31))
    U = stored(np.linalg.qr(g.standard_normal((n, k)))[0] + 2e-3 * g.standard_normal((n, k)) /
               np.sqrt(n), storage)
    B = stored(np.linalg.qr(g.standard_normal((d, k)))[0] + 2e-3 * g.standard_normal((d, k)) /
               np.sqrt(d), storage)
    s = stored(np.sqrt(n) * np.arange(1, k + 1) ** -1.0, torch.float32)
    h = m.LowRankHistory(d, r, n, storage=storage)
    set_state(h, U, s, B, np.arange(n), folds=16)
    m.reorth(h)
    U2, s2, B2, _, (k2, n2, folds, st) = state(h)
    assert (k2, n2, folds, st) == (k, n, 0, 0)
    Ur, sr, Br = oreo.reorth(U, s, B)
    np.testing.assert_allclose(s2, sr, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U2, s2, B2), of.low_rank_product(U, s, B)) < tol
    if storage == torch.float32:
        assert oreo.orthogonality_error(U2) < 1e-4
        assert oreo.orthogonality_error(B2) < 1e-4
    else:
        # bf16 factors are orthonormal up to bf16 rounding: the floor is the oracle's orthonormal
        # result rounded to bf16. The tensor-core rotation applies a bf16 rotation matrix, which
        # adds about as much again, hence the factor 1.5.
        for got, ref in ((U2, Ur), (B2, Br)):
            assert oreo.orthogonality_error(got) < 1.5 * oreo.orthogonality_error(
                stored(ref, torch.bfloat16))


def test_reorth_bf16_removes_drift():
    """Factors drifted ten times further than in the parity test come back near orthonormal."""
    m = kv()
    n, d, r, k = 4096, 1024, 256, 256
    g = np.random.Generator(np.random.PCG64(37))
    U = stored(np.linalg.qr(g.standard_normal((n, k)))[0] + 2e-2 * g.standard_normal((n, k)) /
               np.sqrt(n), torch.bfloat16)
    B = stored(np.linalg.qr(g.standard_normal((d, k)))[0] + 2e-2 * g.standard_normal((d, k)) /
               np.sqrt(d), torch.bfloat16)
    s = stored(np.sqrt(n) * np.arange(1, k + 1) ** -1.0, torch.float32)
    h = m.LowRankHistory(d, r, n, storage=torch.bfloat16)
    set_state(h, U, s, B, np.arange(n), folds=16)
    m.reorth(h)
    U2, s2, B2, _, (_, _, _, st) = state(h)
    assert st == 0
    Ur, sr, Br = oreo.reorth(U, s, B)
    np.testing.assert_allclose(s2, sr, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U2, s2, B2), of.low_rank_product(U, s, B)) < 2e-2
    # The rotation matrices are bf16 tensor-core operands, so the result is orthonormal to about
    # 2^-9 ||T||_F (~0.04 here, per-pair cosines ~1e-4) rather than to the floor of bf16 rounding
    # of the factors alone (~0.01).
    for got, ref, before in ((U2, Ur, U), (B2, Br, B)):
        err = oreo.orthogonality_error(got)
        assert err < 5.0 * oreo.orthogonality_error(stored(ref, torch.bfloat16))
        assert err < 0.4 * oreo.orthogonality_error(before)


def test_reorth_partial_rank_after_folds():
    m = kv()
    import synth
    X = stored(synth.lowrank_rows(512, 128, 1.0, 0.0, seed=0, rank=12), torch.float32)
    h = m.LowRankHistory(128, 16, 512, storage=torch.float32)
    Xd = torch.as_tensor(X, dtype=torch.float32, device="cuda")
    for i in range(10):
        m.fold_block(h, Xd[i * 16:(i + 1) * 16].contiguous(),
                     torch.arange(i * 16, (i + 1) * 16, dtype=torch.int32, device="cuda"))
    U, s, B, _, (k, n, _, _) = state(h)
    m.reorth(h)
    U2, s2, B2, _, (k2, n2, folds, st) = state(h)
    assert (k2, n2, folds, st) == (k, n, 0, 0)
    assert of.rel_fro(of.low_rank_product(U2, s2, B2), of.low_rank_product(U, s, B)) < 1e-4


@pytest.mark.parametrize("f_dtype", [torch.float32, torch.bfloat16])
def test_bf16_partial_rank_with_stale_workspace(f_dtype):
    """A bf16 history of rank k < r_max = 128: the tensor-core projection (bf16 blocks) and
    rotations of the fold and of the re-orthogonalisation run over all r columns and whole
    r x (r + b) and r x r operands, so with every workspace filled with NaN bytes before the call,
    the columns beyond k must come out zero and the factors finite; the represented rows follow
    the oracle's folds (tau_rel = 1e-2 keeps the rank of the rank-40 rows) and are unchanged by the
    re-orthogonalisation."""
    import synth
    m = kv()
    d, r, b, n = 256, 128, 64, 512
    X = stored(synth.lowrank_rows(n, d, 1.0, 0.0, seed=9, rank=40), f_dtype)
    h = m.LowRankHistory(d, r, n, storage=torch.bfloat16)
    Xd = torch.as_tensor(X, dtype=f_dtype, device="cuda")
    wsf = torch.empty(m.fold_workspace_size(1, d, r, b), dtype=torch.uint8, device="cuda")
    Uo, so, Bo = of.empty_history(d)
    for i in range(n // b):
        wsf.fill_(255)
        m.fold_block(h, Xd[i * b:(i + 1) * b].contiguous(),
                     torch.arange(i * b, (i + 1) * b, dtype=torch.int32, device="cuda"),
                     tau_rel=1e-2, ws=wsf)
        res = of.fold_block(Uo, so, Bo, X[i * b:(i + 1) * b], r, 1e-2)
        Uo, so, Bo = res.U, res.sigma, res.B
    U, s, B, _, (k, nn, _, st) = state(h)
    assert st == 0 and nn == n and k == so.shape[0] and k < r
    assert bool((h.U[:n, k:] == 0).all()) and bool((h.B[:, k:] == 0).all())
    assert bool(torch.isfinite(h.U[:n]).all()) and bool(torch.isfinite(h.B).all())
    assert of.rel_fro(of.low_rank_product(U, s, B), of.low_rank_product(Uo, so, Bo)) < 2e-2
    wsr = torch.full((m.reorth_workspace_size(1, d, r, n),), 255, dtype=torch.uint8,
                     device="cuda")
    m.reorth(h, ws=wsr)
    U2, s2, B2, _, (k2, n2, folds, st2) = state(h)
    assert (k2, n2, folds, st2) == (k, n, 0, 0)
    assert bool((h.U[:n, k:] == 0).all()) and bool((h.B[:, k:] == 0).all())
    assert bool(torch.isfinite(h.U[:n]).all()) and bool(torch.isfinite(h.B).all())
    assert of.rel_fro(of.low_rank_product(U2, s2, B2), of.low_rank_product(U, s, B)) < 2e-2
