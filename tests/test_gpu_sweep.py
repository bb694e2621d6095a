"""GPU parity over the sweep shapes: rank budget r in {128, 256, 384} x fold block b in
{32, 64, 128} at d = 1024, bf16 storage -- one fold from a known state, then a
re-orthogonalisation of the result, each against the float64 oracle started from the exact stored
state. The spectrum decays like i^-0.6 (value-like), which leaves a clear gap at the truncation
boundary (the precondition is asserted), so the kept subspace is well defined."""

import numpy as np
import pytest
import torch

from gpu_util import kv, np64, set_state, state, stored, synthetic_history
from oracle import fold as of
from oracle import reorth as oreo

pytestmark = pytest.mark.gpu

N, D = 2048, 1024


def _setup(m, r, b, storage):
    U0, s0, B0 = synthetic_history(N, D, r, seed=100 + r + b, exponent=0.6, dtype=storage)
    g = np.random.Generator(np.random.PCG64(7 + r + b))
    coords = g.standard_normal((b, r)) * np.arange(1, r + 1) ** -0.6 * 3
    F = stored(coords @ B0.T + 0.002 * g.standard_normal((b, D)), storage)
    h = m.LowRankHistory(D, r, N + b, storage=storage)
    set_state(h, U0, s0, B0, np.arange(N))
    return h, U0, s0, B0, F


@pytest.mark.parametrize("r", [128, 256, 384])
@pytest.mark.parametrize("b", [32, 64, 128])
def test_fold_then_reorth_sweep(r, b):
    m = kv()
    h, U0, s0, B0, F = _setup(m, r, b, torch.bfloat16)
    m.fold_block(h, torch.as_tensor(F, dtype=torch.bfloat16, device="cuda"),
                 torch.arange(N, N + b, dtype=torch.int32, device="cuda"))
    U1, s1, B1, pos, (k1, n1, folds, st) = state(h)
    res = of.fold_block(U0, s0, B0, F, r)
    cs = res.core_sigma
    assert (cs[res.k_new - 1] - cs[res.k_new]) / cs[0] > 1e-3  # precondition: a clear gap
    assert (k1, n1, folds, st) == (res.k_new, N + b, 1, 0)
    np.testing.assert_allclose(s1, res.sigma, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U1, s1, B1),
                      of.low_rank_product(res.U, res.sigma, res.B)) < 2e-2
    assert np.array_equal(pos, np.arange(N + b))

    m.reorth(h)
    U2, s2, B2, _, (k2, n2, folds2, st2) = state(h)
    assert (k2, n2, folds2, st2) == (k1, n1, 0, 0)
    Ur, sr, Br = oreo.reorth(U1, s1, B1)
    np.testing.assert_allclose(s2, sr, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U2, s2, B2), of.low_rank_product(U1, s1, B1)) < 2e-2


@pytest.mark.parametrize("r,b", [(384, 128), (128, 32)])
def test_fold_sweep_float32(r, b):
    """The same fold in float32 storage, at the float32 tolerance."""
    m = kv()
    h, U0, s0, B0, F = _setup(m, r, b, torch.float32)
    m.fold_block(h, torch.as_tensor(F, dtype=torch.float32, device="cuda"),
                 torch.arange(N, N + b, dtype=torch.int32, device="cuda"))
    U1, s1, B1, _, (k1, n1, _, st) = state(h)
    res = of.fold_block(U0, s0, B0, F, r)
    assert (k1, n1, st) == (res.k_new, N + b, 0)
    np.testing.assert_allclose(s1, res.sigma, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U1, s1, B1),
                      of.low_rank_product(res.U, res.sigma, res.B)) < 1e-4


@pytest.mark.parametrize("r,storage,tol", [(512, torch.float32, 1e-4), (512, torch.bfloat16, 2e-2),
                                            (400, torch.bfloat16, 2e-2)])
def test_reorth_at_the_long_prompt_rank(r, storage, tol):
    """Re-orthogonalisation at r = 512 (the long-prompt workload's rank) and at a rank that is not a
    multiple of 64, from a drifted state (factors perturbed off orthonormality), against the
    oracle: singular values 1e-4, the product kept, the factors orthonormal again."""
    m = kv()
    n = 2048
    U0, s0, B0 = synthetic_history(n, D, r, seed=200 + r, exponent=0.6, dtype=torch.float32)
    g = np.random.Generator(np.random.PCG64(201 + r))
    U0 = stored(U0 + 2e-3 * g.standard_normal(U0.shape) / np.sqrt(n), storage)
    B0 = stored(B0 + 2e-3 * g.standard_normal(B0.shape) / np.sqrt(D), storage)
    h = m.LowRankHistory(D, r, n, storage=storage)
    set_state(h, U0, s0, B0, np.arange(n))
    m.reorth(h)
    U, s, B, _, (k, nn, folds, st) = state(h)
    assert (k, nn, folds, st) == (r, n, 0, 0)
    Ur, sr, Br = oreo.reorth(U0, s0, B0)
    np.testing.assert_allclose(s, sr, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U, s, B), of.low_rank_product(U0, s0, B0)) < tol
    if storage == torch.float32:
        assert oreo.orthogonality_error(U) < 1e-3 and oreo.orthogonality_error(B) < 1e-3
