"""GPU parity of the block fold (Algorithm 2) against the float64 oracle.

Tolerances: float32 storage -> relative Frobenius error of the reconstruction <= 1e-4; bf16
storage -> <= 2e-2 (about 2^-8 relative rounding per stored entry, accumulated over the fold's
rotations); singular values <= 1e-4 relative in both (they are float32 in both modes); positions
bit-exact.
"""

import numpy as np
import pytest
import torch

from gpu_util import bit, kv, np64, set_state, state, stored, synthetic_history
from oracle import fold as of
import synth

pytestmark = pytest.mark.gpu


def _fold_rows(m, h, X, b, nblocks, start=0, dtype=torch.float32):
    Xd = torch.as_tensor(X, dtype=dtype, device="cuda")
    for i in range(start, start + nblocks):
        F = Xd[i * b:(i + 1) * b].contiguous()
        p = torch.arange(i * b, (i + 1) * b, dtype=torch.int32, device="cuda")
        m.fold_block(h, F, p)


def test_config1_trajectory_float32():
    """Tiny single-matrix fold: d = 128, 512 rows, b = 16, r = 16, w = 32 -> 30 folds."""
    m = kv()
    X = stored(synth.lowrank_rows(512, 128, 1.0, 0.01, seed=0), torch.float32)
    h = m.LowRankHistory(128, 16, 512, storage=torch.float32)
    _fold_rows(m, h, X, 16, 30)
    U, s, B, pos, (k, n, folds, st) = state(h)
    assert (k, n, folds, st) == (16, 480, 30, 0)
    Uo, so, Bo, _ = of.fold_stream(X[:480], 16, 16)
    assert of.rel_fro(of.low_rank_product(U, s, B), of.low_rank_product(Uo, so, Bo)) < 1e-4
    np.testing.assert_allclose(s, so, rtol=1e-4)
    assert np.array_equal(pos, np.arange(480))


def test_noiseless_rank_fits_reproduces_batch_svd():
    m = kv()
    X = stored(synth.lowrank_rows(512, 128, 1.0, 0.0, seed=0, rank=12), torch.float32)
    h = m.LowRankHistory(128, 16, 512, storage=torch.float32)
    _fold_rows(m, h, X, 16, 30)
    U, s, B, pos, (k, n, folds, st) = state(h)
    assert k == 12 and n == 480 and st == 0          # numerically-zero residuals are not added
    assert of.rel_fro(of.low_rank_product(U, s, B), X[:480]) < 1e-4
    _, s_ref, _ = of.truncated_svd(X[:480], 12)
    np.testing.assert_allclose(s, s_ref, rtol=1e-4)


def test_full_width_rank_skips_residual():
    m = kv()
    X = stored(synth.lowrank_rows(96, 16, 0.5, 0.05, seed=3), torch.float32)
    h = m.LowRankHistory(16, 16, 96, storage=torch.float32)
    _fold_rows(m, h, X, 8, 12)
    U, s, B, _, (k, n, _, st) = state(h)
    assert k == 16 and n == 96 and st == 0
    assert of.rel_fro(of.low_rank_product(U, s, B), X) < 1e-4
    Uo, so, Bo, _ = of.fold_stream(X, 8, 16)
    np.testing.assert_allclose(s, so, rtol=1e-4)


@pytest.mark.parametrize("storage,tol", [(torch.float32, 1e-4), (torch.bfloat16, 2e-2)])
def test_single_fold_config2_shape(storage, tol):
    """One fold at d = 1024, r = 256, b = 64 from a GPU-built history; the oracle starts from the
    exact stored state (upcast)."""
    m = kv()
    d, r, b = 1024, 256, 64
    X = stored(synth.lowrank_rows(26 * b, d, 1.2, 0.02, seed=1), storage)
    h = m.LowRankHistory(d, r, 2048, storage=storage)
    _fold_rows(m, h, X, b, 25, dtype=storage)
    U0, s0, B0, _, (k0, n0, _, st0) = state(h)
    assert st0 == 0 and k0 == r and n0 == 25 * b
    F = X[25 * b:26 * b]
    _fold_rows(m, h, X, b, 1, start=25, dtype=storage)
    U1, s1, B1, pos, (k1, n1, _, st1) = state(h)
    assert st1 == 0 and k1 == r and n1 == 26 * b
    res = of.fold_block(U0, s0, B0, F, r)
    assert res.p == b
    np.testing.assert_allclose(s1, res.sigma, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U1, s1, B1), of.low_rank_product(res.U, res.sigma,
                                                                              res.B)) < tol
    assert np.array_equal(pos, np.arange(26 * b))


def test_full_size_fold_sampled_rows():
    """n = 16384, d = 1024, r = 256, b = 64, bf16 storage -- the benchmark's per-history shape.
    sigma in full, reconstructed rows on a sample."""
    m = kv()
    n, d, r, b = 16384, 1024, 256, 64
    U0, s0, B0 = synthetic_history(n, d, r, seed=5, dtype=torch.bfloat16)
    h = m.LowRankHistory(d, r, n + b, storage=torch.bfloat16)
    set_state(h, U0, s0, B0, np.arange(n))
    g = np.random.Generator(np.random.PCG64(6))
    coords = g.standard_normal((b, r)) * np.arange(1, r + 1) ** -1.2
    F = stored(coords @ B0.T + 0.02 * g.standard_normal((b, d)), torch.bfloat16)
    m.fold_block(h, torch.as_tensor(F, dtype=torch.bfloat16, device="cuda"),
                 torch.arange(n, n + b, dtype=torch.int32, device="cuda"))
    k1, n1, _, st = h.status()
    assert (k1, n1, st) == (r, n + b, 0)
    res = of.fold_block(U0, s0, B0, F, r)
    s1 = np64(h.sigma)
    np.testing.assert_allclose(s1, res.sigma, rtol=1e-4)
    rows = np.r_[g.choice(n, 512, replace=False), np.arange(n, n + b)]
    U1 = np64(h.U[torch.as_tensor(rows)])
    B1 = np64(h.B)
    got = (U1 * s1) @ B1.T
    ref = (res.U[rows] * res.sigma) @ res.B.T
    assert of.rel_fro(got, ref) < 2e-2


def test_batched_equals_single():
    m = kv()
    d, r, b = 256, 64, 32
    Xs = [stored(synth.lowrank_rows(6 * b, d, 1.0, 0.02, seed=10 + i), torch.bfloat16)
          for i in range(3)]
    single = [m.LowRankHistory(d, r, 6 * b) for _ in range(3)]
    batched = [m.LowRankHistory(d, r, 6 * b) for _ in range(3)]
    for i in range(3):
        _fold_rows(m, single[i], Xs[i], b, 6, dtype=torch.bfloat16)
    Xd = [torch.as_tensor(X, dtype=torch.bfloat16, device="cuda") for X in Xs]
    for j in range(6):
        Fs = [x[j * b:(j + 1) * b].contiguous() for x in Xd]
        ps = [torch.arange(j * b, (j + 1) * b, dtype=torch.int32, device="cuda")] * 3
        m.fold_block_batched(batched, Fs, ps)
    for a, c in zip(single, batched):
        assert a.status() == c.status()
        assert torch.equal(a.U, c.U) and torch.equal(a.B, c.B) and torch.equal(a.sigma, c.sigma)


def test_capacity_overflow_is_a_recorded_no_op():
    m = kv()
    X = stored(synth.lowrank_rows(48, 128, 1.0, 0.01, seed=0), torch.float32)
    h = m.LowRankHistory(128, 16, 32, storage=torch.float32)
    _fold_rows(m, h, X, 16, 2)
    before = (h.U.clone(), h.B.clone(), h.sigma.clone())
    _fold_rows(m, h, X, 16, 1, start=2)
    k, n, folds, st = h.status()
    assert n == 32 and folds == 2 and st == bit(4)
    assert torch.equal(before[0], h.U) and torch.equal(before[1], h.B)


def test_nonfinite_block_is_flagged():
    m = kv()
    X = stored(synth.lowrank_rows(32, 128, 1.0, 0.01, seed=0), torch.float32)
    X[20, 5] = np.nan
    h = m.LowRankHistory(128, 16, 64, storage=torch.float32)
    _fold_rows(m, h, X, 16, 2)
    _, _, _, st = h.status()
    assert st & bit(5)


def test_fold_after_event_waits_before_writing_factors():
    """iskv_fold_block_batched_after: a reconstruction issued on another stream, held back there by
    a long spin, must read the factors from before the fold; the fold's result equals the plain
    fold's bit for bit."""
    m = kv()
    d, r, b, n = 256, 64, 64, 1024
    import synth
    X = stored(synth.lowrank_rows(n + b, d, 1.0, 0.02, seed=41), torch.float32)
    Xd = torch.as_tensor(X, dtype=torch.bfloat16, device="cuda")
    pos = torch.arange(n + b, dtype=torch.int32, device="cuda")

    def built():
        h = m.LowRankHistory(d, r, n + b, storage=torch.bfloat16)
        for i in range(0, n, b):
            m.fold_block(h, Xd[i:i + b].contiguous(), pos[i:i + b].contiguous())
        return h

    ha, hb = built(), built()
    exact = torch.zeros(0, d, dtype=torch.bfloat16, device="cuda")
    epos = torch.zeros(0, dtype=torch.int32, device="cuda")
    # The two streams' calls in flight together take workspaces of their own.
    wsr = torch.empty(m.reconstruct_workspace_size(1, d, r), dtype=torch.uint8, device="cuda")
    wsf = torch.empty(m.fold_workspace_size(1, d, r, b), dtype=torch.uint8, device="cuda")
    want = m.reconstruct(ha, exact, epos, n, 2, 128, False, ws=wsr)  # before any new fold
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        torch.cuda._sleep(200_000_000)                               # ~0.1 s at 2 GHz
        got = m.reconstruct(hb, exact, epos, n, 2, 128, False, ws=wsr, stream=side)
        ev = torch.cuda.Event()
        ev.record(side)
    F = Xd[n:n + b].contiguous()
    m.fold_block_batched([hb], [F], [pos[n:n + b].contiguous()], ws=wsf, factors_ready=ev)
    m.fold_block(ha, F, pos[n:n + b].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    for x, y in ((ha.U, hb.U), (ha.B, hb.B), (ha.sigma, hb.sigma), (ha.meta, hb.meta)):
        assert torch.equal(x, y)
