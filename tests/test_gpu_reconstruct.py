"""GPU parity of reconstruction + RoPE (Algorithm 3 steps 7-8) against the float64 oracle."""

import numpy as np
import pytest
import torch

from gpu_util import bit, kv, np64, set_state, stored, synthetic_history
from oracle import fold as of
from oracle import reconstruct as orec

pytestmark = pytest.mark.gpu


def _case(m, n, n_exact, k, storage, seed, d=1024, r=256):
    U, s, B = synthetic_history(n, d, r, seed=seed, dtype=storage)
    U, s, B = U[:, :k], s[:k], B[:, :k]
    g = np.random.Generator(np.random.PCG64(seed + 1))
    perm = g.permutation(n + n_exact)
    pos, epos = perm[:n], perm[n:]
    exact = g.standard_normal((n_exact, d))
    h = m.LowRankHistory(d, r, n, storage=storage)
    set_state(h, U, s, B, pos)
    return h, U, s, B, pos, epos, exact


@pytest.mark.parametrize("storage,out_dtype,rope,tol", [
    (torch.float32, torch.float32, True, 1e-5),
    (torch.float32, torch.float32, False, 1e-5),
    (torch.bfloat16, torch.bfloat16, True, 2e-2),
    (torch.bfloat16, torch.float32, True, 1e-5),
])
def test_reconstruct_parity(storage, out_dtype, rope, tol):
    m = kv()
    n, n_exact, H, hd = 3000, 200, 8, 128
    h, U, s, B, pos, epos, exact = _case(m, n, n_exact, 256, storage, seed=21)
    ex = stored(exact, out_dtype if out_dtype == torch.bfloat16 else torch.float32)
    out = m.reconstruct(h, torch.as_tensor(ex, dtype=torch.float32, device="cuda"),
                        torch.as_tensor(epos, dtype=torch.int32, device="cuda"), n + n_exact, H,
                        hd, rope, 500000.0, out_dtype=out_dtype)
    ref = orec.reconstruct(U, s, B, pos, ex, epos, n + n_exact, H, hd, rope, 500000.0)
    assert of.rel_fro(np64(out), ref) < tol
    assert h.status()[3] == 0


def test_partial_rank_and_untouched_rows():
    m = kv()
    n, H, hd = 500, 8, 128
    h, U, s, B, pos, epos, exact = _case(m, n, 0, 100, torch.float32, seed=22)
    out = torch.full((n + 50, 1024), 7.0, dtype=torch.float32, device="cuda")
    pos2 = np.random.Generator(np.random.PCG64(3)).permutation(n)  # rows n.. stay untouched
    h.pos[:n] = torch.as_tensor(pos2, dtype=torch.int32)
    m.reconstruct(h, None, None, n + 50, H, hd, True, 500000.0, out=out)
    ref = orec.reconstruct(U, s, B, pos2, np.zeros((0, 1024)), np.zeros(0, dtype=int), n + 50, H,
                           hd, True, 500000.0, fill=7.0)
    assert of.rel_fro(np64(out), ref) < 1e-5
    assert torch.all(out[n:] == 7.0)


def test_out_of_range_position_is_skipped_and_flagged():
    m = kv()
    h, U, s, B, pos, epos, exact = _case(m, 64, 0, 32, torch.float32, seed=23)
    h.pos[5] = 10_000
    out = torch.zeros(64, 1024, device="cuda")
    m.reconstruct(h, None, None, 64, 8, 128, False, out=out, out_dtype=torch.float32)
    assert h.status()[3] & bit(2)


def test_full_size_sampled_rows():
    """n = 16384 compressed rows at d = 1024, r = 256 (bf16) plus 128 exact rows, RoPE theta
    500000; compare a sample of rows against the oracle's row-by-row definition."""
    m = kv()
    n, n_exact, H, hd = 16384, 128, 8, 128
    h, U, s, B, pos, epos, exact = _case(m, n, n_exact, 256, torch.bfloat16, seed=24)
    ex = stored(exact, torch.bfloat16)
    out = m.reconstruct(h, torch.as_tensor(ex, dtype=torch.bfloat16, device="cuda"),
                        torch.as_tensor(epos, dtype=torch.int32, device="cuda"), n + n_exact, H,
                        hd, True, 500000.0, out_dtype=torch.bfloat16)
    g = np.random.Generator(np.random.PCG64(25))
    rows = g.choice(n, 400, replace=False)
    ref = orec.reconstruct(U[rows], s, B, pos[rows], ex[:16], epos[:16], n + n_exact, H, hd, True,
                           500000.0)
    got = np64(out)
    sel = np.r_[pos[rows], epos[:16]]
    assert of.rel_fro(got[sel], ref[sel]) < 2e-2


@pytest.mark.parametrize("d,r,H", [(1024, 256, 8), (384, 128, 3), (512, 64, 4), (256, 192, 2)])
def test_batched_tensor_core_shapes(d, r, H):
    """Several bf16 histories in one call (row counts with ragged last tiles, one of a single row,
    one below full rank, keys and values mixed): every history's dense output against the oracle,
    rows at no position left as they were."""
    m = kv()
    ns, ks = [700, 1, 129, 256], [r, r, r - 17, r]
    hs, ref, outs, n_total = [], [], [], []
    for i, (n, k) in enumerate(zip(ns, ks)):
        k = min(k, n)  # a history's rank is at most its row count
        U, s, B = synthetic_history(n, d, r, seed=40 + i, dtype=torch.bfloat16)
        U, s, B = U[:, :k], s[:k], B[:, :k]
        g = np.random.Generator(np.random.PCG64(50 + i))
        nt = n + 37
        pos = g.permutation(nt)[:n]
        h = m.LowRankHistory(d, r, n + 5, storage=torch.bfloat16)
        set_state(h, U, s, B, pos)
        rope = i % 2 == 0
        ref.append(orec.reconstruct(U, s, B, pos, np.zeros((0, d)), np.zeros(0, dtype=int), nt, H,
                                    d // H, rope, 500000.0, fill=3.0))
        outs.append(torch.full((nt, d), 3.0, dtype=torch.bfloat16, device="cuda"))
        hs.append(h)
        n_total.append(nt)
    m.reconstruct_batched(hs, [None] * 4, [None] * 4, n_total, H, d // H,
                          [i % 2 == 0 for i in range(4)], 500000.0, outs=outs)
    for h, o, rf, n, nt in zip(hs, outs, ref, ns, n_total):
        got = np64(o)
        assert of.rel_fro(got, rf) < 2e-2
        untouched = np.setdiff1d(np.arange(nt), h.pos[:n].cpu().numpy())
        assert np.all(got[untouched] == 3.0)
        assert h.status()[3] == 0


def test_positions_in_order_with_gaps():
    """Rows stored in position order -- a gapped prefix (like compressed prompt rows around kept
    blocks) and then consecutive decode positions -- at n = 16384 (128 tiles per history, so a
    row's position usually advances by exactly one tile between units). Sampled rows against the
    oracle, each row to within bf16 output rounding."""
    m = kv()
    n, H, hd = 16384, 8, 128
    U, s, B = synthetic_history(n, 1024, 256, seed=26, dtype=torch.bfloat16)
    g = np.random.Generator(np.random.PCG64(27))
    head = np.sort(g.choice(12000, 6000, replace=False))          # gapped, increasing
    pos = np.r_[head, 12000 + np.arange(n - 6000)]                # then consecutive
    n_total = int(pos[-1]) + 1
    h = m.LowRankHistory(1024, 256, n, storage=torch.bfloat16)
    set_state(h, U, s, B, pos)
    out = m.reconstruct(h, None, None, n_total, H, hd, True, 500000.0, out_dtype=torch.bfloat16)
    rows = np.r_[g.choice(n, 600, replace=False), n - 1, 6000, 5999]
    ref = orec.reconstruct(U[rows], s, B, pos[rows], np.zeros((0, 1024)), np.zeros(0, dtype=int),
                           n_total, H, hd, True, 500000.0)[pos[rows]]
    got = np64(out)[pos[rows]]
    row_err = np.linalg.norm(got - ref, axis=1) / np.linalg.norm(ref, axis=1)
    assert row_err.max() < 4e-3
    assert h.status()[3] == 0
