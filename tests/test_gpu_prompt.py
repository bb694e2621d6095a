"""GPU parity of the prompt compression (Algorithm 1 step 7) and of the long-prompt flow through
the C ABI: prompt-block selection on post-RoPE keys, the prefill partition of each side, the
compression of the remaining prompt rows into the side's history, then decode steps of the cache
policy, against the float64 oracle.

Tolerances: float32 factors 1e-4 (relative Frobenius of the represented rows, singular values
1e-4 relative); positions and row counts bit-exact.
"""

import numpy as np
import pytest
import torch

from gpu_util import kv, np64, state, stored
from oracle import fold as of
from oracle import policy as op
from oracle import reconstruct as orec
from oracle import rope as orope
from oracle import select as osel
import synth

pytestmark = pytest.mark.gpu


def _oracle_blocks(X, b, r, tau=0.0):
    """The oracle's block folds in the device's order: full blocks of b rows, then the short rest."""
    U, s, B = of.empty_history(X.shape[1])
    n = X.shape[0]
    for i in range(0, n, b):
        res = of.fold_block(U, s, B, X[i:min(i + b, n)], r, tau)
        U, s, B = res.U, res.sigma, res.B
    return U, s, B


def test_compress_prompt_block_folds_with_short_last_blocks():
    """Three histories in one call: 1000 rows (15 blocks of 64 and 40 more), 525 rows (8 blocks and
    13 more: a last block of 13 rows padded to 16) and 320 rows (5 whole blocks)."""
    m = kv()
    d, r, b = 256, 32, 64
    ns = (1000, 525, 320)
    Xs = [stored(synth.lowrank_rows(n, d, 1.0, 0.02, seed=300 + n), torch.float32) for n in ns]
    hs = [m.LowRankHistory(d, r, n + 16, storage=torch.float32) for n in ns]
    rows = [torch.as_tensor(X, dtype=torch.float32, device="cuda") for X in Xs]
    pos = [torch.as_tensor(7 + 3 * np.arange(n), dtype=torch.int32, device="cuda") for n in ns]
    m.compress_prompt(hs, rows, pos, block=b)
    for h, X, n in zip(hs, Xs, ns):
        U, s, B, p, (k, nn, _, st) = state(h)
        assert st == 0 and nn == n and k == r
        np.testing.assert_array_equal(p, 7 + 3 * np.arange(n))
        Uo, so, Bo = _oracle_blocks(X, b, r)
        np.testing.assert_allclose(s, so, rtol=1e-4)
        assert of.rel_fro(of.low_rank_product(U, s, B), of.low_rank_product(Uo, so, Bo)) < 1e-4


def test_compress_prompt_reaches_the_batch_svd_when_no_fold_truncates_early():
    """600 rows at r = 512 with folds of 128 rows (the long-prompt workload's rank and block): only
    the last fold truncates, so the history is the rank-512 truncated SVD of all the rows."""
    m = kv()
    d, r, b, n = 1024, 512, 128, 600
    X = stored(synth.lowrank_rows(n, d, 0.6, 0.02, seed=310), torch.float32)
    h = m.LowRankHistory(d, r, n + 8, storage=torch.float32)
    m.compress_prompt(h, torch.as_tensor(X, dtype=torch.float32, device="cuda"),
                      torch.arange(n, dtype=torch.int32, device="cuda"), block=b)
    U, s, B, _, (k, nn, _, st) = state(h)
    Ut, st_, Bt = of.truncated_svd(X, r)
    assert st == 0 and (k, nn) == (r, n)
    np.testing.assert_allclose(s, st_, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U, s, B), of.low_rank_product(Ut, st_, Bt)) < 1e-4


def test_long_prompt_flow_through_the_c_abi():
    """A 3000-token prompt: selection (8-token blocks, 4 per head here, union over 8 heads, 4-block
    suffix, values within 32 tokens) on post-RoPE keys with outlier blocks, the keys' pre-RoPE rows
    being the inverse rotation; each side's prefill partition; iskv_compress_prompt at r = 512 in
    blocks of 128 (about 2700 key rows and 1250 value rows: an incremental compression, compared
    with the oracle's block folds in the same order); then 400 decode steps (W = 128, b = 128,
    re-orthogonalisation every 256 folded rows) through the cache step. The schedule, positions,
    exact tables, factors and reconstruction against the policy oracle."""
    m = kv()
    L, H, hd, W, b, r, R, T = 3000, 8, 128, 128, 128, 512, 256, 400
    d = H * hd
    post, _ = synth.outlier_prompt_keys(L, H, hd, seed=320)
    post = stored(post, torch.float32)
    keys_dev = torch.as_tensor(post, dtype=torch.float32, device="cuda")
    sel = m.select_prompt_blocks(keys_dev, 8, 4, 4, 32)
    torch.cuda.synchronize()
    ref_sel = osel.select_prompt_blocks(post, 8, 4, 4, 32)
    c = sel["counts"].cpu().numpy()
    PK = sel["P_K"][:c[0]].cpu().numpy()
    PV = sel["P_V"][:c[1]].cpu().numpy()
    np.testing.assert_array_equal(PK, ref_sel["P_K"])
    np.testing.assert_array_equal(PV, ref_sel["P_V"])
    XK = stored(np.vstack([orope.apply_rope(post.reshape(L, d), -np.arange(L), H, hd, 500000.0),
                           synth.lowrank_rows(T, d, 1.2, 0.02, seed=321)]), torch.float32)
    XV = stored(synth.lowrank_rows(L + T, d, 0.6, 0.02, seed=322), torch.float32)
    n_cap = L + T + 8
    for kind, X, P, w0 in (("K", XK, PK, 0), ("V", XV, PV, W)):
        Xd = torch.as_tensor(X, dtype=torch.float32, device="cuda")
        t = m.ExactTable(d, L + 2 * W, window=W, block=b, reorth_rows=R, dtype=torch.float32)
        comp_rows, comp_pos = m.cache_prefill(t, Xd[:L].contiguous(),
                                              torch.as_tensor(P, dtype=torch.int32,
                                                              device="cuda"), w0)
        h = m.LowRankHistory(d, r, n_cap, storage=torch.float32)
        m.compress_prompt(h, comp_rows, comp_pos, block=b)
        assert comp_pos.numel() > r + b                # folds truncate before the last one
        init = _oracle_blocks(X[comp_pos.cpu().numpy()], b, r)
        ref = op.run_decode(X[:L], X[L:], P, w0, W, b, r, R, init_history=init)
        batch = m.CacheBatch([t], [h])
        for i in range(T):
            folded, reorthed = batch.step(Xd[L + i:L + i + 1].contiguous())
            acts = [a[0] for a in ref["steps"][i]]
            assert folded[0] == (1 if "fold" in acts else 0) and reorthed[0] == ("reorth" in acts)
        assert any(a[0] == "reorth" for acts in ref["steps"] for a in acts)
        U, s, B, pos, (k, n, _, st) = state(h)
        Uo, so, Bo, poso = ref["history"]
        assert st == 0 and (k, n) == (so.shape[0], poso.shape[0])
        np.testing.assert_array_equal(pos, poso)
        np.testing.assert_allclose(s, so, rtol=1e-4)
        assert of.rel_fro(of.low_rank_product(U, s, B), of.low_rank_product(Uo, so, Bo)) < 1e-4
        rows, epos = t.exact()
        assert epos.cpu().tolist() == ref["exact"][1].tolist()
        out = m.reconstruct(h, rows, epos, L + T, H, hd, kind == "K", 500000.0,
                            out_dtype=torch.float32)
        want = orec.reconstruct(Uo, so, Bo, poso, ref["exact"][0], ref["exact"][1], L + T, H, hd,
                                kind == "K", 500000.0)
        assert of.rel_fro(np64(out), want) < 1e-4
