"""Pins for the cache-policy oracle (Section 3.1, Section 3.2, Algorithm 1 steps 5-8, Algorithm 3
steps 1-6): a schedule worked by hand, a closed form, a reduction to the pinned block stream, the
partition invariants, and exact recovery of rank-deficient data."""

import json
import math
import os

import numpy as np
import pytest

from conftest import GOLDEN
from oracle import fold as of
from oracle import policy as op
from oracle import reconstruct as orec
import synth


def _golden():
    with open(os.path.join(GOLDEN, "policy_small.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden(), ids=lambda c: c["name"][:6])
def test_hand_worked_schedule(case):
    side, comp = op.new_side(case["L"], case["protected"], case["init_window"], case["window"],
                             case["block"], case["reorth_rows"], case.get("refit_rows", 0))
    assert side.prot == case["prefill"]["prot"]
    assert side.live == case["prefill"]["live"]
    assert comp == case["prefill"]["comp"]
    for i in range(case["decode_steps"]):
        t = case["L"] + i
        acts = op.append(side, t)
        assert [list(a[:1]) + [list(a[1])] if len(a) > 1 else list(a) for a in acts] == \
            case["steps"][str(t)], t
    assert op.exact_positions(side) == case["final"]["exact"]
    assert comp + side.compressed == case["final"]["history"]


@pytest.mark.parametrize("L,W,b", [(10, 4, 2), (1000, 128, 64), (37, 16, 8), (5, 0, 8)])
def test_empty_window_closed_form(L, W, b):
    """Keys (empty window at prefill, protected rows inside the prompt only): the j-th fold comes
    with position L - 1 + W + j b and merges positions L + (j-1) b .. L + j b - 1."""
    side, _ = op.new_side(L, [L - 1], 0, W, b, 0)
    folds = []
    for t in range(L, L + W + 6 * b - 1):    # just before the sixth fold
        for a in op.append(side, t):
            folds.append((t, a[1]))
    assert len(folds) == 5
    for j, (t, blk) in enumerate(folds, start=1):
        assert t == L - 1 + W + j * b
        assert blk == list(range(L + (j - 1) * b, L + j * b))


def test_no_prompt_no_window_reduces_to_block_stream():
    """Empty prompt and W = 0: every b decode rows are folded as they arrive, which is the pinned
    block stream ``fold_stream``; the rows after the last full block stay exact."""
    d, b, r = 24, 4, 6
    X = synth.lowrank_rows(30, d, 1.0, 0.05, seed=3)
    out = op.run_decode(np.zeros((0, d)), X, [], 0, 0, b, r, 0)
    U, s, B, pos = out["history"]
    Us, ss, Bs, _ = of.fold_stream(X, b, r)
    np.testing.assert_array_equal(U, Us)
    np.testing.assert_array_equal(s, ss)
    np.testing.assert_array_equal(B, Bs)
    np.testing.assert_array_equal(pos, np.arange(28))
    np.testing.assert_array_equal(out["exact"][1], [28, 29])
    np.testing.assert_array_equal(out["exact"][0], X[28:])


@pytest.mark.parametrize("seed", range(6))
def test_partition_invariants(seed):
    g = synth.rng(100 + seed)
    L = int(g.integers(0, 300))
    W = int(g.integers(0, 40))
    b = int(g.choice([1, 2, 8, 16]))
    w0 = int(g.integers(0, W + 1))
    R = int(g.choice([0, b, 3 * b, 5 * b + 1]))
    F = int(g.choice([0, b, 2 * b, 3]))
    P = np.flatnonzero(g.random(L) < 0.2).tolist()
    side, comp = op.new_side(L, P, w0, W, b, R, F)
    n_refit = 0
    n_folds = n_reorth = 0
    for t in range(L, L + 400):
        acts = op.append(side, t)
        for a in acts:
            if a[0] in ("fold", "refit"):
                blk = a[1]
                assert len(blk) == (b if a[0] == "fold" else F) and blk == sorted(blk)
                assert all(p not in P and p <= t - W for p in blk)
                if a[0] == "fold":
                    assert n_refit == (1 if F else 0)        # the refit comes first
                    n_folds += 1
                else:
                    n_refit += 1
            else:
                n_reorth += 1
        assert len(side.pending()) < (b if side.refit_done else F)
        exact = set(op.exact_positions(side))
        everything = sorted(list(exact) + comp + side.compressed)
        assert everything == list(range(t + 1))                          # a partition of 0..t
        # the window is exact, except prompt rows compressed at prefill (outside the initial window)
        assert all(p in exact for p in range(max(0, t - W + 1, L - w0), t + 1))
        assert set(side.prot) == set(P)
    if R:
        assert n_reorth == n_folds // math.ceil(R / b)
    else:
        assert n_reorth == 0


def test_rank_deficient_rows_are_recovered():
    """Rows of rank below the budget: the history represents every compressed row exactly, the exact
    table holds the stored rows, and reconstruction returns the whole sequence."""
    d, r, b, W, L, T = 32, 10, 4, 6, 40, 50
    g = synth.rng(9)
    X = g.standard_normal((L + T, 5)) @ g.standard_normal((5, d))
    P = [0, 3, 4, 20, 38, 39]
    out = op.run_decode(X[:L], X[L:], P, 6, W, b, r, 8)
    U, s, B, pos = out["history"]
    np.testing.assert_allclose(of.low_rank_product(U, s, B), X[pos], atol=1e-9)
    rows, epos = out["exact"]
    np.testing.assert_array_equal(rows, X[epos])
    full = orec.reconstruct(U, s, B, pos, rows, epos, L + T, 1, d, False, 500000.0)
    np.testing.assert_allclose(full, X, atol=1e-9)


def test_refit_of_an_empty_history_is_the_untruncated_block_stream():
    """Algorithm 3 step 3 with nothing compressed yet (a short prompt, fully protected): the rank-r
    SVD of the first r_V pending rows equals folding them in blocks with rank budget r >= r_V, since
    no fold then truncates. This is how the device carries out the refit."""
    d, b, r, rv = 40, 4, 16, 12
    X = synth.lowrank_rows(rv, d, 0.7, 0.05, seed=21)
    U, s, B = op.refit(*of.empty_history(d), X, r)
    Uf, sf, Bf, _ = of.fold_stream(X, b, r)
    np.testing.assert_allclose(s, sf, rtol=1e-12)
    np.testing.assert_allclose(of.low_rank_product(U, s, B), of.low_rank_product(Uf, sf, Bf),
                               atol=1e-12)
    np.testing.assert_allclose(of.low_rank_product(U, s, B), X, atol=1e-12)


def test_refit_keeps_history_rows_then_new_rows():
    """The refit factors the history's rows followed by the new rows: with enough rank both come
    back exactly, in that order."""
    d = 30
    g = synth.rng(22)
    basis = g.standard_normal((4, d))
    Xh = g.standard_normal((20, 4)) @ basis
    F = g.standard_normal((6, 4)) @ basis
    Uh, sh, Bh = of.truncated_svd(Xh, 4)
    U, s, B = op.refit(Uh, sh, Bh, F, 8)
    np.testing.assert_allclose(of.low_rank_product(U, s, B), np.concatenate([Xh, F]), atol=1e-10)
    # rank 1: the best rank-1 approximation of the stacked rows (Eckart-Young)
    U1, s1, B1 = op.refit(Uh, sh, Bh, F, 1)
    sv = np.linalg.svd(np.concatenate([Xh, F]), compute_uv=False)
    assert s1[0] == pytest.approx(sv[0], rel=1e-12)


def test_argument_errors():
    with pytest.raises(ValueError):
        op.new_side(10, [1], 5, 4, 2, 0)          # init window longer than the window
    with pytest.raises(ValueError):
        op.prefill_partition(10, [3, 3], 0)       # repeated protected position
    with pytest.raises(ValueError):
        op.prefill_partition(10, [10], 0)         # outside the prompt
    side, _ = op.new_side(10, [], 0, 4, 2, 0)
    with pytest.raises(ValueError):
        op.append(side, 12)                        # positions arrive one at a time


def test_policy_then_attention_equals_dense_attention():
    """Algorithm 3 steps 1-9 compose: with K and V rows of rank below the budget, attention over the
    policy's K and V (different protected sets, so row i of the two histories is not the same
    token) equals attention over the dense sequence."""
    from oracle import attention as oatt
    from oracle import rope

    d, hd, n_kv, r, b, W, L, T = 64, 32, 2, 8, 4, 6, 30, 40
    g = synth.rng(31)
    K = g.standard_normal((L + T, 4)) @ g.standard_normal((4, d))
    V = g.standard_normal((L + T, 3)) @ g.standard_normal((3, d))
    PK = [0, 1, 27, 28, 29]
    PV = [0, 1, 2, 5, 26, 27, 28, 29]
    ok = op.run_decode(K[:L], K[L:], PK, 0, W, b, r, 8)
    ov = op.run_decode(V[:L], V[L:], PV, W, W, b, r, 8, refit_rows=8)
    assert ok["history"][3].tolist() != ov["history"][3].tolist()
    q = g.standard_normal((4, hd))
    n = L + T
    got = oatt.decode_attention(ok["history"], ov["history"], ok["exact"][0], ok["exact"][1],
                                ov["exact"][0], ov["exact"][1], n, q, n_kv, hd)
    Kr = rope.apply_rope(K, np.arange(n), n_kv, hd, 500000.0)
    want = np.zeros((4, hd))
    for j in range(4):
        h = j // 2
        s = Kr[:, h * hd:(h + 1) * hd] @ q[j] / np.sqrt(hd)
        p = np.exp(s - s.max())
        want[j] = (p / p.sum()) @ V[:, h * hd:(h + 1) * hd]
    np.testing.assert_allclose(got, want, atol=1e-9)
