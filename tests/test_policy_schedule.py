"""CPU checks of the cache step's host-side schedule against the policy oracle (Section 3.2,
Algorithm 3 steps 1-6): ``iskv_cache_plan`` runs the same per-table decision and host-mirror update
that ``iskv_cache_step`` uses, without a device, so the schedule -- which step folds, refits or
re-orthogonalises each table, and the live positions, counters and history rows afterwards -- is
compared with the oracle step by step over random cases."""

import ctypes
import json
import os

import numpy as np
import pytest

from conftest import GOLDEN
from oracle import policy as op
import synth

D, R, NCAP = 1024, 256, 1 << 20


def _lib():
    from kv_cache_online_b200 import build
    build.build()
    from kv_cache_online_b200 import _lib as L
    return L, L.load()


class _Table:
    """An exact-row table whose host mirror starts where the oracle's prefill leaves it. The device
    pointers are placeholders: the dry run never dereferences them."""

    def __init__(self, L, side, comp, window, block, reorth_rows, refit_rows):
        self.live = (ctypes.c_int32 * (window + max(block, refit_rows)))(*side.live)
        self.t = L.IskvExactTable(D, window, block, reorth_rows, 1, refit_rows, 1 << 30, 0x100000,
                                  0x200000, ctypes.cast(self.live, ctypes.POINTER(ctypes.c_int32)),
                                  window + max(block, refit_rows), len(side.prot), len(side.live),
                                  side.last, 0, len(comp), int(refit_rows == 0))

    def mirror(self):
        t = self.t
        return (list(self.live[:t.n_live]), t.last, t.fold_rows, t.hist_rows, bool(t.refit_done))


def _expect(acts):
    kinds = [a[0] for a in acts]
    return (2 if "refit" in kinds else 1 if "fold" in kinds else 0), int("reorth" in kinds)


def _drive(L, lib, cases, steps):
    """Step every (oracle side, table) pair together through ``steps`` positions."""
    tabs = [c[1] for c in cases]
    arr = (ctypes.POINTER(L.IskvExactTable) * len(tabs))(*[ctypes.pointer(t.t) for t in tabs])
    folded = (ctypes.c_int32 * len(tabs))()
    reorthed = (ctypes.c_int32 * len(tabs))()
    for _ in range(steps):
        assert lib.iskv_cache_plan(arr, len(tabs), R, NCAP, 1, folded, reorthed) == 0, \
            lib.iskv_last_error()
        for k, (side, tab, comp) in enumerate(cases):
            acts = op.append(side, side.last + 1)
            assert (folded[k], reorthed[k]) == _expect(acts), (k, side.last)
            assert tab.mirror() == (side.live, side.last, side.fold_rows,
                                    len(comp) + len(side.compressed), side.refit_done), k


@pytest.mark.parametrize("seed", range(8))
def test_schedule_matches_oracle(seed):
    L_, lib = _lib()
    g = synth.rng(500 + seed)
    b = int(g.choice([8, 16, 64]))
    W = int(g.integers(0, 200))
    cases = []
    for _ in range(6):
        L = int(g.integers(0, 400))
        w0 = int(g.integers(0, W + 1))
        R_ = int(g.choice([0, b, 3 * b, 5 * b + 8]))
        F = int(g.choice([0, b, 2 * b] + ([4 * b] if 4 * b <= 128 else [])))
        P = np.flatnonzero(g.random(L) < g.choice([0.05, 0.3, 1.0])).tolist()
        side, comp = op.new_side(L, P, w0, W, b, R_, F)
        cases.append((side, _Table(L_, side, comp, W, b, R_, F), comp))
    _drive(L_, lib, cases, 700)


@pytest.mark.parametrize("name", [c["name"] for c in json.load(open(
    os.path.join(GOLDEN, "policy_small.json")))["cases"]])
def test_schedule_on_hand_worked_cases(name):
    """The hand-worked schedules, with the block and window scaled by 8 (the fold takes blocks of
    8 rows at least): every position becomes 8 positions, so each step of the worked case is 8 steps
    here and the decisions fall on the last of them."""
    L_, lib = _lib()
    case = [c for c in json.load(open(os.path.join(GOLDEN, "policy_small.json")))["cases"]
            if c["name"] == name][0]
    s = 8
    L = case["L"] * s
    P = [p * s + j for p in case["protected"] for j in range(s)]
    side, comp = op.new_side(L, P, case["init_window"] * s, case["window"] * s,
                             case["block"] * s, case["reorth_rows"] * s,
                             case.get("refit_rows", 0) * s)
    _drive(L_, lib, [(side, _Table(L_, side, comp, case["window"] * s, case["block"] * s,
                                   case["reorth_rows"] * s, case.get("refit_rows", 0) * s),
                      comp)], case["decode_steps"] * s)
    assert op.exact_positions(side)[:len(P)] == P


def test_refused_step_changes_nothing():
    """A first refit due on a history that already holds compressed rows runs through a wide
    history of rank r + refit_rows - block when that rank is at most 512 (136 rows at r = 256,
    b = 8: rank 384); 280 rows would need rank 528 and are refused, leaving the mirror as it was.
    An empty history takes 136 rows as untruncated folds."""
    L_, lib = _lib()
    for rows, hist_rows, want in ((280, 100, 2), (136, 100, 0), (136, 0, 0)):
        side, comp = op.new_side(0, [], 0, 0, 8, 0, rows)
        tab = _Table(L_, side, comp, 0, 8, 0, rows)
        tab.t.hist_rows = hist_rows
        arr = (ctypes.POINTER(L_.IskvExactTable) * 1)(ctypes.pointer(tab.t))
        folded = (ctypes.c_int32 * 1)()
        for _ in range(rows - 1):
            assert lib.iskv_cache_plan(arr, 1, R, NCAP, 1, folded, None) == 0
        before = tab.mirror()
        assert lib.iskv_cache_plan(arr, 1, R, NCAP, 1, folded, None) == want
        if want:
            assert b"wide history" in lib.iskv_last_error()
            assert tab.mirror() == before
        else:
            assert folded[0] == 2 and tab.t.n_live == 0 and tab.t.hist_rows == hist_rows + rows


def test_history_capacity_is_checked_before_the_fold():
    L_, lib = _lib()
    side, comp = op.new_side(0, [], 0, 0, 8, 0, 0)
    tab = _Table(L_, side, comp, 0, 8, 0, 0)
    arr = (ctypes.POINTER(L_.IskvExactTable) * 1)(ctypes.pointer(tab.t))
    for _ in range(7):
        assert lib.iskv_cache_plan(arr, 1, R, 12, 1, None, None) == 0
    assert lib.iskv_cache_plan(arr, 1, R, 12, 1, None, None) == 0      # 8 rows into 12
    for _ in range(7):
        assert lib.iskv_cache_plan(arr, 1, R, 12, 1, None, None) == 0
    before = tab.mirror()
    assert lib.iskv_cache_plan(arr, 1, R, 12, 1, None, None) == 4      # 16 > 12
    assert tab.mirror() == before


def test_cache_batch_plan_through_the_binding():
    """``CacheBatch.plan`` (host memory only, so CPU tensors serve): keys with an empty prompt,
    W = 4, b = 8 -- the first fold comes with position W + b - 1 = 11, then every 8 positions."""
    _lib()
    import torch

    import kv_cache_online_b200 as m
    tabs = [m.ExactTable(64, 64, window=4, block=8, reorth_rows=16, dtype=torch.bfloat16,
                         device="cpu") for _ in range(2)]
    for t in tabs:
        t.t.last = -1
    hists = [m.LowRankHistory(64, 16, 64, storage=torch.bfloat16, device="cpu") for _ in range(2)]
    batch = m.CacheBatch(tabs, hists)
    seen = []
    for pos in range(30):
        folded, reorthed = batch.plan(advance=True)
        if folded[0]:
            seen.append((pos, folded[0], reorthed[0]))
        assert folded == [folded[0]] * 2
    assert seen == [(11, 1, False), (19, 1, True), (27, 1, False)]
    assert tabs[0].live_positions() == list(range(24, 30)) and tabs[0].t.hist_rows == 24


def test_zero_row_refit_counts_as_done():
    """A table without a refit (refit_rows = 0) folds regular blocks even if its mirror says the
    refit is still to come."""
    L_, lib = _lib()
    side, comp = op.new_side(0, [], 0, 0, 8, 0, 0)
    tab = _Table(L_, side, comp, 0, 8, 0, 0)
    tab.t.refit_done = 0
    arr = (ctypes.POINTER(L_.IskvExactTable) * 1)(ctypes.pointer(tab.t))
    folded = (ctypes.c_int32 * 1)()
    got = []
    for _ in range(16):
        assert lib.iskv_cache_plan(arr, 1, R, NCAP, 1, folded, None) == 0
        got.append(folded[0])
    assert got == [0] * 7 + [1] + [0] * 7 + [1] and tab.t.refit_done == 1
