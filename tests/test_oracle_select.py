"""Pins for the prompt-block selection oracle (Section 3.1, Algorithm 1 steps 2-4).

The brute force below recomputes every score with explicit Python loops over tokens and features,
and decides membership by counting, for each candidate block, how many blocks precede it in the
(score, index) order -- no sort, no vectorised numpy.
"""

import math

import numpy as np
import pytest

from oracle import select as osel
import synth


def _brute(keys, block, per_head, suffix_blocks, v_radius):
    L, H, hd = keys.shape
    nb = L // block
    n_cand = max(nb - suffix_blocks, 0)
    scores = [[0.0] * n_cand for _ in range(H)]
    for h in range(H):
        for j in range(n_cand):
            toks = [[float(keys[j * block + t, h, c]) for c in range(hd)] for t in range(block)]
            mean = [sum(toks[t][c] for t in range(block)) / block for c in range(hd)]
            mn = math.sqrt(sum(v * v for v in mean))
            best = None
            for t in range(block):
                dot = sum(toks[t][c] * mean[c] for c in range(hd))
                kn = math.sqrt(sum(v * v for v in toks[t]))
                cos = dot / max(kn * mn, 1e-30)
                best = cos if best is None else min(best, cos)
            scores[h][j] = best
    protected = set(range(n_cand * block, L))
    picked_all = []
    for h in range(H):
        picked = []
        for j in range(n_cand):
            ahead = sum(1 for i in range(n_cand)
                        if (scores[h][i], i) < (scores[h][j], j))
            if ahead < per_head:
                picked.append(j)
                protected.update(range(j * block, (j + 1) * block))
        picked_all.append(picked)
    pk = sorted(protected)
    pv = sorted({q for p in pk for q in range(p - v_radius, p + v_radius + 1) if 0 <= q < L})
    return scores, picked_all, pk, pv


@pytest.mark.parametrize("L,H,hd,per_head,seed", [(77, 2, 8, 3, 0), (130, 2, 6, 5, 1),
                                                  (64, 1, 4, 100, 2), (256, 2, 16, 7, 3)])
def test_selection_matches_brute_force(L, H, hd, per_head, seed):
    keys, _ = synth.outlier_prompt_keys(L, H, hd, seed, outlier_frac=0.15)
    ref_s, ref_h, ref_pk, ref_pv = _brute(keys, 8, per_head, 4, 5)
    out = osel.select_prompt_blocks(keys, 8, per_head, 4, 5)
    np.testing.assert_allclose(out["scores"], np.array(ref_s).reshape(H, -1), rtol=1e-12,
                               atol=1e-15)
    for h in range(H):
        assert list(out["head_blocks"][h]) == ref_h[h]
    assert list(out["P_K"]) == ref_pk
    assert list(out["P_V"]) == ref_pv


def test_short_prompt_is_all_suffix():
    keys, _ = synth.outlier_prompt_keys(39, 2, 8, 4)
    out = osel.select_prompt_blocks(keys)
    assert out["n_cand"] == 0
    assert list(out["P_K"]) == list(range(39))
    assert list(out["P_V"]) == list(range(39))


def test_fewer_candidates_than_budget_takes_all():
    keys, _ = synth.outlier_prompt_keys(8 * 50 + 3, 2, 8, 5)
    out = osel.select_prompt_blocks(keys, per_head=128)
    assert out["n_cand"] == 46
    for hb in out["head_blocks"]:
        assert list(hb) == list(range(46))
    assert list(out["P_K"]) == list(range(403))


def test_outlier_blocks_are_picked_first():
    keys, mask = synth.outlier_prompt_keys(8 * 400, 4, 32, 6, outlier_frac=0.05)
    out = osel.select_prompt_blocks(keys, per_head=20, v_radius=2)
    for h in range(4):
        assert set(np.flatnonzero(mask[h])) <= set(out["head_blocks"][h])
        assert out["scores"][h][mask[h][:out["n_cand"]]].max() < 0.6
        assert np.median(out["scores"][h]) > 0.9


def test_zero_key_scores_zero():
    keys = np.ones((48, 1, 4))
    keys[3, 0, :] = 0.0
    out = osel.select_prompt_blocks(keys, per_head=1, v_radius=0)
    assert out["scores"][0][0] == 0.0
    assert out["scores"][0][1:].min() == pytest.approx(1.0)
    assert list(out["head_blocks"][0]) == [0]
