"""Pins for the decode-attention oracle (Algorithm 3 step 9 over the cache of steps 7-8)."""

import math

import numpy as np
import pytest

from oracle import attention as oatt
from oracle import reconstruct as orec
from oracle import rope
import synth


def _factors(g, n, d, k, pos):
    U = np.linalg.qr(g.standard_normal((n, k)))[0]
    B = np.linalg.qr(g.standard_normal((d, k)))[0]
    s = np.geomspace(4.0, 0.5, k)
    return U, s, B, np.asarray(pos)


def test_single_position_returns_its_value():
    """One cached position: softmax of one score is 1, the output is that value row."""
    g = synth.rng(1)
    d, hd, H, nq = 16, 8, 2, 4
    kf = _factors(g, 1, d, 1, [0])
    vf = _factors(g, 1, d, 1, [0])
    q = g.standard_normal((nq, hd))
    out = oatt.decode_attention(kf, vf, np.zeros((0, d)), [], np.zeros((0, d)), [], 1, q, H, hd)
    V = (vf[0] * vf[1]) @ vf[2].T
    for j in range(nq):
        h = j // (nq // H)
        np.testing.assert_allclose(out[j], V[0, h * hd:(h + 1) * hd], atol=1e-14)


def test_zero_scale_averages_values():
    """scale = 0 makes every score equal: the output is the mean value over all positions,
    exact rows included."""
    g = synth.rng(2)
    n, d, hd, H, nq, k = 12, 16, 8, 2, 2, 3
    kf = _factors(g, n, d, k, np.arange(0, 2 * n, 2))
    vf = _factors(g, n, d, k, np.arange(0, 2 * n, 2))
    ex = g.standard_normal((n, d))
    epos = np.arange(1, 2 * n, 2)
    q = g.standard_normal((nq, hd))
    out = oatt.decode_attention(kf, vf, ex, epos, ex, epos, 2 * n, q, H, hd, scale=0.0)
    V = orec.reconstruct(vf[0], vf[1], vf[2], vf[3], ex, epos, 2 * n, H, hd, False)
    for j in range(nq):
        np.testing.assert_allclose(out[j], V[:, j * hd:(j + 1) * hd].mean(axis=0), atol=1e-13)


def test_query_matching_one_rotated_key_picks_it():
    """Keys are rotated by their own positions: a query equal to one key's post-RoPE value (scaled
    up) puts almost all weight on that position, even though the pre-RoPE keys are identical."""
    d, hd, H, nq, n = 8, 8, 1, 1, 6
    key = np.zeros((1, d))
    key[0, 0] = 1.0
    Kex = np.repeat(key, n, axis=0)                   # identical pre-RoPE keys
    pos = np.arange(n) * 7
    Vex = np.eye(n, d) if n <= d else None
    target = 3
    q = 60.0 * rope.apply_rope(key, [pos[target]], H, hd, 10000.0)
    out = oatt.decode_attention(
        (np.zeros((0, 1)), np.zeros(1), np.zeros((d, 1)), np.zeros(0, dtype=int)),
        (np.zeros((0, 1)), np.zeros(1), np.zeros((d, 1)), np.zeros(0, dtype=int)),
        Kex, pos, Vex, pos, int(pos[-1]) + 1, q, H, hd, theta=10000.0, scale=1.0)
    assert out[0, target] > 0.99
    # and without rotation every key would score the same
    assert abs(out[0].sum() - 1.0) < 1e-12


def test_gqa_maps_query_heads_to_their_kv_head():
    """With one position, query head j returns KV head j // group of the value row."""
    d, hd, H, nq = 32, 8, 4, 8
    V = np.arange(d, dtype=np.float64)[None, :]
    K = np.ones((1, d))
    q = synth.rng(3).standard_normal((nq, hd))
    out = oatt.decode_attention(
        (np.zeros((0, 1)), np.zeros(1), np.zeros((d, 1)), np.zeros(0, dtype=int)),
        (np.zeros((0, 1)), np.zeros(1), np.zeros((d, 1)), np.zeros(0, dtype=int)),
        K, [0], V, [0], 1, q, H, hd)
    for j in range(nq):
        h = j // 2
        np.testing.assert_array_equal(out[j], V[0, h * hd:(h + 1) * hd])


def test_matches_scalar_loops_on_a_small_cache():
    """Vectorised oracle vs an independent scalar-loop restatement on a mixed compressed/exact
    cache with RoPE."""
    g = synth.rng(4)
    n, d, hd, H, nq, k, ne = 10, 16, 8, 2, 4, 4, 5
    perm = g.permutation(n + ne)
    kf = _factors(g, n, d, k, perm[:n])
    vf = _factors(g, n, d, k, perm[:n])
    Kex, Vex = g.standard_normal((ne, d)), g.standard_normal((ne, d))
    q = g.standard_normal((nq, hd))
    out = oatt.decode_attention(kf, vf, Kex, perm[n:], Vex, perm[n:], n + ne, q, H, hd, 500.0)
    K = orec.reconstruct(*kf, Kex, perm[n:], n + ne, H, hd, True, 500.0)
    V = orec.reconstruct(*vf, Vex, perm[n:], n + ne, H, hd, False)
    ref = oatt.decode_attention_loops(K.tolist(), V.tolist(), q.tolist(), H, hd, 1 / math.sqrt(hd))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)


def test_mismatched_k_and_v_positions_rejected():
    g = synth.rng(5)
    d, hd, H = 8, 8, 1
    kf = _factors(g, 3, d, 2, [0, 1, 2])
    vf = _factors(g, 2, d, 2, [0, 1])
    with pytest.raises(ValueError):
        oatt.decode_attention(kf, vf, np.zeros((0, d)), [], np.zeros((0, d)), [], 3,
                              g.standard_normal((1, hd)), H, hd)
