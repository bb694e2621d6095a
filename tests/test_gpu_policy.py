"""GPU parity of the cache policy (Section 3.1, Section 3.2, Algorithm 1 steps 5-8, Algorithm 3
steps 1-6) against the oracle: the prefill partition bit for bit, then decode steps whose schedule
(which tables fold or re-orthogonalise in which step), exact-row tables and history positions match
exactly and whose factors, reconstruction and decode attention match within the fp32 / bf16
tolerances."""

import numpy as np
import pytest
import torch

from gpu_util import kv, np64, set_state, state, stored
from oracle import attention as oatt
from oracle import fold as of
from oracle import policy as op
from oracle import reconstruct as orec
import synth

pytestmark = pytest.mark.gpu


def _protected(L, seed, frac=0.08, suffix=36):
    g = np.random.Generator(np.random.PCG64(seed))
    mask = g.random(L) < frac
    mask[max(0, L - suffix):] = True
    return np.flatnonzero(mask)


def _widen(P, L, radius):
    near = np.zeros(L, dtype=bool)
    for p in P:
        near[max(0, p - radius):min(L, p + radius + 1)] = True
    return np.flatnonzero(near)


@pytest.mark.parametrize("L,frac,init_window,xdt,tdt", [
    (5000, 0.1, 128, torch.float32, torch.float32),
    (5000, 0.1, 0, torch.bfloat16, torch.bfloat16),
    (3000, 0.3, 100, torch.float32, torch.bfloat16),
    (50, 0.2, 128, torch.bfloat16, torch.bfloat16),     # prompt shorter than the window
    (700, 0.0, 64, torch.float32, torch.float32),       # nothing protected
    (400, 1.0, 128, torch.float32, torch.float32),      # everything protected
    (0, 0.0, 0, torch.float32, torch.float32),          # empty prompt
])
def test_prefill_partition(L, frac, init_window, xdt, tdt):
    m = kv()
    d = 256
    g = np.random.Generator(np.random.PCG64(L + init_window))
    X = torch.as_tensor(g.standard_normal((max(L, 1), d)), dtype=xdt, device="cuda")[:L].contiguous()
    P = np.flatnonzero(g.random(L) < frac) if frac < 1 else np.arange(L)
    t = m.ExactTable(d, L + 128, window=128, block=64, dtype=tdt)
    comp_rows, comp_pos = m.cache_prefill(t, X, torch.as_tensor(P, dtype=torch.int32,
                                                                 device="cuda"), init_window)
    prot, live, comp = op.prefill_partition(L, P.tolist(), init_window)
    assert (t.t.n_prot, t.t.n_live, t.t.last, t.t.hist_rows) == (len(prot), len(live), L - 1,
                                                                  len(comp))
    assert t.live_positions() == live
    rows, pos = t.exact()
    assert pos.cpu().tolist() == prot + live
    assert torch.equal(rows, X[pos.long()].to(tdt))
    assert comp_pos.cpu().tolist() == comp
    assert torch.equal(comp_rows, X[comp_pos.long()])


def test_prefill_rejects_unordered_protected_positions():
    m = kv()
    X = torch.zeros(100, 256, device="cuda")
    t = m.ExactTable(256, 512, window=32, block=16, dtype=torch.float32)
    with pytest.raises(m.IskvError, match="ascending"):
        m.cache_prefill(t, X, torch.tensor([5, 3, 90], dtype=torch.int32, device="cuda"), 32)
    with pytest.raises(m.IskvError, match="ascending"):
        m.cache_prefill(t, X, torch.tensor([5, 100], dtype=torch.int32, device="cuda"), 32)


def _run(m, *, d, r, b, W, R, Ls, T, storage, seed, tol, suffix=36, refit=0, v_all=None,
         rv=None):
    """Two sequences x (K, V) = four tables stepped together through T decode steps, against four
    oracle runs started from the same stored prompt factors. With ``refit`` > 0 the value sides run
    the first refit of ``refit`` rows; ``v_all`` (default: when refitting) protects their whole
    prompt (a short prompt), so that their history is empty at the refit. ``rv`` gives the value
    sides their own rank budget; the key and value tables then step as two batches (a batched
    step takes histories of one rank)."""
    v_all = bool(refit) if v_all is None else v_all
    rv = r if rv is None else rv
    sides = []
    for s, L in enumerate(Ls):
        PK = _protected(L, seed + s, suffix=suffix)
        PV = np.arange(L) if v_all else _widen(PK, L, 4)
        for kind, P, w0, ex in (("K", PK, 0, 1.1), ("V", PV, min(W, L), 0.7)):
            X = stored(synth.lowrank_rows(L + T, d, ex, 0.02, seed=seed + 10 * s + len(sides)),
                       storage)
            sides.append(dict(kind=kind, L=L, P=P, w0=w0, X=X, F=refit if kind == "V" else 0,
                              r=rv if kind == "V" else r))
    n_cap = max(L for L in Ls) + T
    tabs, hists, refs = [], [], []
    for sd in sides:
        L = sd["L"]
        Xd = torch.as_tensor(sd["X"], dtype=storage, device="cuda")
        t = m.ExactTable(d, 1024, window=W, block=b, reorth_rows=R, dtype=storage,
                         refit_rows=sd["F"])
        comp_rows, comp_pos = m.cache_prefill(t, Xd[:L].contiguous(),
                                              torch.as_tensor(sd["P"], dtype=torch.int32,
                                                              device="cuda"), sd["w0"])
        if comp_pos.numel():
            U0, s0, B0 = of.truncated_svd(sd["X"][comp_pos.cpu().numpy()], sd["r"])
        else:
            U0, s0, B0 = of.empty_history(d)
        U0, s0, B0 = stored(U0, storage), stored(s0, torch.float32), stored(B0, storage)
        h = m.LowRankHistory(d, sd["r"], n_cap, storage=storage)
        set_state(h, U0, s0, B0, comp_pos.cpu().numpy())
        ref = op.run_decode(sd["X"][:L], sd["X"][L:], sd["P"], sd["w0"], W, b, sd["r"], R,
                            init_history=(U0, s0, B0), refit_rows=sd["F"])
        sd["Xd"] = Xd
        tabs.append(t)
        hists.append(h)
        refs.append(ref)
    groups = [list(range(len(sides)))] if rv == r else [
        [k for k, sd in enumerate(sides) if sd["kind"] == kind] for kind in ("K", "V")]
    batches = [m.CacheBatch([tabs[k] for k in g], [hists[k] for k in g]) for g in groups]
    for i in range(T):
        folded, reorthed = [0] * len(sides), [False] * len(sides)
        for g, batch in zip(groups, batches):
            rows = torch.stack([sides[k]["Xd"][sides[k]["L"] + i] for k in g]).contiguous()
            fo, re = batch.step(rows)
            for j, k in enumerate(g):
                folded[k], reorthed[k] = fo[j], re[j]
        for k, ref in enumerate(refs):
            acts = [a[0] for a in ref["steps"][i]]
            assert folded[k] == (2 if "refit" in acts else 1 if "fold" in acts else 0), (i, k)
            assert reorthed[k] == ("reorth" in acts), (i, k)
    for sd, t, h, ref in zip(sides, tabs, hists, refs):
        U, s, B, pos, (k, n, _, st) = state(h)
        Uo, so, Bo, poso = ref["history"]
        assert st == 0
        assert (k, n) == (so.shape[0], poso.shape[0])
        np.testing.assert_array_equal(pos, poso)
        assert of.rel_fro(of.low_rank_product(U, s, B), of.low_rank_product(Uo, so, Bo)) < tol
        rows, epos = t.exact()
        assert epos.cpu().tolist() == ref["exact"][1].tolist()
        np.testing.assert_array_equal(np64(rows), ref["exact"][0])
        assert t.live_positions() == ref["side"].live
        n_total = sd["L"] + T
        out = m.reconstruct(h, rows, epos, n_total, d // 128, 128, sd["kind"] == "K", 500000.0,
                            out_dtype=torch.float32)
        want = orec.reconstruct(Uo, so, Bo, poso, ref["exact"][0], ref["exact"][1], n_total,
                                d // 128, 128, sd["kind"] == "K", 500000.0)
        assert of.rel_fro(np64(out), want) < tol
    return sides, tabs, hists, refs


def test_decode_policy_fp32():
    m = kv()
    d, T = 256, 130
    # An 8-token suffix leaves unprotected rows in the value window at prefill.
    sides, tabs, hists, refs = _run(m, d=d, r=32, b=16, W=24, R=32, Ls=(300, 180), T=T,
                                    storage=torch.float32, seed=70, tol=1e-4, suffix=8)
    assert tabs[1].t.n_prot > 0 and refs[1]["side"].compressed
    # Decode attention of sequence 0 straight from its K and V tables (Algorithm 3 steps 7-9).
    g = np.random.Generator(np.random.PCG64(71))
    q = stored(40 * g.standard_normal((8, 128)) / np.sqrt(128), torch.float32)
    n_total = sides[0]["L"] + T
    kr, kp = tabs[0].exact()
    vr, vp = tabs[1].exact()
    out = m.decode_attention(hists[0], hists[1], kr, kp, vr, vp, n_total,
                             torch.as_tensor(q, dtype=torch.float32, device="cuda"), 2, 128)
    rk, rv = refs[0], refs[1]
    want = oatt.decode_attention(rk["history"], rv["history"], rk["exact"][0], rk["exact"][1],
                                 rv["exact"][0], rv["exact"][1], n_total, q, 2, 128)
    assert float(np.linalg.norm(np64(out) - want) / np.linalg.norm(want)) < 1e-4


def _refits(refs, tabs):
    for k in (1, 3):
        assert any(a[0] == "refit" for acts in refs[k]["steps"] for a in acts)
        assert tabs[k].t.refit_done == 1


def test_decode_policy_value_first_refit():
    """Short prompts whose values are all protected: the value sides wait for 32 pending rows, refit
    them into their empty histories (one 32-row fold at r = 32), then fold 16-row blocks; the key
    sides fold from the start."""
    m = kv()
    sides, tabs, hists, refs = _run(m, d=256, r=32, b=16, W=24, R=32, Ls=(120, 90), T=150,
                                    storage=torch.float32, seed=80, tol=1e-4, refit=32)
    _refits(refs, tabs)


def test_refit_of_a_compressed_history_in_one_fold():
    """Prompts with compressed values: the refit factors the history's rows followed by the 32
    pending rows, truncated to r = 32 -- one 32-row fold on the device."""
    m = kv()
    sides, tabs, hists, refs = _run(m, d=256, r=32, b=16, W=24, R=32, Ls=(300, 180), T=150,
                                    storage=torch.float32, seed=83, tol=1e-4, suffix=8, refit=32,
                                    v_all=False)
    _refits(refs, tabs)
    assert all(len(refs[k]["comp"]) > 0 for k in (1, 3))


def test_refit_by_untruncated_block_folds():
    """A 144-row refit (more than one fold takes) of empty histories at r = 160: nine 16-row folds
    in one step, none of which truncates."""
    m = kv()
    sides, tabs, hists, refs = _run(m, d=256, r=160, b=16, W=24, R=64, Ls=(60, 50), T=200,
                                    storage=torch.float32, seed=86, tol=1e-4, refit=144)
    _refits(refs, tabs)


def test_refit_of_a_compressed_history_through_a_wide_history():
    """The pages' value refit (Section 3.2, Algorithm 3 step 3): r_V = 256 pending rows into a
    history that already holds compressed prompt rows, at d = 1024, r = 256, b = 64 -- four 64-row
    folds into a wide history of rank 448 (none truncates before the last), whose top 256
    components come back: the rank-256 SVD of the history's rows followed by the refit rows."""
    m = kv()
    sides, tabs, hists, refs = _run(m, d=1024, r=256, b=64, W=128, R=256, Ls=(600, 450), T=450,
                                    storage=torch.float32, seed=88, tol=1e-4, suffix=8,
                                    refit=256, v_all=False)
    _refits(refs, tabs)
    assert all(len(refs[k]["comp"]) > 0 for k in (1, 3))


def test_refit_that_runs_neither_way_is_refused():
    """144 rows (more than one fold takes) into a history that already holds compressed rows, where
    the wide history would need rank 160 + 144 - 16 = 288 > d = 256."""
    m = kv()
    d, b, rv = 256, 16, 144
    X = torch.randn(300, d, device="cuda")
    t = m.ExactTable(d, 512, window=8, block=b, reorth_rows=0, dtype=torch.float32, refit_rows=rv)
    comp, comp_pos = m.cache_prefill(t, X[:100].contiguous(),
                                     torch.arange(90, 100, dtype=torch.int32, device="cuda"), 8)
    assert t.t.hist_rows == 90 and t.t.refit_done == 0
    h = m.LowRankHistory(d, 160, 400, storage=torch.float32)
    for i in range(100, 100 + 8 + rv - 1):
        m.cache_step([t], [h], X[i:i + 1].contiguous())
    last = t.t.last
    with pytest.raises(m.IskvError, match="empty history"):
        m.cache_step([t], [h], X[last + 1:last + 2].contiguous())
    assert t.t.last == last                          # the refused step changed nothing


def test_decode_policy_bf16_model_width():
    """d = 1024 (8 KV heads x 128), r = 64, b = 64, W = 128, re-orthogonalisation every 128 rows."""
    m = kv()
    _run(m, d=1024, r=64, b=64, W=128, R=128, Ls=(600, 450), T=300, storage=torch.bfloat16,
         seed=90, tol=2e-2)


def _attention_check(m, sides, tabs, hists, refs, T, n_kv, tol, seed):
    """Decode attention of sequence 0 straight from its K and V tables (Algorithm 3 steps 7-9)."""
    g = np.random.Generator(np.random.PCG64(seed))
    q = stored(40 * g.standard_normal((4 * n_kv, 128)) / np.sqrt(128), torch.float32)
    n_total = sides[0]["L"] + T
    kr, kp = tabs[0].exact()
    vr, vp = tabs[1].exact()
    out = m.decode_attention(hists[0], hists[1], kr, kp, vr, vp, n_total,
                             torch.as_tensor(q, dtype=torch.float32, device="cuda"), n_kv, 128)
    assert hists[0].status()[3] == 0 and hists[1].status()[3] == 0
    rk, rv = refs[0], refs[1]
    want = oatt.decode_attention(rk["history"], rv["history"], rk["exact"][0], rk["exact"][1],
                                 rv["exact"][0], rv["exact"][1], n_total, q, n_kv, 128)
    assert float(np.linalg.norm(np64(out) - want) / np.linalg.norm(want)) < tol


def test_decode_policy_different_key_and_value_ranks_fp32():
    """Keys at r = 32 and values at r = 48 (Section 8's separate K / V ranks): the key and value
    tables step as two batches, then decode attention reads a K history and a V history of
    different rank."""
    m = kv()
    T = 130
    sides, tabs, hists, refs = _run(m, d=256, r=32, rv=48, b=16, W=24, R=32, Ls=(300, 180), T=T,
                                    storage=torch.float32, seed=75, tol=1e-4, suffix=8)
    assert hists[0].r_max == 32 and hists[1].r_max == 48
    _attention_check(m, sides, tabs, hists, refs, T, 2, 1e-4, 76)


def test_decode_policy_different_key_and_value_ranks_bf16_model_width():
    """d = 1024 (8 KV heads x 128), keys at r = 256 and values at r = 128, b = 64, W = 128, bf16:
    the tensor-core score and value kernels each at their own rank."""
    m = kv()
    T = 200
    sides, tabs, hists, refs = _run(m, d=1024, r=256, rv=128, b=64, W=128, R=256, Ls=(600, 450),
                                    T=T, storage=torch.bfloat16, seed=95, tol=2e-2)
    _attention_check(m, sides, tabs, hists, refs, T, 8, 2e-2, 96)
