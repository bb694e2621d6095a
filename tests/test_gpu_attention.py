"""GPU parity of decode attention over the compressed cache (Algorithm 3 steps 7-9) against the
float64 oracle."""

import numpy as np
import pytest
import torch

from gpu_util import bit, kv, set_state, stored, synthetic_history
from oracle import attention as oatt

pytestmark = pytest.mark.gpu


def _case(m, *, n, d, r, k, n_kv, hd, n_q, prompt, window, storage, exact_dtype, seed,
          gap=1, qscale=48.0, theta=500000.0, n_cap=None, offsets=None):
    """K and V histories at the same positions (compressed rows every `gap` positions after the
    prompt, shifted by `offsets` if given, the other positions exact), exact prompt and window
    rows, one query."""
    g = np.random.Generator(np.random.PCG64(seed))
    Uk, sk, Bk = synthetic_history(n, d, k, seed, 1.2, storage)
    Uv, sv, Bv = synthetic_history(n, d, k, seed + 1, 0.6, storage)
    comp = prompt + gap * np.arange(n) + (0 if offsets is None else offsets)
    n_total = int(comp[-1]) + 1 + window
    exact = np.setdiff1d(np.arange(n_total), comp)
    cap = n + 8 if n_cap is None else n_cap
    hk = m.LowRankHistory(d, r, cap, storage=storage)
    hv = m.LowRankHistory(d, r, cap, storage=storage)
    set_state(hk, Uk, sk, Bk, comp)
    set_state(hv, Uv, sv, Bv, comp)
    Kex = stored(0.3 * g.standard_normal((exact.size, d)), exact_dtype)
    Vex = stored(0.3 * g.standard_normal((exact.size, d)), exact_dtype)
    q = stored(qscale * g.standard_normal((n_q, hd)) / np.sqrt(hd), torch.float32)
    dev = "cuda"
    t = lambda a, dt: torch.as_tensor(a, dtype=dt, device=dev).contiguous()
    args = dict(k_exact=t(Kex, exact_dtype), k_exact_pos=t(exact, torch.int32),
                v_exact=t(Vex, exact_dtype), v_exact_pos=t(exact, torch.int32),
                n_total=n_total, q=t(q, torch.float32))
    ref = oatt.decode_attention((Uk, sk, Bk, comp), (Uv, sv, Bv, comp), Kex, exact, Vex, exact,
                                n_total, q, n_kv, hd, theta)
    return hk, hv, args, ref


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("storage,tol", [(torch.float32, 1e-4), (torch.bfloat16, 2e-2)])
def test_attention_parity(storage, tol):
    m = kv()
    hk, hv, a, ref = _case(m, n=700, d=256, r=32, k=32, n_kv=2, hd=128, n_q=8, prompt=40,
                           window=24, storage=storage, exact_dtype=torch.float32, seed=11, gap=2)
    out = m.decode_attention(hk, hv, a["k_exact"], a["k_exact_pos"], a["v_exact"],
                             a["v_exact_pos"], a["n_total"], a["q"], 2, 128)
    assert hk.status()[3] == 0 and hv.status()[3] == 0
    assert _rel(out.double().cpu().numpy(), ref) < tol


@pytest.mark.parametrize("n_q", [8, 16, 32, 64])
def test_tensor_core_scores_grouped_query_shapes(n_q):
    """bf16 factors at the model shape (8 KV heads x 128, r = 256): the tensor-core scores kernel
    with 1, 2, 4 and 8 query heads per KV head, a ragged row count and bf16 exact rows."""
    m = kv()
    hk, hv, a, ref = _case(m, n=1000, d=1024, r=256, k=256, n_kv=8, hd=128, n_q=n_q, prompt=512,
                           window=128, storage=torch.bfloat16, exact_dtype=torch.bfloat16,
                           seed=20 + n_q)
    out = m.decode_attention(hk, hv, a["k_exact"], a["k_exact_pos"], a["v_exact"],
                             a["v_exact_pos"], a["n_total"], a["q"], 8, 128)
    assert hk.status()[3] == 0 and hv.status()[3] == 0
    assert _rel(out.double().cpu().numpy(), ref) < 2e-2


@pytest.mark.parametrize("layout", ["consecutive", "gapped", "jumps"])
def test_tensor_core_scores_position_layouts(layout):
    """The tensor-core scores kernel rotates a warp's 32 keys by angle addition when their
    positions are consecutive and each key on its own otherwise: consecutive positions, every
    third position, and runs broken inside a warp (rows 40 and 150), over a short history whose
    every key weighs in the softmax, with a ragged last tile."""
    m = kv()
    n = 300
    offsets = None
    if layout == "jumps":
        offsets = np.where(np.arange(n) >= 40, 7, 0) + np.where(np.arange(n) >= 150, 13, 0)
    hk, hv, a, ref = _case(m, n=n, d=1024, r=256, k=256, n_kv=8, hd=128, n_q=32, prompt=8,
                           window=8, storage=torch.bfloat16, exact_dtype=torch.bfloat16, seed=71,
                           gap=3 if layout == "gapped" else 1, offsets=offsets)
    out = m.decode_attention(hk, hv, a["k_exact"], a["k_exact_pos"], a["v_exact"],
                             a["v_exact_pos"], a["n_total"], a["q"], 8, 128)
    assert hk.status()[3] == 0 and hv.status()[3] == 0
    assert _rel(out.double().cpu().numpy(), ref) < 2e-2


def test_full_size_layer():
    """One layer at n = 16384 compressed rows with the 640 exact rows of the benchmark."""
    m = kv()
    hk, hv, a, ref = _case(m, n=16384, d=1024, r=256, k=256, n_kv=8, hd=128, n_q=32, prompt=512,
                           window=128, storage=torch.bfloat16, exact_dtype=torch.bfloat16, seed=5)
    out = m.decode_attention(hk, hv, a["k_exact"], a["k_exact_pos"], a["v_exact"],
                             a["v_exact_pos"], a["n_total"], a["q"], 8, 128)
    assert hk.status()[3] == 0 and hv.status()[3] == 0
    assert _rel(out.double().cpu().numpy(), ref) < 2e-2


def test_batched_equals_single():
    m = kv()
    cases = [_case(m, n=n, d=1024, r=256, k=kk, n_kv=8, hd=128, n_q=32, prompt=64, window=32,
                   storage=torch.bfloat16, exact_dtype=torch.bfloat16, seed=40 + n, n_cap=1600)
             for n, kk in ((900, 256), (1500, 200))]
    outs = m.decode_attention_batched(
        [c[0] for c in cases], [c[1] for c in cases], [c[2]["k_exact"] for c in cases],
        [c[2]["k_exact_pos"] for c in cases], [c[2]["v_exact"] for c in cases],
        [c[2]["v_exact_pos"] for c in cases], [c[2]["n_total"] for c in cases],
        [c[2]["q"] for c in cases], 8, 128)
    for (hk, hv, a, ref), o in zip(cases, outs):
        single = m.decode_attention(hk, hv, a["k_exact"], a["k_exact_pos"], a["v_exact"],
                                    a["v_exact_pos"], a["n_total"], a["q"], 8, 128)
        assert torch.equal(single, o)
        assert _rel(o.double().cpu().numpy(), ref) < 2e-2


def test_batched_tile_ranges_cross_histories():
    """Six histories of different lengths, prompts and windows in one call. The tensor-core
    kernels cut the tiles of all histories into contiguous per-CTA ranges, so ranges run from
    the end of one history into the next: every history's output must equal its own call."""
    m = kv()
    spec = ((1000, 64, 32), (2500, 100, 16), (3100, 8, 64), (1800, 300, 8), (3900, 40, 40),
            (700, 16, 128))
    cases = [_case(m, n=n, d=1024, r=256, k=256, n_kv=8, hd=128, n_q=32, prompt=pr, window=wi,
                   storage=torch.bfloat16, exact_dtype=torch.bfloat16, seed=90 + i, n_cap=4096)
             for i, (n, pr, wi) in enumerate(spec)]
    outs = m.decode_attention_batched(
        [c[0] for c in cases], [c[1] for c in cases], [c[2]["k_exact"] for c in cases],
        [c[2]["k_exact_pos"] for c in cases], [c[2]["v_exact"] for c in cases],
        [c[2]["v_exact_pos"] for c in cases], [c[2]["n_total"] for c in cases],
        [c[2]["q"] for c in cases], 8, 128)
    for (hk, hv, a, ref), o in zip(cases, outs):
        single = m.decode_attention(hk, hv, a["k_exact"], a["k_exact_pos"], a["v_exact"],
                                    a["v_exact_pos"], a["n_total"], a["q"], 8, 128)
        assert hk.status()[3] == 0 and hv.status()[3] == 0
        assert torch.equal(single, o)
        assert _rel(o.double().cpu().numpy(), ref) < 2e-2


def test_key_without_value_is_flagged():
    """A key position whose value row is missing leaves probability mass unaccounted: SHAPE."""
    m = kv()
    hk, hv, a, _ = _case(m, n=300, d=256, r=32, k=32, n_kv=2, hd=128, n_q=4, prompt=16, window=8,
                         storage=torch.float32, exact_dtype=torch.float32, seed=3, qscale=0.0)
    keep = a["v_exact_pos"].numel() - 8
    m.decode_attention(hk, hv, a["k_exact"], a["k_exact_pos"], a["v_exact"][:keep].contiguous(),
                       a["v_exact_pos"][:keep].contiguous(), a["n_total"], a["q"], 2, 128)
    assert hv.status()[3] & bit(2)


@pytest.mark.parametrize("storage,rk,rv,tol", [(torch.float32, 32, 48, 1e-4),
                                               (torch.bfloat16, 256, 128, 2e-2),
                                               (torch.bfloat16, 128, 256, 2e-2)])
def test_keys_and_values_of_different_rank(storage, rk, rv, tol):
    """A K history and a V history with their own rank budgets (Section 8's separate K / V
    ranks), both full to their budget."""
    m = kv()
    d, n_kv, n = (256, 2, 700) if storage == torch.float32 else (1024, 8, 1200)
    g = np.random.Generator(np.random.PCG64(rk + rv))
    Uk, sk, Bk = synthetic_history(n, d, rk, 61, 1.2, storage)
    Uv, sv, Bv = synthetic_history(n, d, rv, 62, 0.6, storage)
    prompt, window = 64, 32
    n_total = prompt + n + window
    comp = prompt + np.arange(n)
    exact = np.setdiff1d(np.arange(n_total), comp)
    hk = m.LowRankHistory(d, rk, n + 8, storage=storage)
    hv = m.LowRankHistory(d, rv, n + 8, storage=storage)
    set_state(hk, Uk, sk, Bk, comp)
    set_state(hv, Uv, sv, Bv, comp)
    Kex = stored(0.3 * g.standard_normal((exact.size, d)), storage)
    Vex = stored(0.3 * g.standard_normal((exact.size, d)), storage)
    q = stored(48 * g.standard_normal((4 * n_kv, 128)) / np.sqrt(128), torch.float32)
    t = lambda a, dt: torch.as_tensor(a, dtype=dt, device="cuda").contiguous()
    out = m.decode_attention(hk, hv, t(Kex, storage), t(exact, torch.int32), t(Vex, storage),
                             t(exact, torch.int32), n_total, t(q, torch.float32), n_kv, 128)
    ref = oatt.decode_attention((Uk, sk, Bk, comp), (Uv, sv, Bv, comp), Kex, exact, Vex, exact,
                                n_total, q, n_kv, 128, 500000.0)
    assert hk.status()[3] == 0 and hv.status()[3] == 0
    assert _rel(out.double().cpu().numpy(), ref) < tol
