"""fp16 factors and outputs (Section 7.3 of the pages: fp16 factors overflowed on long generations
and the run went to NaN). Here sigma stays float32 and U, B have orthonormal columns, so stored
factors stay below 1; the fp16 overflow risk moves to the reconstructed cache, where it is detected
and recorded as ISKV_ERR_NONFINITE. Parity tolerance: fp16 keeps 11 significant bits (relative
rounding 2^-11 ~ 4.9e-4 per stored element), so 5e-3 relative Frobenius error."""

import numpy as np
import pytest
import torch

from gpu_util import bit, kv, np64, set_state, state, stored, synthetic_history
from oracle import attention as oatt
from oracle import fold as of
from oracle import reconstruct as orec
from oracle import reorth as oreo
import synth

pytestmark = pytest.mark.gpu

F16 = torch.float16


def test_fold_trajectory_fp16_factors():
    """The tiny fold trajectory (d = 128, b = 16, r = 16, 30 folds) with fp16 U and B."""
    m = kv()
    X = stored(synth.lowrank_rows(512, 128, 1.0, 0.01, seed=0), torch.float32)
    h = m.LowRankHistory(128, 16, 512, storage=F16)
    Xd = torch.as_tensor(X, dtype=torch.float32, device="cuda")
    for i in range(30):
        m.fold_block(h, Xd[i * 16:(i + 1) * 16].contiguous(),
                     torch.arange(i * 16, (i + 1) * 16, dtype=torch.int32, device="cuda"))
    U, s, B, pos, (k, n, folds, st) = state(h)
    assert (k, n, folds, st) == (16, 480, 30, 0)
    Uo, so, Bo, _ = of.fold_stream(X[:480], 16, 16)
    assert of.rel_fro(of.low_rank_product(U, s, B), of.low_rank_product(Uo, so, Bo)) < 5e-3
    np.testing.assert_allclose(s, so, rtol=1e-3)


def test_reorth_fp16_factors():
    m = kv()
    n, d, r, k = 2048, 512, 128, 128
    g = np.random.Generator(np.random.PCG64(12))
    U = stored(np.linalg.qr(g.standard_normal((n, k)))[0] + 1e-2 * g.standard_normal((n, k)) /
               np.sqrt(n), F16)
    B = stored(np.linalg.qr(g.standard_normal((d, k)))[0] + 1e-2 * g.standard_normal((d, k)) /
               np.sqrt(d), F16)
    s = stored(np.sqrt(n) * np.arange(1, k + 1) ** -1.0, torch.float32)
    h = m.LowRankHistory(d, r, n, storage=F16)
    set_state(h, U, s, B, np.arange(n), folds=16)
    m.reorth(h)
    U2, s2, B2, _, (k2, n2, folds, st) = state(h)
    assert (k2, n2, folds, st) == (k, n, 0, 0)
    Ur, sr, Br = oreo.reorth(U, s, B)
    np.testing.assert_allclose(s2, sr, rtol=1e-4)
    assert of.rel_fro(of.low_rank_product(U2, s2, B2), of.low_rank_product(U, s, B)) < 5e-3
    for got, ref in ((U2, Ur), (B2, Br)):
        assert oreo.orthogonality_error(got) < 1.5 * oreo.orthogonality_error(stored(ref, F16))


@pytest.mark.parametrize("storage", [F16, torch.bfloat16])
def test_reconstruct_into_fp16(storage):
    m = kv()
    n, n_exact, H, hd, d, r = 2000, 100, 8, 128, 1024, 128
    U, s, B = synthetic_history(n, d, r, seed=31, dtype=storage)
    g = np.random.Generator(np.random.PCG64(32))
    perm = g.permutation(n + n_exact)
    pos, epos = perm[:n], perm[n:]
    exact = stored(g.standard_normal((n_exact, d)), F16)
    h = m.LowRankHistory(d, r, n, storage=storage)
    set_state(h, U, s, B, pos)
    out = m.reconstruct(h, torch.as_tensor(exact, dtype=F16, device="cuda"),
                        torch.as_tensor(epos, dtype=torch.int32, device="cuda"), n + n_exact, H,
                        hd, True, 500000.0, out_dtype=F16)
    ref = orec.reconstruct(U, s, B, pos, exact, epos, n + n_exact, H, hd, True, 500000.0)
    assert of.rel_fro(np64(out), ref) < 5e-3
    assert h.status()[3] == 0


def test_fp16_overflow_in_reconstruction_is_flagged():
    """Singular values large enough that reconstructed rows exceed 65504: the fp16 output holds
    infinities and the history records NONFINITE; the same history reconstructed into bf16 does
    not (bf16 shares float32's exponent range)."""
    m = kv()
    n, d, r, H, hd = 600, 256, 32, 2, 128
    U, s, B = synthetic_history(n, d, r, seed=41, dtype=F16)
    s = s * 1e7
    h = m.LowRankHistory(d, r, n, storage=F16)
    set_state(h, U, s, B, np.arange(n))
    m.reconstruct(h, None, None, n, H, hd, False, 500000.0, out_dtype=torch.bfloat16)
    assert h.status()[3] == 0
    out = m.reconstruct(h, None, None, n, H, hd, False, 500000.0, out_dtype=F16)
    assert torch.isinf(out).any()
    assert h.status()[3] & bit(5)


def test_attention_fp16_factors():
    m = kv()
    n, d, r, k, n_kv, hd, n_q = 600, 256, 32, 32, 2, 128, 8
    Uk, sk, Bk = synthetic_history(n, d, k, 51, 1.2, F16)
    Uv, sv, Bv = synthetic_history(n, d, k, 52, 0.6, F16)
    g = np.random.Generator(np.random.PCG64(53))
    n_total = n + 48
    comp = np.arange(24, 24 + n)
    exact = np.setdiff1d(np.arange(n_total), comp)
    hk = m.LowRankHistory(d, r, n, storage=F16)
    hv = m.LowRankHistory(d, r, n, storage=F16)
    set_state(hk, Uk, sk, Bk, comp)
    set_state(hv, Uv, sv, Bv, comp)
    Kex = stored(0.3 * g.standard_normal((exact.size, d)), F16)
    Vex = stored(0.3 * g.standard_normal((exact.size, d)), F16)
    q = stored(48 * g.standard_normal((n_q, hd)) / np.sqrt(hd), torch.float32)
    t = lambda a, dt: torch.as_tensor(a, dtype=dt, device="cuda").contiguous()
    out = m.decode_attention(hk, hv, t(Kex, F16), t(exact, torch.int32), t(Vex, F16),
                             t(exact, torch.int32), n_total, t(q, torch.float32), n_kv, hd)
    ref = oatt.decode_attention((Uk, sk, Bk, comp), (Uv, sv, Bv, comp), Kex, exact, Vex, exact,
                                n_total, q, n_kv, hd)
    assert hk.status()[3] == 0 and hv.status()[3] == 0
    assert float(np.linalg.norm(np64(out) - ref) / np.linalg.norm(ref)) < 5e-3
