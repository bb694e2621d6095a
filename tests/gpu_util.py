"""Helpers for the GPU parity tests: library import, host copies, synthetic histories."""

import numpy as np
import pytest
import torch


def kv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_online_b200 import build
    build.build()
    import kv_cache_online_b200 as m
    return m


def np64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def state(h):
    """Host float64 copies of (U[:n, :k], sigma[:k], B[:, :k], pos[:n]) and the meta word."""
    k, n, folds, st = h.status()
    return (np64(h.U[:n, :k]), np64(h.sigma[:k]), np64(h.B[:, :k]), h.pos[:n].cpu().numpy(),
            (k, n, folds, st))


def set_state(h, U, sigma, B, pos, folds=0):
    """Write a history's factors (host arrays) into its device tensors."""
    n, k = U.shape
    h.U.zero_()
    h.B.zero_()
    h.sigma.zero_()
    h.U[:n, :k] = torch.as_tensor(U, dtype=h.U.dtype)
    h.B[:, :k] = torch.as_tensor(B, dtype=h.B.dtype)
    h.sigma[:k] = torch.as_tensor(sigma, dtype=torch.float32)
    h.pos[:n] = torch.as_tensor(pos, dtype=torch.int32)
    h.meta.copy_(torch.tensor([k, n, folds, 0], dtype=torch.int64))
    torch.cuda.synchronize()


def stored(x, dtype):
    """Round a host array through a torch dtype and back to float64 (the values a kernel sees)."""
    return torch.as_tensor(np.asarray(x), dtype=dtype).to(torch.float64).numpy()


def synthetic_history(n, d, k, seed, exponent=1.2, dtype=torch.float32):
    """Orthonormal-column U, B and a power-law sigma scaled like a history of n rows."""
    g = np.random.Generator(np.random.PCG64(seed))
    U = np.linalg.qr(g.standard_normal((n, k)))[0]
    B = np.linalg.qr(g.standard_normal((d, k)))[0]
    sigma = np.sqrt(n) * np.arange(1, k + 1, dtype=np.float64) ** (-exponent)
    return stored(U, dtype), stored(sigma, torch.float32), stored(B, dtype)


def bit(code):
    return 1 << code
