"""Seeded synthetic inputs shared by the tests, the smoke run and the benchmark.

This module draws random numbers and nothing else: it holds none of the compression method's
arithmetic, so that the float64 oracle and the CUDA library can both be fed from it without sharing
any code of the method.

The pages measure on model traces and benchmark suites (MATH-500, AIME, RULER) that are not available
here; these generators stand in for them with the structure the pages describe -- rows with a
power-law singular spectrum plus noise (pre-RoPE keys decay faster than values), and post-RoPE prompt
keys whose 8-token blocks are mostly coherent with a few outlier blocks.
"""

from __future__ import annotations

import numpy as np


def rng(seed: int) -> np.random.Generator:
    """NumPy PCG64 generator."""
    return np.random.Generator(np.random.PCG64(int(seed)))


def random_orthogonal(d: int, g: np.random.Generator) -> np.ndarray:
    """Haar-distributed d x d orthogonal matrix: QR of a Gaussian with the sign of R's diagonal
    moved into Q."""
    A = g.standard_normal((d, d))
    Q, R = np.linalg.qr(A)
    return Q * np.sign(np.diag(R))[None, :]


def power_spectrum(d: int, exponent: float, rank: int | None = None) -> np.ndarray:
    """``s_i = i ** -exponent`` for ``i = 1..d``; zero beyond ``rank`` when given."""
    s = np.arange(1, d + 1, dtype=np.float64) ** (-float(exponent))
    if rank is not None:
        s[int(rank):] = 0.0
    return s


def lowrank_rows(n: int, d: int, exponent: float, noise: float, seed: int,
                 rank: int | None = None, H: np.ndarray | None = None) -> np.ndarray:
    """Rows ``G diag(s) H^T + noise * N(0, 1)`` with ``G`` (n x d) standard normal, ``H`` a random
    d x d orthogonal matrix (drawn from the same seed unless given) and ``s`` a power law.
    Float64, shape (n, d)."""
    g = rng(seed)
    if H is None:
        H = random_orthogonal(d, g)
    s = power_spectrum(d, exponent, rank)
    G = g.standard_normal((n, d))
    X = (G * s[None, :]) @ H.T
    if noise:
        X = X + float(noise) * g.standard_normal((n, d))
    return X


def outlier_prompt_keys(L: int, n_heads: int, head_dim: int, seed: int, outlier_frac: float = 0.05,
                        block: int = 8, coherence: float = 0.1):
    """Post-RoPE prompt keys ``(L, H, hd)``: per head a strong shared mean direction plus small
    noise (block cosines near 1), with ``outlier_frac`` of the full blocks of each head (chosen
    independently per head) replaced by random-direction tokens (block cosines well below 1).
    Returns ``(keys float64, outlier_mask (H, L // block) bool)``."""
    g = rng(seed)
    nb = L // block
    K = np.empty((L, n_heads, head_dim))
    mask = np.zeros((n_heads, nb), dtype=bool)
    for h in range(n_heads):
        mu = g.standard_normal(head_dim)
        mu /= np.linalg.norm(mu)
        scale = 1.0 + 0.1 * g.random(L)
        K[:, h, :] = scale[:, None] * (mu[None, :] + coherence * g.standard_normal((L, head_dim))
                                       / np.sqrt(head_dim))
        n_out = int(round(outlier_frac * nb))
        if n_out:
            blocks = g.choice(nb, size=n_out, replace=False)
            mask[h, blocks] = True
            for j in blocks:
                K[j * block:(j + 1) * block, h, :] = g.standard_normal((block, head_dim))
    return K, mask


def torch_orthonormal(rows: int, cols: int, seed: int, device="cuda", dtype=None):
    """Random ``rows x cols`` matrix with orthonormal columns (QR of a Gaussian), drawn on
    ``device`` with a seeded torch generator. Returned in float32 unless ``dtype`` is given."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    A = torch.randn(rows, cols, generator=gen, device=device, dtype=torch.float32)
    Q, R = torch.linalg.qr(A)
    Q = Q * torch.sign(torch.diagonal(R))[None, :]
    return Q if dtype is None else Q.to(dtype)


def torch_lowrank_rows(n: int, d: int, exponent: float, noise: float, basis, seed: int,
                       device="cuda"):
    """Torch counterpart of ``lowrank_rows`` for large benchmark inputs: ``G diag(s) basis^T +
    noise * N(0,1)`` with ``basis`` a (d x m) matrix with orthonormal columns, float32."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    m = basis.shape[1]
    s = torch.arange(1, m + 1, device=device, dtype=torch.float32) ** (-float(exponent))
    G = torch.randn(n, m, generator=gen, device=device, dtype=torch.float32)
    X = (G * s[None, :]) @ basis.float().T
    if noise:
        X = X + float(noise) * torch.randn(n, d, generator=gen, device=device, dtype=torch.float32)
    return X


class DriftingRows:
    """Rows of ``count`` independent streams whose dominant subspace drifts, drawn on ``device``
    with a seeded torch generator, one block of ``block`` rows per stream at a time.

    Stream i emits ``G diag(s_i) H_i(t)^T + noise * N(0, 1)`` with ``G`` standard normal,
    ``s_i[j] = (j + 1) ** -exponents[i]`` and ``H_i(t) = H_i(0) exp((t / 1024) angle_per_1k S_i)``,
    where ``H_i(0)`` is a random d x d orthogonal matrix and ``S_i`` a random skew-symmetric matrix
    scaled to spectral norm 1 (estimated by power iteration): the subspace turns by about
    ``angle_per_1k`` radians per 1024 rows. ``H`` advances by one block after each call of
    :meth:`next_blocks`. Float32 throughout; returns (count, block, d) tensors."""

    def __init__(self, count: int, d: int, exponents, noise: float, seed: int, block: int,
                 angle_per_1k: float = 0.05, device="cuda"):
        import torch

        self.torch = torch
        self.count, self.d, self.block, self.noise = int(count), int(d), int(block), float(noise)
        self.gen = torch.Generator(device=device)
        self.gen.manual_seed(int(seed))
        self.device = device
        A = torch.randn(self.count, d, d, generator=self.gen, device=device)
        Q, R = torch.linalg.qr(A)
        self.H = Q * torch.sign(torch.diagonal(R, dim1=-2, dim2=-1))[:, None, :]
        A = torch.randn(self.count, d, d, generator=self.gen, device=device)
        S = A - A.transpose(1, 2)
        v = torch.randn(self.count, d, 1, generator=self.gen, device=device)
        for _ in range(30):                       # power iteration on S^T S
            v = S.transpose(1, 2) @ (S @ v)
            v = v / torch.linalg.vector_norm(v, dim=1, keepdim=True)
        snorm = torch.linalg.vector_norm(S @ v, dim=1, keepdim=True)
        S = S / snorm
        self.E = torch.linalg.matrix_exp(S * (float(angle_per_1k) * self.block / 1024.0))
        ex = torch.as_tensor([float(e) for e in exponents], device=device)[:, None]
        j = torch.arange(1, d + 1, device=device, dtype=torch.float32)[None, :]
        self.s = j ** (-ex)                       # (count, d)

    def next_blocks(self):
        torch = self.torch
        G = torch.randn(self.count, self.block, self.d, generator=self.gen, device=self.device)
        X = (G * self.s[:, None, :]) @ self.H.transpose(1, 2)
        if self.noise:
            X = X + self.noise * torch.randn(self.count, self.block, self.d, generator=self.gen,
                                             device=self.device)
        self.H = self.H @ self.E
        return X
