"""Seeded synthetic inputs shared by the CUDA path's tests/benchmarks and the oracle.

This module only *draws* inputs.  It contains none of the Shampoo or PRISM
arithmetic: no Gram statistics, no residuals, no polynomial, no alpha fit, no
matrix function.  Both sides receive the exact same fp32 (or bf16) bytes from
here; the oracle upcasts them to float64, the CUDA path copies them to HBM.

Workloads follow the synthetic spectra the PRISM summary describes
(gist.science "Sintesi Tecnica: PRISM", "Risultati Sperimentali": Gaussian
random matrices and heavy-tailed Marchenko-Pastur spectra) and the Shampoo
tutorial's weight/gradient shapes (algorithm.idocdown.com "Shampoo", §2).

Random streams: ``numpy.random.default_rng`` (PCG64).  A batch member ``i``
of a stream with seed ``s`` draws from ``default_rng((s, i))`` so that any
single block can be regenerated without drawing the others.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "spd_block",
    "spd_batch",
    "singular_spectrum",
    "gaussian",
    "lowrank_noise",
    "lowrank_noise_batch",
    "mp_spd",
    "sketch_stack",
    "to_bf16_bits",
    "bf16_bits_to_f32",
]


def _rng(seed, index=None):
    if index is None:
        return np.random.default_rng(seed)
    return np.random.default_rng((seed, index))


def spd_block(n: int, lam_lo: float, lam_hi: float, seed: int, index: int = 0,
              return_spectrum: bool = False):
    """One SPD matrix A = Q diag(lam) Q^T, stored fp32.

    Q is the orthogonal factor of a QR factorisation of an n x n N(0,1) matrix,
    with column signs fixed so that diag(R) > 0; lam is log-uniform on
    [lam_lo, lam_hi].  A is formed in float64, symmetrised, then rounded to
    fp32 (the rounding keeps exact symmetry).
    """
    g = _rng(seed, index)
    M = g.standard_normal((n, n))
    Q, Rq = np.linalg.qr(M)
    Q = Q * np.sign(np.diag(Rq))[None, :]
    lam = np.exp(g.uniform(np.log(lam_lo), np.log(lam_hi), size=n))
    A = (Q * lam[None, :]) @ Q.T
    A = 0.5 * (A + A.T)
    A32 = A.astype(np.float32)
    if return_spectrum:
        return A32, Q, lam
    return A32


def spd_batch(n: int, batch: int, lam_lo: float, lam_hi: float, seed: int,
              indices=None) -> np.ndarray:
    """A [batch, n, n] fp32 stack of independent :func:`spd_block` draws."""
    idx = range(batch) if indices is None else indices
    out = np.empty((len(idx), n, n), dtype=np.float32)
    for j, i in enumerate(idx):
        out[j] = spd_block(n, lam_lo, lam_hi, seed, i)
    return out


def singular_spectrum(m: int, n: int, sigma_min: float, batch: int, seed: int) -> np.ndarray:
    """[batch, m, n] fp32 matrices U diag(sigma) V^T (m >= n) with U, V the
    orthogonal factors of QR factorisations of N(0,1) matrices (signs fixed)
    and sigma log-uniform on [sigma_min, 1], largest set to 1: the sigma_min
    sweep of the polar iteration."""
    out = np.empty((batch, m, n), dtype=np.float32)
    for b in range(batch):
        g = _rng(seed, b)
        U, Ru = np.linalg.qr(g.standard_normal((m, n)))
        U = U * np.sign(np.diag(Ru))[None, :]
        V, Rv = np.linalg.qr(g.standard_normal((n, n)))
        V = V * np.sign(np.diag(Rv))[None, :]
        sig = np.exp(g.uniform(np.log(sigma_min), 0.0, size=n))
        sig[0] = 1.0
        out[b] = ((U * sig[None, :]) @ V.T).astype(np.float32)
    return out


def gaussian(shape, std: float, seed: int, index=None) -> np.ndarray:
    """N(0, std^2) fp32 array."""
    g = _rng(seed, index)
    return (g.standard_normal(shape) * std).astype(np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 exactly."""
    return (b.astype(np.uint32) << 16).view(np.float32)


def lowrank_noise(m: int, n: int, rank: int, noise: float, seed: int, index: int = 0):
    """U V^T + noise * N(0,1), U: m x rank, V: n x rank, both N(0,1); then
    divided by its Frobenius norm.  Returned as (bf16 bits, fp32 value of those bits)."""
    g = _rng(seed, index)
    U = g.standard_normal((m, rank))
    V = g.standard_normal((n, rank))
    G = U @ V.T + noise * g.standard_normal((m, n))
    G /= np.linalg.norm(G)
    bits = to_bf16_bits(G.astype(np.float32))
    return bits, bf16_bits_to_f32(bits)


def lowrank_noise_batch(m, n, rank, noise, batch, seed, indices=None):
    idx = range(batch) if indices is None else indices
    bits = np.empty((len(idx), m, n), dtype=np.uint16)
    for j, i in enumerate(idx):
        bits[j], _ = lowrank_noise(m, n, rank, noise, seed, i)
    return bits, bf16_bits_to_f32(bits)


def mp_spd(n: int, samples: int, shift: float, seed: int, chunk: int = 2048) -> np.ndarray:
    """A = X X^T / samples + shift * I with X n x samples N(0,1) fp32
    (Marchenko-Pastur spectrum, aspect ratio n/samples).  X is drawn in fp32
    column chunks; the product is accumulated in float64; A is returned fp32."""
    g = _rng(seed)
    A = np.zeros((n, n), dtype=np.float64)
    done = 0
    while done < samples:
        c = min(chunk, samples - done)
        X = g.standard_normal((n, c), dtype=np.float32).astype(np.float64)
        A += X @ X.T
        done += c
    A /= samples
    A[np.diag_indices(n)] += shift
    A = 0.5 * (A + A.T)
    return A.astype(np.float32)


def sketch_stack(K: int, n: int, p: int, seed: int) -> np.ndarray:
    """Gaussian sketch matrices S_k in R^{n x p}, k = 0..K-1, N(0,1), fp32,
    layout [K][n][p] row-major."""
    g = _rng(seed)
    return g.standard_normal((K, n, p), dtype=np.float32)
