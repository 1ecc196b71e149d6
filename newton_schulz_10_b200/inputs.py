"""Seeded synthetic inputs for the Muon-step workloads.

This module only draws random numbers and lays them out; it holds none of the
optimizer's arithmetic. Tests, the bench and the oracle-side scripts all take
their inputs from here, so the CPU oracle and the CUDA library see identical
bits.

Recipe: every array is drawn in float64 from NumPy's PCG64 seeded with
``(seed, stream)`` where ``seed = 1000*workload + 16*layer + matrix`` and the
stream selects the array (0 = W, 1 = G of step 0, 2 = G of step 1, ...), then
rounded to float32 (or to bfloat16 where a workload says so).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

W_STREAM = 0
G_STREAM = 1


def rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(seed), int(stream)]))


def gaussian(shape, std, seed, stream, dtype=np.float32):
    x = rng(seed, stream).standard_normal(shape)
    x *= std
    return x.astype(dtype)


def student_t3(shape, scale, seed, stream, dtype=np.float32):
    """Heavy-tailed entries scale * N / sqrt(chi2_3 / 3) (Student-t, nu = 3)."""
    g = rng(seed, stream)
    z = g.standard_normal(shape)
    chi = g.chisquare(3.0, size=shape)
    z /= np.sqrt(chi / 3.0)
    z *= scale
    return z.astype(dtype)


def random_orthonormal(rows, cols, seed, stream):
    """rows x cols matrix with orthonormal columns (rows >= cols): the Q factor
    of a seeded Gaussian matrix, with column signs fixed by diag(R) > 0."""
    a = rng(seed, stream).standard_normal((rows, cols))
    q, r = np.linalg.qr(a)
    q *= np.sign(np.diag(r))[None, :]
    return q


def to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest-even), returned as uint16 bit
    patterns (NaN kept quiet)."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    nan = np.isnan(x32)
    if np.any(nan):
        rounded = np.where(nan, ((u >> 16) | 0x40).astype(np.uint16), rounded)
    return rounded.reshape(np.shape(x32))


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# Workload shapes
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class MatrixSpec:
    rows: int
    cols: int
    seed: int
    name: str


def gpt124m_layer_set(layers: int = 12, workload: int = 2):
    """GPT-124M-shaped set: per layer four 768x768 attention matrices, one
    768x3072 and one 3072x768 MLP matrix."""
    shapes = [(768, 768)] * 4 + [(768, 3072), (3072, 768)]
    names = ["q", "k", "v", "o", "fc", "proj"]
    return [MatrixSpec(r, c, 1000 * workload + 16 * l + i, f"l{l}.{names[i]}")
            for l in range(layers) for i, (r, c) in enumerate(shapes)]


def llama7b_layer_set(layers: int = 32, workload: int = 5):
    """Llama-7B-shaped set: per layer four 4096x4096 attention matrices, one
    4096x14336 and one 14336x4096 MLP matrix."""
    shapes = [(4096, 4096)] * 4 + [(4096, 14336), (14336, 4096)]
    names = ["q", "k", "v", "o", "up", "down"]
    return [MatrixSpec(r, c, 1000 * workload + 16 * l + i, f"l{l}.{names[i]}")
            for l in range(layers) for i, (r, c) in enumerate(shapes)]


def spectrum_matrix(rows, cols, sigma_min_exp=-4.0, seed=3000):
    """X = U diag(sigma) V^T with seeded orthonormal factors and singular
    values sigma_i = 10**(sigma_min_exp * u_i), u_i ~ U[0, 1) (log-uniform in
    [10**sigma_min_exp, 1]). rows <= cols. Returns (X float64, sigma)."""
    assert rows <= cols
    U = random_orthonormal(rows, rows, seed, 0)
    V = random_orthonormal(cols, rows, seed, 1)
    u = rng(seed, 2).random(rows)
    sigma = 10.0 ** (sigma_min_exp * u)
    return (U * sigma[None, :]) @ V.T, sigma
