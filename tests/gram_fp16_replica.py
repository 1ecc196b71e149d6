"""A CPU replica of the library's fp16 Gram Newton-Schulz arithmetic.

TEST INFRASTRUCTURE, and NOT the oracle: the oracle computes the method in
float64; this module instead reproduces where the CUDA library rounds, so that
precision findings about the fp16 Gram chain can be checked on the CPU. It
imports nothing from the oracle or from the CUDA library.

What it replicates (the Gram iteration of "1. Gram Newton-Schulz" on the
Dion3 page, Theorem 2 with the restart of Algorithm 3, as the library stores
it):

* storage points: X_0 kept as fp16(sqrt(n) X_0), the Gram matrix as
  fp16(n X X^T), Z, Q, Z R and R in fp16, every product accumulated in a
  wider type and rounded once when stored;
* one-triangle products: a product whose exact result is symmetric (X X^T,
  R R, Q Z, Z R, (Z R) Z) is computed on one triangle and mirrored, so the
  stored matrix is exactly symmetric even where the fp16 factors no longer
  commute exactly.

Each knob picks one of several equally valid roundings of the same
algorithm: which triangle is computed (`triangle`), the accumulation type
(`acc`), or no mirroring at all (`triangle="full"`). The tensor cores' own
summation order is one more such choice, so the GPU result is one sample of
the spread these variants show.
"""

from __future__ import annotations

import numpy as np


def _f16(x):
    return np.asarray(x, np.float64).astype(np.float16).astype(np.float64)


def _keep(x):
    return np.asarray(x, np.float64)


def _product(A, B, acc, triangle, sym):
    """A @ B accumulated in `acc`; for symmetric results one triangle is kept
    and mirrored (the diagonal belongs to both)."""
    D = (A.astype(acc) @ B.astype(acc)).astype(np.float64)
    if not sym or triangle == "full":
        return D
    L = np.tril(D) if triangle == "lower" else np.triu(D).T
    return L + np.tril(L, -1).T


def gram_ns_fp16(X, coeffs, eps=1e-7, restart_at=3, acc=np.float32, triangle="lower", fp16=True):
    """Gram Newton-Schulz of a wide X (n <= m) with the library's fp16
    storage points. Returns the float64 values of the fp16 output (NaN/inf
    propagate, as an fp16 overflow would). fp16=False keeps every stored
    value in float64 (the same algebra without rounding)."""
    rnd = _f16 if fp16 else _keep
    X = np.asarray(X, np.float64)
    n = X.shape[0]
    kappa, rho = np.sqrt(n), float(n)
    s = 1.0 / (np.sqrt(np.sum(X * X)) + eps)
    Xs = rnd(kappa * s * X)  # stored operand: sqrt(n) X_0
    I = np.eye(n)

    def mm(A, B, sym, alpha=1.0, C=None, beta=0.0, gamma=0.0):
        D = alpha * _product(A, B, acc, triangle, sym)
        if C is not None:
            D = D + beta * C
        return rnd(D + gamma * I if gamma else D)

    # R_0 = n X_0 X_0^T = (rho / kappa^2) Xs Xs^T
    R = mm(Xs, Xs.T, True, rho / kappa ** 2)
    Q = None
    T = len(coeffs)
    with np.errstate(over="ignore", invalid="ignore"):
        for t, (a, b, c) in enumerate(coeffs, start=1):
            if restart_at and t == restart_at and Q is not None:
                Xs = mm(Q, Xs, False)
                R = mm(Xs, Xs.T, True, rho / kappa ** 2)
                Q = None
            # Z = a I + (b / rho) R + (c / rho^2) R R  (R is stored as rho X X^T)
            Z = mm(R, R, True, c / rho ** 2, R, b / rho, a)
            Q = Z if Q is None else mm(Q, Z, True)
            if t < T and not (restart_at and t + 1 == restart_at):
                ZR = mm(Z, R, True)
                R = mm(ZR, Z, True)
        return mm(Q, Xs, False, 1.0 / kappa)
