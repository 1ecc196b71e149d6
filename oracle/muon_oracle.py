"""Plain, slow fp64 CPU oracle for the Muon optimizer step.

TEST INFRASTRUCTURE. This module is not part of the product path. Only the
test suite (``tests/``), the smoke check in ``__graft_entry__.py`` and the CPU
baseline / reference arm of ``bench.py`` may import or run it. It shares no
code, table or constant with the CUDA library; the two meet only through the
seeded input generators in ``newton_schulz_10_b200/inputs.py``.

Source of every formula: "Dion3: Full-stack orthogonal updates"
(arXiv 2608.11612), as summarised on its web page. Sections used:

* "Muon Update Rule", Eq. (1): M <- mu*M + G ; W <- W - eta*polar(M).
* "Definition 1 (Polar Decomposition)": polar(X) = U V^T for X = U S V^T.
* "NorMuon Variant", Eq. (2): per-row second moment v, O_hat, and the
  Frobenius ratio ||O||_F / ||O_hat||_F.
* "Standard Newton-Schulz": X_{t+1} = a_t X + b_t X X^T X + c_t (X X^T)^2 X,
  with X_0 = X / ||X||_F; and its "FLOP Analysis" T(4 m n^2 + 2 n^3).
* "1. Gram Newton-Schulz": Theorem 2 (p_t(x) = x h_t(x^2); r_0 = x^2, q_0 = 1,
  z_t = h_t(r_{t-1}), r_t = r_{t-1} z_t^2, q_t = q_{t-1} z_t), the "Algorithm
  Structure (Naive Version)" (R_0 = X X^T, iterate, output Q_T X), its FLOP
  count (4T + 3 alpha - 3) n^3, and "Stabilization via Restarting" /
  Algorithm 3 (restart at t = 3 with X_2 = Q_2 X, costing 3(alpha - 1) n^3).
* "3. Dion3 Update Rule", Algorithm 4: top-k rows by l1 norm with
  k = ceil(f n), polar of M[S, :], update W[S, :], error feedback
  M <- mu*M_hat + (M - M_hat).

Readings taken where the page is silent:

* Coefficients (a_t, b_t, c_t) are inputs; the workloads use
  (3.4445, -4.7750, 2.0315) for every t.
* Frobenius normalisation is X / (||X||_F + eps) with eps = 1e-7.
* A tall matrix (rows > cols) is orthogonalised as the transpose of its wide
  transpose, since polar(X^T) = polar(X)^T.
* Dion3 momentum order: M <- M + G, select, O = polar(M[S]), update W[S],
  then M[S] <- mu*M[S] (the page's error feedback replaces M <- mu*M).
* Selection ties go to the lower row index; the index list is ascending.
* NorMuon: v starts at 0, no bias correction, m = columns of O as stored,
  eps is added to sqrt(v); when ||O_hat||_F = 0 the update is zero.
* State W, M, v is float32 between steps (as on the GPU); inside a step all
  arithmetic is float64. The momentum is rounded once, as a fused
  multiply-add would round it.

Parity status: every function below is pinned by ``tests/test_oracle_pins.py``
against closed forms, SVDs, brute force or hand-computed values. The page's
"reformulated intermediate polynomials" of Algorithm 3 are not given, so they
are not implemented (Theorem 2 is used verbatim).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

F64 = np.float64
F32 = np.float32

# ---------------------------------------------------------------------------
# fp32 state helpers
# ---------------------------------------------------------------------------


def fma_f32(a, b, c):
    """Exact fp32 result of a*b + c rounded once to nearest-even.

    Used for the momentum M <- mu*M + G of Eq. (1) so that the float32 state
    matches a fused multiply-add bit for bit. a, b, c are float32 arrays
    (broadcastable). The product of two float32 values is exact in float64;
    the sum is split into s + e exactly (TwoSum), and e only matters when s
    sits exactly halfway between two float32 neighbours.
    """
    a = np.asarray(a, dtype=F32)
    b = np.asarray(b, dtype=F32)
    c = np.asarray(c, dtype=F32)
    p = a.astype(F64) * b.astype(F64)          # exact: 24 + 24 bits < 53
    c64 = c.astype(F64)
    s = p + c64
    bp = s - c64
    bc = s - bp
    e = (p - bp) + (c64 - bc)                  # p + c == s + e exactly
    r = s.astype(F32)                          # round-to-nearest-even of s
    r64 = r.astype(F64)
    toward = np.where(s > r64, F32(np.inf), F32(-np.inf))
    other = np.nextafter(r, toward)            # float32 neighbour on s's side
    other64 = other.astype(F64)
    is_mid = (s != r64) & np.isfinite(other64) & ((s - r64) == (other64 - r64) * 0.5)
    fix = is_mid & (e != 0)
    if np.any(fix):
        up = np.maximum(r, other)
        down = np.minimum(r, other)
        r = np.where(fix, np.where(e > 0, up, down), r)
    return r.astype(F32)


# ---------------------------------------------------------------------------
# FLOP counter (page: "FLOP Analysis of Standard Newton-Schulz" and the
# Gram FLOP analysis, which count a symmetric GEMM of size n as n^3)
# ---------------------------------------------------------------------------


@dataclass
class FlopCounter:
    """Counts the products the oracle performs.

    ``dense`` counts every product (p x q)(q x r) as 2pqr FLOPs.
    ``symmetric`` counts a product whose result is symmetric as pqr (one
    triangle), and any other product as 2pqr, as the page's FLOP formulas do.
    """

    dense: int = 0
    symmetric: int = 0
    products: list = field(default_factory=list)

    def add(self, p: int, q: int, r: int, sym: bool, name: str) -> None:
        self.dense += 2 * p * q * r
        self.symmetric += (p * q * r) if sym else (2 * p * q * r)
        self.products.append((name, p, q, r, sym))


def _mm(A, B, counter, sym, name):
    if counter is not None:
        counter.add(A.shape[0], A.shape[1], B.shape[1], sym, name)
    return A @ B


def _keep(x, store, role):
    """Storage point: identity in exact mode; ``store(x, role)`` when a
    rounding emulation is requested (a diagnostic only)."""
    return x if store is None else store(x, role)


# ---------------------------------------------------------------------------
# Eq. (1) and Definition 1
# ---------------------------------------------------------------------------


def momentum(M, G, mu):
    """Eq. (1), first line: M <- mu*M + G, float32 state, one rounding."""
    return fma_f32(F32(mu), M, G)


def momentum_accumulate(M, G):
    """Dion3 reading of the momentum: M <- M + G (decay moved to the error
    feedback of Algorithm 4, step 4). One float32 rounding."""
    return (np.asarray(M, F32) + np.asarray(G, F32)).astype(F32)


def polar_svd(X):
    """Definition 1: polar(X) = U V^T from the thin SVD X = U S V^T."""
    U, _, Vt = np.linalg.svd(np.asarray(X, F64), full_matrices=False)
    return U @ Vt


def frobenius_normalize(X, eps=1e-7):
    """X_0 = X / (||X||_F + eps) ("Standard Newton-Schulz": the normalisation
    that puts every singular value in [0, 1])."""
    X = np.asarray(X, F64)
    return X / (math.sqrt(float(np.sum(X * X))) + eps)


def _wide(X):
    """Return (X in wide orientation, transposed?) -- alpha = m/n >= 1."""
    if X.shape[0] > X.shape[1]:
        return X.T, True
    return X, False


# ---------------------------------------------------------------------------
# Standard Newton-Schulz
# ---------------------------------------------------------------------------


def ns_iterations(X0, coeffs, counter=None, store=None):
    """T quintic steps on an already normalised wide X0 (n <= m):
    A = X X^T ; B = b A + c A A ; X <- a X + B X."""
    X = X0
    n = X.shape[0]
    for (a, b, c) in coeffs:
        A = _keep(_mm(X, X.T, counter, True, "XXt"), store, "A")
        B = _keep(b * A + c * _mm(A, A, counter, True, "AA"), store, "B")
        X = _keep(a * X + _mm(B, X, counter, False, "BX"), store, "X")
        assert X.shape[0] == n
    return X


def newton_schulz(X, coeffs, eps=1e-7, counter=None, store=None):
    """Standard Newton-Schulz approximation of polar(X) (any orientation)."""
    Xw, tr = _wide(np.asarray(X, F64))
    X0 = _keep(frobenius_normalize(Xw, eps), store, "X0")
    O = ns_iterations(X0, coeffs, counter, store)
    return O.T if tr else O


# ---------------------------------------------------------------------------
# Gram Newton-Schulz (Theorem 2, naive structure, restart of Algorithm 3)
# ---------------------------------------------------------------------------


def h_poly(y, a, b, c):
    """h_t(y) with p_t(x) = x h_t(x^2) for p_t(x) = a x + b x^3 + c x^5."""
    return a + b * y + c * y * y


def compose_scalar(x, coeffs):
    """(p_T o ... o p_1)(x) by direct composition."""
    x = np.asarray(x, F64)
    for (a, b, c) in coeffs:
        x = a * x + b * x ** 3 + c * x ** 5
    return x


def theorem2_q(x, coeffs):
    """q_T of Theorem 2: r_0 = x^2, q_0 = 1, z_t = h_t(r_{t-1}),
    r_t = r_{t-1} z_t^2, q_t = q_{t-1} z_t.  Theorem 2: composition = q_T x."""
    x = np.asarray(x, F64)
    r = x * x
    q = np.ones_like(x)
    for (a, b, c) in coeffs:
        z = h_poly(r, a, b, c)
        r = r * z * z
        q = q * z
    return q


def gram_iterations(X0, coeffs, restart_at=3, counter=None, store=None):
    """Gram Newton-Schulz on a normalised wide X0.

    R_0 = X X^T; for each t: Z_t = a I + b R + c R^2 (the matrix h_t),
    Q_t = Q_{t-1} Z_t (Q_0 = I, so Q_1 = Z_1 costs nothing),
    R_t = Z_t R_{t-1} Z_t (= R_{t-1} Z_t^2, kept in symmetric form; not formed
    after the last step). Output Q_T X.

    Restart (Algorithm 3): with restart_at = r > 0, before step r the current
    Q is applied, X <- Q X, R <- X X^T and Q <- I. R_{r-1} is then never
    formed. restart_at = 0 disables the restart (the naive version).
    """
    X = X0
    n = X.shape[0]
    I = np.eye(n)
    T = len(coeffs)
    R = _keep(_mm(X, X.T, counter, True, "XXt"), store, "R")
    Q = None
    for t, (a, b, c) in enumerate(coeffs, start=1):
        if restart_at and t == restart_at and Q is not None:
            X = _keep(_mm(Q, X, counter, False, "QX"), store, "X")
            R = _keep(_mm(X, X.T, counter, True, "XXt"), store, "R")
            Q = None
        Z = _keep(a * I + b * R + c * _mm(R, R, counter, True, "RR"), store, "Z")
        Q = Z if Q is None else _keep(_mm(Q, Z, counter, True, "QZ"), store, "Q")
        last = t == T
        restart_next = bool(restart_at) and (t + 1 == restart_at)
        if not last and not restart_next:
            ZR = _keep(_mm(Z, R, counter, True, "ZR"), store, "ZR")
            R = _keep(_mm(ZR, Z, counter, True, "ZRZ"), store, "R")
    return _mm(Q, X, counter, False, "QX")


def gram_newton_schulz(X, coeffs, eps=1e-7, restart_at=3, counter=None, store=None):
    """Gram Newton-Schulz approximation of polar(X) (any orientation)."""
    Xw, tr = _wide(np.asarray(X, F64))
    X0 = _keep(frobenius_normalize(Xw, eps), store, "X0")
    O = gram_iterations(X0, coeffs, restart_at, counter, store)
    O = _keep(O, store, "O")
    return O.T if tr else O


# ---------------------------------------------------------------------------
# FLOP formulas as printed on the page (for the counter pins)
# ---------------------------------------------------------------------------


def flops_standard_dense(n, m, T):
    """"FLOP Analysis of Standard Newton-Schulz": T (4 m n^2 + 2 n^3)."""
    return T * (4 * m * n * n + 2 * n ** 3)


def flops_standard_symmetric(n, m, T):
    """Standard NS with symmetric GEMMs: T (3 alpha + 1) n^3 = T (3 m n^2 + n^3)."""
    return T * (3 * m * n * n + n ** 3)


def flops_gram(n, m, T):
    """Gram NS with symmetric GEMMs: (4T + 3 alpha - 3) n^3."""
    return 4 * T * n ** 3 + 3 * m * n * n - 3 * n ** 3


def flops_restart_extra(n, m):
    """Cost of one restart: 3 (alpha - 1) n^3."""
    return 3 * m * n * n - 3 * n ** 3


# ---------------------------------------------------------------------------
# NorMuon, Eq. (2)
# ---------------------------------------------------------------------------


def normuon(O, v, beta2, eps):
    """Eq. (2) on the rows of O (k x m) with their second moments v (k).

    v_i <- beta2 v_i + (1 - beta2) (1/m) sum_j O_ij^2
    O_hat_ij = O_ij / (sqrt(v_i) + eps)
    update direction = (||O||_F / ||O_hat||_F) O_hat

    Returns (v_new, row_scale) with update = row_scale[:, None] * O.
    """
    O = np.asarray(O, F64)
    v = np.asarray(v, F64)
    m = O.shape[1]
    r = np.sum(O * O, axis=1)
    v_new = beta2 * v + (1.0 - beta2) * r / m
    d = 1.0 / (np.sqrt(v_new) + eps)
    norm_o = math.sqrt(float(np.sum(r)))
    norm_ohat = math.sqrt(float(np.sum(d * d * r)))
    ratio = 0.0 if norm_ohat == 0.0 else norm_o / norm_ohat
    return v_new, ratio * d


# ---------------------------------------------------------------------------
# Dion3 selection (Algorithm 4, step 1)
# ---------------------------------------------------------------------------


def rows_for_fraction(n, f_num, f_den):
    """k = ceil(f n) for f = f_num / f_den, in exact integer arithmetic."""
    return (n * f_num + f_den - 1) // f_den


def row_keys(M, norm="l1"):
    """Per-row selection key in float64: sum_j |M_ij| (l1, the page's rule)
    or sum_j M_ij^2 (ordering by the l2 norm)."""
    M = np.asarray(M, F64)
    if norm == "l1":
        return np.sum(np.abs(M), axis=1)
    if norm == "l2":
        return np.sum(M * M, axis=1)
    raise ValueError(norm)


def select_rows(M, k, norm="l1"):
    """Indices of the k rows with the largest key; ties to the lower index;
    returned in ascending order."""
    keys = row_keys(M, norm)
    order = np.argsort(-keys, kind="stable")
    return np.sort(order[:k]).astype(np.int64)


# ---------------------------------------------------------------------------
# Whole steps
# ---------------------------------------------------------------------------


@dataclass
class StepParams:
    mu: float = 0.95
    lr: float = 0.02
    coeffs: tuple = ((3.4445, -4.7750, 2.0315),) * 5
    norm_eps: float = 1e-7
    gram: bool = False
    restart_at: int = 3
    normuon: bool = False
    beta2: float = 0.95
    normuon_eps: float = 1e-8
    k: int | None = None          # Dion3 rows; None = plain Muon
    select_norm: str = "l1"


def orthogonalize(X, p: StepParams, counter=None, store=None):
    if p.gram:
        return gram_newton_schulz(X, p.coeffs, p.norm_eps, p.restart_at, counter, store)
    return newton_schulz(X, p.coeffs, p.norm_eps, counter, store)


def muon_step(W, M, G, v, p: StepParams, store=None):
    """One optimizer step on one matrix.

    Plain Muon (p.k is None): Eq. (1) with optional NorMuon (Eq. (2)).
    Dion3 (p.k given): Algorithm 4 with the momentum reading above.

    Returns dict with the new float32 W, M, v, plus the float64 O (rows as
    selected), the selected indices and the per-row update scales.
    """
    W = np.asarray(W, F32)
    M = np.asarray(M, F32)
    G = np.asarray(G, F32)
    rows = W.shape[0]
    v = np.zeros(rows, F32) if v is None else np.asarray(v, F32)
    if p.k is None:
        M_new = momentum(M, G, p.mu)
        idx = np.arange(rows)
        X = M_new
    else:
        M_new = momentum_accumulate(M, G)
        idx = select_rows(M_new, p.k, p.select_norm)
        X = M_new[idx, :]
    O = orthogonalize(X, p, store=store)
    v_new = v.copy()
    if p.normuon:
        v_rows, scale = normuon(O, v[idx], p.beta2, p.normuon_eps)
        v_new[idx] = v_rows.astype(F32)
    else:
        scale = np.ones(len(idx))
    W_new = W.copy()
    W_new[idx, :] = (W[idx, :].astype(F64) - p.lr * scale[:, None] * O).astype(F32)
    if p.k is not None:
        M_new = M_new.copy()
        M_new[idx, :] = (F32(p.mu) * M_new[idx, :]).astype(F32)
    return {"W": W_new, "M": M_new, "v": v_new, "O": O, "idx": idx, "scale": scale}
