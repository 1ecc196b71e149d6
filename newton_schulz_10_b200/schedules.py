"""Step-dependent Newton-Schulz coefficients.

"Standard Newton-Schulz" of "Dion3: Full-stack orthogonal updates" writes the
iteration with per-step coefficients (a_t, b_t, c_t); the library takes a
table of them (`muon.ns_params(coeffs=...)`). This module builds such a table
for a known range of singular values: step t uses the odd quintic

    p_t(x) = a_t x + b_t x^3 + c_t x^5

that minimises max |1 - p_t(x)| over the interval [l_t, u_t] the singular
values occupy before the step (a minimax, i.e. Chebyshev, approximation of
the constant 1 by the span of x, x^3, x^5, computed by the Remez exchange).
By the alternation theorem the error of the best approximation equioscillates
at four points of [l_t, u_t] with magnitude E_t, so after the step the
singular values lie in [1 - E_t, 1 + E_t], the interval of step t + 1. The
first interval is [lower, 1] for a Frobenius-normalised input (every singular
value is at most 1).

Each interval's upper end is widened by a relative `margin` (default 2%):
the early polynomials are steep, and a singular value that rounding pushes
just above the interval a step was designed for would otherwise be thrown
far outside the next one (with no margin a 2% excess per step diverges; with
2% it stays within [1 - E_T, 1 + E_T]).

Host-side parameter computation only: the iteration itself runs in the
library's kernels with whatever table the caller passes.
"""

from __future__ import annotations

import numpy as np

F64 = np.float64

# The quintic with p(1) = 1 and p'(1) = p''(1) = 0: (15x - 10x^3 + 3x^5) / 8.
CONVERGED = (15.0 / 8.0, -10.0 / 8.0, 3.0 / 8.0)


def _basis(x):
    x = np.asarray(x, F64)
    return np.stack([x, x ** 3, x ** 5], axis=-1)


def _grid(lo: float, hi: float, n: int = 20001) -> np.ndarray:
    """Dense evaluation grid, geometric near a small lower end and uniform
    elsewhere, so both ends of a wide-ratio interval are resolved."""
    g = np.concatenate([np.geomspace(lo, hi, n), np.linspace(lo, hi, n)])
    return np.unique(np.clip(g, lo, hi))


def _alternating_extrema(x: np.ndarray, e: np.ndarray, k: int) -> np.ndarray | None:
    """Indices of k points of x where e has alternating signs and, among
    such choices, large magnitude (the Remez multi-point exchange)."""
    # candidate extrema: interior local extrema of e plus both end points
    cand = [0]
    for i in range(1, len(x) - 1):
        if (e[i] >= e[i - 1] and e[i] >= e[i + 1]) or (e[i] <= e[i - 1] and e[i] <= e[i + 1]):
            cand.append(i)
    cand.append(len(x) - 1)
    # merge runs of equal sign, keeping the largest magnitude of each run
    runs = []
    for i in cand:
        if runs and np.sign(e[i]) == np.sign(e[runs[-1]]):
            if abs(e[i]) > abs(e[runs[-1]]):
                runs[-1] = i
        else:
            runs.append(i)
    # drop runs from the end with the smaller magnitude until k remain
    while len(runs) > k:
        if abs(e[runs[0]]) < abs(e[runs[-1]]):
            runs.pop(0)
        else:
            runs.pop()
    return np.array(runs) if len(runs) == k else None


def _critical_points(coef, lo: float, hi: float) -> list:
    """Interior extrema of 1 - p on (lo, hi): p'(x) = a + 3b x^2 + 5c x^4 is
    a quadratic in y = x^2, so they are square roots of its roots."""
    a, b, c = coef
    if c != 0.0:
        ys = np.roots([5.0 * c, 3.0 * b, a])
    elif b != 0.0:
        ys = np.array([-a / (3.0 * b)])
    else:
        ys = np.array([])
    out = []
    for y in ys:
        if abs(y.imag) <= 1e-12 * max(1.0, abs(y.real)) and lo * lo < y.real < hi * hi:
            out.append(float(np.sqrt(y.real)))
    return sorted(out)


def _max_error(coef, lo: float, hi: float) -> float:
    """max |1 - p(x)| over [lo, hi], attained at an end or a critical point."""
    pts = np.array([lo, *_critical_points(coef, lo, hi), hi])
    return float(np.max(np.abs(1.0 - _basis(pts) @ np.asarray(coef, F64))))


def minimax_quintic(lo: float, hi: float, iters: int = 100, tol: float = 1e-15):
    """(a, b, c) of the odd quintic minimising max |1 - p(x)| on [lo, hi]
    (0 < lo < hi), and that minimal maximum E."""
    if not (0.0 < lo < hi):
        raise ValueError("need 0 < lo < hi")
    # initial reference: Chebyshev extrema of degree 3 mapped to [lo, hi]
    ref = lo + (hi - lo) * 0.5 * (1.0 - np.cos(np.pi * np.arange(4) / 3.0))
    coef = np.zeros(3)
    x = None
    for _ in range(iters):
        # solve p(r_i) + (-1)^i h = 1 on the reference
        A = np.concatenate([_basis(ref), ((-1.0) ** np.arange(4))[:, None]], axis=1)
        sol = np.linalg.solve(A, np.ones(4))
        coef, h = sol[:3], sol[3]
        # exchange: the error's extrema are the two ends and the critical points
        pts = np.array([lo, *_critical_points(coef, lo, hi), hi])
        e = 1.0 - _basis(pts) @ coef
        if len(pts) == 4 and np.all(np.sign(e[1:]) != np.sign(e[:-1])):
            new_ref = pts
        else:
            if x is None:
                x = _grid(lo, hi)
            eg = 1.0 - _basis(x) @ coef
            idx = _alternating_extrema(x, eg, 4)
            if idx is None:
                break
            new_ref = x[idx]
        emax = float(np.max(np.abs(e)))
        if emax - abs(h) <= tol * max(1.0, emax) or np.array_equal(new_ref, ref):
            break
        ref = new_ref
    coef = tuple(float(v) for v in coef)
    return coef, _max_error(coef, lo, hi)


def minimax_schedule(T: int, lower: float, upper: float = 1.0, margin: float = 0.02):
    """T coefficient triples for inputs whose singular values lie in
    [lower, upper]. Each step's interval is the previous step's image
    [1 - E, 1 + E]; `margin` widens the upper end by that relative amount to
    leave room for rounding in half precision (see the module docstring). Returns (coeffs, intervals)
    with intervals[t] = (l_t, u_t) before step t and intervals[T] after."""
    if T < 1 or not (0.0 < lower < upper):
        raise ValueError("need T >= 1 and 0 < lower < upper")
    lo, hi = float(lower), float(upper) * (1.0 + margin)
    coeffs, intervals = [], [(lo, hi)]
    for _ in range(T):
        if hi - lo <= 1e-4 * hi:
            # nearly converged: the Remez system degenerates, and the minimax
            # quintics tend to the one with p(1) = 1, p'(1) = p''(1) = 0
            abc = CONVERGED
            x = np.linspace(lo, hi, 1001)
            E = float(np.max(np.abs(1.0 - _basis(x) @ np.array(abc))))
        else:
            abc, E = minimax_quintic(lo, hi)
        coeffs.append(abc)
        lo, hi = 1.0 - E, (1.0 + E) * (1.0 + margin)
        intervals.append((lo, hi))
    return coeffs, intervals
