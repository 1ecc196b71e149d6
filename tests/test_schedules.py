"""Minimax Newton-Schulz schedules (newton_schulz_10_b200/schedules.py),
pinned by the mathematics rather than by themselves:

- the Chebyshev alternation theorem characterises the best approximation of
  1 by odd quintics on [lo, hi]: the error equioscillates at four points
  with the maximal magnitude, and no other odd quintic does better;
- as the interval shrinks to {1} the minimax quintic tends to the one with
  p(1) = 1, p'(1) = p''(1) = 0, i.e. (15, -10, 3) / 8;
- composing the schedule with the oracle's own scalar composition keeps
  every singular value of [lower, 1] inside the predicted final interval.
"""

import numpy as np
import pytest

import oracle as O
from newton_schulz_10_b200 import schedules as S


def _err(coef, x):
    a, b, c = coef
    return 1.0 - (a * x + b * x ** 3 + c * x ** 5)


@pytest.mark.parametrize("lo,hi", [(0.3, 1.0), (1e-2, 1.0), (1e-3, 1.0), (0.0085, 1.99), (0.45, 1.55)])
def test_alternation_theorem(lo, hi):
    coef, E = S.minimax_quintic(lo, hi)
    x = np.concatenate([np.geomspace(lo, hi, 200001), np.linspace(lo, hi, 200001)])
    e = _err(coef, x)
    assert np.max(np.abs(e)) <= E * (1 + 1e-9)
    # four alternating points reach |e| = E (within the grid's resolution)
    near = np.abs(np.abs(e) - E) <= 1e-6 * max(E, 1e-12)
    signs = np.sign(e[near])
    xs = x[near]
    order = np.argsort(xs)
    alternations = 1 + int(np.sum(signs[order][1:] != signs[order][:-1]))
    assert alternations >= 4
    # and nearby quintics are worse
    rng = np.random.default_rng(0)
    for _ in range(50):
        d = rng.normal(size=3) * 1e-3 * np.abs(coef).max()
        assert np.max(np.abs(_err(np.asarray(coef) + d, x))) > E * (1 - 1e-12)


def test_limit_is_the_converging_quintic():
    prev = None
    for delta in [1e-1, 3e-2, 1e-2]:
        coef, E = S.minimax_quintic(1 - delta, 1 + delta)
        dist = np.max(np.abs(np.asarray(coef) - np.asarray(S.CONVERGED)))
        if prev is not None:
            assert dist < prev
        prev = dist
    assert prev < 0.05
    # (15x - 10x^3 + 3x^5)/8 has p(1) = 1, p'(1) = 0, p''(1) = 0
    a, b, c = S.CONVERGED
    assert a + b + c == 1.0 and a + 3 * b + 5 * c == 0.0 and 6 * b + 20 * c == 0.0


@pytest.mark.parametrize("lower,T", [(1e-3, 5), (1e-3, 8), (1e-5, 10), (1e-5, 12)])
def test_schedule_keeps_singular_values_in_its_intervals(lower, T):
    coeffs, iv = S.minimax_schedule(T, lower)
    assert len(coeffs) == T and len(iv) == T + 1
    x = np.concatenate([np.geomspace(lower, 1.0, 20001), np.linspace(lower, 1.0, 20001)])
    y = x
    for t, abc in enumerate(coeffs):
        y = O.compose_scalar(y, [abc])
        lo, hi = iv[t + 1]
        assert y.min() >= lo - 1e-9 and y.max() <= hi + 1e-9
    # the image intervals shrink towards 1
    widths = [hi - lo for lo, hi in iv]
    assert widths[-1] < widths[0]


def test_converging_schedule_reaches_the_polar_factor():
    """With enough steps the tuned schedule drives every singular value of
    [1e-4, 1] to 1: on a matrix with that spectrum the oracle's NS equals
    the SVD polar factor."""
    coeffs, iv = S.minimax_schedule(12, 1e-4, margin=0.0)
    assert 1 - iv[-1][0] < 1e-10
    rng = np.random.default_rng(3)
    U, _ = np.linalg.qr(rng.normal(size=(24, 24)))
    V, _ = np.linalg.qr(rng.normal(size=(64, 24)))
    sig = np.geomspace(1e-2, 1.0, 24)
    X = (U * sig) @ V.T
    got = O.newton_schulz(X, coeffs)
    assert np.max(np.abs(got - O.polar_svd(X))) < 1e-9


def test_margin_keeps_steep_steps_stable():
    """A 2% excess per step (rounding) stays bounded with the default margin."""
    coeffs, iv = S.minimax_schedule(10, 1e-5)
    y = np.linspace(1e-6, 1.0, 20001)
    for abc in coeffs:
        y = O.compose_scalar(y * 1.02, [abc])
    assert np.all(np.isfinite(y)) and y.max() < 1.2 and y.min() > 0


# ---------------------------------------------------------------------------
# the pins above catch plausible mistakes in the schedule code
# ---------------------------------------------------------------------------

def _one_step_remez(lo, hi, iters=60, tol=1e-13):
    """Mistake: solve on the initial Chebyshev reference, never exchange."""
    return S.minimax_quintic(lo, hi, iters=1)


def _no_alternation(lo, hi, iters=60, tol=1e-13):
    """Mistake: the levelled error term has one sign on every reference point."""
    ref = lo + (hi - lo) * 0.5 * (1.0 - np.cos(np.pi * np.arange(4) / 3.0))
    A = np.concatenate([S._basis(ref), np.ones((4, 1))], axis=1)
    coef = np.linalg.solve(A, np.ones(4))[:3]
    coef = tuple(float(v) for v in coef)
    return coef, S._max_error(coef, lo, hi)


def _stale_intervals(T, lower, upper=1.0, margin=0.02):
    """Mistake: every step designed for the first interval."""
    coeffs, iv = [], [(lower, upper)]
    for _ in range(T):
        abc, E = S.minimax_quintic(lower, upper)
        coeffs.append(abc)
        iv.append((1.0 - E, 1.0 + E))
    return coeffs, iv


def _fails(fn):
    try:
        fn()
    except Exception:  # noqa: BLE001 - any failing pin counts
        return True
    return False


@pytest.mark.parametrize("attr,mutant,pin", [
    ("minimax_quintic", _one_step_remez, lambda: test_alternation_theorem(0.3, 1.0)),
    ("minimax_quintic", _no_alternation, lambda: test_alternation_theorem(1e-2, 1.0)),
    ("minimax_schedule", _stale_intervals, lambda: test_schedule_keeps_singular_values_in_its_intervals(1e-3, 5)),
    ("CONVERGED", (15.0 / 8.0, -10.0 / 8.0, 2.0 / 8.0), test_limit_is_the_converging_quintic),
], ids=["one-step-remez", "no-alternation", "stale-intervals", "wrong-limit"])
def test_planted_schedule_mistake_is_caught(monkeypatch, attr, mutant, pin):
    assert not _fails(pin)
    monkeypatch.setattr(S, attr, mutant)
    assert _fails(pin)
