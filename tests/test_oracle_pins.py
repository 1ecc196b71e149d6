"""Pins of the fp64 oracle against facts fixed by the page and by mathematics.

Each test checks the oracle against something other than itself: a value the
page prints, a hand-derived value, a closed form, an SVD-free
characterisation, or brute force. Source page: "Dion3: Full-stack orthogonal
updates" (arXiv 2608.11612).
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from newton_schulz_10_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")
COEFFS5 = ((3.4445, -4.7750, 2.0315),) * 5
# Textbook converging quintic p(x) = (15x - 10x^3 + 3x^5)/8: p(1) = 1,
# p'(1) = p''(1) = 0, so its iterates converge to polar(X).
CONVERGING = (15 / 8, -10 / 8, 3 / 8)


def load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(np.asarray(b)), 1e-300)


def gaussian(shape, seed):
    return inputs.rng(seed, 0).standard_normal(shape)


# ---------------------------------------------------------------------------
# fp32 fused multiply-add emulation (momentum state)
# ---------------------------------------------------------------------------


def _exact_round_f32(x: Fraction) -> np.float32:
    """Round an exact rational to float32, nearest-even, by bisection over the
    float32 neighbours (independent of the oracle's TwoSum method)."""
    f = np.float32(float(x))  # close, maybe off by one ulp
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    best = min(cands, key=lambda c: (abs(Fraction(float(c)) - x),
                                     int(np.array(c, np.float32).view(np.uint32)) & 1))
    return np.float32(best)


def test_fma_f32_matches_exact_rationals():
    g = inputs.rng(11, 0)
    a = g.standard_normal(3000).astype(np.float32)
    b = g.standard_normal(3000).astype(np.float32)
    c = (g.standard_normal(3000) * 10.0 ** g.integers(-3, 3, 3000)).astype(np.float32)
    got = O.fma_f32(a, b, c)
    for i in range(3000):
        want = _exact_round_f32(Fraction(float(a[i])) * Fraction(float(b[i])) + Fraction(float(c[i])))
        assert got[i] == want, i


def test_fma_f32_midpoint_ties():
    # c = 1, a*b = 2^-24 + 2^-60: a plain double sum rounds to 1 + 2^-24,
    # exactly halfway between 1 and 1 + 2^-23, then ties to 1.0; the exact
    # value is above the midpoint, so the fused result must be 1 + 2^-23.
    a = np.float32(2.0 ** -12 * (1 + 2.0 ** -23))
    b = np.float32(2.0 ** -12 * (1 - 2.0 ** -23))  # a*b = 2^-24 (1 - 2^-46)
    c = np.float32(1.0)
    exact = Fraction(float(a)) * Fraction(float(b)) + 1
    assert O.fma_f32(a, b, c) == _exact_round_f32(exact)
    a2 = np.float32(2.0 ** -12 * (1 + 2.0 ** -23))
    b2 = np.float32(2.0 ** -12 * (1 + 2.0 ** -23))  # a*b = 2^-24 (1 + 2^-22 + 2^-46)
    exact2 = Fraction(float(a2)) * Fraction(float(b2)) + 1
    assert O.fma_f32(a2, b2, c) == _exact_round_f32(exact2)
    # many near-tie cases: c in [1, 2), a*b tiny and near half an ulp
    g = inputs.rng(12, 0)
    for _ in range(500):
        cc = np.float32(1.0 + g.integers(0, 2 ** 23) * 2.0 ** -23)
        aa = np.float32(2.0 ** -12 * (1 + g.integers(-4, 5) * 2.0 ** -23))
        bb = np.float32(2.0 ** -12 * (1 + g.integers(-4, 5) * 2.0 ** -23))
        want = _exact_round_f32(Fraction(float(aa)) * Fraction(float(bb)) + Fraction(float(cc)))
        assert O.fma_f32(aa, bb, cc) == want


def test_momentum_matches_eq1():
    g = inputs.rng(13, 0)
    M = g.standard_normal((7, 9)).astype(np.float32)
    G = g.standard_normal((7, 9)).astype(np.float32)
    got = O.momentum(M, G, 0.95)
    want = (np.float32(0.95).astype(np.float64) * M + G).astype(np.float32)
    # differs from the double-rounded value at most by one float32 ulp
    assert np.all(np.abs(got.astype(np.float64) - want) <= np.spacing(np.abs(want)))


# ---------------------------------------------------------------------------
# Definition 1: polar(X) = U V^T
# ---------------------------------------------------------------------------


def _polar_characterisation(X, P):
    """For full-rank wide X, P = polar(X) iff P has orthonormal rows and
    H = X P^T is symmetric positive definite (X = H P)."""
    n = X.shape[0]
    assert np.allclose(P @ P.T, np.eye(n), atol=1e-10)
    H = X @ P.T
    assert np.allclose(H, H.T, atol=1e-10 * np.abs(H).max())
    assert np.min(np.linalg.eigvalsh((H + H.T) / 2)) > 0
    assert rel(H @ P, X) < 1e-12


@pytest.mark.parametrize("shape", [(4, 8), (16, 64), (5, 5)])
def test_polar_svd_characterisation(shape):
    X = gaussian(shape, 21 + shape[0])
    _polar_characterisation(X, O.polar_svd(X))


def test_polar_svd_2x2_hand_value():
    h = load("hand_values.json")["polar_2x2"]
    t = h["theta"]
    R = np.array([[math.cos(t), -math.sin(t)], [math.sin(t), math.cos(t)]])
    X = R @ np.diag(h["s"])
    assert rel(O.polar_svd(X), R) < 1e-14


@pytest.mark.parametrize("shape", [(4, 8), (16, 64), (8, 8), (24, 10)])
def test_converging_ns_reaches_polar(shape):
    X = gaussian(shape, 31 + shape[0] * 7 + shape[1])
    coeffs = (CONVERGING,) * 60
    P = O.polar_svd(X)
    assert rel(O.newton_schulz(X, coeffs, eps=0.0), P) < 1e-10
    assert rel(O.gram_newton_schulz(X, coeffs, eps=0.0, restart_at=3), P) < 1e-9


# ---------------------------------------------------------------------------
# Standard Newton-Schulz: spectral closed form
# ---------------------------------------------------------------------------


def _known_svd(n, m, seed, smin=1e-3):
    U = inputs.random_orthonormal(n, n, seed, 0)
    V = inputs.random_orthonormal(m, n, seed, 1)
    s = np.sort(10 ** (np.log10(smin) * inputs.rng(seed, 2).random(n)))[::-1]
    return U, s, V


@pytest.mark.parametrize("n,m", [(8, 32), (12, 12), (16, 40)])
def test_ns_spectral_closed_form(n, m):
    """Each step keeps the singular vectors and maps sigma -> p_t(sigma), so
    NS_T(X) = U diag(P(sigma / (||X||_F + eps))) V^T."""
    U, s, V = _known_svd(n, m, 40 + n)
    X = (U * s) @ V.T
    eps = 1e-7
    sn = s / (math.sqrt(np.sum(s * s)) + eps)
    P = np.array([O.compose_scalar(x, COEFFS5) for x in sn])
    want = (U * P) @ V.T
    assert rel(O.newton_schulz(X, COEFFS5, eps), want) < 1e-11
    assert rel(O.newton_schulz(X.T, COEFFS5, eps), want.T) < 1e-11
    assert rel(O.gram_newton_schulz(X, COEFFS5, eps, restart_at=3), want) < 1e-9
    assert rel(O.gram_newton_schulz(X, COEFFS5, eps, restart_at=0), want) < 1e-9


def test_quintic_hand_values():
    h = load("hand_values.json")["quintic_step"]
    for case in h["cases"]:
        got = O.compose_scalar(case["x"], (tuple(h["coeffs"]),))
        assert abs(got - case["px"]) < 1e-15


def test_near_unit_band():
    """With the workload coefficients, 5 steps map [1e-2, 1] into a band
    around 1 (they do not converge to exactly 1); the oracle's output singular
    values must lie in that band."""
    grid = np.geomspace(1e-2, 1.0, 20001)
    band = O.compose_scalar(grid, COEFFS5)
    lo, hi = band.min(), band.max()
    assert 0.65 < lo < 0.7 and 1.1 < hi < 1.2
    X = gaussian((32, 128), 51)
    s = np.linalg.svd(X, compute_uv=False)
    assert s.min() / np.linalg.norm(s) > 1e-2  # the input's spectrum is inside the grid
    sv = np.linalg.svd(O.newton_schulz(X, COEFFS5), compute_uv=False)
    assert np.all(sv >= lo - 1e-9) and np.all(sv <= hi + 1e-9)


def test_orthogonality_error_closed_form():
    """||O O^T - I||_F = sqrt(sum_i (P(sigma_i)^2 - 1)^2) for the spectral
    closed form (used for the reported orthogonality error)."""
    U, s, V = _known_svd(10, 30, 61, smin=1e-4)
    X = (U * s) @ V.T
    sn = s / (math.sqrt(np.sum(s * s)) + 1e-7)
    P = O.compose_scalar(sn, COEFFS5)
    Ob = O.newton_schulz(X, COEFFS5)
    got = np.linalg.norm(Ob @ Ob.T - np.eye(10))
    assert abs(got - math.sqrt(np.sum((P * P - 1) ** 2))) < 1e-10


# ---------------------------------------------------------------------------
# Gram Newton-Schulz: Theorem 2 and equivalence
# ---------------------------------------------------------------------------


def test_theorem2_scalar():
    x = np.linspace(0.0, 1.0, 10001)
    for coeffs in (COEFFS5, (CONVERGING,) * 7,
                   ((3.0, -3.2, 1.2), (2.5, -1.5, 0.5), (1.9, -1.3, 0.4))):
        comp = O.compose_scalar(x, coeffs)
        q = O.theorem2_q(x, coeffs)
        assert np.max(np.abs(comp - q * x)) < 1e-13


@pytest.mark.parametrize("n,m,restart", [(16, 64, 3), (16, 64, 0), (24, 24, 3), (10, 70, 2)])
def test_gram_equals_standard(n, m, restart):
    X = gaussian((n, m), 70 + n + m)
    std = O.newton_schulz(X, COEFFS5)
    gram = O.gram_newton_schulz(X, COEFFS5, restart_at=restart)
    assert rel(gram, std) < 1e-9


def test_time_varying_coefficients():
    coeffs = ((4.0, -5.0, 2.1), (3.4445, -4.7750, 2.0315), (3.0, -3.5, 1.6),
              (2.0, -1.5, 0.55), (1.875, -1.25, 0.375))
    U, s, V = _known_svd(12, 36, 81)
    X = (U * s) @ V.T
    sn = s / (math.sqrt(np.sum(s * s)) + 1e-7)
    want = (U * O.compose_scalar(sn, coeffs)) @ V.T
    assert rel(O.newton_schulz(X, coeffs), want) < 1e-11
    assert rel(O.gram_newton_schulz(X, coeffs), want) < 1e-9


# ---------------------------------------------------------------------------
# FLOP formulas (page numbers)
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("n,m,T", [(8, 32, 5), (16, 16, 5), (8, 56, 3), (12, 48, 7)])
def test_flop_counter_matches_page_formulas(n, m, T):
    coeffs = COEFFS5[:1] * T
    X = gaussian((n, m), 90)
    c = O.FlopCounter()
    O.newton_schulz(X, coeffs, counter=c)
    assert c.dense == O.flops_standard_dense(n, m, T) == T * (4 * m * n * n + 2 * n ** 3)
    assert c.symmetric == O.flops_standard_symmetric(n, m, T) == T * (3 * m * n * n + n ** 3)
    g0 = O.FlopCounter()
    O.gram_newton_schulz(X, coeffs, restart_at=0, counter=g0)
    assert g0.symmetric == O.flops_gram(n, m, T) == (4 * T * n ** 3 + 3 * m * n * n - 3 * n ** 3)
    if T >= 3:
        g3 = O.FlopCounter()
        O.gram_newton_schulz(X, coeffs, restart_at=3, counter=g3)
        assert g3.symmetric - g0.symmetric == O.flops_restart_extra(n, m) == 3 * (m - n) * n * n


def test_page_printed_flop_numbers():
    p = load("page_numbers.json")
    s = p["standard_ns_T5"]
    for alpha in (1, 2, 4, 8):
        n = 6
        assert O.flops_standard_dense(n, alpha * n, s["T"]) == \
            (s["flops_over_n3_per_alpha"] * alpha + s["flops_over_n3_const"]) * n ** 3
    c = O.FlopCounter()
    O.newton_schulz(gaussian((4, 16), 1), COEFFS5, counter=c)
    assert len(c.products) == s["gemm_count"]
    g = p["gram_saving_alpha4_T5"]
    n = 10
    saving = 1 - O.flops_gram(n, g["alpha"] * n, g["T"]) / O.flops_standard_symmetric(n, g["alpha"] * n, g["T"])
    assert round(100 * saving) == g["saving_percent"]
    r = p["restart_extra"]
    assert O.flops_restart_extra(n, 4 * n) == r["per_alpha_minus_1"] * 3 * n ** 3


def test_lr_transfer_norm_fact():
    """||polar(X)||_F^2 = rows for full-rank wide X, the fact behind the page's
    learning-rate transfer eta' = eta / sqrt(f)."""
    X = gaussian((12, 40), 3)
    assert abs(np.linalg.norm(O.polar_svd(X)) ** 2 - 12) < 1e-10
    k = O.rows_for_fraction(12, 1, 4)
    assert abs(np.linalg.norm(O.polar_svd(X[:k])) ** 2 - k) < 1e-10


# ---------------------------------------------------------------------------
# NorMuon (Eq. (2)) by hand
# ---------------------------------------------------------------------------


def test_normuon_hand_values():
    h = load("hand_values.json")["normuon_two_steps"]
    v1, s1 = O.normuon(np.array(h["O1"]), np.array(h["v0"]), h["beta2"], h["eps"])
    assert np.allclose(v1, h["v1"], rtol=0, atol=1e-15)
    assert np.allclose(s1, h["scale1"], rtol=1e-15)
    v2, s2 = O.normuon(np.array(h["O2"]), v1, h["beta2"], h["eps"])
    assert np.allclose(v2, h["v2"], rtol=1e-15)
    d = np.array([1 / math.sqrt(3.75), 1 / math.sqrt(5.25)])
    ratio = math.sqrt(63 / (9.6 + 36 / 7))
    assert np.allclose(s2, ratio * d, rtol=1e-14)


def test_normuon_orthonormal_rows_is_muon():
    """If O has orthonormal rows every row sum of squares is 1, all d_i are
    equal and the ratio cancels them: the NorMuon update equals Muon's."""
    P = O.polar_svd(gaussian((6, 20), 5))
    for v in (np.zeros(6), np.linspace(0.01, 0.3, 6) * 0 + 0.07):
        _, s = O.normuon(P, v, 0.95, 1e-8)
        assert np.allclose(s, 1.0, rtol=1e-12)


def test_normuon_zero_matrix():
    v, s = O.normuon(np.zeros((3, 4)), np.zeros(3), 0.95, 1e-8)
    assert np.all(v == 0) and np.all(s == 0)


# ---------------------------------------------------------------------------
# Dion3 selection (Algorithm 4, step 1)
# ---------------------------------------------------------------------------


def _brute_select(M, k, norm):
    keys = [sum(abs(float(x)) for x in row) if norm == "l1" else sum(float(x) ** 2 for x in row)
            for row in M]
    best = None
    for S in itertools.combinations(range(len(M)), k):
        # a valid top-k set: every chosen key >= every unchosen key, and on
        # equal keys the chosen index is lower
        ok = all((keys[i] > keys[j]) or (keys[i] == keys[j] and i < j)
                 for i in S for j in range(len(M)) if j not in S)
        if ok:
            assert best is None
            best = list(S)
    return best


@pytest.mark.parametrize("norm", ["l1", "l2"])
def test_select_rows_brute_force(norm):
    g = inputs.rng(101, 0)
    for trial in range(30):
        n = int(g.integers(1, 9))
        M = g.standard_normal((n, 5)).astype(np.float32)
        if n >= 3:  # plant exact ties by duplicating rows (also sign flips)
            M[n - 1] = M[0]
            M[1] = -M[0] if norm == "l2" or trial % 2 else M[0]
        for k in range(1, n + 1):
            assert list(O.select_rows(M, k, norm)) == _brute_select(M, k, norm)


def test_rows_for_fraction():
    assert O.rows_for_fraction(8192, 1, 4) == 2048
    assert O.rows_for_fraction(10, 1, 3) == 4
    assert O.rows_for_fraction(9, 1, 3) == 3
    assert O.rows_for_fraction(1, 1, 8) == 1
    assert O.rows_for_fraction(77, 1, 1) == 77
    M = gaussian((9, 4), 7)
    assert list(O.select_rows(M, 9)) == list(range(9))  # f = 1 selects all rows


# ---------------------------------------------------------------------------
# Whole steps
# ---------------------------------------------------------------------------


def test_zero_momentum_leaves_weights():
    W = gaussian((6, 10), 9).astype(np.float32)
    z = np.zeros((6, 10), np.float32)
    for gram in (False, True):
        for normuon in (False, True):
            out = O.muon_step(W, z, z, None, O.StepParams(gram=gram, normuon=normuon))
            assert np.all(out["O"] == 0) and np.array_equal(out["W"], W)


def test_muon_step_is_eq1():
    g = inputs.rng(5, 1)
    W = g.standard_normal((8, 20)).astype(np.float32)
    M = g.standard_normal((8, 20)).astype(np.float32)
    G = g.standard_normal((8, 20)).astype(np.float32)
    p = O.StepParams(lr=0.1)
    out = O.muon_step(W, M, G, None, p)
    M1 = O.fma_f32(np.float32(0.95), M, G)
    assert np.array_equal(out["M"], M1)
    U, s, Vt = np.linalg.svd(M1.astype(np.float64), full_matrices=False)
    sn = s / (np.linalg.norm(s) + 1e-7)
    Ow = (U * O.compose_scalar(sn, p.coeffs)) @ Vt
    # W is float32 state: its rounding (~6e-8 |W|) bounds the match of the step
    assert rel(out["W"].astype(np.float64) - W, -0.1 * Ow) < 1e-5


def test_dion3_full_fraction_equals_muon():
    """With f = 1 (k = rows) and zero initial momentum, Dion3's state is mu
    times Muon's and the weight trajectories agree."""
    g = inputs.rng(6, 1)
    W0 = g.standard_normal((10, 24)).astype(np.float32)
    Wm, Mm = W0.copy(), np.zeros_like(W0)
    Wd, Md = W0.copy(), np.zeros_like(W0)
    for step in range(3):
        G = g.standard_normal(W0.shape).astype(np.float32)
        a = O.muon_step(Wm, Mm, G, None, O.StepParams())
        b = O.muon_step(Wd, Md, G, None, O.StepParams(k=10, gram=True))
        Wm, Mm, Wd, Md = a["W"], a["M"], b["W"], b["M"]
        assert rel(Md, 0.95 * Mm) < 1e-6
        assert rel(Wd - W0, Wm - W0) < 1e-6


def test_dion3_updates_only_selected_rows():
    g = inputs.rng(7, 1)
    W = g.standard_normal((12, 16)).astype(np.float32)
    M = g.standard_normal((12, 16)).astype(np.float32)
    G = g.standard_normal((12, 16)).astype(np.float32)
    out = O.muon_step(W, M, G, np.zeros(12, np.float32), O.StepParams(k=3, normuon=True, gram=True))
    S = out["idx"]
    assert len(S) == 3 and list(S) == sorted(S)
    others = np.setdiff1d(np.arange(12), S)
    M1 = M + G
    assert np.array_equal(out["W"][others], W[others])
    assert np.array_equal(out["M"][others], M1[others])
    assert np.array_equal(out["M"][S], (np.float32(0.95) * M1[S]).astype(np.float32))
    assert np.all(out["v"][others] == 0) and np.all(out["v"][S] > 0)
    # the selected rows are the 3 largest l1 rows of M + G
    l1 = np.abs(M1.astype(np.float64)).sum(1)
    assert set(S) == set(np.argsort(-l1)[:3])


# ---------------------------------------------------------------------------
# Whole steps with NorMuon ("NorMuon Variant", Eq. (2), applied to the
# orthogonalised momentum of Eq. (1) and, for Dion3, to the selected rows of
# Algorithm 4). The expected values come from the spectral closed form of the
# Newton-Schulz output (numpy's SVD of the momentum) and from Eq. (2) written
# out row by row with Python floats, not from the oracle's own code path.
# ---------------------------------------------------------------------------


def _ns_closed_form(X, coeffs, eps=1e-7):
    """NS_T(X) = U diag(P(sigma / (||X||_F + eps))) V^T from numpy's SVD."""
    U, s, Vt = np.linalg.svd(np.asarray(X, np.float64), full_matrices=False)
    sn = s / (math.sqrt(float(np.sum(s * s))) + eps)
    return (U * O.compose_scalar(sn, coeffs)) @ Vt


def _eq2_by_rows(Orows, v_rows, beta2, eps):
    """Eq. (2) one row at a time: v_i <- beta2 v_i + (1 - beta2) mean_j O_ij^2,
    d_i = 1 / (sqrt(v_i) + eps), scale_i = d_i ||O||_F / ||diag(d) O||_F."""
    k, m = Orows.shape
    r = [math.fsum(float(x) * float(x) for x in Orows[i]) for i in range(k)]
    v_new = [beta2 * float(v_rows[i]) + (1.0 - beta2) * r[i] / m for i in range(k)]
    d = [1.0 / (math.sqrt(v) + eps) for v in v_new]
    ratio = math.sqrt(math.fsum(r)) / math.sqrt(math.fsum(d[i] * d[i] * r[i] for i in range(k)))
    return np.array(v_new), np.array([ratio * di for di in d])


@pytest.mark.parametrize("shape", [(8, 20), (20, 8)])
def test_normuon_muon_step_closed_form(shape):
    """Plain Muon with NorMuon: W_i -= lr scale_i O_i for every stored row i,
    v updated in place, with O the closed-form Newton-Schulz output of the
    momentum. Rows of G have unequal norms, so the scales are far from 1 and
    a dropped scale or a mis-scattered v changes the result."""
    rows, cols = shape
    g = inputs.rng(41, rows)
    W = g.standard_normal(shape).astype(np.float32)
    G = (g.standard_normal(shape) * np.linspace(0.2, 3.0, rows)[:, None]).astype(np.float32)
    v0 = (0.01 + 0.2 * g.random(rows)).astype(np.float32)
    p = O.StepParams(lr=0.1, normuon=True, beta2=0.9, normuon_eps=1e-4)
    out = O.muon_step(W, np.zeros(shape, np.float32), G, v0, p)
    # M0 = 0: the momentum 0.95 * 0 + G is G exactly
    assert np.array_equal(out["M"], G)
    Ocf = _ns_closed_form(G, p.coeffs)
    v_want, scale = _eq2_by_rows(Ocf, v0, p.beta2, p.normuon_eps)
    assert np.ptp(scale) > 0.2 * np.mean(scale)
    assert rel(out["v"].astype(np.float64), v_want) < 1e-6
    assert rel(out["W"].astype(np.float64) - W, -p.lr * scale[:, None] * Ocf) < 1e-5


def test_normuon_dion3_step_closed_form():
    """Dion3 with NorMuon (Algorithm 4 with Eq. (2) on the selected rows):
    rows 2, 5, 9 and 11 carry ten times the momentum, so they are the k = 4
    rows with the largest l1 norm. Only those rows of W and v change, v by
    Eq. (2) from its own old values, W by lr scale_i times the closed-form
    polar approximation of M[S]; M[S] is then multiplied by mu."""
    n, m, k = 12, 16, 4
    g = inputs.rng(43, 0)
    W = g.standard_normal((n, m)).astype(np.float32)
    M = g.standard_normal((n, m)).astype(np.float32)
    G = g.standard_normal((n, m)).astype(np.float32)
    S = [2, 5, 9, 11]
    M[S] *= 10.0
    v0 = (0.01 + 0.2 * g.random(n)).astype(np.float32)
    p = O.StepParams(lr=0.1, normuon=True, beta2=0.9, normuon_eps=1e-4, k=k)
    out = O.muon_step(W, M, G, v0, p)
    assert list(out["idx"]) == S
    M1 = (M + G).astype(np.float32)
    Ocf = _ns_closed_form(M1[S], p.coeffs)
    v_rows, scale = _eq2_by_rows(Ocf, v0[S], p.beta2, p.normuon_eps)
    assert np.ptp(scale) > 0.02 * np.mean(scale)
    others = np.setdiff1d(np.arange(n), S)
    assert np.array_equal(out["v"][others], v0[others])
    assert rel(out["v"][S].astype(np.float64), v_rows) < 1e-6
    assert np.array_equal(out["W"][others], W[others])
    assert rel(out["W"][S].astype(np.float64) - W[S], -p.lr * scale[:, None] * Ocf) < 1e-5
    assert np.array_equal(out["M"][S], (np.float32(0.95) * M1[S]).astype(np.float32))
    assert np.array_equal(out["M"][others], M1[others])
