"""The oracle's pins must catch plausible mistakes in it.

Each case plants one mistake in the oracle (a dropped term, a flipped sign, a
swapped operand, a wrong index or order) on the CPU and checks that at least
one pin of tests/test_oracle_pins.py then fails. Nothing here touches the
CUDA library.
"""

import contextlib

import numpy as np
import pytest

import oracle
import oracle.muon_oracle as OM
import test_oracle_pins as pins

F64 = np.float64


@contextlib.contextmanager
def planted(name, fn):
    """Replace oracle function `name` (module global and package export)."""
    old_mod = getattr(OM, name)
    old_pkg = getattr(oracle, name, None)
    setattr(OM, name, fn)
    if old_pkg is not None:
        setattr(oracle, name, fn)
    try:
        yield
    finally:
        setattr(OM, name, old_mod)
        if old_pkg is not None:
            setattr(oracle, name, old_pkg)


def fails(*checks):
    """True if at least one pin check raises (an assertion or an error)."""
    for check in checks:
        try:
            check()
        except Exception:  # noqa: BLE001 - any failure of a pin counts
            return True
    return False


def ns_pins():
    return [lambda: pins.test_ns_spectral_closed_form(8, 32), lambda: pins.test_ns_spectral_closed_form(12, 12),
            pins.test_near_unit_band, pins.test_orthogonality_error_closed_form,
            lambda: pins.test_converging_ns_reaches_polar((16, 64)), pins.test_time_varying_coefficients]


def gram_pins():
    return [lambda: pins.test_gram_equals_standard(16, 64, 3), lambda: pins.test_gram_equals_standard(10, 70, 2),
            lambda: pins.test_gram_equals_standard(16, 64, 0),
            lambda: pins.test_flop_counter_matches_page_formulas(8, 32, 5), pins.test_page_printed_flop_numbers]


def _ns_iter_dropped_cubic(X0, coeffs, counter=None, store=None):
    X = X0
    for (a, b, c) in coeffs:  # mistake: B = b A (the c A^2 term is dropped)
        A = X @ X.T
        X = a * X + (b * A) @ X
    return X


def _ns_iter_flipped_sign(X0, coeffs, counter=None, store=None):
    X = X0
    for (a, b, c) in coeffs:  # mistake: -b
        A = X @ X.T
        X = a * X + (-b * A + c * A @ A) @ X
    return X


def _ns_iter_a_on_both(X0, coeffs, counter=None, store=None):
    X = X0
    for (a, b, c) in coeffs:  # mistake: a multiplies the B X term too
        A = X @ X.T
        X = a * (X + (b * A + c * A @ A) @ X)
    return X


def _normalize_no_root(X, eps=1e-7):
    X = np.asarray(X, F64)
    return X / (float(np.sum(X * X)) + eps)  # mistake: squared norm


def _gram_no_q_update(X0, coeffs, restart_at=3, counter=None, store=None):
    X = X0
    I = np.eye(X.shape[0])
    R = X @ X.T
    Q = I
    for (a, b, c) in coeffs:  # mistake: Q keeps only the last Z
        Z = a * I + b * R + c * R @ R
        Q = Z
        R = Z @ R @ Z
    return Q @ X


def _gram_restart_forgets_q(X0, coeffs, restart_at=3, counter=None, store=None):
    X = X0
    I = np.eye(X.shape[0])
    R = X @ X.T
    Q = I
    for t, (a, b, c) in enumerate(coeffs, start=1):
        if restart_at and t == restart_at:  # mistake: restart without applying Q to X
            R = X @ X.T
            Q = I
        Z = a * I + b * R + c * R @ R
        Q = Q @ Z
        R = Z @ R @ Z
    return Q @ X


def _theorem2_wrong_r(x, coeffs):
    x = np.asarray(x, F64)
    r = x * x
    q = np.ones_like(x)
    for (a, b, c) in coeffs:
        z = OM.h_poly(r, a, b, c)
        r = r * z  # mistake: z instead of z^2
        q = q * z
    return q


def _normuon_no_mean(O, v, beta2, eps):
    O = np.asarray(O, F64)
    r = np.sum(O * O, axis=1)
    v_new = beta2 * v + (1 - beta2) * r  # mistake: no 1/m
    d = 1.0 / (np.sqrt(v_new) + eps)
    no, nh = np.sqrt(np.sum(r)), np.sqrt(np.sum(d * d * r))
    return v_new, (no / nh if nh else 0.0) * d


def _normuon_inverted_ratio(O, v, beta2, eps):
    O = np.asarray(O, F64)
    m = O.shape[1]
    r = np.sum(O * O, axis=1)
    v_new = beta2 * v + (1 - beta2) * r / m
    d = 1.0 / (np.sqrt(v_new) + eps)
    no, nh = np.sqrt(np.sum(r)), np.sqrt(np.sum(d * d * r))
    return v_new, (nh / no if no else 0.0) * d  # mistake: inverted ratio


def _select_ties_high(M, k, norm="l1"):
    keys = OM.row_keys(M, norm)
    order = np.lexsort((-np.arange(len(keys)), -keys))  # mistake: ties to the higher index
    return np.sort(order[:k])


def _select_smallest(M, k, norm="l1"):
    keys = OM.row_keys(M, norm)
    return np.sort(np.argsort(keys, kind="stable")[:k])  # mistake: smallest keys


def _momentum_swapped(M, G, mu):
    return OM.fma_f32(np.float32(mu), G, M)  # mistake: mu*G + M


def _fma_double_rounded(a, b, c):
    return (np.asarray(a, F64) * np.asarray(b, F64) + np.asarray(c, F64)).astype(np.float32)


def _compose_missing_quintic(x, coeffs):
    x = np.asarray(x, F64)
    for (a, b, c) in coeffs:
        x = a * x + b * x ** 3  # mistake: no x^5 term
    return x


def _polar_u_only(X):
    U, _, Vt = np.linalg.svd(np.asarray(X, F64), full_matrices=False)
    return U  # mistake: U instead of U V^T


def _step_mutant(drop_scale=False, scatter_first=False, read_first=False):
    """The oracle's whole step with one planted mistake in its NorMuon branch."""
    def step(W, M, G, v, p, store=None):
        W = np.asarray(W, np.float32)
        M = np.asarray(M, np.float32)
        G = np.asarray(G, np.float32)
        rows = W.shape[0]
        v = np.zeros(rows, np.float32) if v is None else np.asarray(v, np.float32)
        if p.k is None:
            M_new = OM.momentum(M, G, p.mu)
            idx = np.arange(rows)
        else:
            M_new = OM.momentum_accumulate(M, G)
            idx = OM.select_rows(M_new, p.k, p.select_norm)
        Ow = OM.orthogonalize(M_new[idx, :], p, store=store)
        v_new = v.copy()
        k = len(idx)
        src = np.arange(k) if read_first else idx          # mistake: v of the first k rows
        v_rows, scale = OM.normuon(Ow, v[src], p.beta2, p.normuon_eps)
        v_new[np.arange(k) if scatter_first else idx] = v_rows.astype(np.float32)  # mistake: wrong rows
        if drop_scale:
            scale = np.ones(k)                              # mistake: W -= lr O
        W_new = W.copy()
        W_new[idx, :] = (W[idx, :].astype(F64) - p.lr * scale[:, None] * Ow).astype(np.float32)
        if p.k is not None:
            M_new = M_new.copy()
            M_new[idx, :] = (np.float32(p.mu) * M_new[idx, :]).astype(np.float32)
        return {"W": W_new, "M": M_new, "v": v_new, "O": Ow, "idx": idx, "scale": scale}
    step.__name__ = ("_step_drop_scale" if drop_scale else "_step_v_scatter_first" if scatter_first
                     else "_step_v_read_first")
    return step


def normuon_step_pins():
    return [lambda: pins.test_normuon_muon_step_closed_form((8, 20)),
            lambda: pins.test_normuon_muon_step_closed_form((20, 8)),
            pins.test_normuon_dion3_step_closed_form]


CASES = [
    ("ns_iterations", _ns_iter_dropped_cubic, ns_pins),
    ("ns_iterations", _ns_iter_flipped_sign, ns_pins),
    ("ns_iterations", _ns_iter_a_on_both, ns_pins),
    ("frobenius_normalize", _normalize_no_root, ns_pins),
    ("gram_iterations", _gram_no_q_update, gram_pins),
    ("gram_iterations", _gram_restart_forgets_q, gram_pins),
    ("theorem2_q", _theorem2_wrong_r, lambda: [pins.test_theorem2_scalar]),
    ("compose_scalar", _compose_missing_quintic,
     lambda: [pins.test_quintic_hand_values, pins.test_theorem2_scalar]),
    ("normuon", _normuon_no_mean, lambda: [pins.test_normuon_hand_values]),
    ("normuon", _normuon_inverted_ratio,
     lambda: [pins.test_normuon_hand_values, pins.test_normuon_orthonormal_rows_is_muon]),
    ("select_rows", _select_ties_high, lambda: [lambda: pins.test_select_rows_brute_force("l1")]),
    ("select_rows", _select_smallest, lambda: [lambda: pins.test_select_rows_brute_force("l2")]),
    ("momentum", _momentum_swapped, lambda: [pins.test_momentum_matches_eq1, pins.test_muon_step_is_eq1]),
    ("fma_f32", _fma_double_rounded, lambda: [pins.test_fma_f32_midpoint_ties]),
    ("polar_svd", _polar_u_only,
     lambda: [lambda: pins.test_polar_svd_characterisation((4, 8)), pins.test_polar_svd_2x2_hand_value]),
    ("muon_step", _step_mutant(drop_scale=True), normuon_step_pins),
    ("muon_step", _step_mutant(scatter_first=True), lambda: [pins.test_normuon_dion3_step_closed_form]),
    ("muon_step", _step_mutant(read_first=True), lambda: [pins.test_normuon_dion3_step_closed_form]),
]


@pytest.mark.parametrize("name,mutant,checks", CASES, ids=[f"{c[0]}:{c[1].__name__}" for c in CASES])
def test_planted_mistake_is_caught(name, mutant, checks):
    # the pins pass on the real oracle ...
    assert not fails(*checks())
    # ... and at least one fails once the mistake is planted
    with planted(name, mutant):
        assert fails(*checks()), f"no pin caught {mutant.__name__}"
