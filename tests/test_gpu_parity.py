"""Parity of the CUDA library (through its C ABI) with the fp64 oracle.

Tolerances (relative Frobenius error): 1e-4 on fp32 paths, 2e-2 on
bf16/fp16 Newton-Schulz outputs and on the weight change of a bf16 step;
row-selection indices and the fp32 momentum state are compared bit for bit.
"""

import os

import numpy as np
import pytest
import torch

import oracle as O
from newton_schulz_10_b200 import inputs
from newton_schulz_10_b200 import muon as mu

from gpu_util import COEFFS5, bf16_values, dev, gauss, host, rel

pytestmark = pytest.mark.gpu

TOL32 = 1e-4
TOL16 = 2e-2


@pytest.fixture(autouse=True)
def _gpu(cuda):
    yield
    torch.cuda.synchronize()


def status_of(ws) -> int:
    torch.cuda.synchronize()
    return int(ws[:4].view(torch.int32).item())


# ---------------------------------------------------------------------------
# ns_polar / gram_ns_polar
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("shape", [(256, 1024), (300, 100), (17, 33), (1, 40), (64, 64)])
def test_ns_polar_fp32(shape):
    X = gauss(shape, 100 + shape[0])
    Og, ws = mu.ns_polar(dev(X), mu.ns_params(compute=mu.F32))
    assert status_of(ws) == mu.OK
    assert rel(host(Og), O.newton_schulz(X.astype(np.float64), COEFFS5)) < TOL32


BF16_SHAPES = [(128, 512), (200, 520), (520, 200), (64, 64), (300, 300), (1, 96), (96, 1), (8, 4096),
               (768, 3072), (3072, 768), (130, 130), (256, 257)]


@pytest.mark.parametrize("shape", BF16_SHAPES)
def test_ns_polar_bf16(shape):
    X = gauss(shape, 200 + shape[0] + shape[1])
    Og, ws = mu.ns_polar(dev(X), mu.ns_params(compute=mu.BF16), out_dtype=torch.float32)
    assert status_of(ws) == mu.OK
    assert rel(host(Og), O.newton_schulz(X.astype(np.float64), COEFFS5)) < TOL16


def test_ns_polar_bf16_input_output():
    X32 = gauss((192, 640), 7)
    Xb = dev(X32, torch.bfloat16)
    Og, ws = mu.ns_polar(Xb, mu.ns_params(compute=mu.BF16))
    assert Og.dtype == torch.bfloat16 and status_of(ws) == mu.OK
    assert rel(host(Og), O.newton_schulz(bf16_values(X32), COEFFS5)) < TOL16


@pytest.mark.parametrize("compute", [mu.F16, mu.BF16, mu.F32])
@pytest.mark.parametrize("restart", [3, 0])
@pytest.mark.parametrize("shape", [(256, 1024), (200, 520), (520, 200), (96, 96)])
def test_gram_ns_polar(compute, restart, shape):
    if compute == mu.BF16 and shape[0] == shape[1]:
        pytest.skip("bf16 Gram on a square Gaussian input exceeds 2e-2 by the algorithm itself "
                    "(see test_gram_bf16_square_matches_emulation)")
    X = gauss(shape, 300 + shape[0])
    p = mu.ns_params(gram=True, restart_at=restart, compute=compute)
    Og, ws = mu.gram_ns_polar(dev(X), p, out_dtype=torch.float32)
    assert status_of(ws) == mu.OK
    want = O.gram_newton_schulz(X.astype(np.float64), COEFFS5, restart_at=restart)
    assert rel(want, O.newton_schulz(X.astype(np.float64), COEFFS5)) < 1e-9
    assert rel(host(Og), want) < (TOL32 if compute == mu.F32 else TOL16)


def _emulate_bf16(x, role):
    return bf16_values(np.asarray(x, np.float32))


@pytest.mark.parametrize("restart", [3, 0])
def test_gram_bf16_square_matches_emulation(restart):
    """A square Gaussian matrix has singular values down to ~0, where T = 5
    steps amplify rounding ~a^5 = 489 times. In bf16 the Gram iteration then
    misses the exact polar factor by more than 2e-2 by the algorithm itself:
    the oracle, rounding to bf16 at the same storage points, misses it by the
    same amount. The GPU result must not be worse than that emulation by more
    than 25%."""
    X = gauss((96, 96), 396)
    exact = O.gram_newton_schulz(X.astype(np.float64), COEFFS5, restart_at=restart)
    emul = O.gram_newton_schulz(X.astype(np.float64), COEFFS5, restart_at=restart, store=_emulate_bf16)
    Og, ws = mu.gram_ns_polar(dev(X), mu.ns_params(gram=True, restart_at=restart, compute=mu.BF16),
                              out_dtype=torch.float32)
    assert status_of(ws) == mu.OK
    e_alg = rel(emul, exact)
    assert e_alg > 2e-2
    assert rel(host(Og), exact) < 1.25 * e_alg


def _emulate_f16(n):
    """fp16 storage as the library stores it: X as sqrt(n) X, R as n R."""
    kappa, rho = np.sqrt(n), float(n)

    def store(x, role):
        x = np.asarray(x, np.float64)
        if role in ("X0", "X"):
            return (x * kappa).astype(np.float16).astype(np.float64) / kappa
        if role in ("R", "ZR"):
            return (x * rho).astype(np.float16).astype(np.float64) / rho
        return x.astype(np.float16).astype(np.float64)
    return store


@pytest.mark.parametrize("gram,compute", [(False, mu.F16), (False, mu.BF16), (True, mu.F16)])
def test_spectrum_matrix(gram, compute):
    """Singular values log-uniform in [1e-4, 1] (the spectrum workload,
    256 x 1024). After normalisation the smallest are ~1e-5, where T = 5
    quintic steps amplify any rounding ~a^5 = 489 times; how far a half
    precision chain lands from the exact polar factor is then set by the
    arithmetic, not by the kernels. Checks: (1) on the well-conditioned
    directions (normalised sigma > 1e-2) the error is < 2e-2; (2) overall the
    GPU is within 25% of the oracle run with the same half-precision storage;
    (3) where that emulated algorithm meets 2e-2 (fp16 standard), the GPU
    meets 2e-2 too."""
    X, _ = inputs.spectrum_matrix(256, 1024, -4.0, seed=31)
    X32 = X.astype(np.float32)
    p = mu.ns_params(gram=gram, compute=compute)
    Og, ws = mu.ns_polar(dev(X32, torch.bfloat16), p, out_dtype=torch.float32)
    assert status_of(ws) == mu.OK
    Xb = bf16_values(X32)
    exact = O.newton_schulz(Xb, COEFFS5)
    store = _emulate_f16(256) if compute == mu.F16 else _emulate_bf16
    emul = (O.gram_newton_schulz(Xb, COEFFS5, store=store) if gram else O.newton_schulz(Xb, COEFFS5, store=store))
    got = host(Og)
    U, s, _ = np.linalg.svd(Xb, full_matrices=False)
    well = (s / np.linalg.norm(s)) > 1e-2
    assert np.linalg.norm((U.T @ (got - exact))[well]) / np.linalg.norm(exact) < TOL16
    e_alg = rel(emul, exact)
    assert rel(got, exact) < 1.25 * max(e_alg, 4e-3)
    if e_alg < TOL16:
        assert rel(got, exact) < TOL16


def test_time_varying_coefficients():
    coeffs = [(4.0, -5.0, 2.1), (3.4445, -4.7750, 2.0315), (3.0, -3.5, 1.6), (2.0, -1.5, 0.55)]
    X = gauss((128, 384), 41)
    for gram in (False, True):
        p = mu.ns_params(T=4, coeffs=coeffs, gram=gram, compute=mu.F32)
        Og, ws = mu.ns_polar(dev(X), p)
        assert rel(host(Og), O.newton_schulz(X.astype(np.float64), coeffs)) < TOL32


def test_zero_matrix_gives_zero():
    Og, ws = mu.ns_polar(torch.zeros(64, 128, device="cuda"), mu.ns_params())
    assert status_of(ws) == mu.OK and torch.count_nonzero(Og).item() == 0


# ---------------------------------------------------------------------------
# select_rows / normuon_scale
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("norm", [mu.NORM_L1, mu.NORM_L2])
def test_select_rows_exact(norm):
    g = inputs.rng(55, 0)
    for n, m in [(1000, 300), (64, 33), (8192, 256), (5, 4)]:
        M = g.standard_normal((n, m)).astype(np.float32)
        M[n // 2] = M[0]          # exact ties
        M[n - 1] = -M[1]
        Md = dev(M)
        for k in sorted({1, max(1, n // 4), n // 2 or 1, n}):
            idx = mu.select_rows(Md, k, norm).cpu().numpy()
            want = O.select_rows(M, k, "l1" if norm == mu.NORM_L1 else "l2")
            assert np.array_equal(idx, want), (n, m, k)


def test_normuon_scale_fp32():
    g = inputs.rng(56, 0)
    Om = g.standard_normal((300, 130)).astype(np.float32)
    v0 = (g.random(300) * 0.01).astype(np.float32)
    v = dev(v0)
    scale = mu.normuon_scale(dev(Om), v, beta2=0.9, eps=1e-8)
    v_want, s_want = O.normuon(Om.astype(np.float64), v0.astype(np.float64), 0.9, 1e-8)
    assert rel(host(v), v_want) < 1e-5
    assert rel(host(scale), s_want) < 1e-5
    # with a row map: only mapped entries of v change
    v2 = dev(np.zeros(500, np.float32))
    rows = dev(np.arange(0, 600, 2)[:300].astype(np.int32), torch.int32)
    mu.normuon_scale(dev(Om), v2, beta2=0.9, eps=1e-8, rows=rows)
    hv = host(v2)
    assert np.all(hv[1::2] == 0)
    v_want2, _ = O.normuon(Om.astype(np.float64), np.zeros(300), 0.9, 1e-8)
    assert rel(hv[0::2][:250], v_want2[:250]) < 1e-5


# ---------------------------------------------------------------------------
# muon_step
# ---------------------------------------------------------------------------


def make_state(shapes, seed, m_std=0.0):
    out = []
    for i, (r, c) in enumerate(shapes):
        W = inputs.gaussian((r, c), 0.02, seed + i, 0)
        G = inputs.gaussian((r, c), 1e-3, seed + i, 1)
        M = inputs.gaussian((r, c), m_std, seed + i, 2) if m_std else np.zeros((r, c), np.float32)
        v = np.zeros(r, np.float32)
        out.append((W, M, G, v))
    return out


def run_step(state, p):
    dmats = [(dev(W), dev(M), dev(G), dev(v)) for (W, M, G, v) in state]
    s = mu.muon_step(dmats, p)
    st = s.device_status()
    return [(host(a), host(b), host(d)) for (a, b, _, d) in dmats], st


def check_step(state, got, sp: O.StepParams, tol, label=""):
    for (W, M, G, v), (Wg, Mg, vg) in zip(state, got):
        want = O.muon_step(W, M, G, v, sp)
        assert np.array_equal(Mg.astype(np.float32), want["M"]), f"{label} momentum state differs"
        dW = Wg - W.astype(np.float64)
        dW_want = want["W"].astype(np.float64) - W.astype(np.float64)
        assert rel(dW, dW_want) < tol, (label, W.shape, rel(dW, dW_want))
        if sp.normuon:
            assert rel(vg, want["v"]) < tol
        if sp.k is not None:
            changed = np.where(np.any(Wg != W, axis=1))[0]
            assert set(changed) <= set(want["idx"].tolist())


def test_step_fp32_single():
    state = make_state([(256, 1024)], 1000, m_std=1e-3)
    p = mu.step_params(ns=mu.ns_params(compute=mu.F32))
    got, st = run_step(state, p)
    assert st == mu.OK
    check_step(state, got, O.StepParams(), TOL32)


MIXED = [(128, 128), (128, 128), (128, 384), (384, 128), (100, 260), (260, 100), (64, 64)]
MIXED_RECT = [(128, 384), (128, 384), (384, 128), (100, 260), (260, 100), (64, 640)]


@pytest.mark.parametrize("gram,compute", [(False, mu.BF16), (True, mu.F16), (True, mu.BF16), (False, mu.F32)])
def test_step_batched(gram, compute):
    # bf16 Gram only on rectangular matrices (square ones: see test_gram_bf16_square_matches_emulation)
    shapes = MIXED_RECT if (gram and compute == mu.BF16) else MIXED
    state = make_state(shapes, 2000, m_std=2e-3)
    p = mu.step_params(ns=mu.ns_params(gram=gram, compute=compute))
    got, st = run_step(state, p)
    assert st == mu.OK
    check_step(state, got, O.StepParams(gram=gram), TOL32 if compute == mu.F32 else TOL16)


@pytest.mark.parametrize("compute", [mu.BF16, mu.F32])
def test_step_normuon(compute):
    state = make_state(MIXED[:5], 3000, m_std=2e-3)
    for i, s in enumerate(state):
        s[3][:] = (inputs.rng(7 + i, 0).random(s[3].shape[0]) * 1e-4).astype(np.float32)
    p = mu.step_params(ns=mu.ns_params(compute=compute), normuon=True, beta2=0.95, normuon_eps=1e-8)
    got, st = run_step(state, p)
    assert st == mu.OK
    check_step(state, got, O.StepParams(normuon=True), TOL32 if compute == mu.F32 else TOL16)


@pytest.mark.parametrize("norm", ["l1", "l2"])
@pytest.mark.parametrize("frac", [(1, 4), (1, 2), (1, 1)])
def test_step_dion3(norm, frac):
    shapes = [(256, 512), (512, 256), (200, 96)]
    state = make_state(shapes, 4000, m_std=3e-3)
    p = mu.step_params(ns=mu.ns_params(gram=True, compute=mu.F16), dion3=True, frac=frac, normuon=True,
                       select_norm=mu.NORM_L1 if norm == "l1" else mu.NORM_L2)
    got, st = run_step(state, p)
    assert st == mu.OK
    for (W, M, G, v), g in zip(state, got):
        k = O.rows_for_fraction(W.shape[0], *frac)
        check_step([(W, M, G, v)], [g], O.StepParams(gram=True, normuon=True, k=k, select_norm=norm), TOL16,
                   f"dion3 {norm} {frac}")


def test_step_zero_and_empty():
    state = make_state([(64, 128)], 5000)
    state[0][2][:] = 0  # zero gradient, zero momentum
    got, st = run_step(state, mu.step_params())
    assert st == mu.OK
    assert np.array_equal(got[0][0], state[0][0].astype(np.float64))


def test_step_nonfinite_reported():
    state = make_state([(64, 128)], 5100)
    state[0][2][3, 5] = np.nan
    _, st = run_step(state, mu.step_params())
    assert st == mu.ERR_NONFINITE


def test_step_deterministic_and_resumable():
    """Two steps in one go equal one step, a save/reload of the state, and a
    second step (bit for bit): fixed reduction orders, no float atomics."""
    shapes = [(128, 384), (384, 128)]
    state = make_state(shapes, 6000, m_std=1e-3)
    G2 = [inputs.gaussian(s, 1e-3, 6100 + i, 1) for i, s in enumerate(shapes)]
    p = mu.step_params(normuon=True)
    d1 = [(dev(W), dev(M), dev(G), dev(v)) for (W, M, G, v) in state]
    s1 = mu.muon_step(d1, p)
    for i, g in enumerate(G2):
        d1[i][2].copy_(dev(g))
    s1()
    ref = [tuple(host(t) for t in (a, b, d)) for (a, b, _, d) in d1]
    # run 1 step, checkpoint to host, restore into fresh buffers, run step 2
    d2 = [(dev(W), dev(M), dev(G), dev(v)) for (W, M, G, v) in state]
    mu.muon_step(d2, p)
    saved = [tuple(t.cpu().clone() for t in m) for m in d2]
    d3 = [tuple(t.cuda() for t in m) for m in saved]
    for i, g in enumerate(G2):
        d3[i][2].copy_(dev(g))
    mu.muon_step(d3, p)
    for r, (a, b, _, d) in zip(ref, d3):
        assert np.array_equal(r[0], host(a)) and np.array_equal(r[1], host(b)) and np.array_equal(r[2], host(d))


def test_step_cuda_graph_matches_eager():
    """A step captured in a CUDA graph and replayed gives the same bits as the
    same step run eagerly (the page captures its step in a graph to remove
    launch overhead at small scale)."""
    shapes = [(128, 384), (384, 128), (64, 64)]
    state = make_state(shapes, 7000, m_std=1e-3)
    p = mu.step_params(normuon=True)
    d1 = [(dev(W), dev(M), dev(G), dev(v)) for (W, M, G, v) in state]
    s1 = mu.Step(d1, p)
    s1()
    s1()
    d2 = [(dev(W), dev(M), dev(G), dev(v)) for (W, M, G, v) in state]
    s2 = mu.Step(d2, p)
    s2()  # first step eagerly (also sets kernel attributes before capture)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        s2(torch.cuda.current_stream())
    graph.replay()
    torch.cuda.synchronize()
    assert s2.device_status() == mu.OK
    for a, b in zip(d1, d2):
        for x, y in zip(a, b):
            assert torch.equal(x, y)


@pytest.mark.parametrize("pair", [True, False])
def test_step_many_tiles_mixed_layouts(pair):
    """More tiles than persistent CTAs (or CTA pairs), with wide, square and
    tall groups (K-major and MN-major operands) sharing every launch: each
    CTA walks many tiles of different layouts through one shared-memory ring,
    the case where producer/consumer phase tracking must hold up."""
    shapes = [(512, 512)] * 40 + [(512, 1536)] * 8 + [(1536, 512)] * 8
    state = make_state(shapes, 8000, m_std=1e-3)
    mu.set_gemm_cta_pair(pair)
    try:
        got, st = run_step(state, mu.step_params())
    finally:
        mu.set_gemm_cta_pair(True)
    assert st == mu.OK, mu.status_str(st)
    idx = [0, 39, 40, 47, 48, 55]
    check_step([state[i] for i in idx], [got[i] for i in idx], O.StepParams(), TOL16)


# ---------------------------------------------------------------------------
# split K: X X^T launches with fewer tiles than CTAs (pairs) and a long K
# ---------------------------------------------------------------------------


def _launches(fn):
    """fn's result and the kernels it queued, in the per-product launch mode
    (the split-K launches these tests count belong to that mode; the fused
    chain never splits K)."""
    mu.set_gemm_chain(False)
    try:
        n0 = mu.kernel_launch_count()
        out = fn()
        torch.cuda.synchronize()
        return out, mu.kernel_launch_count() - n0
    finally:
        mu.set_gemm_chain(os.environ.get("MUON_GEMM_CHAIN") == "1")


@pytest.mark.parametrize("pair", [True, False])
@pytest.mark.parametrize("shape", [(300, 9000), (9000, 300)])
def test_split_k_standard_bf16(pair, shape):
    """n = 300 rows against K = 9000 (ragged in both): X X^T has a handful of
    tiles, so each is split along K into fp32 partials that a second launch
    sums in a fixed order. One reduction launch per X X^T (five)."""
    X = gauss(shape, 9100 + shape[0])
    short = gauss((shape[0], 1000) if shape[0] < shape[1] else (1000, shape[1]), 9200)
    mu.set_gemm_cta_pair(pair)
    try:
        (Og, ws), n_split = _launches(lambda: mu.ns_polar(dev(X), mu.ns_params(compute=mu.BF16),
                                                          out_dtype=torch.float32))
        (_, ws2), n_plain = _launches(lambda: mu.ns_polar(dev(short), mu.ns_params(compute=mu.BF16),
                                                          out_dtype=torch.float32))
        # the same input again: bit-identical (fixed-order reduction)
        Og2, _ = mu.ns_polar(dev(X), mu.ns_params(compute=mu.BF16), out_dtype=torch.float32)
    finally:
        mu.set_gemm_cta_pair(True)
    assert status_of(ws) == mu.OK and status_of(ws2) == mu.OK
    assert n_split - n_plain == 5
    assert torch.equal(Og, Og2)
    assert rel(host(Og), O.newton_schulz(X.astype(np.float64), COEFFS5)) < TOL16


@pytest.mark.parametrize("restart", [3, 0])
def test_split_k_gram_f16(restart):
    """Gram NS in fp16 on 520 x 4200: X X^T (at the start and at the restart)
    is split into parts of 32, 32 and 2 k-blocks (a ragged last part)."""
    X = gauss((520, 4200), 9300)
    p = mu.ns_params(gram=True, restart_at=restart, compute=mu.F16)
    (Og, ws), n_split = _launches(lambda: mu.gram_ns_polar(dev(X), p, out_dtype=torch.float32))
    (_, ws2), n_plain = _launches(lambda: mu.gram_ns_polar(dev(gauss((520, 1000), 9301)), p,
                                                           out_dtype=torch.float32))
    assert status_of(ws) == mu.OK and status_of(ws2) == mu.OK
    assert n_split - n_plain == (2 if restart else 1)
    want = O.gram_newton_schulz(X.astype(np.float64), COEFFS5, restart_at=restart)
    assert rel(host(Og), want) < TOL16


def test_split_k_dion3_batched_step():
    """Dion3 (f = 1/4) + NorMuon + Gram fp16 on two 1024 x 8192 matrices: the
    selected 256 x 8192 pair shares each X X^T launch, split four ways."""
    state = make_state([(1024, 8192), (1024, 8192)], 9400, m_std=1e-3)
    p = mu.step_params(ns=mu.ns_params(gram=True, restart_at=3, compute=mu.F16), normuon=True, dion3=True,
                       frac=(1, 4), select_norm=mu.NORM_L2)
    got, st = run_step(state, p)
    assert st == mu.OK
    k = O.rows_for_fraction(1024, 1, 4)
    check_step(state, got, O.StepParams(gram=True, restart_at=3, normuon=True, k=k, select_norm="l2"), TOL16)


@pytest.mark.parametrize("pair", [True, False])
@pytest.mark.parametrize("gram", [False, True])
def test_narrow_tiles_ragged(pair, gram):
    """Launches too small to fill the GPU run on 128-column tiles (256x128
    per CTA pair, 128x128 per CTA): ragged symmetric n (300, 200) and
    rectangular groups, standard bf16 and Gram fp16, both kernel forms."""
    shapes = [(300, 700), (300, 700), (700, 300), (200, 200), (130, 390)]
    state = make_state(shapes, 9500 + 10 * pair + gram, m_std=1e-3)
    p = mu.step_params(ns=mu.ns_params(gram=gram, restart_at=3, compute=mu.F16 if gram else mu.BF16))
    mu.set_gemm_cta_pair(pair)
    try:
        got, st = run_step(state, p)
    finally:
        mu.set_gemm_cta_pair(True)
    assert st == mu.OK, mu.status_str(st)
    check_step(state, got, O.StepParams(gram=gram, restart_at=3), TOL16)


def _orth(Om):
    Om = np.asarray(Om, np.float64)
    return float(np.linalg.norm(Om @ Om.T - np.eye(Om.shape[0])))


@pytest.mark.parametrize("gram,compute", [(False, mu.BF16), (False, mu.F16), (True, mu.F16)])
def test_minimax_schedule(gram, compute):
    """A tuned per-step schedule (minimax quintics, T = 8 from a lower end of
    1e-2) through the per-step coefficient table, on a 256 x 1024 matrix with
    singular values log-uniform in [1e-2, 1]: parity with the oracle on the
    same table (bounded by the oracle's own half-precision emulation where
    the arithmetic itself misses 2e-2), and an orthogonality error far below
    the fixed coefficients' at T = 5.

    Steeper tables (lower end 1e-3, first-step slope 8.5) make the fp16 Gram
    chain fragile: its products are computed on one triangle and mirrored,
    which keeps the rounding residue of fp16 factors that no longer commute
    exactly, and equally valid roundings then straddle the 2e-2 bound
    (tests/test_gram_fp16_replica.py: a CPU replica of the library's storage
    points and one-triangle products gives 3.0% for the library's choice,
    where the GPU gave 2.9%, and 1.3% for products computed in full; every
    variant stays below 1% with the table from 1e-2)."""
    from newton_schulz_10_b200 import schedules
    X, _ = inputs.spectrum_matrix(256, 1024, -2.0, seed=9600)
    X32 = X.astype(np.float32)
    Xb = bf16_values(X32)
    coeffs, _ = schedules.minimax_schedule(8, 1e-2)
    p = mu.ns_params(T=8, coeffs=coeffs, gram=gram, restart_at=3, compute=compute)
    fn = mu.gram_ns_polar if gram else mu.ns_polar
    Og, ws = fn(dev(X32, torch.bfloat16), p, out_dtype=torch.float32)
    assert status_of(ws) == mu.OK
    got = host(Og)
    exact = O.newton_schulz(Xb, coeffs)
    store = _emulate_bf16 if compute == mu.BF16 else _emulate_f16(256)
    emul = (O.gram_newton_schulz(Xb, coeffs, restart_at=3, store=store) if gram
            else O.newton_schulz(Xb, coeffs, store=store))
    e_alg = rel(emul, exact)
    assert rel(got, exact) < (TOL16 if e_alg < TOL16 else 1.25 * e_alg), (rel(got, exact), e_alg)
    assert _orth(got) < 0.1 * _orth(O.newton_schulz(Xb, COEFFS5))


@pytest.mark.parametrize("gram", [False, True])
def test_nonfinite_output_is_reported(gram):
    """p(x) = 300 x for three steps multiplies every singular value by
    2.7e7, past the fp16 range: the polar output and the step's update must
    report MUON_ERR_NONFINITE instead of passing inf or NaN on as MUON_OK.
    The same table in bf16 stays finite and reports MUON_OK."""
    X = gauss((256, 1024), 9700)
    table = [(300.0, 0.0, 0.0)] * 3
    fn = mu.gram_ns_polar if gram else mu.ns_polar
    _, ws = fn(dev(X, torch.bfloat16), mu.ns_params(T=3, coeffs=table, gram=gram, compute=mu.F16),
               out_dtype=torch.float32)
    assert status_of(ws) == mu.ERR_NONFINITE
    _, ws = fn(dev(X, torch.bfloat16), mu.ns_params(T=3, coeffs=table, gram=gram, compute=mu.BF16),
               out_dtype=torch.float32)
    assert status_of(ws) == mu.OK
    state = make_state([(256, 1024)], 9710, m_std=1e-3)
    _, st = run_step(state, mu.step_params(ns=mu.ns_params(T=3, coeffs=table, gram=gram, compute=mu.F16)))
    assert st == mu.ERR_NONFINITE


def test_step_events_record_phases():
    """muon_step_events records the caller's five events at the phase
    boundaries of an ordinary step (fresh torch events included: they get a
    CUDA handle before the call), without changing the step: the state equals
    a muon_step run's bit for bit, and the phase times are positive and add up
    to the span of the first and last event."""
    state = make_state(MIXED, 7800, m_std=1e-3)
    p = mu.step_params(normuon=True)
    d1 = [(dev(W), dev(M), dev(G), dev(v)) for (W, M, G, v) in state]
    d2 = [tuple(t.clone() for t in m) for m in d1]
    mu.muon_step(d1, p)
    s2 = mu.Step(d2, p)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    s2.timed(ev)
    torch.cuda.synchronize()
    assert s2.device_status() == mu.OK
    for a, b in zip(d1, d2):
        for x, y in zip(a, b):
            assert torch.equal(x, y)
    phases = [ev[i].elapsed_time(ev[i + 1]) for i in range(4)]
    assert phases[1] > 0 and all(t >= 0 for t in phases)
    assert abs(sum(phases) - ev[0].elapsed_time(ev[4])) < 1e-3 * max(1.0, sum(phases))
