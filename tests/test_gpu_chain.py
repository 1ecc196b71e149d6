"""The fused Newton-Schulz chain (muon_set_gemm_chain(1)) against the oracle
and against the per-product launches.

In the fused chain every product of a chain (all shape groups together) runs
in one persistent launch, or a few when the products need more kernel
parameters than one launch holds; a tile of a product waits, matrix by
matrix, on completion counters of the previous product. These tests run the
small and ragged cases of the parity suite with it: standard and Gram
chains (restart on and off), wide and tall matrices, several shape groups in
one chain, Dion3 with NorMuon, long chains that need several launches,
CUDA-graph replay, and a bounded wait that runs out.
"""

import os

import numpy as np
import pytest
import torch

import oracle as O
from newton_schulz_10_b200 import inputs
from newton_schulz_10_b200 import muon as mu

from gpu_util import COEFFS5, dev, gauss, host, rel
from test_gpu_parity import MIXED, MIXED_RECT, TOL16, check_step, make_state, run_step, status_of

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def chain_mode(cuda):
    mu.set_gemm_chain(True)
    yield
    torch.cuda.synchronize()
    mu.set_gemm_chain(os.environ.get("MUON_GEMM_CHAIN") == "1")


@pytest.mark.parametrize("shape", [(256, 1024), (300, 100), (200, 520), (520, 200), (96, 96), (2048, 8192)])
def test_chain_ns_polar_bf16(shape):
    X = gauss(shape, 7100 + shape[0])
    Og, ws = mu.ns_polar(dev(X), mu.ns_params(compute=mu.BF16), out_dtype=torch.float32)
    assert status_of(ws) == mu.OK
    assert rel(host(Og), O.newton_schulz(X.astype(np.float64), COEFFS5)) < TOL16
    mu.set_gemm_chain(False)  # the per-product launches, for comparison
    Ol, ws = mu.ns_polar(dev(X), mu.ns_params(compute=mu.BF16), out_dtype=torch.float32)
    assert status_of(ws) == mu.OK
    assert rel(host(Og), host(Ol)) < 1e-2


@pytest.mark.parametrize("restart", [3, 0])
@pytest.mark.parametrize("shape", [(256, 1024), (200, 520), (520, 200), (2048, 8192)])
def test_chain_gram_ns_polar_f16(restart, shape):
    X = gauss(shape, 7200 + shape[0])
    p = mu.ns_params(gram=True, restart_at=restart, compute=mu.F16)
    Og, ws = mu.gram_ns_polar(dev(X), p, out_dtype=torch.float32)
    assert status_of(ws) == mu.OK
    want = O.gram_newton_schulz(X.astype(np.float64), COEFFS5, restart_at=restart)
    assert rel(host(Og), want) < TOL16


def test_chain_long_schedule_spans_launches():
    """T = 16 standard steps with four shape groups: 48 products x 4 groups
    exceed one launch's jobs, so the chain continues over several launches."""
    from newton_schulz_10_b200 import schedules
    coeffs, _ = schedules.minimax_schedule(16, 1e-2)
    shapes = [(128, 384), (384, 128), (100, 260), (64, 640)]
    state = make_state(shapes, 7300, m_std=2e-3)
    p = mu.step_params(ns=mu.ns_params(T=16, coeffs=coeffs, gram=False, compute=mu.BF16))
    got, st = run_step(state, p)
    assert st == mu.OK
    check_step(state, got, O.StepParams(coeffs=tuple(map(tuple, coeffs))), TOL16, "T=16 chain")


@pytest.mark.parametrize("gram,compute", [(False, mu.BF16), (True, mu.F16), (True, mu.BF16)])
def test_chain_step_batched(gram, compute):
    shapes = MIXED_RECT if (gram and compute == mu.BF16) else MIXED
    state = make_state(shapes, 7400, m_std=2e-3)
    p = mu.step_params(ns=mu.ns_params(gram=gram, compute=compute))
    got, st = run_step(state, p)
    assert st == mu.OK
    check_step(state, got, O.StepParams(gram=gram), TOL16, "chain batched")


def test_chain_step_dion3_normuon():
    shapes = [(256, 512), (512, 256), (200, 96)]
    state = make_state(shapes, 7500, m_std=3e-3)
    p = mu.step_params(ns=mu.ns_params(gram=True, compute=mu.F16), dion3=True, frac=(1, 4), normuon=True)
    got, st = run_step(state, p)
    assert st == mu.OK
    for (W, M, G, v), g in zip(state, got):
        k = O.rows_for_fraction(W.shape[0], 1, 4)
        check_step([(W, M, G, v)], [g], O.StepParams(gram=True, normuon=True, k=k), TOL16, "chain dion3")


def test_chain_cuda_graph_matches_eager():
    state = make_state(MIXED, 7600, m_std=2e-3)
    dm = [(dev(W), dev(M), dev(G), dev(v)) for (W, M, G, v) in state]
    de = [tuple(t.clone() for t in m) for m in dm]
    p = mu.step_params(ns=mu.ns_params(compute=mu.BF16))
    step_g = mu.Step(dm, p)
    step_e = mu.Step(de, p)
    step_g()  # first step eagerly on both (also sets kernel attributes before capture)
    step_e()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step_g(torch.cuda.current_stream())
    for _ in range(2):
        graph.replay()
        step_e()
    torch.cuda.synchronize()
    assert step_g.device_status() == mu.OK and step_e.device_status() == mu.OK
    for a, b in zip(dm, de):
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_chain_bounded_wait_reports_timeout_and_recovers():
    X = inputs.gaussian((1024, 8192), 1.0, 7700, 0)
    Xd = torch.from_numpy(X).cuda()
    try:
        mu.set_wait_timeout_ns(1)
        _, ws = mu.ns_polar(Xd, mu.ns_params())
        assert status_of(ws) == mu.ERR_TIMEOUT
    finally:
        mu.set_wait_timeout_ns(0)
    Og, ws = mu.ns_polar(Xd, mu.ns_params(), out_dtype=torch.float32)
    assert status_of(ws) == mu.OK
    assert rel(host(Og), O.newton_schulz(X.astype(np.float64), COEFFS5)) < TOL16
