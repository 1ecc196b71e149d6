"""Parity at the full workload sizes, in the launch configuration bench.py
times (all matrices of a layer set in one batched step).

- GPT-124M layer set: every one of the 72 matrices against the oracle.
- 8192 x 28672 Dion3 (f = 1/4, l1 rows) + NorMuon, Gram NS in fp16: the whole
  momentum state bit for bit (which fixes the selection), the weight change
  and NorMuon's second moments.
- 4096 x 16384 spectrum matrix (singular values log-uniform in [1e-4, 1]):
  standard NS in bf16 and fp16, Gram NS in fp16, against the exact fp64
  result; bounded by the oracle's own half-precision emulation at this size
  (tests/golden/spectrum_4096x16384_emulated.json) and exact to 2e-2 on the
  well-conditioned directions.
- Llama-7B layer set, NorMuon off and on: the whole 192-matrix step on the
  GPU, layer 0 (six matrices, drawn by the NumPy recipe) checked against the
  oracle; the other layers are drawn on the device.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle as O
from newton_schulz_10_b200 import inputs
from newton_schulz_10_b200 import muon as mu

from gpu_util import COEFFS5, bf16_values, host, rel

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

GOLD = os.path.join(os.path.dirname(__file__), "golden")
TOL16 = 2e-2


@pytest.fixture(autouse=True)
def _gpu(cuda):
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _check_matrix(W, M, G, v, got, sp, label):
    want = O.muon_step(W, M, G, v, sp)
    Wg, Mg, vg = got
    assert np.array_equal(Mg, want["M"]), f"{label}: momentum state differs"
    dW = Wg.astype(np.float64) - W
    dW_want = want["W"].astype(np.float64) - W
    e = rel(dW, dW_want)
    assert e < TOL16, (label, e)
    if sp.normuon:
        # v_i = beta2 v_i + (1 - beta2) sum_j O_ij^2 / m is quadratic in the
        # Newton-Schulz output: a relative error eps in O's rows is about
        # 2 eps in v, so the 2e-2 bound of half-precision NS outputs is 4e-2
        # here
        assert rel(vg, want["v"]) < 2 * TOL16, (label, rel(vg, want["v"]))
    return e


def test_gpt124m_full_step():
    specs = inputs.gpt124m_layer_set()
    host_state, dmats = [], []
    for s in specs:
        W = inputs.gaussian((s.rows, s.cols), 0.02, s.seed, inputs.W_STREAM)
        G = inputs.gaussian((s.rows, s.cols), 1e-3, s.seed, inputs.G_STREAM)
        M = np.zeros_like(W)
        v = np.zeros(s.rows, np.float32)
        host_state.append((W, M, G, v))
        dmats.append(tuple(torch.from_numpy(a).cuda() for a in (W, M, G, v)))
    step = mu.muon_step(dmats, mu.step_params())
    assert step.device_status() == mu.OK
    worst = 0.0
    for s, (W, M, G, v), d in zip(specs, host_state, dmats):
        got = (d[0].cpu().numpy(), d[1].cpu().numpy(), d[3].cpu().numpy())
        worst = max(worst, _check_matrix(W, M, G, v, got, O.StepParams(), s.name))
    print(f"gpt124m: worst relative dW error {worst:.3e}")


def test_dion3_8192x28672():
    shape = (8192, 28672)
    W = inputs.gaussian(shape, 0.02, 4000, inputs.W_STREAM)
    G = inputs.student_t3(shape, 1e-3, 4000, inputs.G_STREAM)
    M = np.zeros(shape, np.float32)
    v = np.zeros(shape[0], np.float32)
    d = [torch.from_numpy(a).cuda() for a in (W, M, G, v)]
    p = mu.step_params(ns=mu.ns_params(gram=True, restart_at=3, compute=mu.F16), normuon=True, dion3=True,
                       frac=(1, 4), select_norm=mu.NORM_L1)
    step = mu.muon_step([tuple(d)], p)
    assert step.device_status() == mu.OK
    got = (d[0].cpu().numpy(), d[1].cpu().numpy(), d[3].cpu().numpy())
    del d
    k = O.rows_for_fraction(shape[0], 1, 4)
    sp = O.StepParams(gram=True, restart_at=3, normuon=True, k=k, select_norm="l1")
    e = _check_matrix(W, M, G, v, got, sp, "dion3")
    changed = np.where(np.any(got[0] != W, axis=1))[0]
    assert len(changed) == k
    print(f"dion3 8192x28672: relative dW error {e:.3e}")


@pytest.mark.parametrize("name,gram,compute", [("standard_bf16", False, mu.BF16), ("standard_f16", False, mu.F16),
                                               ("gram_f16_restart3", True, mu.F16)])
def test_spectrum_4096x16384(name, gram, compute):
    with open(os.path.join(GOLD, "spectrum_4096x16384_emulated.json")) as f:
        bounds = json.load(f)
    n, m, seed = 4096, 16384, bounds["seed"]
    X, sigma = inputs.spectrum_matrix(n, m, -4.0, seed=seed)
    U = inputs.random_orthonormal(n, n, seed, 0)  # the left factor X was built from
    X32 = X.astype(np.float32)
    del X
    Xd = torch.from_numpy(X32).cuda().to(torch.bfloat16)
    Og, ws = mu.ns_polar(Xd, mu.ns_params(gram=gram, restart_at=3, compute=compute), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == mu.OK
    got = host(Og)
    del Og, ws, Xd
    exact = _spectrum_exact(X32)
    err = rel(got, exact)
    well = sigma / np.linalg.norm(sigma) > 1e-2
    err_well = np.linalg.norm((U.T @ (got - exact))[well]) / np.linalg.norm(exact)
    print(f"spectrum {name}: error {err:.4f} (emulated algorithm {bounds[name]:.4f}), "
          f"well-conditioned directions {err_well:.4f}")
    assert err_well < TOL16
    assert err < 1.25 * bounds[name]
    if bounds[name] < TOL16:
        assert err < TOL16


_EXACT = {}


def _spectrum_exact(X32):
    key = X32.shape
    if key not in _EXACT:
        _EXACT[key] = O.newton_schulz(bf16_values(X32), COEFFS5)
    return _EXACT[key]


@pytest.mark.parametrize("normuon,gram", [(False, False), (True, False), (False, True)],
                         ids=["normuon_off", "normuon_on", "gram_f16"])
def test_llama7b_sampled_layer0(normuon, gram):
    """The Llama-7B workload with NorMuon off and then on (Eq. (2) on every
    row, v from zero), and with Gram Newton-Schulz in fp16 (restart 3): the
    whole 192-matrix step on the GPU, layer 0 against the oracle (momentum
    bit for bit, dW and v within 2e-2)."""
    specs = inputs.llama7b_layer_set()
    layer0 = [s for s in specs if s.name.startswith("l0.")]
    host_state = {}
    dmats = []
    for s in specs:
        shape = (s.rows, s.cols)
        if s.name.startswith("l0."):
            W = inputs.gaussian(shape, 0.02, s.seed, inputs.W_STREAM)
            G = inputs.student_t3(shape, 1e-3, s.seed, inputs.G_STREAM)
            host_state[s.name] = (W, np.zeros(shape, np.float32), G, np.zeros(s.rows, np.float32))
            dmats.append(tuple(torch.from_numpy(a).cuda() for a in host_state[s.name]))
        else:
            g = torch.Generator(device="cuda")
            g.manual_seed(s.seed)
            W = torch.randn(shape, device="cuda", generator=g) * 0.02
            G = torch.randn(shape, device="cuda", generator=g) * 1e-3
            dmats.append((W, torch.zeros(shape, device="cuda"), G, torch.zeros(s.rows, device="cuda")))
    ns = mu.ns_params(gram=True, restart_at=3, compute=mu.F16) if gram else mu.ns_params()
    step = mu.muon_step(dmats, mu.step_params(ns=ns, normuon=normuon, beta2=0.95, normuon_eps=1e-8))
    assert step.device_status() == mu.OK
    got = {s.name: (d[0].cpu().numpy(), d[1].cpu().numpy(), d[3].cpu().numpy())
           for s, d in zip(specs, dmats) if s.name.startswith("l0.")}
    del dmats, step
    for s in layer0:
        e = _check_matrix(*host_state[s.name], got[s.name], O.StepParams(normuon=normuon, gram=gram), s.name)
        label = "Gram fp16" if gram else f"NorMuon {'on' if normuon else 'off'}"
        print(f"llama7b {s.name} ({label}): relative dW error {e:.3e}")
