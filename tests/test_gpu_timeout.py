"""Failure detection without faulting the GPU: every device-side wait in the
tensor-core GEMM is bounded. With the bound set to 1 ns the first wait that is
not already satisfied gives up: the kernel records MUON_ERR_TIMEOUT, stops,
drains its in-flight copies and MMAs and frees its tensor memory. The
context stays usable: with the default bound restored the same call succeeds."""

import os

import numpy as np
import pytest
import torch

import oracle as O
from newton_schulz_10_b200 import inputs
from newton_schulz_10_b200 import muon as mu

from gpu_util import COEFFS5, host, rel

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cta_pair", [True, False], ids=["cta_pair", "single_cta"])
def test_bounded_wait_reports_timeout_and_recovers(cuda, cta_pair):
    # K = 8192 in the first product: its first tile's mainloop alone outlasts
    # the 1 ns bound, so the epilogue's first wait cannot be satisfied in time.
    # In the CTA-pair form the early stop reaches both CTAs of a pair and the
    # leader drains every operand copy either CTA issued before they exit.
    X = inputs.gaussian((1024, 8192), 1.0, 77, 0)
    Xd = torch.from_numpy(X).cuda()
    default_pair = os.environ.get("MUON_GEMM_CTA_PAIR") != "0"
    try:
        mu.set_gemm_cta_pair(cta_pair)
        mu.set_wait_timeout_ns(1)
        _, ws = mu.ns_polar(Xd, mu.ns_params())
        torch.cuda.synchronize()
        st = int(ws[:4].view(torch.int32).item())
        assert st == mu.ERR_TIMEOUT, mu.status_str(st)
    finally:
        mu.set_wait_timeout_ns(0)  # back to the default bound
    try:
        Og, ws = mu.ns_polar(Xd, mu.ns_params(), out_dtype=torch.float32)
        torch.cuda.synchronize()
    finally:
        mu.set_gemm_cta_pair(default_pair)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == mu.OK
    assert rel(host(Og), O.newton_schulz(X.astype(np.float64), COEFFS5)) < 2e-2
