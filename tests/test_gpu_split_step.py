"""muon_momentum + muon_orthogonalize + muon_apply_update against muon_step.

The three entry points split the step at the two places where a multi-GPU
caller moves data between GPUs ("4. Megabatched Communication" of the Dion3
page: momentum shards go to the GPU that owns the matrix, orthogonalised rows
come back). On one GPU the three calls in sequence must give the same W, M
and v as muon_step, bit for bit, for every variant of the step.
"""

import numpy as np
import pytest
import torch

from newton_schulz_10_b200 import muon as mu

from gpu_util import dev
from test_gpu_parity import MIXED, make_state

pytestmark = pytest.mark.gpu

VARIANTS = {
    "muon_bf16": dict(ns=dict(compute=mu.BF16)),
    "muon_bf16_normuon": dict(ns=dict(compute=mu.BF16), normuon=True),
    "gram_f16": dict(ns=dict(gram=True, compute=mu.F16)),
    "dion3_gram_f16_normuon": dict(ns=dict(gram=True, compute=mu.F16), dion3=True, frac=(1, 4), normuon=True),
    "dion3_bf16_l2": dict(ns=dict(compute=mu.BF16), dion3=True, frac=(1, 3), select_norm=mu.NORM_L2),
    "muon_f32": dict(ns=dict(compute=mu.F32)),
}


def _params(v):
    kw = {k: x for k, x in v.items() if k != "ns"}
    return mu.step_params(ns=mu.ns_params(**v["ns"]), **kw)


@pytest.mark.parametrize("name", list(VARIANTS))
def test_three_calls_equal_muon_step(cuda, name):
    shapes = MIXED if VARIANTS[name]["ns"]["compute"] != mu.F32 else MIXED[:4]
    state = make_state(shapes, 8100, m_std=2e-3)
    for i, s in enumerate(state):
        s[3][:] = np.linspace(1e-5, 1e-4, s[3].shape[0], dtype=np.float32)
    p = _params(VARIANTS[name])
    a = [tuple(dev(x) for x in s) for s in state]
    b = [tuple(t.clone() for t in m) for m in a]
    for _ in range(2):  # two steps: the second starts from nonzero momentum and v
        step = mu.muon_step(a, p)
        assert step.device_status() == mu.OK
        mu.momentum(b, p)
        O = [torch.empty(W.shape, dtype=mu.operand_dtype(p), device="cuda") for (W, _, _, _) in b]
        scale = [torch.empty(W.shape[0], dtype=torch.float32, device="cuda") for (W, _, _, _) in b]
        sel = [torch.empty(W.shape[0], dtype=torch.int32, device="cuda") for (W, _, _, _) in b] if p.dion3 else None
        ws = mu.orthogonalize([(None, M, None, v) for (_, M, _, v) in b], p, O, scale, sel)
        mu.apply_update(b, p, O, scale, sel)
        torch.cuda.synchronize()
        assert int(ws[:4].view(torch.int32).item()) == mu.OK
        for x, y in zip(a, b):
            for t1, t2 in zip(x, y):
                assert torch.equal(t1, t2), name
        if p.dion3:
            for (W, _, _, _), f in zip(b, sel):
                k = mu.rows_for_fraction(W.shape[0], p.frac_num, p.frac_den)
                assert int(f.sum().item()) == k
