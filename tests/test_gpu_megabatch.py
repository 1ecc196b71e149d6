"""The megabatched step on the GPU with the library's arithmetic.

One process, one GPU, an NCCL process group of one rank: the all-to-alls are
local, and the module runs muon_momentum, muon_orthogonalize and
muon_apply_update around them. The result must equal muon_step bit for bit.
(The exchange between several ranks is tested on the CPU with gloo in
test_megabatch.py; this run has a single GPU.)
"""

import datetime
import os
import socket

import pytest
import torch

from newton_schulz_10_b200 import megabatch
from newton_schulz_10_b200 import muon as mu

from gpu_util import dev
from test_gpu_parity import MIXED, make_state

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_group(cuda):
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    yield
    torch.cuda.synchronize()
    dist.destroy_process_group()


@pytest.mark.parametrize("variant", ["muon_bf16", "dion3_normuon_f16"])
def test_megabatched_step_one_rank_equals_muon_step(nccl_group, variant):
    if variant == "muon_bf16":
        p = mu.step_params(ns=mu.ns_params(compute=mu.BF16))
    else:
        p = mu.step_params(ns=mu.ns_params(gram=True, compute=mu.F16), dion3=True, frac=(1, 4), normuon=True)
    state = make_state(MIXED, 8300, m_std=2e-3)
    a = [tuple(dev(x) for x in s) for s in state]
    b = [tuple(t.clone() for t in m) for m in a]
    step = megabatch.MegabatchedStep(b, [tuple(W.shape) for (W, _, _, _) in b], params=p)
    for _ in range(2):
        mu.muon_step(a, p)
        step()
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        for t1, t2 in zip(x, y):
            assert torch.equal(t1, t2)
