"""select_rows_noalloc: the selection entry point that allocates nothing.

It is for callers that cannot allocate device memory when they select rows
(a pre-carved memory pool, a runtime that forbids cudaMalloc after start-up,
a plain C host). This file is collected last on purpose, so that a run that
stops at the first failure has run every other test before it; it also passes
on its own in a fresh process.
"""

import numpy as np
import pytest

from newton_schulz_10_b200 import inputs
from newton_schulz_10_b200 import muon as mu

FAKE = 1 << 20  # aligned non-NULL address, never dereferenced by host checks


def test_noalloc_rejects_too_many_rows():
    L = mu.lib()
    assert L.select_rows_noalloc(FAKE, 65537, 8, 4, mu.NORM_L1, FAKE, None, None) == mu.ERR_SHAPE
    assert L.select_rows_noalloc(FAKE, 100, 8, 0, mu.NORM_L1, FAKE, None, None) == mu.ERR_SHAPE
    assert L.select_rows_noalloc(FAKE, 100, 8, 101, mu.NORM_L1, FAKE, None, None) == mu.ERR_SHAPE
    assert L.select_rows_noalloc(FAKE + 4, 100, 8, 4, mu.NORM_L1, FAKE, None, None) == mu.ERR_ALIGN


@pytest.mark.gpu
def test_noalloc_matches_select_rows_two_calls(cuda):
    import torch

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # two calls in a row through the C ABI: a large one, then a smaller one
    # that must not see the first call's leftovers in the shared scratch
    for call, (n, m, k, norm) in enumerate([(4096, 384, 1024, mu.NORM_L1), (1000, 96, 250, mu.NORM_L2)]):
        g = inputs.rng(900 + call, 0)
        M = g.standard_normal((n, m)).astype(np.float32)
        M[n // 3] = M[5]  # an exact tie
        Md = torch.from_numpy(M).cuda()
        want = mu.select_rows(Md, k, norm)
        got = mu.select_rows_noalloc(Md, k, norm, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == mu.OK
        assert torch.equal(got, want), call


@pytest.mark.gpu
def test_noalloc_largest_size_bit_exact(cuda):
    """n = 65536, the most rows the fixed scratch holds: its per-row sums and
    keys then fill the array end to end. Two calls in a row (l1, then l2)
    match select_rows bit for bit."""
    import torch

    n, m, k = 65536, 8, 16384
    g = inputs.rng(905, 0)
    M = g.standard_normal((n, m)).astype(np.float32)
    M[n - 1] = M[0]      # an exact tie at the far end of the scratch
    M[n // 2] = -M[7]
    Md = torch.from_numpy(M).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for norm in (mu.NORM_L1, mu.NORM_L2):
        want = mu.select_rows(Md, k, norm)
        got = mu.select_rows_noalloc(Md, k, norm, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == mu.OK
        assert torch.equal(got, want), norm
