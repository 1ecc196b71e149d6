"""bench.py's algorithmic FLOP counts (the numerator of every reported
TFLOP/s and roofline fraction) equal the oracle's FLOP formulas, which the
oracle pins check against the page's printed numbers."""

import importlib.util
import os
import sys

import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


@pytest.mark.parametrize("n,m,T", [(768, 768, 5), (768, 3072, 5), (4096, 16384, 5), (2048, 28672, 5),
                                   (4096, 16384, 10), (256, 1024, 5)])
def test_ns_flops_match_the_oracle_formulas(bench, n, m, T):
    assert bench.ns_flops(n, m, T, False) == O.flops_standard_symmetric(n, m, T)
    assert bench.ns_flops(n, m, T, True, restart_at=0) == O.flops_gram(n, m, T)
    assert bench.ns_flops(n, m, T, True, restart_at=3) == O.flops_gram(n, m, T) + O.flops_restart_extra(n, m)
