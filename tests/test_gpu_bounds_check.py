"""The bounds-checked debug build (-DMUON_BOUNDS_CHECK) on the parity suite's
small and ragged cases.

That build adds device-side index checks to the global accesses of the row
kernels, the split-K reduction and the GEMM epilogue's C loads; a failed
check writes MUON_ERR_INVALID_ARG to the status word (and skips the access)
instead of trapping. Every parity test asserts status MUON_OK, so running
them against libmuon_check.so shows that no index of these kernels leaves its
matrix on shapes with ragged tails, tall and wide orientations, split K and
narrow tiles.
"""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = ("ns_polar or gram_ns_polar or select_rows_exact or normuon_scale or step_batched or step_normuon "
         "or step_dion3 or split_k or narrow_tiles or many_tiles or zero_and_empty or loaded_library")


def test_loaded_library_is_the_requested_variant():
    from newton_schulz_10_b200 import muon as mu
    want = "libmuon_check.so" if os.environ.get("MUON_BOUNDS_CHECK") == "1" else "libmuon.so"
    assert os.path.basename(mu.lib()._name) == want


@pytest.mark.gpu
def test_parity_cases_under_bounds_checked_build(cuda):
    from newton_schulz_10_b200 import build
    build.build(debug=True)
    env = dict(os.environ, MUON_BOUNDS_CHECK="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu or not gpu",
           os.path.join(ROOT, "tests", "test_gpu_parity.py"), os.path.join(ROOT, "tests", "test_gpu_bounds_check.py"),
           "-k", CASES]
    r = subprocess.run(cmd, env=env, cwd=ROOT, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
