import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload, minutes of CPU time")
    # MUON_GEMM_CTA_PAIR=0 runs the suite on the single-CTA GEMM kernel;
    # MUON_GEMM_CHAIN=1 runs every Newton-Schulz chain as a fused chain
    if os.environ.get("MUON_GEMM_CTA_PAIR") == "0":
        from newton_schulz_10_b200 import muon
        muon.set_gemm_cta_pair(False)
    if os.environ.get("MUON_GEMM_CHAIN") == "1":
        from newton_schulz_10_b200 import muon
        muon.set_gemm_chain(True)


@pytest.fixture(scope="session")
def cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
