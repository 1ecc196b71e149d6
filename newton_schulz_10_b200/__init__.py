"""Muon optimizer step on one NVIDIA B200 (sm_100a).

The computation lives in ``libmuon.so`` (hand-written CUDA: tcgen05/TMEM
tensor-core GEMMs fed by TMA, and vectorised memory-bound kernels) behind the
C ABI declared in ``include/muon.h``. ``newton_schulz_10_b200.muon`` is the
thin ctypes binding; ``newton_schulz_10_b200.inputs`` generates the seeded
synthetic workloads.
"""

__all__ = ["muon", "inputs", "build"]
