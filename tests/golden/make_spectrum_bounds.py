"""Writes spectrum_4096x16384_emulated.json: how far the Newton-Schulz
algorithms land from the exact fp64 result when their stored matrices are
rounded to half precision, on the 4096 x 16384 spectrum workload (singular
values log-uniform in [1e-4, 1], input rounded to bf16).

Uses only the oracle (its rounding hook) and the input generator. The GPU
test compares its own error with these numbers: the kernels may not add more
than a small margin to what the arithmetic itself loses.

  python tests/golden/make_spectrum_bounds.py
"""

import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
from newton_schulz_10_b200 import inputs  # noqa: E402

COEFFS5 = ((3.4445, -4.7750, 2.0315),) * 5


def bf16(x):
    return inputs.bf16_bits_to_f32(inputs.to_bf16_bits(np.asarray(x, np.float32))).astype(np.float64)


def store_bf16(x, role):
    return bf16(x)


def store_f16(n):
    kappa, rho = np.sqrt(n), float(n)

    def store(x, role):
        if role in ("X0", "X"):
            return (x * kappa).astype(np.float16).astype(np.float64) / kappa
        if role in ("R", "ZR"):
            return (x * rho).astype(np.float16).astype(np.float64) / rho
        return x.astype(np.float16).astype(np.float64)
    return store


def rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def main():
    n, m, seed = 4096, 16384, 3000
    t = time.time()
    X, sigma = inputs.spectrum_matrix(n, m, -4.0, seed=seed)
    Xb = bf16(X)
    del X
    exact = O.newton_schulz(Xb, COEFFS5)
    out = {"_source": "tests/golden/make_spectrum_bounds.py (oracle only)", "shape": [n, m], "seed": seed,
           "coeffs": list(COEFFS5[0]), "T": 5}
    out["standard_bf16"] = rel(O.newton_schulz(Xb, COEFFS5, store=store_bf16), exact)
    out["standard_f16"] = rel(O.newton_schulz(Xb, COEFFS5, store=store_f16(n)), exact)
    out["gram_f16_restart3"] = rel(O.gram_newton_schulz(Xb, COEFFS5, restart_at=3, store=store_f16(n)), exact)
    out["orthogonality_exact"] = float(np.linalg.norm(exact @ exact.T - np.eye(n)))
    out["seconds"] = round(time.time() - t, 1)
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "spectrum_4096x16384_emulated.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
