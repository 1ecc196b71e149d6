"""Helpers shared by the GPU parity tests (no method arithmetic here)."""

import numpy as np
import torch

from newton_schulz_10_b200 import inputs

COEFFS5 = ((3.4445, -4.7750, 2.0315),) * 5


def rel(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def dev(x: np.ndarray, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(dtype).contiguous()


def host(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_values(x32: np.ndarray) -> np.ndarray:
    """Values of the bf16 rounding of x32, as float64."""
    return inputs.bf16_bits_to_f32(inputs.to_bf16_bits(x32)).astype(np.float64)


def gauss(shape, seed, std=1.0):
    return inputs.gaussian(shape, std, seed, 0)
