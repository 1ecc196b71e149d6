"""The seeded input recipes (newton_schulz_10_b200/inputs.py) produce what
the workloads state, checked against independent references: the SVD for the
constructed spectrum, torch's bf16 cast for the rounding helper, and the
Student-t distribution for the heavy-tailed gradients."""

import numpy as np
import pytest
import torch
from scipy import stats

from newton_schulz_10_b200 import inputs


def test_spectrum_matrix_has_the_stated_singular_values():
    X, sigma = inputs.spectrum_matrix(64, 256, -4.0, seed=11)
    s = np.linalg.svd(X, compute_uv=False)
    assert np.allclose(np.sort(s), np.sort(sigma), rtol=1e-10, atol=1e-14)
    assert sigma.min() >= 1e-4 and sigma.max() <= 1.0
    # log-uniform: log10(sigma) / -4 is uniform on [0, 1)
    assert stats.kstest(np.log10(sigma) / -4.0, "uniform").pvalue > 1e-3


def test_random_orthonormal_columns():
    Q = inputs.random_orthonormal(200, 64, 5, 1)
    assert np.allclose(Q.T @ Q, np.eye(64), atol=1e-12)
    assert Q.shape == (200, 64)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 10.0 ** rng.integers(-20, 20, 10000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0, 3.4e38, 1e-40], np.float32)])
    ours = inputs.bf16_bits_to_f32(inputs.to_bf16_bits(x))
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("scale", [1e-3, 1.0])
def test_student_t3_distribution(scale):
    z = inputs.student_t3((400000,), scale, 7, 1).astype(np.float64) / scale
    assert stats.kstest(z, stats.t(df=3).cdf).pvalue > 1e-3


def test_gaussian_moments_and_determinism():
    a = inputs.gaussian((1000, 100), 0.02, 3, 0)
    b = inputs.gaussian((1000, 100), 0.02, 3, 0)
    assert np.array_equal(a, b) and a.dtype == np.float32
    assert abs(a.mean()) < 1e-3 and abs(a.std() / 0.02 - 1) < 0.01
    assert not np.array_equal(a, inputs.gaussian((1000, 100), 0.02, 3, 1))
