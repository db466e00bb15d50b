"""Pins for the oracle's block Hadamard rotation (CPU)."""
import numpy as np
import pytest
import scipy.linalg

from nvfp4_block_numerics_b200 import inputs


@pytest.mark.parametrize("n", [16, 32, 64, 128])
def test_rotation_matches_scipy_hadamard(orc, n):
    """Against SciPy's Hadamard matrix (an independent Sylvester construction)."""
    x = inputs.laplace_bf16(inputs.rng_for(n, "pin", "had"), 5, 2 * n, outlier_channels=(1,), outlier_scale=40)
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    ref = (xf.reshape(5, 2, n) @ H * (1.0 / np.sqrt(n))).astype(np.float32).reshape(5, 2 * n)
    assert np.array_equal(orc.hadamard_rotate(x, n), ref)


@pytest.mark.parametrize("n", [16, 32, 64, 128])
def test_rotation_is_orthonormal(orc, n):
    # unit vectors map to the rows of H / sqrt(n); the norm of every block is preserved
    e = np.eye(n, dtype=np.float32)
    y = orc.hadamard_rotate(e, n).astype(np.float64)
    assert np.allclose(y @ y.T, np.eye(n), atol=1e-6)
    assert np.allclose(np.abs(y), 1 / np.sqrt(n), rtol=1e-7)
    x = np.random.default_rng(n).standard_normal((3, 4 * n)).astype(np.float32)
    yb = orc.hadamard_rotate(x, n).reshape(3, 4, n).astype(np.float64)
    xb = x.reshape(3, 4, n).astype(np.float64)
    assert np.allclose((yb ** 2).sum(-1), (xb ** 2).sum(-1), rtol=1e-6)
    # applying the rotation twice gives the input back (H H = n I)
    assert np.allclose(orc.hadamard_rotate(orc.hadamard_rotate(x, n), n), x, rtol=1e-5, atol=1e-6)


def test_rotation_flattens_an_outlier(orc):
    """One large value spreads evenly over its block: the effect the FP4 overview relies
    on before FP4 quantization (section 2.1)."""
    x = np.zeros((1, 128), np.float32)
    x[0, 5] = 64.0
    y = orc.hadamard_rotate(x, 128)
    assert np.allclose(np.abs(y), 64.0 / np.sqrt(128), rtol=1e-7)
