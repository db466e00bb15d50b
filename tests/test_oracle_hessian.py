"""Pins for the oracle's local Hessian H_b = sum_t x_b^T x_b (CPU)."""
import numpy as np

from nvfp4_block_numerics_b200 import inputs


def _x(seed, T, K, **kw):
    return inputs.laplace_bf16(inputs.rng_for(seed, "pin", f"H{T}x{K}"), T, K, **kw)


def test_hessian_matches_numpy_matmul(orc):
    x = _x(1, 300, 96, outlier_channels=(5, 40), outlier_scale=30)
    H = orc.hessian_accum(x)
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64)
    for b in range(6):
        xb = xf[:, 16 * b:16 * b + 16]
        np.testing.assert_allclose(H[b], xb.T @ xb, rtol=1e-13, atol=0)
    # a transposed or shifted block would not match: blocks differ from each other
    assert not np.allclose(H[0], H[1])


def test_hessian_invariants(orc):
    x = _x(2, 513, 64)
    H = orc.hessian_accum(x)
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64)
    for b in range(4):
        assert np.array_equal(H[b], H[b].T)                            # symmetric
        ev = np.linalg.eigvalsh(H[b])
        assert ev.min() >= -1e-12 * np.trace(H[b])                       # PSD
        np.testing.assert_allclose(np.trace(H[b]), (xf[:, 16 * b:16 * b + 16] ** 2).sum(), rtol=1e-13)


def test_hessian_additive_over_token_batches_and_accumulates(orc):
    x = _x(3, 200, 32)
    full = orc.hessian_accum(x)
    H = orc.hessian_accum(np.ascontiguousarray(x[:77]))
    H = orc.hessian_accum(np.ascontiguousarray(x[77:]), H)             # += semantics
    np.testing.assert_allclose(H, full, rtol=1e-13)


def test_hessian_leading_dimension(orc):
    x = _x(4, 50, 80)
    sub = np.ascontiguousarray(x[:, :48])
    np.testing.assert_array_equal(orc.hessian_accum(x, cols=48), orc.hessian_accum(sub))
