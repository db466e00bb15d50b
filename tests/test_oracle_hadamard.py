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


# ---------------------------------------------------------------- pins of the exact reading
def _rn32_fraction(F):
    """RN32 of an exact rational, decided by exact distances to the two nearest FP32 values
    (ties to the even significand); independent of the oracle's integer rounding."""
    from fractions import Fraction

    f = np.float32(float(F))
    if not np.isfinite(f):
        return f
    cands = {f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))}
    best = None
    for c in cands:
        if not np.isfinite(c):
            continue
        d = abs(Fraction(float(c)) - F)
        key = (d, int(np.array([c], np.float32).view(np.uint32)[0]) & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


@pytest.mark.parametrize("n", [32, 128])
def test_rotation_reading_in_exact_rationals(orc, n):
    """y = RN32(RN64(sum) * RN64(1/sqrt(n))) recomputed with exact rationals: the sum of
    the BF16 values exactly, RN64 of it and of the product by Python's correctly rounded
    rational-to-float conversion, and RN32 by exact distances.  n = 32 and 128 make
    1/sqrt(n) irrational, so the reading's rounding order is what is pinned."""
    from fractions import Fraction

    x = inputs.laplace_bf16(inputs.rng_for(n, "pin", "had-exact"), 3, 2 * n, outlier_channels=(2,),
                            outlier_scale=300)
    xf = inputs.bf16_bits_to_f32(x)
    H = scipy.linalg.hadamard(n)
    c = Fraction(float(np.float64(1.0) / np.sqrt(np.float64(n))))
    got = orc.hadamard_rotate(x, n)
    for r in range(3):
        for blk in range(2):
            v = [Fraction(float(t)) for t in xf[r, blk * n:(blk + 1) * n]]
            for j in range(n):
                s = sum((v[i] if H[i, j] > 0 else -v[i]) for i in range(n))
                s64 = Fraction(float(s))                         # RN64 of the exact sum
                p64 = Fraction(float(s64 * c))                   # RN64 of the exact product
                want = _rn32_fraction(p64)
                assert got[r, blk * n + j] == want, (r, blk, j)


def test_rn32_of_integers(orc):
    """The oracle's exact-integer rounding against numpy's single rounding of values that
    FP64 holds exactly, and at the FP32 edges (subnormals, the largest finite, overflow)."""
    rng = np.random.default_rng(5)
    for _ in range(2000):
        N = int(rng.integers(-(1 << 52), 1 << 52))
        k = int(rng.integers(-200, 100))
        with np.errstate(over="ignore"):
            want = np.float32(float(N) * 2.0 ** k)
        assert orc._rn32_of_int(N, k) == float(want)
    assert orc._rn32_of_int(3, -150) == 2.0 ** -148                # 1.5 * 2^-149 -> ties to even (2 ulp)
    assert orc._rn32_of_int(1, -150) == 0.0                        # half the smallest subnormal: tie to 0
    assert orc._rn32_of_int((1 << 24) - 1, 104) == float(np.float32(3.4028234663852886e38))
    assert orc._rn32_of_int((1 << 25) - 1, 103) == float("inf")    # rounds up past the largest finite


def _hadamard2_exact(B, n):
    """H B H^T / n in exact rationals, each entry rounded to FP32 by exact distances."""
    from fractions import Fraction

    H = scipy.linalg.hadamard(n)
    F = [[Fraction(float(v)) for v in row] for row in B]
    out = np.empty((n, n), np.float32)
    for i in range(n):
        for j in range(n):
            s = sum(F[k][l] * (H[i, k] * H[j, l]) for k in range(n) for l in range(n))
            out[i, j] = _rn32_fraction(s / n)
    return out


@pytest.mark.parametrize("n", [16, 32])
def test_two_sided_rotation_in_exact_rationals(orc, n):
    """Every entry of H B H^T / n for a BF16 tile and an FP32 tile, recomputed in exact
    rationals with SciPy's Hadamard matrix; one FP32 tile spans ~140 binades, so the
    oracle's integer path is pinned too."""
    rng = np.random.default_rng(n)
    wb = inputs.f32_to_bf16_bits((rng.standard_normal((n, n)) * 0.02).astype(np.float32))
    assert np.array_equal(orc.hadamard2_rotate(wb, n), _hadamard2_exact(inputs.bf16_bits_to_f32(wb), n))
    wf = (rng.standard_normal((n, n)) * np.exp2(rng.integers(-70, 70, (n, n)))).astype(np.float32)
    assert np.array_equal(orc.hadamard2_rotate(wf, n), _hadamard2_exact(wf, n))


@pytest.mark.parametrize("n", [16, 32])
def test_two_sided_rotation_properties(orc, n):
    """Orthogonality (a tile of the identity maps to itself), a single value spreads to
    +-b/n with the sign pattern H_ik H_jl, energy is preserved, and the rotation is its own
    inverse (H H^T = n I) up to the FP32 rounding of the intermediate."""
    I = np.tile(np.eye(n, dtype=np.float32), (2, 3))
    assert np.array_equal(orc.hadamard2_rotate(I, n), I)
    B = np.zeros((n, n), np.float32)
    B[3, 5] = 48.0
    H = scipy.linalg.hadamard(n)
    assert np.array_equal(orc.hadamard2_rotate(B, n), (48.0 / n * np.outer(H[:, 3], H[:, 5])).astype(np.float32))
    w = np.random.default_rng(7).standard_normal((2 * n, 3 * n)).astype(np.float32)
    y = orc.hadamard2_rotate(w, n)
    tiles = lambda a: a.reshape(2, n, 3, n).transpose(0, 2, 1, 3).astype(np.float64)
    assert np.allclose((tiles(y) ** 2).sum((-1, -2)), (tiles(w) ** 2).sum((-1, -2)), rtol=1e-6)
    assert np.allclose(orc.hadamard2_rotate(y, n), w, rtol=1e-5, atol=1e-6)
