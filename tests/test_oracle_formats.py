"""Pins for the oracle's number formats and encoders (CPU only).

Each check compares the oracle with something independent of it: the values the
pages print (golden fixtures), torch's float8/bf16/fp16 conversions, or exact
rational arithmetic in ``tests/exact.py``.
"""
from fractions import Fraction as Fr

import numpy as np
import pytest
import torch

import exact as X

pytestmark = pytest.mark.filterwarnings("ignore")


def test_e2m1_grid_matches_page(orc):
    # FP4 overview 1.1 lists the magnitudes; the sign bit mirrors them.
    assert [Fr(orc.e2m1_value(c)) for c in range(8)] == X.GRID
    for c in range(8):
        assert orc.e2m1_value(c | 8) == -orc.e2m1_value(c)
    assert np.signbit(orc.e2m1_value(8))  # code 0x8 is -0


def test_e4m3_decode_matches_torch(orc):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().tolist()
    for c in range(256):
        v = orc.e4m3_value(c)
        if np.isnan(ref[c]):
            assert np.isnan(v), c
        else:
            assert v == ref[c] and np.signbit(v) == np.signbit(ref[c]), c


def test_e4m3_facts_from_pages(orc):
    kv = X.golden_kv("e4m3_facts.txt")
    finite = [orc.e4m3_value(c) for c in range(128) if not np.isnan(orc.e4m3_value(c))]
    assert max(finite) == float(kv["e4m3_max"])                 # 448
    assert max(X.GRID) == int(kv["e2m1_max"])                   # 6
    assert int(kv["e4m3_max"]) * int(kv["e2m1_max"]) == int(kv["per_tensor_divisor"])
    # the 7-bit code space has 128 points; 127 are finite candidates (0x7F is NaN)
    assert len(finite) == int(kv["code_space_nonneg"]) - 1
    assert all(a < b for a, b in zip(finite, finite[1:]))


def test_e8m0_decode_matches_torch(orc):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).float().tolist()
    for c in range(255):
        assert orc.e8m0_value(c) == ref[c], c
    assert np.isnan(orc.e8m0_value(255))


def _fp32_neighbors(v: float):
    f = np.float32(v)
    return [float(np.nextafter(f, np.float32(-np.inf))), float(f), float(np.nextafter(f, np.float32(np.inf)))]


def test_e4m3_encode_matches_torch_cast(orc):
    """den = 1: the exact quotient is the FP32 input itself, so torch's single-rounding
    float32 -> e4m3fn cast (RNE) is the reference, below its NaN overflow at 464."""
    rng = np.random.default_rng(1)
    vals = list(rng.uniform(0, 464, 3000).astype(np.float32))
    vals += list(np.exp2(rng.uniform(-14, 8.85, 3000)).astype(np.float32))
    e4 = [float(v) for v in X.E4M3]
    for a, b in zip(e4, e4[1:]):
        vals += _fp32_neighbors((a + b) / 2)                   # midpoints and +-1 ulp
    vals = [float(v) for v in vals if 0 <= v < 464]
    t = torch.tensor(vals, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).tolist()
    for v, ref in zip(vals, t):
        assert orc.e4m3_encode(v, 1.0) == ref, v


def test_e4m3_encode_exact_quotient(orc):
    """num/den with den = 6*s2 (s2 an FP32 value): brute force nearest in exact rationals,
    including saturation above 448 and quotients that sit exactly on a midpoint."""
    rng = np.random.default_rng(2)
    e4 = X.E4M3
    cases = []
    for _ in range(1500):
        s2 = X.f32(np.exp2(rng.uniform(-30, 10)) * rng.uniform(1, 2))
        num = X.f32(rng.uniform(0, 600) * 6 * s2)
        cases.append((num, s2))
    for k in range(0, 126, 5):                                   # exact midpoints
        s2 = 0.125
        mid = (e4[k] + e4[k + 1]) / 2
        num = mid * 6 * Fr(s2)
        if X.rn32(num) == num:
            cases.append((float(num), s2))
    cases.append((0.0, 1.0))
    cases.append((1e30, 1e-30))
    for num, s2 in cases:
        ref = X.e4m3_code(Fr(num), 6 * Fr(s2))
        assert orc.e4m3_encode(num, 6.0 * s2) == ref, (num, s2)
    assert orc.e4m3_encode(5.0, 0.0) == 0  # zero second-level scale


def test_e2m1_encode_exact(orc):
    rng = np.random.default_rng(3)
    cases = []
    for _ in range(4000):
        S = X.f32(np.exp2(rng.uniform(-40, 40)) * rng.uniform(1, 2))
        x = X.f32(rng.uniform(-7, 7) * S)
        cases.append((x, S))
    mids = [(X.GRID[k] + X.GRID[k + 1]) / 2 for k in range(7)]
    for S in (1.0, X.f32(0.3), X.f32(1.2345678), 2.0 ** -140, 3.0 * 2 ** -149):
        for m in mids:
            v = m * Fr(S)
            for x in _fp32_neighbors(float(v)):
                cases.append((x, S))
                cases.append((-x, S))
    cases += [(0.0, 1.0), (-0.0, 1.0), (-1e-30, 1.0), (5.0, 0.0), (-5.0, 0.0), (1e30, 1.0)]
    for x, S in cases:
        ref = X.e2m1_code(x, Fr(S))
        assert orc.e2m1_encode(x, S) == ref, (x, S)


def test_s2_single_rounding(orc):
    rng = np.random.default_rng(4)
    amaxes = list(np.exp2(rng.uniform(-126, 127, 3000)).astype(np.float32))
    amaxes += [np.float32(2688.0 * 2.0 ** k) for k in range(-100, 100, 7)]
    amaxes += [np.float32(1.0), np.float32(0.0), np.float32(1e-45), np.float32(3.4e38)]
    for a in amaxes:
        a = float(a)
        ref = X.rn32(Fr(a) / 2688)
        assert Fr(orc.s2_from_amax(a)) == ref, a
    for k in range(-100, 100, 7):
        assert orc.s2_from_amax(2688.0 * 2.0 ** k) == 2.0 ** k


def test_f32_to_bf16_and_f16_match_torch(orc):
    rng = np.random.default_rng(5)
    bits = rng.integers(0, 2 ** 32, 20000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    extra = np.array([65504.0, 65519.99, 65520.0, 65536.0, 6e-8, 3e-8, 2.0 ** -24, 2.0 ** -25,
                      3.3895314e38, 3.4028235e38, 0.0, -0.0, 1.0, 1.00390625, 1.0 + 2 ** -9],
                     dtype=np.float32)
    f = np.concatenate([f, extra, -extra])
    tb = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    th = torch.from_numpy(f.copy()).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    for v, b, h in zip(f.tolist(), tb.tolist(), th.tolist()):
        assert orc.f32_to_bf16(v) == b, v
        assert orc.f32_to_f16(v) == h, v
