"""Pins for the oracle's format variants: MXFP4 (32-element blocks, E8M0 scales) and
FP8 E4M3 with a static per-tensor scale (CPU)."""
from fractions import Fraction as Fr

import numpy as np
import torch

import exact as X
from nvfp4_block_numerics_b200 import inputs


# ------------------------------------------------------------------ MXFP4
def _mx_block_exact(xs):
    a = max(abs(Fr(float(v))) for v in xs)
    if a == 0:
        return 0, [8 if np.signbit(v) else 0 for v in xs]          # all-zero block: code 0, signs kept
    e = max(min(X.floor_log2(a) - 2, 127), -127)
    S = Fr(2) ** e
    return e + 127, [X.e2m1_code(v, S) for v in xs]


def test_mxfp4_brute_force_rationals(orc):
    rng = np.random.default_rng(31)
    w = (rng.standard_normal((6, 96)) * 0.05).astype(np.float32)
    w[1, :32] *= 1e-30                       # tiny values: exponent far below 0
    w[2, 32:64] = 0.0
    w[3, 64:96] = -0.0
    # plant exact E2M1 rounding midpoints of each block's scale
    for b in range(3):
        code, _ = _mx_block_exact([float(v) for v in w[4, 32 * b:32 * b + 32]])
        S = Fr(2) ** (code - 127)
        w[4, 32 * b + 7] = X.f32(Fr(5, 4) * S)
        w[4, 32 * b + 9] = X.f32(-Fr(5, 2) * S)
    for x in (w, inputs.f32_to_bf16_bits(w)):
        q, e8, flags = orc.mxfp4_quant(np.ascontiguousarray(x))
        assert flags == 0
        xf = x if x.dtype == np.float32 else inputs.bf16_bits_to_f32(x)
        for r in range(xf.shape[0]):
            for b in range(3):
                code, nibs = _mx_block_exact([float(v) for v in xf[r, 32 * b:32 * b + 32]])
                assert e8[r, b] == code, (r, b)
                packed = [nibs[2 * k] | (nibs[2 * k + 1] << 4) for k in range(16)]
                assert q[r, 16 * b:16 * b + 16].tolist() == packed


def test_mxfp4_closed_forms_and_flags(orc):
    k = -5
    grid = np.array([6, 4, 3, 2, 1.5, 1, 0.5, 0] * 4, np.float32) * np.float32(2.0 ** k)
    big = grid.copy()
    big[0] = np.float32(7.9 * 2.0 ** k)       # floor(log2) unchanged: saturates to 6 * 2^k
    x = np.stack([grid, big, np.zeros(32, np.float32)])
    q, e8, flags = orc.mxfp4_quant(x)
    assert e8[:, 0].tolist() == [127 + k, 127 + k, 0] and flags == 0
    back = orc.mxfp4_dequant(q, e8, "fp32")
    assert np.array_equal(back[0], grid)                     # grid values come back exactly
    assert back[1, 0] == np.float32(6 * 2.0 ** k)
    q, e8, flags = orc.mxfp4_quant(np.array([[np.nan] + [1.0] * 31], np.float32))
    assert e8[0, 0] == 0xFF and flags & orc.FLAG_NONFINITE


def test_mxfp4_dequant_matches_torch_e8m0(orc):
    rng = np.random.default_rng(32)
    q = rng.integers(0, 256, (5, 64), dtype=np.uint8)
    e8 = rng.integers(100, 150, (5, 4), dtype=np.uint8)
    got = orc.mxfp4_dequant(q, e8, "fp32")
    grid = torch.tensor([float(X.e2m1_signed_value(c)) for c in range(16)], dtype=torch.float64)
    t = torch.from_numpy(q.astype(np.int64))
    nib = torch.stack([t & 15, t >> 4], -1).reshape(5, -1)
    sc = torch.from_numpy(e8.copy()).view(torch.float8_e8m0fnu).double().repeat_interleave(32, 1)
    assert np.array_equal(got, (grid[nib] * sc).float().numpy())


def test_mxfp4_then_cast_is_lossless_in_window(orc):
    """MXFP4 quantization followed by the closed-form cast (MXFP4 to NVFP4 guide, section
    2): every in-window block dequantizes to the same values in both formats."""
    x = inputs.laplace_bf16(inputs.rng_for(33, "pin", "mxcast"), 24, 256, outlier_channels=(3,), outlier_scale=60)
    q, e8, _ = orc.mxfp4_quant(x)
    res = orc.mxfp4_to_nvfp4(q, e8)
    mx = orc.mxfp4_dequant(q, e8, "fp32")
    nv = orc.dequant(res["nv_q"], res["nv_scales"], res["s2"], "fp32")
    kmax = res["k_max"]
    inwin = np.repeat((kmax - (e8.astype(int) - 127)) <= 17, 32, axis=1)
    assert np.array_equal(mx.view(np.uint32)[inwin], nv.view(np.uint32)[inwin])


# ------------------------------------------------------------------ FP8 E4M3, static per-tensor scale
def test_fp8_brute_force_rationals(orc):
    rng = np.random.default_rng(34)
    x = (rng.laplace(size=(4, 40)) * 3).astype(np.float32)
    amax = float(np.abs(x).max())
    s = X.rn32(Fr(amax) / 448)
    # plant midpoints between E4M3 values, and values above the calibrated amax
    x[1, 0] = X.f32((X.E4M3[40] + X.E4M3[41]) / 2 * s)
    x[1, 1] = X.f32(-(X.E4M3[41] + X.E4M3[42]) / 2 * s)
    x[2, 5] = np.float32(amax * 3)
    for xin in (x, inputs.f32_to_bf16_bits(x)):
        q, s_got, flags = orc.fp8_quant(np.ascontiguousarray(xin), amax)
        assert Fr(s_got) == s and flags == 0
        xf = xin if xin.dtype == np.float32 else inputs.bf16_bits_to_f32(xin)
        for v, c in zip(xf.ravel(), q.ravel()):
            exp = (0x80 if np.signbit(v) else 0) | X.e4m3_code(abs(Fr(float(v))), s)
            assert c == exp, (v, c, exp)
    q, _, _ = orc.fp8_quant(x, amax)
    assert q[2, 5] & 0x7F == 0x7E                          # saturates at 448
    assert q[1, 0] == 40 and q[1, 1] == 0x80 | 42          # ties to the even code


def test_fp8_zero_scale_and_dequant(orc):
    x = np.array([[1.0, -2.0, -0.0, 0.0]], np.float32)
    q, s, _ = orc.fp8_quant(x, 0.0)
    assert s == 0.0 and q.tolist() == [[0, 0x80, 0x80, 0]]
    q, s, _ = orc.fp8_quant(x, 448.0)                      # s = 1: values are E4M3 already
    assert s == 1.0 and np.array_equal(orc.fp8_dequant(q, s), x.astype(np.float64))
