"""Pins for the oracle's amax, dynamic activation quantization and dequantization (CPU)."""
from fractions import Fraction as Fr

import numpy as np
import torch

import exact as X
from nvfp4_block_numerics_b200 import inputs


def _bf16(vals) -> np.ndarray:
    return inputs.f32_to_bf16_bits(np.asarray(vals, np.float32))


def test_amax_is_numpy_max_abs(orc):
    x = inputs.laplace_bf16(inputs.rng_for(7, "pin", "amax"), 37, 48, outlier_channels=(3,), outlier_scale=80)
    a, f = orc.tensor_amax(x)
    assert a == float(np.abs(inputs.bf16_bits_to_f32(x)).max()) and f == 0
    w = np.random.default_rng(8).standard_normal((5, 33)).astype(np.float32)
    a, f = orc.tensor_amax(w)
    assert a == float(np.abs(w).max()) and f == 0
    a, f = orc.tensor_amax(np.array([1.0, np.nan, -3.0], np.float32))
    assert a == 3.0 and f & orc.FLAG_NONFINITE
    a, f = orc.tensor_amax(np.array([1.0, -np.inf], np.float32))
    assert a == np.inf and f & orc.FLAG_NONFINITE
    assert orc.tensor_amax(np.zeros(0, np.uint16))[0] == 0.0


def test_act_quant_brute_force(orc):
    """Every block of a small Laplace input, decided again in exact rationals."""
    r = inputs.rng_for(9, "pin", "act")
    x = inputs.laplace_bf16(r, 6, 96, outlier_channels=(7, 50), outlier_scale=30, zero_block_frac=0.1)
    amax, _ = orc.tensor_amax(x)
    q, sc, s2, flags = orc.act_quant(x, amax)
    assert flags == 0
    s2r = X.rn32(Fr(amax) / 2688)
    assert Fr(s2) == s2r
    xf = inputs.bf16_bits_to_f32(x)
    for i in range(x.shape[0]):
        for b in range(x.shape[1] // 16):
            code, S, nibs = X.act_quant_block([float(v) for v in xf[i, 16 * b:16 * b + 16]], s2r)
            assert sc[i, b] == code
            packed = [nibs[2 * k] | (nibs[2 * k + 1] << 4) for k in range(8)]
            assert q[i, 8 * b:8 * b + 8].tolist() == packed


def test_act_quant_calibrated_amax_saturates_and_zero_amax(orc):
    x = _bf16([[100.0] + [1.0] * 15, [-0.0] * 8 + [-1e-3] * 8])
    q, sc, s2, _ = orc.act_quant(x, 1.0)          # calibrated amax far below the data
    assert sc[0, 0] == 0x7E                        # block scale saturates at 448
    q, sc, s2, _ = orc.act_quant(x, 0.0)
    assert s2 == 0.0 and (sc == 0).all()
    # zero scale: magnitude 0, sign kept (8 for negatives / -0)
    nib = np.stack([q & 15, q >> 4], -1).reshape(2, 16)
    assert (nib[0] == 0).all() and (nib[1] == 8).all()


def test_act_quant_packing_order(orc):
    # s2 = 1 (amax = 2688); a block whose max is 6 gets scale 1.0 (code 0x38).
    vals = [6.0, 0.5, -1.0, 2.0, 3.0, -4.0, 1.5, 0.0] * 2
    x = _bf16([vals])
    q, sc, s2, _ = orc.act_quant(x, 2688.0)
    assert s2 == 1.0 and sc[0, 0] == 0x38 and X.E4M3[0x38] == 1
    # element 2i in the low nibble, 2i+1 in the high one
    assert q[0, 0] == (0x7 | (0x1 << 4))
    assert q[0, 1] == (0xA | (0x4 << 4))
    assert q[0, 2] == (0x5 | (0xE << 4))
    assert q[0, 3] == (0x3 | (0x0 << 4))


def test_round_trip_properties(orc):
    """Dequantized values lie on +-grid*S, the error is at most half a grid gap, and a
    block whose max equals 6*S reconstructs that max exactly (FLOW 3.4 / 5.4)."""
    r = inputs.rng_for(10, "pin", "rt")
    x = inputs.laplace_bf16(r, 64, 128, outlier_channels=(1, 99), outlier_scale=50, zero_block_frac=0.05)
    amax, _ = orc.tensor_amax(x)
    q, sc, s2, _ = orc.act_quant(x, amax)
    dq = orc.dequant(q, sc, s2, "fp32")
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64)
    S = (torch.tensor(sc.reshape(-1)).view(torch.float8_e4m3fn).float() * torch.tensor(s2)).numpy()
    S = np.repeat(S.reshape(64, 8), 16, axis=1).astype(np.float64)
    grid = np.array([float(g) for g in X.GRID])
    # DQ2 rounds v*S once to FP32, so |dq| is one of RN32(g*S), g on the grid
    cand = (grid.astype(np.float32)[None, None, :] * S.astype(np.float32)[..., None]).astype(np.float64)
    assert np.all(np.any(np.abs(dq)[..., None] == cand, axis=-1))
    gaps = np.diff(grid)
    # half gap at |x|/S: nearest-grid rounding; saturation cannot occur (amax is exact)
    idx = np.clip(np.searchsorted(grid, np.minimum(np.abs(xf) / np.where(S > 0, S, 1), 6), side="right") - 1, 0, 6)
    assert np.all(np.abs(xf - dq) <= gaps[idx] / 2 * S + 2.0 ** -23 * np.abs(dq) + 1e-30)
    # a block whose max is exactly 6*S reconstructs that max exactly
    x2 = _bf16([[6.0 * 0.5] + [0.25] * 15])
    q2, s2c, s22, _ = orc.act_quant(x2, 2688.0 * 0.5)
    d2 = orc.dequant(q2, s2c, s22, "fp32")
    assert d2[0, 0] == 3.0


def test_dequant_matches_torch_two_step(orc):
    """DQ1 then DQ2 computed with torch float32 ops and torch's bf16/fp16 casts."""
    rng = np.random.default_rng(11)
    rows, cols = 9, 64
    q = rng.integers(0, 256, (rows, cols // 2), dtype=np.uint8)
    sc = rng.integers(0, 127, (rows, cols // 16), dtype=np.uint8)
    for s2 in (X.f32(0.0123), 1.0, X.f32(3.3e-3), X.f32(1e30), 2.0 ** -130):
        nib = np.stack([q & 15, q >> 4], -1).reshape(rows, cols)
        v = torch.tensor([float(X.e2m1_signed_value(int(c))) for c in nib.reshape(-1)],
                         dtype=torch.float32).reshape(rows, cols)
        neg_zero = torch.tensor((nib.reshape(-1) == 8)).reshape(rows, cols)
        v = torch.where(neg_zero, torch.tensor(-0.0), v)
        S = torch.tensor(sc).view(torch.float8_e4m3fn).float() * torch.tensor(s2, dtype=torch.float32)
        y = v * S.repeat_interleave(16, dim=1)
        ref32 = y.numpy()
        out32 = orc.dequant(q, sc, s2, "fp32")
        assert np.array_equal(out32.view(np.uint32), ref32.view(np.uint32))
        outb = orc.dequant(q, sc, s2, "bf16")
        assert np.array_equal(outb, y.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
        outh = orc.dequant(q, sc, s2, "fp16")
        assert np.array_equal(outh, y.to(torch.float16).view(torch.int16).numpy().view(np.uint16))


# ------------------------------------------------------------ RTN weight quantization
def test_rtn_quant_fp32_brute_force(orc):
    """FP32 weights (with exact rounding midpoints planted) decided again in exact rationals."""
    r = np.random.default_rng(21)
    w = (r.standard_normal((5, 64)) * 0.02).astype(np.float32)
    w[1, 3] = 0.9                                      # an outlier sets amax
    amax, _ = orc.tensor_amax(w)
    s2r = X.rn32(Fr(amax) / 2688)
    # plant elements exactly on E2M1 decision boundaries of their block's scale
    for b in range(4):
        blk = [float(v) for v in w[2, 16 * b:16 * b + 16]]
        code, S, _ = X.act_quant_block(blk, s2r)
        w[2, 16 * b + 5] = X.f32(Fr(5, 4) * S) if b % 2 else X.f32(-Fr(3, 4) * S)
    q, sc, s2, flags = orc.rtn_quant(w, amax)
    assert flags == 0 and Fr(s2) == s2r
    for i in range(w.shape[0]):
        for b in range(w.shape[1] // 16):
            code, S, nibs = X.act_quant_block([float(v) for v in w[i, 16 * b:16 * b + 16]], s2r)
            assert sc[i, b] == code
            assert q[i, 8 * b:8 * b + 8].tolist() == [nibs[2 * k] | (nibs[2 * k + 1] << 4) for k in range(8)]


def test_rtn_quant_bf16_matches_activation_quantizer(orc):
    x = inputs.laplace_bf16(inputs.rng_for(22, "pin", "rtn"), 9, 80, outlier_channels=(2,), outlier_scale=40)
    amax, _ = orc.tensor_amax(x)
    a = orc.act_quant(x, amax)
    b = orc.rtn_quant(x, amax)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and a[2] == b[2]
    # the same values as FP32 give the same codes
    c = orc.rtn_quant(inputs.bf16_bits_to_f32(x).copy(), amax)
    assert np.array_equal(a[0], c[0]) and np.array_equal(a[1], c[1])


# ------------------------------------------------------------ fake quantize-dequantize
def test_fake_qdq_grid_block_roundtrips_exactly(orc):
    """amax = 2688 gives s2 = 1; a block of grid values times a power-of-two S whose
    largest magnitude is 6S gets block scale S and comes back bit-exact."""
    rows = []
    for k, S in enumerate((0.25, 1.0, 4.0, 32.0)):
        v = np.array([6, -0.5, 1, -1.5, 2, 3, -4, 0, 0.5, -6, 4, 1.5, -2, -3, 1, -1], np.float32)
        rows.append(np.roll(v, k) * np.float32(S))
    x = inputs.f32_to_bf16_bits(np.stack(rows).reshape(1, -1).astype(np.float32))
    out, s2, flags = orc.fake_qdq(x, 2688.0)
    assert s2 == 1.0 and flags == 0
    assert np.array_equal(out, x)


def test_fake_qdq_error_within_half_grid_step(orc):
    x = inputs.laplace_bf16(inputs.rng_for(23, "pin", "qdq"), 7, 96, outlier_channels=(11,), outlier_scale=25)
    amax, _ = orc.tensor_amax(x)
    y32, s2, _ = orc.fake_qdq(x, amax, "fp32")
    ybf, _, _ = orc.fake_qdq(x, amax, "bf16")
    q, sc, _, _ = orc.act_quant(x, amax)
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64)
    S = np.repeat(np.array([[orc.e4m3_value(int(c)) for c in row] for row in sc]) * s2, 16, axis=1)
    a = np.abs(xf) / S
    half = np.where(a <= 2, 0.25, np.where(a <= 4, 0.5, 1.0)) * S
    assert np.all(np.abs(xf - y32) <= half * (1 + 1e-6) + (a - 6).clip(0) * S)
    # the BF16 output is the FP32 dequantized value rounded to BF16
    assert np.array_equal(ybf, inputs.f32_to_bf16_bits(y32.astype(np.float32)))
