"""Exhaustive checks of the FP4 and FP8 encoders on the GPU against the oracle's.

Every code the library emits is the nearest representable value to an exact quotient,
decided on the device by a bracket of two FP32 products and an exact fix-up near the
rounding boundaries.  The tests here feed EVERY FP32 bit pattern of the binades around
the decision boundaries (both signs) through the device quantizers and compare each code
with the oracle's exact-comparison encoders, at scales chosen to stress that decision:
s2 = RN32(752 / 2688) (a short rational, whose products land near midpoints often),
power-of-two scales (exact ties), an arbitrary scale, and scales below 2^-100 and above
2^100 (where the kernels switch to their FP64 decisions).

  * E2M1 (element codes): nv4_weight_quant_rtn on FP32 blocks whose first element
    saturates the block scale (a calibrated amax below the data, [FLOW] 3.4-3.5), so
    every block has the same E4M3 scale 448 and S = RN32(448 * s2); the other 15
    elements of the block are the patterns, |x| / S from 2^-7 to 2^6 (the E2M1
    boundaries 0.25 .. 5 with three binades on each side, and saturation).
  * E4M3 (FP8 elements): nv4_fp8_quant with s = RN32(amax / 448), every pattern with
    |x| / s from 2^-14 to 2^12 (the E4M3 boundaries 2^-10 .. 464 with three binades on
    each side) for positive x, three binades for negative x.
  * E4M3 block scales: every FP32 value within 2^12 ulps of each of the 126 decision
    points a_b = midpoint * 6 * s2 of the block-scale encoder (a dense window, not every
    pattern of the binades).
"""
import numpy as np
import pytest
import torch

import gpu_util as G
from nvfp4_block_numerics_b200 import binding as nv4

pytestmark = pytest.mark.gpu

MANT = 1 << 23


def _binade(E: int, negative: bool = False) -> np.ndarray:
    """Every FP32 pattern with biased exponent field E (2^23 values)."""
    bits = (np.uint32(E) << np.uint32(23)) | np.arange(MANT, dtype=np.uint32)
    if negative:
        bits |= np.uint32(0x80000000)
    return bits.view(np.float32)


def _exp_field(v: float) -> int:
    return int((np.array([v], np.float32).view(np.uint32)[0] >> 23) & 0xFF)


E2M1_AMAX = [2688.0, 752.0, 0.8137, 6.0 * 2.0 ** -102, 6.0 * 2.0 ** 101]


@pytest.mark.parametrize("amax", E2M1_AMAX)
def test_e2m1_every_pattern_near_boundaries(orc, amax):
    amax = float(np.float32(amax))
    s2 = orc.s2_from_amax(amax)
    S = float(np.float32(448.0) * np.float32(s2))          # the saturated block scale, RN32(448 * s2)
    big = np.float32(4.0 * amax)                           # a_b / (6 s2) > 448: every block saturates
    eS = _exp_field(S)
    per_row, cols = 15 * 16, 256
    d_amax = torch.tensor([amax], dtype=torch.float32, device=G.DEV)
    checked = 0
    for E in range(eS - 7, eS + 6):
        for neg in (False, True):
            pat = _binade(E, neg)
            rows = -(-pat.size // per_row)
            fill = np.resize(pat, rows * per_row).reshape(rows, 16, 15)
            w = np.empty((rows, 16, 16), np.float32)
            w[:, :, 0] = big
            w[:, :, 1:] = fill
            w = w.reshape(rows, cols)
            q, sc, s2g = nv4.weight_quant_rtn(G.f32_dev(w), d_amax)
            qr, scr, s2r, _ = orc.rtn_quant(w, amax)
            assert s2g.item() == s2r
            assert np.all(G.host(sc) == 0x7E), "every block must saturate to the scale code 448"
            got = G.host(q)
            if not np.array_equal(got, qr):
                bad = np.argwhere(got != qr)[:5]
                r, c = bad[0]
                x = w[r, 2 * c:2 * c + 2]
                raise AssertionError(f"E2M1 mismatch at S={S!r}: x={x.tolist()} gpu={got[r, c]:#x} "
                                     f"oracle={qr[r, c]:#x} ({len(np.argwhere(got != qr))} bytes differ)")
            checked += pat.size
    print(f"E2M1 S={S:.6g}: {checked} patterns, all codes equal")


FP8_AMAX = [448.0, 752.0, 0.0371]


@pytest.mark.parametrize("amax", FP8_AMAX)
def test_e4m3_every_pattern_near_boundaries(orc, amax):
    amax = float(np.float32(amax))
    s = float(np.float32(amax) / np.float32(448.0))
    es = _exp_field(s)
    d_amax = torch.tensor([amax], dtype=torch.float32, device=G.DEV)
    cols = 4096
    checked = 0
    for E in range(es - 14, es + 12):
        for neg in ((False, True) if E in (es - 11, es, es + 8) else (False,)):
            x = _binade(E, neg).reshape(-1, cols)
            xd = G.f32_dev(x)
            q = torch.empty(x.shape, dtype=torch.uint8, device=G.DEV)
            sc = torch.empty(1, dtype=torch.float32, device=G.DEV)
            nv4.nv4_fp8_quant(xd, d_amax, q, sc)
            qr, sr, _ = orc.fp8_quant(x, amax)
            assert sc.item() == sr
            got = G.host(q)
            if not np.array_equal(got, qr):
                bad = np.argwhere(got != qr)[:5]
                r, c = bad[0]
                raise AssertionError(f"E4M3 mismatch at s={s!r}: x={x[r, c]!r} gpu={got[r, c]:#x} "
                                     f"oracle={qr[r, c]:#x} ({len(np.argwhere(got != qr))} differ)")
            checked += x.size
    print(f"E4M3 s={s:.6g}: {checked} patterns, all codes equal")


@pytest.mark.parametrize("amax", [2688.0, 752.0, 1.7e-3])
def test_block_scale_dense_windows(orc, amax):
    """The block-scale encoder E4M3(a_b / (6 s2)) at every FP32 a_b within 2^12 ulps of
    each of its 126 decision points (midpoints between adjacent E4M3 values, and the
    saturation edge above 448); the block's other elements are a_b scaled by 0.3."""
    amax = float(np.float32(amax))
    s2 = np.float32(orc.s2_from_amax(amax))
    vals = np.array([orc.e4m3_value(c) for c in range(127)], np.float64)
    mids = np.concatenate([(vals[:-1] + vals[1:]) / 2, [464.0]])          # 126 decision points
    centers = (mids * 6.0 * float(s2)).astype(np.float32).view(np.int32)
    off = np.arange(-4096, 4096, dtype=np.int32)
    a = (centers[:, None] + off[None, :]).reshape(-1)
    a = a[a > 0].view(np.float32)
    a = a[np.isfinite(a)]
    blk = np.empty((a.size, 16), np.float32)
    blk[:, 0] = a
    blk[:, 1:] = (a * np.float32(0.3))[:, None] * np.linspace(-1, 1, 15, dtype=np.float32)[None, :]
    rows = a.size // 16
    w = np.ascontiguousarray(blk[:rows * 16].reshape(rows, 256))
    d_amax = torch.tensor([amax], dtype=torch.float32, device=G.DEV)
    q, sc, _ = nv4.weight_quant_rtn(G.f32_dev(w), d_amax)
    qr, scr, _, _ = orc.rtn_quant(w, amax)
    assert np.array_equal(G.host(sc), scr), int((G.host(sc) != scr).sum())
    assert np.array_equal(G.host(q), qr), int((G.host(q) != qr).sum())
    print(f"block scales s2={float(s2):.6g}: {rows * 16} blocks, all scales and codes equal")
