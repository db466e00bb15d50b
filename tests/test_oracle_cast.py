"""Pins for the oracle's closed-form MXFP4 -> NVFP4 cast (CPU).

Reference facts: global_amax = 6*448*2^(k_max-8), in-window bit identity for
k_max - k_j <= 17, fallback beyond (MXFP4 to NVFP4 conversion guide, section 2);
scale bytes double (DSpark recipe, stage 3; FP4 overview, table 1.2).
"""
from fractions import Fraction as Fr

import numpy as np
import pytest
import torch

import exact as X
from nvfp4_block_numerics_b200 import inputs

KV = X.golden_kv("cast_window.txt")
WINDOW = int(KV["window"])


def _dequant_mx(mx_q, e8m0):
    """MXFP4 dequant with torch: e2m1 value * 2^(code-127), FP32."""
    grid = torch.tensor([float(X.e2m1_signed_value(c)) for c in range(16)], dtype=torch.float32)
    grid[8] = -0.0
    q = torch.from_numpy(mx_q.astype(np.int64))
    nib = torch.stack([q & 15, q >> 4], -1).reshape(q.shape[0], -1)
    v = grid[nib]
    scale = torch.from_numpy(e8m0.copy()).view(torch.float8_e8m0fnu).float()
    return v * scale.repeat_interleave(32, dim=1)


def _dequant_nv(nv_q, nv_s, s2):
    grid = torch.tensor([float(X.e2m1_signed_value(c)) for c in range(16)], dtype=torch.float32)
    grid[8] = -0.0
    q = torch.from_numpy(nv_q.astype(np.int64))
    nib = torch.stack([q & 15, q >> 4], -1).reshape(q.shape[0], -1)
    S = torch.from_numpy(nv_s.copy()).view(torch.float8_e4m3fn).float() * torch.tensor(s2, dtype=torch.float32)
    return grid[nib] * S.repeat_interleave(16, dim=1)


def test_global_amax_formula(orc):
    fac, off = int(KV["global_amax_factor"]), int(KV["global_exponent_offset"])
    for kmax in (-127, -40, -8, 0, 7, 60, 116):
        e = np.full((1, 1), 127 + kmax, np.uint8)
        res = orc.mxfp4_to_nvfp4(np.zeros((1, 16), np.uint8), e)
        assert res["k_max"] == kmax
        assert Fr(res["global_amax"]) == fac * Fr(2) ** (kmax - off)
        assert Fr(res["s2"]) == Fr(2) ** (kmax - off)
        assert res["flags"] == 0
    res = orc.mxfp4_to_nvfp4(np.zeros((1, 16), np.uint8), np.full((1, 1), 127 + 125, np.uint8))
    assert res["flags"] & orc.FLAG_OVERFLOW                  # 2688*2^117 exceeds FP32


def test_in_window_bit_identity_and_scale_bytes(orc):
    mx_q, e8m0 = inputs.mxfp4_matrix(inputs.rng_for(1, "pin", "cast"), 48, 256, fallback_frac=0.02)
    res = orc.mxfp4_to_nvfp4(mx_q, e8m0)
    kmax = int(e8m0.max()) - 127
    assert res["nv_scales"].size == 2 * e8m0.size            # scale bytes double
    mx = _dequant_mx(mx_q, e8m0).numpy()
    nv = _dequant_nv(res["nv_q"], res["nv_scales"], res["s2"]).numpy()
    inwin = np.repeat((kmax - (e8m0.astype(int) - 127)) <= WINDOW, 2, axis=1)
    mx16 = mx.reshape(48, -1, 16).view(np.uint32)
    nv16 = nv.reshape(48, -1, 16).view(np.uint32)
    same = np.all(mx16 == nv16, axis=-1)
    assert np.all(same[inwin])                              # every in-window block is lossless
    # nibbles of in-window blocks are reused unchanged
    qb = mx_q.reshape(48, -1, 8)
    assert np.array_equal(res["nv_q"].reshape(48, -1, 8)[inwin], qb[inwin])
    c = res["counts"]
    assert c[0] == inwin.sum() and c[1] == (~inwin).sum() and c[2] == same.sum()
    assert c[1] > 0


def test_window_edge(orc):
    # k_max = 0 (code 127); blocks at exactly 17 below stay exact, 18 below fall back
    mx_q = np.full((1, 64), 0x77, np.uint8)                   # every element 6.0
    e8m0 = np.array([[127, 127 - WINDOW, 127 - WINDOW - 1, 127 - 3]], np.uint8)
    res = orc.mxfp4_to_nvfp4(mx_q, e8m0)
    assert res["counts"].tolist() == [6, 2, 6]
    s = res["nv_scales"][0]
    # in window: the scale encodes 2^(k_j - k_max + 8) exactly
    vals = torch.from_numpy(s.copy()).view(torch.float8_e4m3fn).float().tolist()
    assert vals[0] == vals[1] == 2.0 ** 8 and vals[2] == vals[3] == 2.0 ** -9
    assert vals[6] == vals[7] == 2.0 ** 5


def test_fallback_blocks_follow_the_quantizer_rules(orc):
    mx_q, e8m0 = inputs.mxfp4_matrix(inputs.rng_for(2, "pin", "castfb"), 16, 512, fallback_frac=0.05)
    res = orc.mxfp4_to_nvfp4(mx_q, e8m0)
    kmax = int(e8m0.max()) - 127
    s2 = Fr(2) ** (kmax - 8)
    mx = _dequant_mx(mx_q, e8m0).numpy()
    n_fb = 0
    for r in range(16):
        for j in range(512 // 32):
            if kmax - (int(e8m0[r, j]) - 127) <= WINDOW:
                continue
            for h in range(2):
                b = 2 * j + h
                vals = [float(v) for v in mx[r, 16 * b:16 * b + 16]]
                code, S, nibs = X.act_quant_block(vals, s2)
                assert res["nv_scales"][r, b] == code
                packed = [nibs[2 * k] | (nibs[2 * k + 1] << 4) for k in range(8)]
                assert res["nv_q"][r, 8 * b:8 * b + 8].tolist() == packed
                n_fb += 1
    assert n_fb > 0


def test_e8m0_nan_rejected(orc):
    with pytest.raises(ValueError):
        orc.mxfp4_to_nvfp4(np.zeros((1, 16), np.uint8), np.array([[255]], np.uint8))


def test_storage_cost_table(orc):
    rows = {ln.split()[0]: ln.split()[1:] for ln in X.golden_lines("format_table.txt")}
    for fmt in ("MXFP4", "NVFP4"):
        g, sbits, bpp = int(rows[fmt][0]), int(rows[fmt][1]), float(rows[fmt][2])
        assert 4 + sbits / g == bpp


def test_grouped_scale2_window_follows_the_group_max(orc):
    """Two matrices sharing one scale_2 (the conversion guide's w1/w3 of routed experts):
    the one holding the group's largest exponent casts as it does alone; the other uses
    the shared s2, so its blocks exactly 17 below the GROUP maximum stay lossless and
    those 18 below fall back, although alone they would all be in window."""
    a_q = np.full((1, 64), 0x77, np.uint8)                    # every element 6.0
    a_e = np.array([[127, 120, 127, 110]], np.uint8)          # k_max(A) = 0
    b_q = np.full((1, 64), 0x35, np.uint8)                    # elements 3.0 and 1.5 (codes 5, 3)
    b_e = np.array([[127 - WINDOW, 127 - WINDOW - 1, 127 - WINDOW - 1, 127 - 14]], np.uint8)
    alone_a, alone_b = orc.mxfp4_to_nvfp4(a_q, a_e), orc.mxfp4_to_nvfp4(b_q, b_e)
    ga, gb = orc.mxfp4_to_nvfp4_group([(a_q, a_e), (b_q, b_e)])
    assert alone_b["counts"].tolist()[:2] == [8, 0]             # alone: k_max(B) = -14, all in window
    for k in ("nv_q", "nv_scales"):
        assert np.array_equal(ga[k], alone_a[k])
    assert ga["s2"] == gb["s2"] == alone_a["s2"] and ga["global_amax"] == gb["global_amax"]
    assert gb["k_max"] == 0
    assert gb["counts"].tolist() == [4, 4, 4]                   # blocks 0 and 3 in window, 1 and 2 fall back
    mx = _dequant_mx(b_q, b_e).numpy().reshape(-1, 16).view(np.uint32)
    nv = _dequant_nv(gb["nv_q"], gb["nv_scales"], gb["s2"]).numpy().reshape(-1, 16).view(np.uint32)
    assert np.all(mx[[0, 1, 6, 7]] == nv[[0, 1, 6, 7]])
    # fallback blocks: 3.0 * 2^-18 and 1.5 * 2^-18 against s2 = 2^-8 are far below the
    # smallest E4M3 block scale (2^-9 * 2^-8), so they become zero blocks (scale code 0)
    assert (gb["nv_scales"][0, 2:6] == 0).all()
    # a group of one is the plain cast
    (solo,) = orc.mxfp4_to_nvfp4_group([(b_q, b_e)])
    assert np.array_equal(solo["nv_q"], alone_b["nv_q"]) and solo["s2"] == alone_b["s2"]
