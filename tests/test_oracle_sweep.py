"""Pins for the oracle's Hessian-weighted E4M3 scale sweep (CPU).

The brute force below is written independently of the oracle: E2M1 rounding by
exact rational distances (tests/exact.py), S_c from torch's E4M3 decode and a
float32 multiply, the quadratic form by numpy.
"""
from fractions import Fraction as Fr

import numpy as np
import torch

import exact as X
from nvfp4_block_numerics_b200 import inputs

E4_F32 = torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()


def brute_block(w: np.ndarray, H: np.ndarray, s2: float):
    """All 127 candidate costs, dequantized blocks and codes of one block."""
    S_all = E4_F32 * np.float32(s2)                       # RN32(e4m3(c) * s2)
    costs, deqs, qs = [], [], []
    for c in range(127):
        S = Fr(float(S_all[c]))
        q = [X.e2m1_code(float(v), S) for v in w]
        d = [X.e2m1_signed_value(k) * S for k in q]
        e = np.array([float(Fr(float(v)) - dd) for v, dd in zip(w, d)])
        costs.append(float(e @ H @ e))
        deqs.append(tuple(d))
        qs.append(q)
    costs = np.array(costs)
    best = int(np.argmin(costs))                            # first minimum = lowest code
    other = [costs[c] for c in range(127) if deqs[c] != deqs[best]]
    return best, qs[best], costs[best], (min(other) if other else np.inf), costs


def _pack(q):
    return [q[2 * k] | (q[2 * k + 1] << 4) for k in range(8)]


def _psd_blocks(seed, nblk, T=64):
    x = inputs.laplace_bf16(inputs.rng_for(seed, "pin", "sweepH"), T, 16 * nblk, outlier_channels=(2,),
                            outlier_scale=20)
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64)
    return np.stack([xf[:, 16 * b:16 * b + 16].T @ xf[:, 16 * b:16 * b + 16] for b in range(nblk)])


def test_sweep_matches_brute_force(orc):
    H = _psd_blocks(1, 3)
    r = np.random.default_rng(2)
    w32 = (r.standard_normal((5, 48)) * 0.02).astype(np.float32)
    w32[:, 7] *= 20
    for w in (w32, inputs.f32_to_bf16_bits(w32)):
        amax, _ = orc.tensor_amax(w)
        res = orc.scale_sweep(w, H, amax)
        wf = w if w.dtype == np.float32 else inputs.bf16_bits_to_f32(w)
        s2 = orc.s2_from_amax(amax)
        for i in range(5):
            for b in range(3):
                best, q, c1, c2, costs = brute_block(wf[i, 16 * b:16 * b + 16], H[b], s2)
                srt = np.sort(costs)
                if srt[1] - srt[0] <= 1e-9 * srt[1]:
                    continue                                # fp64 summation-order near tie
                assert res["codes"][i, b] == best
                assert res["q"][i, 8 * b:8 * b + 8].tolist() == _pack(q)
                np.testing.assert_allclose(res["cost1"][i, b], c1, rtol=1e-12)
                np.testing.assert_allclose(res["cost2"][i, b], c2, rtol=1e-12)


def test_sweep_identity_hessian_is_mse_search_and_scale_invariant(orc):
    r = np.random.default_rng(3)
    w = (r.standard_normal((4, 32)) * 0.05).astype(np.float32)
    amax, _ = orc.tensor_amax(w)
    s2 = orc.s2_from_amax(amax)
    I = np.stack([np.eye(16)] * 2)
    res = orc.scale_sweep(w, I, amax)
    res3 = orc.scale_sweep(w, 3.0 * I, amax)
    assert np.array_equal(res["codes"], res3["codes"])
    np.testing.assert_allclose(res3["cost1"], 3 * res["cost1"], rtol=1e-13)
    for i in range(4):
        for b in range(2):
            blk = w[i, 16 * b:16 * b + 16].astype(np.float64)
            mse = []
            for c in range(127):
                S = float(E4_F32[c] * np.float32(s2))
                deq = [float(X.e2m1_signed_value(X.e2m1_code(float(v), Fr(S))) * Fr(S)) for v in blk]
                mse.append(float(np.sum((blk - np.array(deq)) ** 2)))
            assert res["codes"][i, b] == int(np.argmin(mse))


def test_sweep_degenerate_blocks(orc):
    H = _psd_blocks(4, 2)
    w = np.zeros((2, 32), np.float32)
    w[1, 16:] = (np.random.default_rng(5).standard_normal(16) * 0.1).astype(np.float32)
    Hz = H.copy()
    Hz[1] = 0.0
    res = orc.scale_sweep(w, Hz, 1.0)
    # zero block: every code dequantizes to zeros -> code 0, cost 0, no different block
    assert res["codes"][0, 0] == 0 and res["cost1"][0, 0] == 0 and np.isinf(res["cost2"][0, 0])
    # dead input channels (H_b = 0): every cost is 0 -> lowest code
    assert res["codes"][1, 1] == 0 and res["cost1"][1, 1] == 0 and res["cost2"][1, 1] == 0


def test_sweep_exactly_representable_block_picks_lowest_zero_cost_code(orc):
    H = _psd_blocks(6, 1)
    amax = 2688.0 * 2.0 ** -5                    # s2 = 2^-5
    s2 = orc.s2_from_amax(amax)
    r = np.random.default_rng(7)
    for c in (0x30, 0x38, 0x41, 0x4B, 0x55):
        S = float(E4_F32[c] * np.float32(s2))
        g = r.choice([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], 16) * r.choice([-1, 1], 16)
        g[3] = 6.0
        w = (g * S).astype(np.float32)[None, :]
        assert np.array_equal(w[0].astype(np.float64), g * S)
        res = orc.scale_sweep(w, H, amax)
        best, q, c1, c2, costs = brute_block(w[0], H[0], s2)
        zero = [k for k in range(127) if costs[k] == 0.0]
        assert costs[c] == 0.0 and zero[0] <= c
        assert res["codes"][0, 0] == zero[0] == best and res["cost1"][0, 0] == 0.0


def test_sweep_beats_or_ties_round_to_nearest_scale(orc):
    """The max-calibrated (RTN) block scale is one of the candidates, so the winner's
    cost is never above it (calibration note, section 2 steps 1 and 3)."""
    H = _psd_blocks(8, 4)
    w = (np.random.default_rng(9).standard_normal((6, 64)) * 0.02).astype(np.float32)
    amax, _ = orc.tensor_amax(w)
    s2 = orc.s2_from_amax(amax)
    res = orc.scale_sweep(w, H, amax)
    for i in range(6):
        for b in range(4):
            blk = w[i, 16 * b:16 * b + 16]
            rtn = X.e4m3_code(max(abs(Fr(float(v))) for v in blk), 6 * Fr(s2))
            _, _, _, _, costs = brute_block(blk, H[b], s2)
            assert res["cost1"][i, b] <= costs[rtn] * (1 + 1e-12)
