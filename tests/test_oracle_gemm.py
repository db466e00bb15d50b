"""Pins for the oracle's NVFP4 x NVFP4 GEMM and the MMA scale-factor layout (CPU)."""
from fractions import Fraction as Fr

import numpy as np
import torch

import exact as X


def _rand_operand(rng, rows, k, code_hi=0x7E):
    q = rng.integers(0, 256, (rows, k // 2), dtype=np.uint8)
    sc = rng.integers(0, code_hi + 1, (rows, k // 16), dtype=np.uint8)
    return q, sc


def test_gemm_brute_force_rationals(orc):
    """Every output of a small product, recomputed in exact rationals from the E2M1 grid
    and torch's E4M3 decoding (no oracle table involved)."""
    rng = np.random.default_rng(1)
    qa, sa = _rand_operand(rng, 3, 48)
    qb, sb = _rand_operand(rng, 4, 48)
    s2a, s2b = float(np.float32(0.0123)), float(np.float32(3.7e-3))
    D, Dabs = orc.gemm_nvfp4(qa, sa, s2a, qb, sb, s2b)

    def deq(q, sc, s2):
        rows = []
        for r in range(q.shape[0]):
            row = []
            for k in range(q.shape[1] * 2):
                b = int(q[r, k // 2])
                code = b >> 4 if k & 1 else b & 15
                row.append(X.e2m1_signed_value(code) * X.E4M3[int(sc[r, k // 16])] * Fr(s2))
            rows.append(row)
        return rows

    A, B = deq(qa, sa, s2a), deq(qb, sb, s2b)
    for m in range(3):
        for n in range(4):
            ex = sum(a * b for a, b in zip(A[m], B[n]))
            mag = sum(abs(a * b) for a, b in zip(A[m], B[n]))
            assert abs(Fr(D[m, n]) - ex) <= Fr(1, 2 ** 50) * mag
            assert Fr(Dabs[m, n]) == mag or abs(Fr(Dabs[m, n]) - mag) <= Fr(1, 2 ** 50) * mag


def test_gemm_matches_torch_float8_decode(orc):
    """Against an independent dequantization with torch's float8 E4M3 decoding and a
    float64 matmul: agreement to FP64 rounding."""
    rng = np.random.default_rng(2)
    qa, sa = _rand_operand(rng, 37, 256)
    qb, sb = _rand_operand(rng, 29, 256)
    grid = torch.tensor([float(X.e2m1_signed_value(c)) for c in range(16)], dtype=torch.float64)

    def deq(q, sc, s2):
        t = torch.from_numpy(q.astype(np.int64))
        nib = torch.stack([t & 15, t >> 4], -1).reshape(t.shape[0], -1)
        s = torch.from_numpy(sc.copy()).view(torch.float8_e4m3fn).double().repeat_interleave(16, 1)
        return grid[nib] * s * s2

    A, B = deq(qa, sa, 0.5), deq(qb, sb, 2.0 ** -7)
    D, _ = orc.gemm_nvfp4(qa, sa, 0.5, qb, sb, 2.0 ** -7)
    ref = (A @ B.T).numpy()
    assert np.allclose(D, ref, rtol=0, atol=1e-12 * A.abs().max().item() * B.abs().max().item() * 256)
    # an identity-like case: B has one nonzero element per row, so D picks columns of A
    qb = np.zeros((4, 128), np.uint8)
    sb = np.full((4, 16), 0x38, np.uint8)                 # E4M3 1.0
    for n in range(4):
        qb[n, 5 * n] = 0x02                                # element 10n = 1.0 (low nibble code 2)
    D, _ = orc.gemm_nvfp4(qa, sa, 1.0, qb, sb, 1.0)
    A1 = deq(qa, sa, 1.0).numpy()
    assert np.array_equal(D, A1[:, [0, 10, 20, 30]])


def test_mma_scale_layout_positions(orc):
    sc = np.arange(200 * 9, dtype=np.int64).reshape(200, 9) % 251 + 1
    out = orc.scales_to_mma_layout(sc.astype(np.uint8))
    assert out.size == 2 * 3 * 512                         # rows pad to 256, 9 scales pad to 12
    assert out[0] == sc[0, 0] and out[16] == sc[1, 0] and out[4] == sc[32, 0]
    assert out[512 + 16 + 4 + 1] == sc[33, 5]              # atom (0, 1), r = 33, j = 5
    assert out[(1 * 3 + 2) * 512 + 16 * 7 + 4 * 1 + 0] == sc[128 + 32 + 7, 8]
    # a bijection onto the unpadded part, zeros elsewhere
    assert np.count_nonzero(out) == sc.size
    assert sorted(out[out != 0].tolist()) == sorted(sc.astype(np.uint8).ravel().tolist())
