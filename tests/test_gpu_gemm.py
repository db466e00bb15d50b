"""GPU parity of the W4A4 GEMM (tcgen05 kind::mxf4nvf4) and of the MMA scale layout.

Operands come from the oracle (random codes, or the oracle's own quantizers), never
from the CUDA path.  The expected product is the oracle's exact FP64 product of the
dequantized operands.  Error bound, from the arithmetic: the products e2m1 * e4m3 *
e2m1 * e4m3 are exact; the FP32 accumulation adds K/64 MMA partial sums (each of 64
exact products) and so errs by at most ~(K/64 + 4) * 2^-24 * sum|a||b|; the epilogue
multiplies by RN32(s2_A * s2_B) (two more roundings of 2^-24) and, for BF16 output,
rounds to 8 significant bits (2^-8 relative).
"""
import numpy as np
import pytest
import torch

import gpu_util as G
from nvfp4_block_numerics_b200 import binding as nv4
from nvfp4_block_numerics_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols", [(1, 16), (200, 144), (128, 256), (300, 1040)])
def test_mma_scale_layout_matches_oracle(orc, rows, cols):
    sc = np.random.default_rng(rows + cols).integers(0, 256, (rows, cols // 16), dtype=np.uint8)
    got = G.host(nv4.mma_scales(G.u8_dev(sc)))
    assert np.array_equal(got, orc.scales_to_mma_layout(sc))


def _random_operand(rng, rows, K, lo=0x20, hi=0x48):
    q = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    sc = rng.integers(lo, hi + 1, (rows, K // 16), dtype=np.uint8)
    return q, sc


def _check(orc, qa, sa, s2a, qb, sb, s2b, dtypes=(torch.float32, torch.bfloat16)):
    M, K = qa.shape[0], 2 * qa.shape[1]
    D, Dabs = orc.gemm_nvfp4(qa, sa, s2a, qb, sb, s2b)
    da = torch.tensor([s2a], dtype=torch.float32, device=G.DEV)
    db = torch.tensor([s2b], dtype=torch.float32, device=G.DEV)
    acc = (K / 64 + 4) * 2.0 ** -24 * Dabs + 2.0 ** -22 * np.abs(D) + 1e-38
    stats = {}
    for dt in dtypes:
        f = G.flags_dev()
        out = nv4.gemm_nvfp4(G.u8_dev(qa), G.u8_dev(sa), da, G.u8_dev(qb), G.u8_dev(sb), db, dtype=dt, d_flags=f)
        torch.cuda.synchronize()
        assert f.item() == 0
        got = out.float().cpu().numpy().astype(np.float64)
        err = np.abs(got - D)
        bound = acc + (2.0 ** -8 * np.abs(D) if dt == torch.bfloat16 else 0.0)
        ratio = float((err / np.where(Dabs > 0, Dabs, 1.0)).max())
        stats[str(dt)] = ratio
        assert np.all(err <= bound), (dt, float((err - bound).max()), ratio)
    print("gemm", qa.shape[0], qb.shape[0], K, "max |err| / sum|ab|:", stats)


def test_gemm_single_tile(orc):
    rng = np.random.default_rng(11)
    qa, sa = _random_operand(rng, 128, 256)
    qb, sb = _random_operand(rng, 128, 256)
    _check(orc, qa, sa, 1.0, qb, sb, 1.0)


def test_gemm_unit_scales_exact(orc):
    """All scales 1.0 and s2 = 1: every product is a multiple of 1/4 and the sums are
    small integers / 4, exact in FP32, so the FP32 output equals the oracle exactly."""
    rng = np.random.default_rng(12)
    qa = rng.integers(0, 256, (128, 128), dtype=np.uint8)
    qb = rng.integers(0, 256, (256, 128), dtype=np.uint8)
    sa = np.full((128, 16), 0x38, np.uint8)
    sb = np.full((256, 16), 0x38, np.uint8)
    D, _ = orc.gemm_nvfp4(qa, sa, 1.0, qb, sb, 1.0)
    one = torch.ones(1, dtype=torch.float32, device=G.DEV)
    out = nv4.gemm_nvfp4(G.u8_dev(qa), G.u8_dev(sa), one, G.u8_dev(qb), G.u8_dev(sb), one, dtype=torch.float32)
    assert np.array_equal(out.cpu().numpy().astype(np.float64), D)


def test_gemm_multi_tile_random(orc):
    rng = np.random.default_rng(13)
    qa, sa = _random_operand(rng, 384, 1024, lo=0x08, hi=0x7E)
    qb, sb = _random_operand(rng, 256, 1024, lo=0x08, hi=0x7E)
    _check(orc, qa, sa, float(np.float32(3.1e-3)), qb, sb, float(np.float32(0.021)))


def test_gemm_narrow_tiles(orc):
    """N a multiple of 128 but not of 256: the 128-wide tile variant."""
    rng = np.random.default_rng(15)
    qa, sa = _random_operand(rng, 256, 768, lo=0x08, hi=0x7E)
    qb, sb = _random_operand(rng, 384, 768, lo=0x08, hi=0x7E)
    _check(orc, qa, sa, 1.0, qb, sb, float(np.float32(1e-3)))


def test_gemm_quantized_layer(orc):
    """Activations quantized by the oracle's dynamic quantizer, weights by its RTN
    quantizer: the W4A4 product of a 256-token batch through a 2048 -> 512 projection."""
    x = inputs.c2_shape(256, 2048)
    qa, sa, s2a, _ = orc.act_quant(x, orc.tensor_amax(x)[0])
    w = inputs.c3_layer(0, which=("W_q",))["W_q"][:512]
    qb, sb, s2b, _ = orc.rtn_quant(np.ascontiguousarray(w), orc.tensor_amax(w)[0])
    _check(orc, qa, sa, s2a, qb, sb, s2b)


def test_gemm_large(orc):
    rng = np.random.default_rng(14)
    qa, sa = _random_operand(rng, 1024, 4096)
    qb, sb = _random_operand(rng, 1024, 4096)
    _check(orc, qa, sa, 0.5, qb, sb, 0.25, dtypes=(torch.float32,))


# Persistent paths: the grid is min(tiles, resident CTAs or CTA pairs), so these shapes give
# every CTA (pair) several output tiles.  M and N multiples of 256 run the CTA-pair kernel
# (256 x 256 tiles, 5-stage ring); other shapes the single-CTA kernel (128 x 256 tiles when
# N allows, else 128 x 128; 4-stage ring).  Stage counts per tile of 1, 2, 3 and 5 move the
# rings' phases across tile boundaries in different ways; the accumulator hand-off between
# the epilogue and the next tile's MMAs and the teardown drain run on every CTA.
@pytest.mark.parametrize("M,N,K", [
    (4096, 4096, 512),    # pairs: 16 x 16 = 256 tiles 256 x 256, ~3.5 per pair, 2 stages per tile
    (4096, 4096, 256),    # pairs: 1 stage per tile, the ring wraps every 5 tiles
    (4096, 4096, 1280),   # pairs: 5 stages per tile, the ring's period
    (3968, 4096, 512),    # single CTA: 31 x 16 = 496 tiles 128 x 256 (M not a multiple of 256)
    (3968, 4096, 256),    # single CTA, 1 stage per tile: the ring wraps every 4 tiles
    (4096, 3968, 512),    # single CTA: 32 x 31 = 992 tiles 128 x 128 (N not a multiple of 256)
    (2048, 3968, 768),    # single CTA: 496 tiles 128 x 128, 3 stages per tile
    (256, 256, 256),      # pairs: a single tile, one pair of CTAs
    (512, 768, 512),      # pairs: 2 x 3 tiles, fewer tiles than pairs
])
def test_gemm_persistent_multi_tile(orc, M, N, K):
    rng = np.random.default_rng(M + N + K)
    qa, sa = _random_operand(rng, M, K, lo=0x08, hi=0x7E)
    qb, sb = _random_operand(rng, N, K, lo=0x08, hi=0x7E)
    _check(orc, qa, sa, float(np.float32(0.37)), qb, sb, float(np.float32(1.9e-2)))
