"""GPU parity of the format variants against the oracle: MXFP4 quantization and
dequantization (bit-exact), FP8 E4M3 static per-tensor quantization and dequantization
(bit-exact), and the MXFP4 -> NVFP4 chain through the cast kernel."""
import numpy as np
import pytest
import torch

import gpu_util as G
from nvfp4_block_numerics_b200 import binding as nv4
from nvfp4_block_numerics_b200 import inputs

pytestmark = pytest.mark.gpu


def _dev(x):
    return G.f32_dev(x) if x.dtype == np.float32 else G.bf16_dev(x)


def _mx_check(orc, x):
    xd = _dev(x)
    f = G.flags_dev()
    q, e8 = nv4.mxfp4_quant(xd, d_flags=f)
    rq, re8, rf = orc.mxfp4_quant(np.ascontiguousarray(x))
    torch.cuda.synchronize()
    assert f.item() == rf
    assert np.array_equal(G.host(e8), re8)
    assert np.array_equal(G.host(q), rq)
    for dt, name in ((torch.bfloat16, "bf16"), (torch.float16, "fp16"), (torch.float32, "fp32")):
        out = torch.empty(tuple(x.shape), dtype=dt, device=G.DEV)
        nv4.nv4_mxfp4_dequant(q, e8, out)
        ref = orc.mxfp4_dequant(rq, re8, name)
        got = G.host(out)
        if name == "fp32":
            got, ref = got.view(np.uint32), ref.view(np.uint32)
        assert np.array_equal(got, ref), name


@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 96), (129, 160), (300, 1024)])
def test_mxfp4_small_ragged(orc, rows, cols):
    r = np.random.default_rng(rows * cols)
    w = (r.laplace(size=(rows, cols)) * 0.03).astype(np.float32)
    w[:, 1] *= 80.0
    w[::4, :32] = 0.0
    w[1::5, 32:64] = -0.0
    w[2::7, :32] *= np.float32(1e-35)                     # subnormal block maxima
    _mx_check(orc, w)
    _mx_check(orc, inputs.f32_to_bf16_bits(w))


def test_mxfp4_edge_values(orc):
    k = 3
    g = np.array([0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, 6, 7.9, -0.25, -5, -6, 1e-30, -0.0, 4] * 2, np.float32)
    x = np.stack([g * np.float32(2.0 ** k), g * np.float32(2.0 ** -130), g * np.float32(2.0 ** 120),
                  np.full(32, np.float32(3.4e38))])
    _mx_check(orc, x)


def test_mxfp4_layer_shapes(orc):
    _mx_check(orc, inputs.c2_shape(4096, 7168))
    _mx_check(orc, inputs.c3_layer(0, which=("W_q",))["W_q"])


def test_mxfp4_quant_then_cast(orc):
    """The GPU MXFP4 quantizer feeding the GPU cast: in-window blocks dequantize to the
    MXFP4 values exactly; the whole chain matches the oracle chain."""
    x = inputs.c2_shape(256, 4096)
    xd = G.bf16_dev(x)
    q, e8 = nv4.mxfp4_quant(xd)
    nvq, nvs, ga, s2 = nv4.mxfp4_to_nvfp4(q, e8)
    rq, re8, _ = orc.mxfp4_quant(x)
    ref = orc.mxfp4_to_nvfp4(rq, re8)
    torch.cuda.synchronize()
    assert np.array_equal(G.host(nvq), ref["nv_q"]) and np.array_equal(G.host(nvs), ref["nv_scales"])
    assert s2.item() == ref["s2"]


def _fp8_check(orc, x, amax=None):
    xd = _dev(x)
    if amax is None:
        amax = orc.tensor_amax(x)[0]
    d_amax = torch.tensor([amax], dtype=torch.float32, device=G.DEV)
    f = G.flags_dev()
    q, sc = nv4.fp8_quant(xd, d_amax, d_flags=f)
    rq, rs, rf = orc.fp8_quant(np.ascontiguousarray(x), amax)
    torch.cuda.synchronize()
    assert sc.item() == rs and f.item() == rf
    assert np.array_equal(G.host(q), rq)
    for dt in (torch.bfloat16, torch.float16, torch.float32):
        out = torch.empty(tuple(x.shape), dtype=dt, device=G.DEV)
        nv4.nv4_fp8_dequant(q, sc, out)
        exact = orc.fp8_dequant(rq, rs)
        ref = torch.from_numpy(exact.astype(np.float32)).to(dt)            # RN32, then RN to the output type
        assert torch.equal(out.cpu().view(torch.int16 if dt != torch.float32 else torch.int32),
                           ref.view(torch.int16 if dt != torch.float32 else torch.int32)), dt


@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 48), (129, 80), (300, 1024)])
def test_fp8_small_ragged(orc, rows, cols):
    r = np.random.default_rng(rows + 7 * cols)
    x = (r.laplace(size=(rows, cols)) * 2).astype(np.float32)
    x[0, 0] = -0.0
    _fp8_check(orc, x)
    _fp8_check(orc, inputs.f32_to_bf16_bits(x))
    _fp8_check(orc, x, amax=float(np.abs(x).max()) / 4)                    # values beyond the static amax
    _fp8_check(orc, x, amax=0.0)


def test_fp8_degenerate_scales_and_layer(orc):
    r = np.random.default_rng(9)
    x = (r.standard_normal((4, 64)) * 1e-35).astype(np.float32)
    _fp8_check(orc, x)                                                      # s far below 2^-100: exact path
    _fp8_check(orc, inputs.c2_shape(4096, 4096))


def _e4m3_values():
    c = np.arange(127)
    e, m = c >> 3, c & 7
    return np.where(e == 0, m * 2.0 ** -9, (1 + m / 8) * 2.0 ** (e - 7.0))


@pytest.mark.parametrize("amax", [752.0, 1000.0, 336.0, 3.3e-3, 123456.7])
def test_fp8_near_midpoints(orc, amax):
    """Inputs on, just below and just above every E4M3 midpoint times s (both signs), so
    the exact decision runs in both directions and on ties; amax = 752 and 336 give an s
    close to or equal to a short rational (336 / 448 = 0.75 exactly: true ties)."""
    _, s, _ = orc.fp8_quant(np.zeros((1, 16), np.float32), amax)
    v = _e4m3_values()
    t = 0.5 * (v[:-1] + v[1:]) * float(s)                                   # exact in FP64
    x = np.float32(t)
    x = np.concatenate([x, np.nextafter(x, np.float32(np.inf)), np.nextafter(x, np.float32(0))])
    x = np.concatenate([x, -x])
    x = np.pad(x, (0, -len(x) % 16)).astype(np.float32).reshape(-1, 16)
    _fp8_check(orc, x, amax)
    _fp8_check(orc, inputs.f32_to_bf16_bits(x), amax)
    # BF16 Laplace data with outlier channels at a static amax of 752: about one element in
    # a hundred straddles a midpoint
    xl = inputs.laplace_bf16(inputs.rng_for(0, "gpu", "fp8ties"), 257, 1024, outlier_channels=(5, 900),
                             outlier_scale=50.0, zero_block_frac=0.01)
    _fp8_check(orc, xl, amax)


# ------------------------------------------------------------------ block Hadamard + FP4
@pytest.mark.parametrize("n", [16, 32, 64, 128])
def test_hadamard_quant_matches_oracle(orc, n):
    x = inputs.laplace_bf16(inputs.rng_for(n, "gpu", "had"), 129, 512, outlier_channels=(3, 200), outlier_scale=50,
                            zero_block_frac=0.02)
    xd = G.bf16_dev(x)
    y = orc.hadamard_rotate(x, n)
    # amax of the rotated tensor
    amax = torch.zeros(1, dtype=torch.float32, device=G.DEV)
    nv4.nv4_hadamard_amax(xd, n, amax)
    assert amax.item() == float(np.abs(y).max())
    # MXFP4 of the rotated values
    q, e8 = nv4.hadamard_mxfp4_quant(xd, n)
    rq, re8, _ = orc.mxfp4_quant(y)
    assert np.array_equal(G.host(e8), re8) and np.array_equal(G.host(q), rq)
    # NVFP4 of the rotated values (two passes)
    q, sc, s2, _ = nv4.hadamard_nvfp4_quant(xd, n)
    nq, nsc, ns2, _ = orc.rtn_quant(y, float(np.abs(y).max()))
    assert s2.item() == ns2
    assert np.array_equal(G.host(sc), nsc) and np.array_equal(G.host(q), nq)


@pytest.mark.parametrize("n", [16, 32, 64, 128])
@pytest.mark.parametrize("pad", [8, 64])
def test_hadamard_quant_strided_rows(orc, n, pad):
    """Rows inside a wider buffer (row pitch cols + pad), 37 rows so that the last warp of
    segments is only partly live: amax, MXFP4 and NVFP4 of the rotated rows as the oracle
    gives them, and the padding columns never read into the result."""
    rows, cols = 37, 384
    xc = inputs.laplace_bf16(inputs.rng_for(n + pad, "gpu", "had_ld"), rows, cols, outlier_channels=(5, 300),
                             outlier_scale=40, zero_block_frac=0.02)
    x = np.full((rows, cols + pad), 0x7FC0, np.uint16)           # NaN padding: must stay out of every result
    x[:, :cols] = xc
    xd = G.bf16_dev(x)[:, :cols]
    y = orc.hadamard_rotate(xc, n)
    f = G.flags_dev()
    amax = torch.zeros(1, dtype=torch.float32, device=G.DEV)
    nv4.nv4_hadamard_amax(xd, n, amax, f)
    q, e8 = nv4.hadamard_mxfp4_quant(xd, n, d_flags=f)
    qn, sc, s2, _ = nv4.hadamard_nvfp4_quant(xd, n, d_flags=f)
    rq, re8, _ = orc.mxfp4_quant(y)
    nq, nsc, ns2, _ = orc.rtn_quant(y, float(np.abs(y).max()))
    torch.cuda.synchronize()
    assert f.item() == 0 and amax.item() == float(np.abs(y).max())
    assert np.array_equal(G.host(e8), re8) and np.array_equal(G.host(q), rq)
    assert s2.item() == ns2 and np.array_equal(G.host(sc), nsc) and np.array_equal(G.host(qn), nq)


def test_hadamard_quant_layer_shape(orc):
    x = inputs.c2_shape(4096, 7168)
    rows = np.sort(np.random.default_rng(1).choice(4096, 64, replace=False))
    xd = G.bf16_dev(x)
    q, e8 = nv4.hadamard_mxfp4_quant(xd, 128)
    rq, re8, _ = orc.mxfp4_quant(orc.hadamard_rotate(np.ascontiguousarray(x[rows]), 128))
    assert np.array_equal(G.host(e8)[rows], re8) and np.array_equal(G.host(q)[rows], rq)


@pytest.mark.filterwarnings("ignore:overflow encountered in cast")      # the oracle's RN32 of the overflowing sum
@pytest.mark.parametrize("n", [16, 32, 64, 128])
def test_hadamard_quant_nonfinite_overflow_tiny(orc, n):
    """A NaN and an Inf input (every output of their block turns non-finite), a block of
    BF16 values near the top of the range whose rotated sum overflows FP32, and a row of
    BF16 subnormals: MXFP4 codes and scales (0xFF for non-finite blocks) and the non-finite
    flag as the oracle gives them, and the amax pass skipping NaN but keeping Inf."""
    x = inputs.laplace_bf16(inputs.rng_for(n, "gpu", "had_nf"), 6, 512, outlier_channels=(9,), outlier_scale=30)
    x[1, 7] = 0x7FC0                                             # NaN
    x[2, 300] = 0x7F80                                           # +Inf
    x[3, 0:128] = 0x7F61                                         # ~3.0e38: the block's first sum overflows
    x[4, :] = inputs.f32_to_bf16_bits((np.arange(512) % 97 - 48).astype(np.float32) * np.float32(2.0 ** -133))
    x[5, 256:384] = 0                                            # an all-zero block
    xd = G.bf16_dev(x)
    y = orc.hadamard_rotate(x, n)
    f = G.flags_dev()
    q, e8 = nv4.hadamard_mxfp4_quant(xd, n, d_flags=f)
    rq, re8, rf = orc.mxfp4_quant(y)
    torch.cuda.synchronize()
    assert np.array_equal(G.host(e8), re8) and np.array_equal(G.host(q), rq)
    assert (re8 == 0xFF).any() and f.item() == rf
    amax = torch.zeros(1, dtype=torch.float32, device=G.DEV)
    nv4.nv4_hadamard_amax(xd, n, amax)
    assert amax.item() == float(np.nanmax(np.abs(y)))


# ---------------------------------------------------------------- two-sided block Hadamard of weight tiles
def _w_dev(w):
    return G.f32_dev(w) if w.dtype == np.float32 else G.bf16_dev(w)


def _two_sided_check(orc, w, n, ld_pad=0):
    """Rotated values bit for bit, then their amax, MXFP4 and NVFP4 codes, against the
    oracle's rotation followed by its plain quantizers."""
    y = orc.hadamard2_rotate(w, n)
    wd = _w_dev(w)
    if ld_pad:
        big = torch.zeros((w.shape[0], w.shape[1] + ld_pad), dtype=wd.dtype, device=G.DEV)
        big[:, :w.shape[1]] = wd
        wd = big[:, :w.shape[1]]
    f = G.flags_dev()
    got = nv4.hadamard2_rotate(wd, n, d_flags=f)
    torch.cuda.synchronize()
    assert f.item() == 0
    assert np.array_equal(G.host(got).view(np.uint32), y.view(np.uint32))
    amax = torch.zeros(1, dtype=torch.float32, device=G.DEV)
    nv4.nv4_hadamard2_amax(wd, n, amax)
    assert amax.item() == float(np.abs(y).max())
    q, e8 = nv4.hadamard2_mxfp4_quant(wd, n)
    rq, re8, _ = orc.mxfp4_quant(y)
    assert np.array_equal(G.host(e8), re8) and np.array_equal(G.host(q), rq)
    q, sc, s2, _ = nv4.hadamard2_nvfp4_quant(wd, n)
    nq, nsc, ns2, _ = orc.rtn_quant(y, float(np.abs(y).max()))
    assert s2.item() == ns2
    assert np.array_equal(G.host(sc), nsc) and np.array_equal(G.host(q), nq)


@pytest.mark.parametrize("n", [16, 32])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_two_sided_hadamard_matches_oracle(orc, n, dtype):
    rng = np.random.default_rng(n)
    w = (rng.standard_normal((160, 224)) * 0.02).astype(np.float32)
    w[5, 17] = 3.0                                     # an outlier, spread over its tile
    w[32:64, 32:64] = 0.0                              # an all-zero tile
    w[96:96 + n, 64:96] = np.float32(1e-3)             # a constant tile: one nonzero per column pair
    if dtype == "bf16":
        w = inputs.f32_to_bf16_bits(w)
    _two_sided_check(orc, w, n)
    _two_sided_check(orc, w, n, ld_pad=32)


def test_two_sided_hadamard_layer_weights(orc):
    """The Gemma-like layer's q projection [2048, 2048] BF16, 32 x 32 tiles."""
    w = inputs.c3_layer(0, which=("W_q",))["W_q"]
    _two_sided_check(orc, w, 32)


def test_two_sided_hadamard_nonfinite_and_empty(orc):
    w = np.zeros((32, 64), np.float32)
    w[3, 40] = np.inf
    f = G.flags_dev()
    nv4.hadamard2_rotate(G.f32_dev(w), 32, d_flags=f)
    torch.cuda.synchronize()
    assert f.item() & 1
    empty = torch.empty((0, 64), dtype=torch.float32, device=G.DEV)
    assert nv4.hadamard2_rotate(empty, 16).shape == (0, 64)
