"""Out-of-bounds write checks on the GPU (memory-safety checks without a sanitizer).

Every output of every entry point is placed inside a larger device buffer with 256-byte
guard regions before and after it, filled with a canary byte.  The calls run on ragged
shapes (row counts that are not multiples of any tile, few 16-element blocks per row),
and afterwards both guard regions must still hold the canary, and the output must equal
the one written into a plain tensor (whose values the parity tests check against the
oracle).  A kernel that writes past either end of any output fails here."""
import numpy as np
import pytest
import torch

import gpu_util as G
from nvfp4_block_numerics_b200 import binding as nv4
from nvfp4_block_numerics_b200 import inputs

pytestmark = pytest.mark.gpu

GUARD = 256
CANARY = 0xA5


class Guarded:
    """A tensor of `shape` and `dtype` at offset GUARD of a canary-filled byte buffer."""

    def __init__(self, shape, dtype, fill=None):
        elt = torch.empty((), dtype=dtype).element_size()
        self.n = int(np.prod(shape)) * elt
        self.buf = torch.full((GUARD + self.n + GUARD,), CANARY, dtype=torch.uint8, device=G.DEV)
        self.t = self.buf[GUARD:GUARD + self.n].view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self) -> bool:
        torch.cuda.synchronize()
        return bool((self.buf[:GUARD] == CANARY).all()) and bool((self.buf[GUARD + self.n:] == CANARY).all())


def _x(rows, cols, seed=0, dtype=torch.bfloat16):
    bits = inputs.laplace_bf16(inputs.rng_for(seed, "guard", f"{rows}x{cols}"), rows, cols,
                               outlier_channels=(1,), outlier_scale=30.0)
    x = G.bf16_dev(bits)
    return x if dtype == torch.bfloat16 else x.float()


SHAPES = [(1, 16), (37, 48), (129, 80), (300, 208)]


@pytest.mark.parametrize("rows,cols", SHAPES)
def test_guards_quantizers(rows, cols):
    x = _x(rows, cols)
    amax = nv4.tensor_amax(x)
    # activation quantization
    q, sc = Guarded((rows, cols // 2), torch.uint8), Guarded((rows, cols // 16), torch.uint8)
    s2 = Guarded((1,), torch.float32)
    nv4.nv4_act_quant(x, amax, q.t, sc.t, s2.t)
    qr, scr, s2r = nv4.act_quant(x, amax)
    assert q.intact() and sc.intact() and s2.intact()
    assert torch.equal(q.t, qr) and torch.equal(sc.t, scr) and torch.equal(s2.t, s2r)
    # dequantization, all three output types
    for dt in (torch.bfloat16, torch.float16, torch.float32):
        out = Guarded((rows, cols), dt)
        nv4.nv4_dequant(qr, scr, s2r, out.t)
        assert out.intact() and torch.equal(out.t, nv4.dequant(qr, scr, s2r, dt))
    # RTN weight quantization of FP32 input
    xf = x.float()
    q, sc, s2 = Guarded((rows, cols // 2), torch.uint8), Guarded((rows, cols // 16), torch.uint8), Guarded((1,), torch.float32)
    nv4.nv4_weight_quant_rtn(xf, amax, q.t, sc.t, s2.t)
    qr, scr, _ = nv4.weight_quant_rtn(xf, amax)
    assert q.intact() and sc.intact() and s2.intact() and torch.equal(q.t, qr) and torch.equal(sc.t, scr)
    # fused fake quantize-dequantize
    for dt in (torch.bfloat16, torch.float32):
        out, s2 = Guarded((rows, cols), dt), Guarded((1,), torch.float32)
        nv4.nv4_fake_qdq(x, amax, out.t, s2.t)
        assert out.intact() and s2.intact() and torch.equal(out.t, nv4.fake_qdq(x, amax, dt)[0])
    # FP8
    q, s = Guarded((rows, cols), torch.uint8), Guarded((1,), torch.float32)
    nv4.nv4_fp8_quant(x, amax, q.t, s.t)
    qr, sr = nv4.fp8_quant(x, amax)
    assert q.intact() and s.intact() and torch.equal(q.t, qr)
    out = Guarded((rows, cols), torch.bfloat16)
    nv4.nv4_fp8_dequant(qr, sr, out.t)
    assert out.intact()
    # MXFP4 (32-element blocks)
    if cols % 32 == 0:
        q, e = Guarded((rows, cols // 2), torch.uint8), Guarded((rows, cols // 32), torch.uint8)
        nv4.nv4_mxfp4_quant(x, q.t, e.t)
        qr, er = nv4.mxfp4_quant(x)
        assert q.intact() and e.intact() and torch.equal(q.t, qr) and torch.equal(e.t, er)
        out = Guarded((rows, cols), torch.float32)
        nv4.nv4_mxfp4_dequant(qr, er, out.t)
        assert out.intact()


@pytest.mark.parametrize("rows", [1, 37, 300])
def test_guards_hadamard(rows):
    x = _x(rows, 256, seed=3)
    for n in (16, 128):
        q, e = Guarded((rows, 128), torch.uint8), Guarded((rows, 8), torch.uint8)
        nv4.nv4_hadamard_mxfp4_quant(x, n, q.t, e.t)
        assert q.intact() and e.intact()
        qr, er = nv4.hadamard_mxfp4_quant(x, n)
        assert torch.equal(q.t, qr) and torch.equal(e.t, er)
        amax = torch.zeros(1, dtype=torch.float32, device=G.DEV)
        nv4.nv4_hadamard_amax(x, n, amax)
        q, sc, s2 = Guarded((rows, 128), torch.uint8), Guarded((rows, 16), torch.uint8), Guarded((1,), torch.float32)
        nv4.nv4_hadamard_nvfp4_quant(x, n, amax, q.t, sc.t, s2.t)
        assert q.intact() and sc.intact() and s2.intact()


@pytest.mark.parametrize("tokens,cols", [(1, 16), (37, 80), (300, 208), (1000, 1040)])
def test_guards_hessian(tokens, cols):
    x = _x(tokens, cols, seed=4)
    H = Guarded((cols // 16, 16, 16), torch.float32, fill=torch.zeros(cols // 16, 16, 16))
    nv4.nv4_hessian_accum(x, H.t)
    assert H.intact() and torch.equal(H.t, nv4.hessian_accum(x))


@pytest.mark.parametrize("rows,cols", SHAPES)
def test_guards_sweep(orc, rows, cols):
    w = (np.random.default_rng(rows).standard_normal((rows, cols)) * 0.02).astype(np.float32)
    x = inputs.laplace_bf16(inputs.rng_for(cols, "guard", "sweepX"), 4096, cols)
    H = G.f32_dev(orc.hessian_accum(x).astype(np.float32))
    for wd in (G.f32_dev(w), G.f32_dev(w).bfloat16()):
        amax = nv4.tensor_amax(wd)
        nb = cols // 16
        codes, q = Guarded((rows, nb), torch.uint8), Guarded((rows, cols // 2), torch.uint8)
        c1, c2 = Guarded((rows, nb), torch.float32), Guarded((rows, nb), torch.float32)
        nv4.nv4_scale_sweep(wd, H, amax, codes.t, q.t, c1.t, c2.t)
        assert codes.intact() and q.intact() and c1.intact() and c2.intact()
        cr, qr, c1r, c2r = nv4.scale_sweep(wd, H, amax)
        assert torch.equal(codes.t, cr) and torch.equal(q.t, qr) and torch.equal(c1.t, c1r)


@pytest.mark.parametrize("rows,cols", [(1, 32), (37, 96), (300, 2880)])
def test_guards_cast(rows, cols):
    mq, e8 = inputs.mxfp4_matrix(inputs.rng_for(rows, "guard", "cast"), rows, cols)
    mqd, e8d = G.u8_dev(mq), G.u8_dev(e8)
    nq, ns = Guarded((rows, cols // 2), torch.uint8), Guarded((rows, cols // 16), torch.uint8)
    ga, s2 = Guarded((1,), torch.float32), Guarded((1,), torch.float32)
    cnt = Guarded((3,), torch.int64, fill=torch.zeros(3, dtype=torch.int64))
    nv4.nv4_mxfp4_to_nvfp4(mqd, e8d, nq.t, ns.t, ga.t, s2.t, cnt.t)
    assert nq.intact() and ns.intact() and ga.intact() and s2.intact() and cnt.intact()
    nqr, nsr, _, _ = nv4.mxfp4_to_nvfp4(mqd, e8d)
    assert torch.equal(nq.t, nqr) and torch.equal(ns.t, nsr)


@pytest.mark.parametrize("M,N,K,ldd", [(128, 128, 256, 128), (256, 384, 512, 400), (384, 256, 768, 264),
                                         (256, 512, 512, 520)])   # the last: the CTA-pair kernel
def test_guards_gemm_and_scale_layout(M, N, K, ldd):
    g = torch.Generator(device=G.DEV).manual_seed(M + N + K)
    qa = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=G.DEV, generator=g)
    qb = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=G.DEV, generator=g)
    sa = torch.randint(0x30, 0x40, (M, K // 16), dtype=torch.uint8, device=G.DEV, generator=g)
    sb = torch.randint(0x30, 0x40, (N, K // 16), dtype=torch.uint8, device=G.DEV, generator=g)
    fa = Guarded((nv4.nv4_mma_scale_bytes(M, K),), torch.uint8)
    nv4.nv4_scales_to_mma_layout(sa, fa.t)
    assert fa.intact() and torch.equal(fa.t, nv4.mma_scales(sa))
    fb = nv4.mma_scales(sb)
    one = torch.ones(1, dtype=torch.float32, device=G.DEV)
    for dt in (torch.bfloat16, torch.float32):
        full = Guarded((M, ldd), dt, fill=torch.zeros(M, ldd))
        out = full.t[:, :N]
        f = G.flags_dev()
        nv4.nv4_gemm_nvfp4(qa, fa.t, one, qb, fb, one, out, f)
        assert f.item() == 0 and full.intact()
        assert torch.all(full.t[:, N:] == 0), "the GEMM wrote into the row padding beyond N"
        assert torch.equal(out, nv4.gemm_nvfp4(qa, sa, one, qb, sb, one, dtype=dt))


@pytest.mark.parametrize("n,rows", [(16, 16), (32, 96), (16, 208)])
def test_guards_two_sided_hadamard(n, rows):
    cols = 96
    w = _x(rows, cols, seed=5, dtype=torch.float32)
    out = Guarded((rows, cols), torch.float32)
    nv4.nv4_hadamard2_rotate(w, n, out.t)
    assert out.intact() and torch.equal(out.t, nv4.hadamard2_rotate(w, n))
    q, e = Guarded((rows, cols // 2), torch.uint8), Guarded((rows, cols // 32), torch.uint8)
    nv4.nv4_hadamard2_mxfp4_quant(w, n, q.t, e.t)
    assert q.intact() and e.intact()
    amax = torch.zeros(1, dtype=torch.float32, device=G.DEV)
    nv4.nv4_hadamard2_amax(w, n, amax)
    q, sc, s2 = Guarded((rows, cols // 2), torch.uint8), Guarded((rows, cols // 16), torch.uint8), Guarded((1,), torch.float32)
    nv4.nv4_hadamard2_nvfp4_quant(w, n, amax, q.t, sc.t, s2.t)
    assert q.intact() and sc.intact() and s2.intact()
    qr, scr, _, _ = nv4.hadamard2_nvfp4_quant(w, n)
    assert torch.equal(q.t, qr) and torch.equal(sc.t, scr)
