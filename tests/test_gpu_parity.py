"""GPU parity of every libnv4 entry point against the CPU oracle.

Small, ragged cases are compared element by element; the workloads' full sizes
run in the same launch configuration as the benchmark and are compared on
sampled rows (or in full where the oracle is fast enough).  Rules: integer and
byte outputs bit-exact; H within 1e-5 relative Frobenius of the FP64 oracle;
sweep codes bit-exact outside near ties (< 0.1% of blocks may differ).
"""
import numpy as np
import pytest
import torch

import gpu_util as G
from nvfp4_block_numerics_b200 import binding as nv4
from nvfp4_block_numerics_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv4.lib()


# ------------------------------------------------------------------ self-test
def test_selftest_conversions():
    out = torch.zeros(64, dtype=torch.int32, device=G.DEV)
    nv4.nv4_selftest(out)
    v = out.cpu().numpy().view(np.uint32)
    print("selftest:", [hex(int(x)) for x in v[:10]])
    assert v[0] == 0, [hex(int(x)) for x in v[:10]]


# ------------------------------------------------------------------ amax
@pytest.mark.parametrize("n", [1, 7, 8, 9, 1000, 4096 + 5, 1 << 20])
def test_amax_bf16_sizes(orc, n):
    x = inputs.laplace_bf16(inputs.rng_for(n, "gpu", "amax"), 1, n, outlier_channels=(n // 2,), outlier_scale=70)
    a = nv4.tensor_amax(G.bf16_dev(x.reshape(-1)))
    assert a.item() == orc.tensor_amax(x)[0]


def test_amax_f32_running_max_and_flags(orc):
    w = (np.random.default_rng(1).standard_normal(12345) * 0.02).astype(np.float32)
    d = torch.zeros(1, dtype=torch.float32, device=G.DEV)
    f = G.flags_dev()
    nv4.nv4_tensor_amax(G.f32_dev(w[:5000]), d, f)
    nv4.nv4_tensor_amax(G.f32_dev(w[5000:]), d, f)          # running max across batches
    assert d.item() == orc.tensor_amax(w)[0] and f.item() == 0
    wn = w.copy()
    wn[77] = np.nan
    d2 = torch.zeros(1, dtype=torch.float32, device=G.DEV)
    nv4.nv4_tensor_amax(G.f32_dev(wn), d2, f)
    assert d2.item() == orc.tensor_amax(wn)[0] and f.item() & nv4.FLAG_NONFINITE
    xb = inputs.f32_to_bf16_bits(w)
    xb[3] = 0x7FC0
    f3 = G.flags_dev()
    d3 = nv4.tensor_amax(G.bf16_dev(xb), d_flags=f3)
    assert d3.item() == orc.tensor_amax(xb)[0] and f3.item() & nv4.FLAG_NONFINITE


# ------------------------------------------------------------------ act quant / dequant
def _act_check(orc, x_bits, amax=None, rows_sample=None, ld_pad=0):
    rows, cols = x_bits.shape
    xs = x_bits
    if ld_pad:
        xs = np.zeros((rows, cols + ld_pad), np.uint16)
        xs[:, :cols] = x_bits
    xd = G.bf16_dev(xs)[:, :cols]
    f = G.flags_dev()
    if amax is None:
        d_amax = nv4.tensor_amax(G.bf16_dev(x_bits))
        amax = orc.tensor_amax(x_bits)[0]
        assert d_amax.item() == amax
    else:
        d_amax = torch.tensor([amax], dtype=torch.float32, device=G.DEV)
    q, sc, s2 = nv4.act_quant(xd, d_amax, d_flags=f)
    outs = {dt: nv4.dequant(q, sc, s2, dt) for dt in (torch.bfloat16, torch.float16, torch.float32)}
    torch.cuda.synchronize()
    idx = np.arange(rows) if rows_sample is None else rows_sample
    xr = np.ascontiguousarray(x_bits[idx])
    oq, osc, os2, of = orc.act_quant(xr, amax)
    assert s2.item() == os2 and f.item() == of
    qg, scg = G.host(q)[idx], G.host(sc)[idx]
    assert np.array_equal(scg, osc), np.argwhere(scg != osc)[:5]
    assert np.array_equal(qg, oq), np.argwhere(qg != oq)[:5]
    for dt, name in ((torch.bfloat16, "bf16"), (torch.float16, "fp16"), (torch.float32, "fp32")):
        ref = orc.dequant(oq, osc, os2, name)
        got = G.host(outs[dt])[idx]
        if name == "fp32":
            got, ref = got.view(np.uint32), ref.view(np.uint32)
        assert np.array_equal(got, ref), name


@pytest.mark.parametrize("rows,cols,pad", [(1, 16, 0), (3, 48, 8), (37, 96, 0), (130, 272, 16), (5, 2048, 0)])
def test_act_quant_small_ragged(orc, rows, cols, pad):
    x = inputs.laplace_bf16(inputs.rng_for(rows * cols, "gpu", "act"), rows, cols, outlier_channels=(1,),
                            outlier_scale=50, zero_block_frac=0.05)
    _act_check(orc, x, ld_pad=pad)


def test_act_quant_tiny_config(orc):
    _act_check(orc, inputs.c1_tiny_linear(0)["X"])


def test_act_quant_edge_values(orc):
    S = 1.0  # amax 2688 -> s2 = 1
    g = [0.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, -0.0, -0.25, -0.75, -5.0, 1e-30, -1e-30]
    rows = [g, [v * 0.5 for v in g], [448.0 * 6] + [0.0] * 15, [-0.0] * 16, [3.0] * 16]
    x = inputs.f32_to_bf16_bits(np.array(rows, np.float32))
    _act_check(orc, x, amax=2688.0 * S)
    _act_check(orc, x, amax=0.0)            # s2 = 0: sign-only codes
    _act_check(orc, x, amax=1.0)            # calibrated amax below the data: saturation


def test_empty_inputs_still_write_the_second_level_scale(orc):
    """A tensor with no rows (or no columns) quantizes nothing, but the second-level scale
    is still an output: s2 = RN32(amax / 2688) ([FLOW] 3.4), and RN32(amax / 448) for FP8.
    The outputs start as NaN so that an unwritten scale shows."""
    amax = torch.tensor([2688.0 * 0.375], dtype=torch.float32, device=G.DEV)
    want = orc.s2_from_amax(2688.0 * 0.375)
    nan = lambda: torch.full((1,), float("nan"), dtype=torch.float32, device=G.DEV)
    u8 = lambda *shape: torch.empty(shape, dtype=torch.uint8, device=G.DEV)
    for rows, cols in ((0, 32), (5, 0)):
        x = torch.empty((rows, cols), dtype=torch.bfloat16, device=G.DEV)
        s2 = nan()
        nv4.nv4_act_quant(x, amax, u8(rows, cols // 2), u8(rows, cols // 16), s2)
        assert s2.item() == want
        s2 = nan()
        nv4.nv4_weight_quant_rtn(x.float(), amax, u8(rows, cols // 2), u8(rows, cols // 16), s2)
        assert s2.item() == want
        s2 = nan()
        nv4.nv4_fake_qdq(x, amax, torch.empty((rows, cols), dtype=torch.float32, device=G.DEV), s2)
        assert s2.item() == want
        sc = nan()
        nv4.nv4_fp8_quant(x, amax, u8(rows, cols), sc)
        assert sc.item() == float(np.float32(2688.0 * 0.375) / np.float32(448.0))
    s2 = nan()
    nv4.nv4_hadamard_nvfp4_quant(torch.empty((0, 128), dtype=torch.bfloat16, device=G.DEV), 32, amax,
                                 u8(0, 64), u8(0, 8), s2)
    assert s2.item() == want
    # a batched call mixing an empty job with a full one
    x = G.bf16_dev(inputs.c2_shape(16, 2048))
    s2a, s2b = nan(), nan()
    a2 = nv4.tensor_amax(x)
    nv4.nv4_act_quant_batched([
        dict(x=torch.empty((0, 64), dtype=torch.bfloat16, device=G.DEV), d_amax=amax, q=u8(0, 32), scales=u8(0, 4),
             d_s2=s2a),
        dict(x=x, d_amax=a2, q=u8(16, 1024), scales=u8(16, 128), d_s2=s2b)])
    torch.cuda.synchronize()
    assert s2a.item() == want and s2b.item() == orc.s2_from_amax(a2.item())


@pytest.mark.parametrize("T,C", inputs.C2_SHAPES)
def test_act_quant_config_shapes(orc, T, C):
    x = inputs.c2_shape(T, C)
    sample = None if T <= 4096 else np.sort(np.random.default_rng(T + C).choice(T, 512, replace=False))
    _act_check(orc, x, rows_sample=sample)


def test_act_path_batched_matches_single_and_oracle(orc):
    """The batched amax, act quant and dequant entries over the 15 activation shapes
    (rows capped at 300 so the oracle checks every row), one of them strided and one
    empty: bit for bit the single-tensor calls and the oracle."""
    xs = [inputs.c2_shape(min(T, 300), C) for (T, C) in inputs.C2_SHAPES]
    xs[4] = xs[4].copy()
    xs[4][7, 100] = 0x7FC0                                   # a NaN: skipped by the amax, flagged
    dev = []
    for i, x in enumerate(xs):
        if i == 7:                                           # rows of a wider buffer (ld > cols)
            buf = np.zeros((x.shape[0], x.shape[1] + 64), np.uint16)
            buf[:, :x.shape[1]] = x
            dev.append(G.bf16_dev(buf)[:, :x.shape[1]])
        else:
            dev.append(G.bf16_dev(x))
    empty = torch.empty((0, 64), dtype=torch.bfloat16, device=G.DEV)
    n = len(xs)

    def outputs():
        return ([torch.empty((x.shape[0], x.shape[1] // 2), dtype=torch.uint8, device=G.DEV) for x in xs],
                [torch.empty((x.shape[0], x.shape[1] // 16), dtype=torch.uint8, device=G.DEV) for x in xs],
                [torch.empty(tuple(x.shape), dtype=torch.bfloat16, device=G.DEV) for x in xs])

    # batched (the amax needs contiguous tensors: the strided one goes through its copy)
    fb = G.flags_dev()
    am_b, s2_b = torch.zeros(n + 1, device=G.DEV), torch.zeros(n + 1, device=G.DEV)
    qb, scb, ob = outputs()
    nv4.nv4_tensor_amax_batched([d.contiguous() for d in dev] + [empty], [am_b[i:i + 1] for i in range(n + 1)], fb)
    nv4.nv4_act_quant_batched([dict(x=dev[i], d_amax=am_b[i:i + 1], q=qb[i], scales=scb[i], d_s2=s2_b[i:i + 1])
                               for i in range(n)], fb)
    nv4.nv4_dequant_batched([dict(q=qb[i], scales=scb[i], d_s2=s2_b[i:i + 1], out=ob[i]) for i in range(n)])
    # one call per tensor
    fs = G.flags_dev()
    am_s, s2_s = torch.zeros(n, device=G.DEV), torch.zeros(n, device=G.DEV)
    qs, scs, os_ = outputs()
    for i in range(n):
        nv4.nv4_tensor_amax(dev[i].contiguous(), am_s[i:i + 1], fs)
        nv4.nv4_act_quant(dev[i], am_s[i:i + 1], qs[i], scs[i], s2_s[i:i + 1], fs)
        nv4.nv4_dequant(qs[i], scs[i], s2_s[i:i + 1], os_[i])
    torch.cuda.synchronize()
    assert fb.item() == fs.item() == nv4.FLAG_NONFINITE
    assert am_b[n].item() == 0.0                             # the empty job
    assert torch.equal(am_b[:n], am_s) and torch.equal(s2_b[:n], s2_s)
    for i, x in enumerate(xs):
        assert torch.equal(qb[i], qs[i]) and torch.equal(scb[i], scs[i]), i
        assert torch.equal(ob[i].view(torch.int16), os_[i].view(torch.int16)), i      # bit patterns (NaN blocks)
        amax, _ = orc.tensor_amax(x)
        assert am_b[i].item() == amax, i
        oq, osc, os2, _ = orc.act_quant(x, amax)
        assert s2_b[i].item() == os2
        gq, gsc, go, ro = G.host(qb[i]), G.host(scb[i]), G.host(ob[i]), orc.dequant(oq, osc, os2, "bf16")
        if i == 4:                                           # the NaN block's outputs are unspecified
            gq[7, 48:56] = oq[7, 48:56]
            gsc[7, 6] = osc[7, 6]
            go[7, 96:112] = ro[7, 96:112]
        assert np.array_equal(gq, oq) and np.array_equal(gsc, osc), i
        assert np.array_equal(go, ro), i


def test_amax_batched_fp32_and_tails(orc):
    r = np.random.default_rng(12)
    xs = [(r.laplace(size=n) * 3).astype(np.float32) for n in (1, 3, 4, 5, 4096 * 4 + 3, 70001)]
    xs[3][2] = np.float32(np.inf)
    d = [G.f32_dev(x) for x in xs]
    am = torch.zeros(len(xs), device=G.DEV)
    f = G.flags_dev()
    nv4.nv4_tensor_amax_batched(d, [am[i:i + 1] for i in range(len(xs))], f)
    torch.cuda.synchronize()
    assert f.item() == nv4.FLAG_NONFINITE
    for i, x in enumerate(xs):
        assert am[i].item() == orc.tensor_amax(x)[0], i


def test_dequant_random_codes(orc):
    rng = np.random.default_rng(3)
    q = rng.integers(0, 256, (33, 40), dtype=np.uint8)
    sc = rng.integers(0, 127, (33, 5), dtype=np.uint8)
    for s2 in (0.0123, 1.0, 3.3e-3, 2.0 ** -130, 1e30):
        s2 = float(np.float32(s2))
        d_s2 = torch.tensor([s2], dtype=torch.float32, device=G.DEV)
        for dt, name in ((torch.bfloat16, "bf16"), (torch.float16, "fp16"), (torch.float32, "fp32")):
            got = G.host(nv4.dequant(G.u8_dev(q), G.u8_dev(sc), d_s2, dt))
            ref = orc.dequant(q, sc, s2, name)
            if name == "fp32":
                got, ref = got.view(np.uint32), ref.view(np.uint32)
            assert np.array_equal(got, ref), (s2, name)


# ------------------------------------------------------------------ RTN weight quantization
def _rtn_check(orc, w, amax=None, ld_pad=0):
    rows, cols = w.shape
    wd_full = G.f32_dev(np.pad(w, ((0, 0), (0, ld_pad)))) if w.dtype == np.float32 else \
        G.bf16_dev(np.pad(w, ((0, 0), (0, ld_pad))))
    wd = wd_full[:, :cols]
    if amax is None:
        amax = orc.tensor_amax(w)[0]
    d_amax = torch.tensor([amax], dtype=torch.float32, device=G.DEV)
    f = G.flags_dev()
    q, sc, s2 = nv4.weight_quant_rtn(wd, d_amax, d_flags=f)
    rq, rsc, rs2, rf = orc.rtn_quant(w, amax)
    torch.cuda.synchronize()
    assert s2.item() == rs2 and f.item() == rf
    assert np.array_equal(G.host(sc), rsc)
    assert np.array_equal(G.host(q), rq)


@pytest.mark.parametrize("rows,cols,pad", [(1, 16, 0), (3, 48, 8), (129, 80, 0), (300, 256, 16)])
def test_weight_quant_rtn_small_ragged(orc, rows, cols, pad):
    r = np.random.default_rng(rows + cols)
    w = (r.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    w[:, 1] *= 40.0
    w[::5, :16] = 0.0
    w[1::7, 16:32] = -0.0
    _rtn_check(orc, w, ld_pad=pad)
    _rtn_check(orc, inputs.f32_to_bf16_bits(w), ld_pad=pad)


def test_weight_quant_rtn_edge_values(orc):
    g = [0.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, -0.0, -0.25, -0.75, -5.0, 1e-30, -1e-30]
    w = np.array([g, [v * 0.5 for v in g], [448.0 * 6] + [0.0] * 15, [3.0] * 16], np.float32)
    w = np.concatenate([w, np.nextafter(w, np.float32(np.inf))], axis=1)     # one ulp above each boundary
    for amax in (2688.0, 0.0, 1.0, float(np.float32(2688.0 * 1.37))):
        _rtn_check(orc, w, amax=amax)


def test_weight_quant_rtn_layer_weights(orc):
    d = inputs.c3_layer(0, which=("W_q", "W_gate"))
    _rtn_check(orc, d["W_q"])
    _rtn_check(orc, d["W_gate"])
    _rtn_check(orc, inputs.c1_tiny_linear(0)["W"])


@pytest.mark.parametrize("fp32", [False, True])
def test_weight_quant_rtn_batched(orc, fp32):
    """One batched launch over ragged weights (row pitch padding, a one-row tensor, zero
    blocks, a static amax below the data's) equals the oracle's RTN per tensor."""
    shapes = [(1, 16, 0), (3, 48, 8), (129, 80, 0), (300, 256, 16), (70, 2048, 0), (17, 176, 24)]
    ws, jobs, amaxes = [], [], []
    n = len(shapes)
    am = torch.zeros(n, device=G.DEV)
    s2 = torch.zeros(n, device=G.DEV)
    for i, (rows, cols, pad) in enumerate(shapes):
        r = np.random.default_rng(77 + i)
        w = (r.standard_normal((rows, cols + pad)) * float(10.0 ** r.uniform(-3, 1))).astype(np.float32)
        w[:, :cols] *= np.repeat(r.random((rows, cols // 16)) >= 0.1, 16, axis=1)   # zero blocks
        if not fp32:
            w = inputs.f32_to_bf16_bits(w)
        wd = (G.f32_dev(w) if fp32 else G.bf16_dev(w))[:, :cols]
        w = np.ascontiguousarray(w[:, :cols])
        a = float(orc.tensor_amax(w)[0]) * (0.5 if i == 4 else 1.0)
        am[i] = a
        ws.append(w)
        amaxes.append(a)
        jobs.append(dict(w=wd, d_amax=am[i:i + 1], d_s2=s2[i:i + 1],
                         q=torch.empty((rows, cols // 2), dtype=torch.uint8, device=G.DEV),
                         scales=torch.empty((rows, cols // 16), dtype=torch.uint8, device=G.DEV)))
    f = G.flags_dev()
    nv4.nv4_weight_quant_rtn_batched(jobs, f)
    torch.cuda.synchronize()
    rflags = 0
    for i, (w, a, j) in enumerate(zip(ws, amaxes, jobs)):
        rq, rsc, rs2, rf = orc.rtn_quant(w, a)
        rflags |= rf
        assert s2[i].item() == rs2, i
        assert np.array_equal(G.host(j["scales"]), rsc), i
        assert np.array_equal(G.host(j["q"]), rq), i
    assert f.item() == rflags


# ------------------------------------------------------------------ fused fake quantize-dequantize
def _qdq_check(orc, x, amax=None, ld_pad=0, out_pad=0):
    rows, cols = x.shape
    xd = G.bf16_dev(np.pad(x, ((0, 0), (0, ld_pad))))[:, :cols]
    if amax is None:
        amax = orc.tensor_amax(x)[0]
    d_amax = torch.tensor([amax], dtype=torch.float32, device=G.DEV)
    for dt, name in ((torch.bfloat16, "bf16"), (torch.float16, "fp16"), (torch.float32, "fp32")):
        out = torch.full((rows, cols + out_pad), 7.0, dtype=dt, device=G.DEV)[:, :cols]
        s2 = torch.empty(1, dtype=torch.float32, device=G.DEV)
        f = G.flags_dev()
        nv4.nv4_fake_qdq(xd, d_amax, out, s2, f)
        ref, rs2, rf = orc.fake_qdq(x, amax, name)
        torch.cuda.synchronize()
        got = G.host(out.contiguous())
        if name == "fp32":
            got, ref = got.view(np.uint32), ref.view(np.uint32)
        assert s2.item() == rs2 and f.item() == rf
        assert np.array_equal(got, ref), name
        if out_pad:                                   # the padding columns are untouched
            assert (G.host(out.as_strided((rows, out_pad), (cols + out_pad, 1), cols).float()) == 7.0).all()


@pytest.mark.parametrize("rows,cols,pad", [(1, 16, 0), (3, 48, 8), (129, 80, 0), (300, 256, 16)])
def test_fake_qdq_small_ragged(orc, rows, cols, pad):
    x = inputs.laplace_bf16(inputs.rng_for(rows * cols, "gpu", "qdq"), rows, cols, outlier_channels=(1,),
                            outlier_scale=50, zero_block_frac=0.05)
    _qdq_check(orc, x, ld_pad=pad, out_pad=pad)


def test_fake_qdq_edge_values_and_in_place(orc):
    g = [0.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, -0.0, -0.25, -0.75, -5.0, 1e-30, -1e-30]
    x = inputs.f32_to_bf16_bits(np.array([g, [v * 0.5 for v in g], [448.0 * 6] + [0.0] * 15, [-0.0] * 16],
                                         np.float32))
    for amax in (2688.0, 0.0, 1.0):
        _qdq_check(orc, x, amax=amax)
    # in place, BF16 over the input
    y = inputs.c2_shape(256, 2048)
    yd = G.bf16_dev(y)
    d_amax = nv4.tensor_amax(yd)
    s2 = torch.empty(1, dtype=torch.float32, device=G.DEV)
    nv4.nv4_fake_qdq(yd, d_amax, yd, s2)
    ref, _, _ = orc.fake_qdq(y, orc.tensor_amax(y)[0], "bf16")
    assert np.array_equal(G.host(yd), ref)


@pytest.mark.parametrize("T,C", [(16, 2048), (4096, 4096), (65536, 7168)])
def test_fake_qdq_config_shapes(orc, T, C):
    """Against the oracle (sampled rows at the largest size) and against the separate
    act-quant + dequant kernels (whole tensor, bit for bit)."""
    x = inputs.c2_shape(T, C)
    xd = G.bf16_dev(x)
    d_amax = nv4.tensor_amax(xd)
    out, s2 = nv4.fake_qdq(xd, d_amax)
    q, sc, s2b = nv4.act_quant(xd, d_amax)
    two = nv4.dequant(q, sc, s2b)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), two.view(torch.int16))
    rows = np.arange(T) if T <= 4096 else np.sort(np.random.default_rng(T).choice(T, 256, replace=False))
    xs = np.ascontiguousarray(x[rows])
    q_r, sc_r, s2_r, _ = orc.act_quant(xs, orc.tensor_amax(x)[0])
    ref = orc.dequant(q_r, sc_r, s2_r, "bf16")
    assert np.array_equal(G.host(out)[rows], ref)


# ------------------------------------------------------------------ Hessian
def _hess_check(orc, x_bits, ld_pad=0, tol=1e-5):
    T, K = x_bits.shape
    xs = x_bits
    if ld_pad:
        xs = np.zeros((T, K + ld_pad), np.uint16)
        xs[:, :K] = x_bits
    xd = G.bf16_dev(xs)[:, :K]
    f = G.flags_dev()
    H = nv4.hessian_accum(xd, d_flags=f)
    ref = orc.hessian_accum(x_bits)
    Hg = G.host(H).reshape(ref.shape)
    assert f.item() == 0
    rel = G.hessian_rel_err(Hg, ref)
    blk = max(G.hessian_rel_err(Hg[b], ref[b]) for b in range(ref.shape[0]))
    print(f"H {T}x{K}: rel Frobenius {rel:.2e}, worst block {blk:.2e}")
    assert rel <= tol
    return H, ref


@pytest.mark.parametrize("T,K,pad", [(1, 16, 0), (63, 48, 8), (64, 64, 0), (1000, 80, 0), (4097, 272, 8)])
def test_hessian_small_ragged(orc, T, K, pad):
    x = inputs.laplace_bf16(inputs.rng_for(T * K, "gpu", "H"), T, K, outlier_channels=(2,), outlier_scale=30)
    _hess_check(orc, x, ld_pad=pad)


def test_hessian_accumulates_and_is_deterministic(orc):
    x = inputs.c1_tiny_linear(0)["X"]
    xd = G.bf16_dev(x)
    H1 = nv4.hessian_accum(xd)
    H2 = nv4.hessian_accum(xd)
    assert torch.equal(H1, H2)                      # bit-reproducible
    nv4.hessian_accum(xd, H1)                       # += semantics
    ref = orc.hessian_accum(x)
    assert G.hessian_rel_err(G.host(H1).reshape(ref.shape), 2 * ref) <= 1e-5


def test_hessian_gemma_layer_full(orc):
    d = inputs.c3_layer(0, which=("X",))
    _hess_check(orc, d["X"])


def test_hessian_gemma_down_full(orc):
    d = inputs.c3_layer(0, which=("X_down",))
    _hess_check(orc, d["X_down"])


def test_hessian_moe_batched(orc):
    xs, Hs, refs = [], [], []
    for e in range(64):
        d = inputs.c4_expert(e, which=("X", "X_down"))
        for name in ("X", "X_down"):
            xs.append(G.bf16_dev(d[name]))
            Hs.append(torch.zeros((d[name].shape[1] // 16, 16, 16), dtype=torch.float32, device=G.DEV))
            if e in (0, 31, 63):
                refs.append((len(xs) - 1, d[name]))
    f = G.flags_dev()
    nv4.nv4_hessian_accum_batched(xs, Hs, f)
    torch.cuda.synchronize()
    assert f.item() == 0
    for i, xb in refs:
        ref = orc.hessian_accum(xb)
        assert G.hessian_rel_err(G.host(Hs[i]).reshape(ref.shape), ref) <= 1e-5


# ------------------------------------------------------------------ sweep
def _sweep_check(orc, w, H64, rows_sample=None):
    """w: float32 or uint16 (bf16 bits) host array; H64: float64 oracle Hessian."""
    H32 = H64.astype(np.float32)
    Hin = H32.astype(np.float64)                    # both sides consume the same FP32 H
    wd = G.f32_dev(w) if w.dtype == np.float32 else G.bf16_dev(w)
    d_amax = nv4.tensor_amax(wd)
    amax = orc.tensor_amax(w)[0]
    assert d_amax.item() == amax
    f = G.flags_dev()
    codes, q, c1, c2 = nv4.scale_sweep(wd, G.f32_dev(H32), d_amax, d_flags=f)
    # without the runner-up output the bounds prune against the best cost: the same
    # winners and nibbles, bit for bit
    codes_only, q_only, _, _ = nv4.scale_sweep(wd, G.f32_dev(H32), d_amax, with_costs=False, d_flags=f)
    torch.cuda.synchronize()
    assert f.item() == 0
    assert torch.equal(codes_only, codes) and torch.equal(q_only, q)
    ref = orc.scale_sweep(w, Hin, amax, rows=rows_sample)
    idx = ref["rows"]
    stats = G.sweep_parity(G.host(codes)[idx], G.host(q)[idx], G.host(c1)[idx], ref, c2_gpu=G.host(c2)[idx])
    print("sweep", w.shape, stats)
    assert stats["mismatch_frac"] < 1e-3
    return stats


def test_sweep_tiny_config(orc):
    d = inputs.c1_tiny_linear(0)
    _sweep_check(orc, d["W"], orc.hessian_accum(d["X"]))


@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 48), (129, 80), (300, 256)])
def test_sweep_small_ragged(orc, rows, cols):
    r = np.random.default_rng(rows * cols)
    w = (r.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    x = inputs.laplace_bf16(inputs.rng_for(cols, "gpu", "sweepX"), 200, cols, outlier_channels=(1,), outlier_scale=20)
    H = orc.hessian_accum(x)
    _sweep_check(orc, w, H)
    _sweep_check(orc, inputs.f32_to_bf16_bits(w), H)


@pytest.mark.parametrize("fp32", [False, True])
def test_sweep_multi_tile_ctas(orc, fp32):
    """Enough row tiles that each CTA takes several tiles of 128 rows (at most 4 for BF16
    weights, 3 for FP32), with a ragged last group and a ragged last tile: the rows on every
    tile boundary and every row of the last 400 (the whole last group) equal the oracle's."""
    rows, cols = 3900, 4096                           # 31 row tiles, the last of 60 rows
    tiles = -(-rows // 128) * (cols // 16)
    per = min(tiles // (torch.cuda.get_device_properties(0).multi_processor_count * 16), 3 if fp32 else 4)
    assert per >= 3 and -(-rows // 128) % per != 0   # several tiles per CTA, a short last group
    r = np.random.default_rng(91 + fp32)
    w = (r.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    w[:: 37, int(r.integers(0, cols))] *= 25.0
    if not fp32:
        w = inputs.f32_to_bf16_bits(w)
    x = inputs.laplace_bf16(inputs.rng_for(93, "gpu", "sweepmt"), 384, cols, outlier_channels=(5, 700), outlier_scale=20)
    H = orc.hessian_accum(x)
    edges = [k * 128 + d for k in range(1, rows // 128 + 1) for d in (-1, 0)]
    sample = sorted(set(e for e in edges if e < rows) | set(range(rows - 400, rows)) | {0})
    _sweep_check(orc, w, H, rows_sample=sample)


def test_sweep_degenerate_blocks(orc):
    w = np.zeros((4, 32), np.float32)
    w[1, :16] = 0.5
    w[2, 16:] = np.array([0, .5, 1, 1.5, 2, 3, 4, 6] * 2, np.float32) * np.float32(0.25)
    w[3, 16:] = -0.0
    H = np.stack([np.eye(16), np.zeros((16, 16))])
    _sweep_check(orc, w, H)


def _bound_regime_hessians(rng, tokens=4096, corr_noise=1.0):
    """Six block columns that exercise every branch of the sweep's lower bounds."""
    cols = 96
    x = rng.laplace(size=(tokens, cols))
    x[:, 16:32] = x[:, 16:17] + corr_noise * rng.standard_normal((tokens, 16))   # correlated: bound off
    x[:, 32:48:3] = 0.0                                                     # dead channels: zero rows
    x[:, 80] *= 1000.0                                                      # one huge channel
    xb = inputs.f32_to_bf16_bits(x.astype(np.float32))
    H = np.asarray(inputs.bf16_bits_to_f32(xb), np.float64)
    H = np.einsum("tbi,tbj->bij", H.reshape(tokens, 6, 16), H.reshape(tokens, 6, 16))
    A = rng.standard_normal((16, 16))
    H[3] = (A + A.T) * tokens / 4.0                                         # indefinite: costs can be negative
    H[4] = H[0] + np.triu(rng.standard_normal((16, 16)), 1) * tokens / 50.0  # not symmetric
    return H


def _bound_regime_weights(rng, rows=300, cols=96):
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    w[::7, 5] *= 60.0                                 # one outlier per block: clipping can win
    w[1::11, 48:64] = 0.0                             # all-zero blocks
    w[2::11, 48:64] = -0.0
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -6, -4, -3, -2, -1.5, -1, -.5, -0.0], np.float32)
    w[3::13, 64:80] = grid * np.float32(0.01)         # blocks exact at some scale: cost 0
    w[4::13, 0:16] = np.float32(1e-12)                # far below the smallest candidate scale
    return w


def test_sweep_bound_regimes(orc):
    rng = np.random.default_rng(77)
    H = _bound_regime_hessians(rng)
    w = _bound_regime_weights(rng)
    _sweep_check(orc, w, H)
    _sweep_check(orc, inputs.f32_to_bf16_bits(w), H)


def test_sweep_ill_conditioned_hessian(orc):
    """A near rank-one H_b (channels equal up to 1e-3 noise, rho far below 0): FP32 costs
    could err by ~1e-3 relative here, so such a column is searched with FP64 costs.  The
    plain parity rule holds on every column: codes exact outside near ties of 1e-5."""
    rng = np.random.default_rng(79)
    H = _bound_regime_hessians(rng, corr_noise=1e-3)
    w = _bound_regime_weights(rng)
    _sweep_check(orc, w, H)
    _sweep_check(orc, inputs.f32_to_bf16_bits(w), H)


def _gershgorin_hessians(rng, rhos, tokens=8192):
    """Block columns H_b = D^1/2 (I + (1 - rho) S) D^1/2 with S symmetric, zero on the
    diagonal, random signs and largest absolute row sum exactly 1: the sweep's
    Gershgorin bound of H_b is rho (up to FP32 rounding of H_b), and H_b is positive
    definite.  Channel variances D spread over two binades, scaled by the token count
    as a sum of X^T X would be."""
    blocks = []
    for rho in rhos:
        S = rng.standard_normal((16, 16)) * rng.uniform(0.2, 1.0, (16, 16))
        S = np.triu(S, 1)
        S = S + S.T
        S /= np.abs(S).sum(1).max()
        d = tokens * 4.0 ** rng.uniform(-1, 1, 16)
        blocks.append(np.sqrt(d)[:, None] * (np.eye(16) + (1.0 - rho) * S) * np.sqrt(d)[None, :])
    return np.stack(blocks)


def test_sweep_small_positive_rho(orc):
    """Columns with rho between 0.05 and 0.55: the bounds stay on, but FP32 costs are
    exact only to ~1.7e-6 (2 - rho) / rho, more than the 1e-5 near-tie tolerance allows
    below rho ~ 0.6.  Blocks whose FP32 runner-up is that close to the winner (and every
    block when the costs are outputs) are searched again in FP64; the plain parity rule
    holds on every column, in both modes (codes + nibbles alone, and with the costs).
    At rho = 0.02 (below 1/32) Gershgorin alone would switch the bounds off; the certified
    lambda_min keeps them on, with FP32 costs whose error bound is not certified, so near
    ties and exact FP32 ties between two codes go to the FP64 search."""
    rng = np.random.default_rng(81)
    H = _gershgorin_hessians(rng, [0.02, 0.05, 0.1, 0.3, 0.55, 0.9])
    w = (rng.standard_normal((2048, 96)) * 0.02).astype(np.float32)
    w[::5, 7] *= 40.0
    st = _sweep_check(orc, w, H)
    _sweep_check(orc, inputs.f32_to_bf16_bits(w), H)
    print("small rho", st)


def _eigen_hessians(rng, lmins, tokens=8192):
    """Block columns whose diagonally scaled matrix has about a given smallest eigenvalue:
    M = Q diag(lambda) Q^T with a random orthogonal Q, lambda_min given and the rest in
    [lambda_min, 2 - lambda_min], rescaled to a unit diagonal (which keeps M positive
    definite but moves its eigenvalues, so lambda_min is measured, not assumed), then
    H_b = S M S with channel scales S over two binades."""
    blocks, lams = [], []
    for lm in lmins:
        q, _ = np.linalg.qr(rng.standard_normal((16, 16)))
        lam = np.concatenate([[lm], rng.uniform(lm, 2.0 - lm, 15)])
        m = (q * lam) @ q.T
        dm = 1.0 / np.sqrt(np.diag(m))
        m = dm[:, None] * m * dm[None, :]
        s = np.sqrt(tokens * 4.0 ** rng.uniform(-1, 1, 16))
        blocks.append(s[:, None] * m * s[None, :])
        lams.append(np.linalg.eigvalsh(m)[0])
    return np.stack(blocks), np.array(lams)


def test_sweep_certified_lambda_min(orc):
    """Block columns with lambda_min of the scaled H_b from ~0.03 to ~0.95 and Gershgorin
    ratios below it (half of them negative): the bounds run on the Cholesky-certified
    lambda_min.  A certificate above the true lambda_min would let the bounds prune
    winners; the plain parity rule and the agreement of both modes, on FP32 and BF16
    weights with outlier elements, show that none was lost."""
    rng = np.random.default_rng(83)
    H, lams = _eigen_hessians(rng, [0.03, 0.06, 0.12, 0.25, 0.5, 0.7, 0.85, 0.95])
    dm = 1.0 / np.sqrt(np.einsum("bii->bi", H))
    M = dm[:, :, None] * H * dm[:, None, :]
    rho = 1.0 - (np.abs(M).sum(2) - 1.0).max(1)
    assert (rho < lams).all() and (rho < 0).sum() >= 4 and lams.min() < 0.05 and lams.max() > 0.9, (rho, lams)
    w = (rng.standard_normal((1024, 128)) * 0.02).astype(np.float32)
    w[::7, 3] *= 30.0
    w[1::11, 77] *= 60.0
    st = _sweep_check(orc, w, H)
    st_b = _sweep_check(orc, inputs.f32_to_bf16_bits(w), H)
    print("certified lambda_min", lams.round(3), "rho", rho.round(2), st, st_b)


def test_sweep_c1_chain_on_device(orc):
    """The tiny Linear's calibration chain with every step on the GPU -- weight amax,
    local Hessian of the activations, sweep with pack ([CAL] section 2 steps 1-3) --
    against the oracle's chain on its FP64 Hessian, under the sweep parity rule."""
    d = inputs.c1_tiny_linear(0)
    X, W = G.bf16_dev(d["X"]), G.f32_dev(d["W"])
    f = G.flags_dev()
    aw = nv4.tensor_amax(W, d_flags=f)
    H = nv4.hessian_accum(X, d_flags=f)
    codes, q, c1, c2 = nv4.scale_sweep(W, H, aw, d_flags=f)
    codes_only, q_only, _, _ = nv4.scale_sweep(W, H, aw, with_costs=False, d_flags=f)
    torch.cuda.synchronize()
    assert f.item() == 0
    assert torch.equal(codes_only, codes) and torch.equal(q_only, q)
    amax_w = orc.tensor_amax(d["W"])[0]
    assert aw.item() == amax_w
    H64 = orc.hessian_accum(d["X"])
    assert G.hessian_rel_err(G.host(H), H64) <= 1e-5
    ref = orc.scale_sweep(d["W"], H64, amax_w)
    st = G.sweep_parity(G.host(codes), G.host(q), G.host(c1), ref, c2_gpu=G.host(c2))
    print("c1 chain", st)
    assert st["mismatch_frac"] < 1e-3


def test_sweep_grouped_scale2(orc):
    """Two matrices sharing one scale_2 (w1/w3 style): both amaxes accumulate into one
    device float (the running-max contract of nv4_tensor_amax), so both sweeps use
    s2 = RN32(max(amax1, amax3) / 2688); the oracle gets that group amax."""
    rng = np.random.default_rng(80)
    x = inputs.laplace_bf16(inputs.rng_for(80, "gpu", "sweepg"), 512, 64)
    H = orc.hessian_accum(x).astype(np.float32)
    w1 = (rng.standard_normal((96, 64)) * 0.02).astype(np.float32)
    w3 = (rng.standard_normal((96, 64)) * 0.05).astype(np.float32)
    d_amax = torch.zeros(1, dtype=torch.float32, device=G.DEV)
    jobs = []
    for w in (w1, w3):
        wd = G.f32_dev(w)
        nv4.nv4_tensor_amax(wd, d_amax)
        jobs.append(dict(w=wd, H=G.f32_dev(H), d_amax_w=d_amax,
                         codes=torch.empty((96, 4), dtype=torch.uint8, device=G.DEV),
                         q=torch.empty((96, 32), dtype=torch.uint8, device=G.DEV),
                         cost1=torch.empty((96, 4), dtype=torch.float32, device=G.DEV),
                         cost2=torch.empty((96, 4), dtype=torch.float32, device=G.DEV)))
    nv4.nv4_scale_sweep_batched(jobs)
    torch.cuda.synchronize()
    amax = max(orc.tensor_amax(w1)[0], orc.tensor_amax(w3)[0])
    assert d_amax.item() == amax
    for w, j in zip((w1, w3), jobs):
        ref = orc.scale_sweep(w, H.astype(np.float64), amax)
        st = G.sweep_parity(G.host(j["codes"]), G.host(j["q"]), G.host(j["cost1"]), ref, c2_gpu=G.host(j["cost2"]))
        assert st["mismatch_frac"] < 1e-3


def test_sweep_work_counter(orc):
    """Bounds on: far fewer than 127 costs per block, both for independent channels and
    for correlated ones (Gershgorin's rho < 0, but lambda_min of the scaled H_b well above
    1/32, which the Cholesky certificate proves); bounds off (a duplicated channel: H_b
    singular): every candidate visited (both halves) and evaluated.  The winners match the
    oracle either way."""
    rng = np.random.default_rng(78)
    x = rng.laplace(size=(2048, 48))
    x[:, 16:48] = x[:, 16:17] + rng.standard_normal((2048, 32))     # correlated channels
    x[:, 33] = x[:, 32]                                              # H_2 singular
    xb = inputs.f32_to_bf16_bits(x.astype(np.float32))
    H = orc.hessian_accum(xb)
    for b in range(3):                                               # what the three columns exercise
        Hs = H[b].astype(np.float32).astype(np.float64)
        dm = 1.0 / np.sqrt(np.diag(Hs))
        M = dm[:, None] * Hs * dm[None, :]
        rho = 1.0 - (np.abs(M).sum(1) - 1.0).max()
        lmin = np.linalg.eigvalsh(M)[0]
        assert (rho > 0.1, rho < 0 and lmin > 0.1, rho < 0 and abs(lmin) < 1e-6)[b], (b, rho, lmin)
    w = (rng.standard_normal((256, 48)) * 0.02).astype(np.float32)
    wd = G.f32_dev(w)
    rows, cols = w.shape
    work = []
    jobs = []
    for b in range(3):
        wb = wd[:, 16 * b:16 * b + 16].contiguous()
        Hb = G.f32_dev(H[b:b + 1].astype(np.float32))
        work.append(torch.zeros(2, dtype=torch.int64, device=G.DEV))
        jobs.append(dict(w=wb, H=Hb, d_amax_w=nv4.tensor_amax(wd),
                         codes=torch.empty((rows, 1), dtype=torch.uint8, device=G.DEV),
                         q=torch.empty((rows, 8), dtype=torch.uint8, device=G.DEV),
                         cost1=torch.empty((rows, 1), dtype=torch.float32, device=G.DEV),
                         cost2=torch.empty((rows, 1), dtype=torch.float32, device=G.DEV), d_work=work[-1]))
    f = G.flags_dev()
    nv4.nv4_scale_sweep_batched(jobs, f)
    torch.cuda.synchronize()
    assert f.item() == 0
    # codes only (no runner-up): pruning against the best cost, fewer costs, same winners
    lean = [torch.zeros(2, dtype=torch.int64, device=G.DEV) for _ in range(2)]
    for b in range(2):
        jb = dict(jobs[b], cost1=None, cost2=None, d_work=lean[b],
                  codes=torch.empty_like(jobs[b]["codes"]), q=torch.empty_like(jobs[b]["q"]))
        nv4.nv4_scale_sweep_batched([jb], f)
        torch.cuda.synchronize()
        assert torch.equal(jb["codes"], jobs[b]["codes"]) and torch.equal(jb["q"], jobs[b]["q"])
    on, corr, off = (w_.cpu().numpy() for w_ in work)
    ln, ln_corr = (w_.cpu().numpy() for w_ in lean)
    print("work with bounds", on, "correlated", corr, "without", off, "codes only", ln, ln_corr)
    assert ln[1] <= on[1] and ln[0] <= on[0]
    # bounds off: both halves of every candidate and every cost; on: a candidate's second
    # half only when its first half leaves it open, a cost only when its whole bound does.
    # The correlated column's FP32 costs are not certified (eta_b > 4e-6): with the costs
    # as outputs every block is searched in FP64; for codes alone the walk prunes, and
    # only near ties go to FP64.
    assert off[0] == 2 * 127 * rows and off[1] == 127 * rows
    assert corr[0] == 2 * 127 * rows and corr[1] == 127 * rows
    for v in (on, ln_corr):
        assert v[1] <= v[0] / 2 <= v[0] <= 2 * 127 * rows and v[1] < 0.25 * 127 * rows
    ref = orc.scale_sweep(w, H.astype(np.float32).astype(np.float64), orc.tensor_amax(w)[0])
    cat = lambda k: np.concatenate([G.host(j[k]) for j in jobs], axis=1)
    st = G.sweep_parity(cat("codes"), cat("q"), cat("cost1"), ref, c2_gpu=cat("cost2"))
    assert st["mismatch_frac"] < 1e-3


def test_sweep_gemma_layer_sampled(orc):
    d = inputs.c3_layer(0)
    H = orc.hessian_accum(d["X"])
    Hd = orc.hessian_accum(d["X_down"])
    rng = np.random.default_rng(5)
    for name, HH in (("W_q", H), ("W_gate", H), ("W_up", H), ("W_down", Hd)):
        w = d[name]
        rows = np.sort(rng.choice(w.shape[0], 48, replace=False))
        _sweep_check(orc, w, HH, rows_sample=rows)


def test_sweep_moe_batched_sampled(orc):
    jobs, checks = [], []
    rng = np.random.default_rng(6)
    for e in range(64):
        d = inputs.c4_expert(e)
        Hx = orc.hessian_accum(d["X"]) if e in (0, 40) else None
        Hxd = orc.hessian_accum(d["X_down"]) if e in (0, 40) else None
        for name, HX in (("W_gate", Hx), ("W_up", Hx), ("W_down", Hxd)):
            w = d[name]
            H32 = (HX if HX is not None else np.broadcast_to(np.eye(16), (w.shape[1] // 16, 16, 16))).astype(np.float32)
            wd = G.bf16_dev(w)
            amax = nv4.tensor_amax(wd)
            rows, cols = w.shape
            job = dict(w=wd, H=G.f32_dev(H32), d_amax_w=amax,
                       codes=torch.empty((rows, cols // 16), dtype=torch.uint8, device=G.DEV),
                       q=torch.empty((rows, cols // 2), dtype=torch.uint8, device=G.DEV),
                       cost1=torch.empty((rows, cols // 16), dtype=torch.float32, device=G.DEV),
                       cost2=torch.empty((rows, cols // 16), dtype=torch.float32, device=G.DEV))
            jobs.append(job)
            if HX is not None:
                checks.append((job, w, H32.astype(np.float64)))
    f = G.flags_dev()
    nv4.nv4_scale_sweep_batched(jobs, f)
    torch.cuda.synchronize()
    assert f.item() == 0
    for job, w, Hin in checks:
        rows = np.sort(rng.choice(w.shape[0], 24, replace=False))
        ref = orc.scale_sweep(w, Hin, orc.tensor_amax(w)[0], rows=rows)
        st = G.sweep_parity(G.host(job["codes"])[rows], G.host(job["q"])[rows], G.host(job["cost1"])[rows], ref,
                            c2_gpu=G.host(job["cost2"])[rows])
        assert st["mismatch_frac"] < 1e-3


# ------------------------------------------------------------------ cast
def _cast_check(orc, mats, in_place=False, groups=None):
    jobs, refs = [], []
    counts = torch.zeros(3, dtype=torch.int64, device=G.DEV)
    f = G.flags_dev()
    groups = [-1] * len(mats) if groups is None else groups
    for (mxq, e8), g in zip(mats, groups):
        mq = G.u8_dev(mxq)
        rows, half = mxq.shape
        jobs.append(dict(mx_q=mq, e8m0=G.u8_dev(e8), nv_q=mq if in_place else torch.empty_like(mq),
                         nv_scales=torch.empty((rows, half // 8), dtype=torch.uint8, device=G.DEV),
                         d_global_amax=torch.empty(1, dtype=torch.float32, device=G.DEV),
                         d_s2=torch.empty(1, dtype=torch.float32, device=G.DEV), group=g))
        if g < 0:
            refs.append(orc.mxfp4_to_nvfp4(mxq, e8))
        else:
            members = [i for i, h in enumerate(groups) if h == g]
            res = orc.mxfp4_to_nvfp4_group([mats[i] for i in members])
            refs.append(res[members.index(len(refs))])
    nv4.nv4_mxfp4_to_nvfp4_batched(jobs, counts, f)
    torch.cuda.synchronize()
    assert f.item() == 0
    tot = np.zeros(3, np.int64)
    for j, r in zip(jobs, refs):
        assert np.array_equal(G.host(j["nv_q"]), r["nv_q"])
        assert np.array_equal(G.host(j["nv_scales"]), r["nv_scales"])
        assert j["d_global_amax"].item() == r["global_amax"] and j["d_s2"].item() == r["s2"]
        tot += r["counts"]
    assert np.array_equal(counts.cpu().numpy(), tot)
    return tot


def test_cast_small_and_edges(orc):
    mats = [inputs.mxfp4_matrix(inputs.rng_for(i, "gpu", "cast"), r, c, fallback_frac=0.05)
            for i, (r, c) in enumerate([(1, 32), (3, 64), (17, 96), (64, 256)])]
    e = np.array([[127, 127 - 17, 127 - 18, 124]], np.uint8)
    mats.append((np.full((1, 64), 0x77, np.uint8), e))
    _cast_check(orc, mats)
    _cast_check(orc, mats, in_place=True)


def test_cast_chunk_tails(orc):
    """Matrices spanning several 2048-block chunks of the streaming kernel, with tails
    that are not whole 16-byte words of E8M0 codes or of scale bytes, fallback blocks
    in every chunk, and more jobs than fit one chunk each."""
    shapes = [(4099, 32), (2049, 64), (1, 2048 * 32), (3, 683 * 32), (129, 160), (2, 4096 * 32 + 32)]
    mats = [inputs.mxfp4_matrix(inputs.rng_for(i, "gpu", "castc"), r, c, fallback_frac=0.03)
            for i, (r, c) in enumerate(shapes)]
    tot = _cast_check(orc, mats)
    assert tot[1] > 0
    _cast_check(orc, mats, in_place=True)
    _cast_check(orc, mats, groups=[0, 1, 0, 1, 0, 1])


def test_cast_extreme_exponents(orc):
    """Fallback blocks under scale_2 values far from 1: tiny exponents (s2 below 2^-100,
    where the block-scale encoder takes its exact path) and large ones (s2 above
    2^100, block scales near the top of FP32)."""
    mats = [inputs.mxfp4_matrix(inputs.rng_for(i, "gpu", "castx"), 64, 256, mean_exp=m, fallback_frac=0.05)
            for i, m in enumerate((-110.0, -100.0, 100.0, 112.0))]
    tot = _cast_check(orc, mats)
    assert tot[1] > 0


def test_cast_grouped_scale2(orc):
    """Matrices sharing one scale_2: the window-edge example, random pairs whose members
    sit apart in the job list, singletons and one-member groups in the same call."""
    win = 17
    a = (np.full((1, 64), 0x77, np.uint8), np.array([[127, 120, 127, 110]], np.uint8))
    b = (np.full((1, 64), 0x35, np.uint8), np.array([[127 - win, 126 - win, 126 - win, 113]], np.uint8))
    rnd = [inputs.mxfp4_matrix(inputs.rng_for(i, "gpu", "castg"), r, c, fallback_frac=0.02, mean_exp=-8.0 - 3 * (i % 2))
           for i, (r, c) in enumerate([(3, 64), (17, 96), (64, 256), (64, 256), (5, 32)])]
    mats = [a, rnd[0], b, rnd[1], rnd[2], rnd[3], rnd[4]]
    groups = [7, 3, 7, -1, 3, 9, 11]
    tot = _cast_check(orc, mats, groups=groups)
    assert tot[1] > 0
    _cast_check(orc, mats, in_place=True, groups=groups)


def test_cast_expert_checkpoint_grouped_pairs(orc):
    mats = [inputs.c5_cast(i) for i in range(32)]
    _cast_check(orc, mats, groups=[i // 2 for i in range(32)])


def test_cast_expert_checkpoint_full(orc):
    mats = [inputs.c5_cast(i) for i in range(32)]
    tot = _cast_check(orc, mats)
    print("cast counts (in-window, fallback, lossless):", tot.tolist(), "lossless fraction", tot[2] / (tot[0] + tot[1]))
    _cast_check(orc, mats, in_place=True)


# ------------------------------------------------------------------ failure detection
def test_bounded_wait_gives_up_and_reports():
    """The bounded-wait path, without any fault: a flag nothing sets makes the wait run
    out (status NV4_FLAG_TIMEOUT after about the limit) and the device stays usable; a
    set flag ends the wait at once."""
    flag = torch.zeros(1, dtype=torch.int32, device=G.DEV)
    status = torch.full((2,), -1, dtype=torch.int32, device=G.DEV)
    nv4.nv4_selftest_wait(flag, 20_000_000, status)            # 20 ms
    torch.cuda.synchronize()
    st = status.cpu().tolist()
    assert st[0] == nv4.FLAG_TIMEOUT and 19_000 <= st[1] <= 2_000_000, st
    flag.fill_(1)
    nv4.nv4_selftest_wait(flag, 20_000_000, status)
    torch.cuda.synchronize()
    st = status.cpu().tolist()
    assert st[0] == 0 and st[1] < 10_000, st
    # the context still works afterwards
    x = torch.ones(4, 16, dtype=torch.bfloat16, device=G.DEV)
    assert nv4.tensor_amax(x).item() == 1.0
