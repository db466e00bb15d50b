"""Seeded randomized parity: many small random shapes, strides and value ranges through
the GPU entry points (single and batched) against the oracle, bit for bit.  Each case's
generator is seeded from its index, so a failure names a reproducible case."""
import numpy as np
import pytest
import torch

import gpu_util as G
from nvfp4_block_numerics_b200 import binding as nv4
from nvfp4_block_numerics_b200 import inputs

pytestmark = pytest.mark.gpu


def _random_act_tensor(r: np.random.Generator):
    """BF16 bits [rows, cols]: Laplace values at a random binade (1e-30 .. 1e30), with
    zero blocks, sign flips and values exactly on E2M1 rounding boundaries of a random
    block scale."""
    rows = int(r.integers(1, 70))
    cols = 16 * int(r.integers(1, 40))
    scale = float(10.0 ** r.uniform(-30, 30))
    x = (r.laplace(size=(rows, cols)) * scale).astype(np.float32)
    nb = rows * cols // 16
    blocks = x.reshape(nb, 16)
    blocks[r.random(nb) < 0.05] = 0.0                               # all-zero blocks
    S = np.float32(scale)
    mids = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]) * S    # ties at a block scale S
    pick = r.random(x.shape) < 0.02
    x[pick] = r.choice(mids, size=int(pick.sum())) * r.choice([-1, 1], size=int(pick.sum()))
    return inputs.f32_to_bf16_bits(x)


@pytest.mark.parametrize("batch", range(8))
def test_fuzz_act_path(orc, batch):
    cases = []
    for k in range(12):
        r = np.random.default_rng(1000 * batch + k)
        x = _random_act_tensor(r)
        rows, cols = x.shape
        pad = int(r.choice([0, 8, 24]))
        buf = np.zeros((rows, cols + pad), np.uint16)
        buf[:, :cols] = x
        xd = G.bf16_dev(buf)[:, :cols]
        static = r.random() < 0.3                                  # a calibrated amax instead of the data's
        amax = float(np.abs((x.astype(np.uint32) << 16).view(np.float32)).max()) * float(r.uniform(0.3, 3.0)) \
            if static else None
        cases.append((x, xd, amax))
    n = len(cases)
    f = G.flags_dev()
    am = torch.zeros(n, device=G.DEV)
    s2 = torch.zeros(n, device=G.DEV)
    for i, (x, xd, amax) in enumerate(cases):
        if amax is not None:
            am[i] = amax
    dyn = [i for i, c in enumerate(cases) if c[2] is None]
    nv4.nv4_tensor_amax_batched([cases[i][1].contiguous() for i in dyn], [am[i:i + 1] for i in dyn], f)
    q = [torch.empty((c[0].shape[0], c[0].shape[1] // 2), dtype=torch.uint8, device=G.DEV) for c in cases]
    sc = [torch.empty((c[0].shape[0], c[0].shape[1] // 16), dtype=torch.uint8, device=G.DEV) for c in cases]
    out = [torch.empty(tuple(c[0].shape), dtype=torch.float32, device=G.DEV) for c in cases]
    nv4.nv4_act_quant_batched([dict(x=c[1], d_amax=am[i:i + 1], q=q[i], scales=sc[i], d_s2=s2[i:i + 1])
                               for i, c in enumerate(cases)], f)
    nv4.nv4_dequant_batched([dict(q=q[i], scales=sc[i], d_s2=s2[i:i + 1], out=out[i]) for i in range(n)])
    torch.cuda.synchronize()
    assert f.item() == 0
    for i, (x, _, amax) in enumerate(cases):
        a = orc.tensor_amax(x)[0] if amax is None else np.float32(amax)
        assert am[i].item() == a, i
        oq, osc, os2, of = orc.act_quant(x, float(a))
        assert s2[i].item() == os2, i
        assert np.array_equal(G.host(sc[i]), osc), (i, np.argwhere(G.host(sc[i]) != osc)[:3])
        assert np.array_equal(G.host(q[i]), oq), (i, np.argwhere(G.host(q[i]) != oq)[:3])
        ref = orc.dequant(oq, osc, os2, "fp32")
        assert np.array_equal(G.host(out[i]).view(np.uint32), ref.view(np.uint32)), i


@pytest.mark.parametrize("batch", range(6))
def test_fuzz_cast(orc, batch):
    mats, groups = [], []
    for k in range(10):
        r = np.random.default_rng(5000 + 100 * batch + k)
        rows, cols = int(r.integers(1, 40)), 32 * int(r.integers(1, 20))
        mean = float(r.uniform(-120, 120))
        mats.append(inputs.mxfp4_matrix(r, rows, cols, mean_exp=mean, std_exp=float(r.uniform(0.5, 6)),
                                        fallback_frac=float(r.choice([0.0, 0.01, 0.2]))))
        groups.append(int(r.choice([-1, -1, 0, 1])))
    jobs, refs = [], []
    counts = torch.zeros(3, dtype=torch.int64, device=G.DEV)
    f = G.flags_dev()
    for (mxq, e8), g in zip(mats, groups):
        mq = G.u8_dev(mxq)
        jobs.append(dict(mx_q=mq, e8m0=G.u8_dev(e8), nv_q=torch.empty_like(mq),
                         nv_scales=torch.empty((mxq.shape[0], mxq.shape[1] // 8), dtype=torch.uint8, device=G.DEV),
                         d_global_amax=torch.empty(1, device=G.DEV), d_s2=torch.empty(1, device=G.DEV), group=g))
    for i, g in enumerate(groups):
        if g < 0:
            refs.append(orc.mxfp4_to_nvfp4(*mats[i]))
        else:
            members = [k for k, h in enumerate(groups) if h == g]
            refs.append(orc.mxfp4_to_nvfp4_group([mats[k] for k in members])[members.index(i)])
    nv4.nv4_mxfp4_to_nvfp4_batched(jobs, counts, f)
    torch.cuda.synchronize()
    tot = np.zeros(3, np.int64)
    for i, (j, ref) in enumerate(zip(jobs, refs)):
        assert np.array_equal(G.host(j["nv_q"]), ref["nv_q"]), i
        assert np.array_equal(G.host(j["nv_scales"]), ref["nv_scales"]), i
        assert j["d_s2"].item() == ref["s2"] and (j["d_global_amax"].item() == ref["global_amax"]
                                                 or not np.isfinite(ref["global_amax"])), i
        tot += ref["counts"]
    assert np.array_equal(counts.cpu().numpy(), tot)


@pytest.mark.parametrize("batch", range(6))
def test_fuzz_sweep(orc, batch):
    """Random small weights and calibration inputs (FP32 and BF16 weights, outlier
    channels, correlated channels, zero blocks): the codes follow the parity rule, the
    codes-only call agrees with the full call bit for bit."""
    for k in range(4):
        r = np.random.default_rng(9000 + 10 * batch + k)
        rows, cols = int(r.integers(1, 50)), 16 * int(r.integers(1, 6))
        x = r.laplace(size=(int(r.integers(16, 200)), cols))
        if r.random() < 0.5:
            x[:, :4] += x[:, 4:5] * float(r.uniform(0, 0.3))          # mildly correlated channels
        x[:, int(r.integers(0, cols))] *= float(r.uniform(1, 50))     # an outlier channel
        H = orc.hessian_accum(inputs.f32_to_bf16_bits(x.astype(np.float32)))
        w = (r.standard_normal((rows, cols)) * float(10.0 ** r.uniform(-3, 1))).astype(np.float32)
        w.reshape(-1, 16)[r.random(rows * cols // 16) < 0.1] = 0.0
        if r.random() < 0.5:
            w = inputs.f32_to_bf16_bits(w)
        H32 = H.astype(np.float32)
        wd = G.f32_dev(w) if w.dtype == np.float32 else G.bf16_dev(w)
        d_amax = nv4.tensor_amax(wd)
        fl = G.flags_dev()
        codes, q, c1, c2 = nv4.scale_sweep(wd, G.f32_dev(H32), d_amax, d_flags=fl)
        co, qo, _, _ = nv4.scale_sweep(wd, G.f32_dev(H32), d_amax, with_costs=False, d_flags=fl)
        torch.cuda.synchronize()
        assert fl.item() == 0
        assert torch.equal(co, codes) and torch.equal(qo, q)
        ref = orc.scale_sweep(w, H32.astype(np.float64), orc.tensor_amax(w)[0])
        st = G.sweep_parity(G.host(codes), G.host(q), G.host(c1), ref, c2_gpu=G.host(c2))
        assert st["near_tie_mismatches"] <= max(1, st["blocks"] // 1000), st


def _random_values(r: np.random.Generator, rows: int, cols: int):
    """FP32 values at a random binade (subnormal BF16 magnitudes included), with zero
    runs and sign flips; returned as FP32 or as BF16 bits."""
    x = (r.laplace(size=(rows, cols)) * float(10.0 ** r.uniform(-40, 35))).astype(np.float32)
    x[r.random(x.shape) < 0.03] = 0.0
    x[:, : int(r.integers(0, cols + 1))] *= np.float32(-1.0)
    return x if r.random() < 0.5 else inputs.f32_to_bf16_bits(x)


@pytest.mark.parametrize("batch", range(4))
def test_fuzz_formats(orc, batch):
    """MXFP4 and FP8 quantization and dequantization on random shapes, dtypes and
    binades, bit for bit against the oracle."""
    for k in range(6):
        r = np.random.default_rng(20000 + 10 * batch + k)
        rows = int(r.integers(1, 60))
        x = _random_values(r, rows, 32 * int(r.integers(1, 24)))
        xd = G.f32_dev(x) if x.dtype == np.float32 else G.bf16_dev(x)
        f = G.flags_dev()
        q, e8 = nv4.mxfp4_quant(xd, d_flags=f)
        rq, re8, rf = orc.mxfp4_quant(x)
        torch.cuda.synchronize()
        assert f.item() == rf and np.array_equal(G.host(e8), re8) and np.array_equal(G.host(q), rq), k
        out = torch.empty(tuple(x.shape), dtype=torch.float32, device=G.DEV)
        nv4.nv4_mxfp4_dequant(q, e8, out)
        ref = orc.mxfp4_dequant(rq, re8, "fp32")
        assert np.array_equal(G.host(out).view(np.uint32), ref.view(np.uint32)), k
        amax = float(orc.tensor_amax(x)[0]) * float(r.choice([1.0, 0.25, 4.0]))
        f = G.flags_dev()
        q8, s8 = nv4.fp8_quant(xd, torch.tensor([amax], dtype=torch.float32, device=G.DEV), d_flags=f)
        rq8, rs8, rf8 = orc.fp8_quant(x, float(np.float32(amax)))
        torch.cuda.synchronize()
        assert s8.item() == rs8 and f.item() == rf8 and np.array_equal(G.host(q8), rq8), k


@pytest.mark.parametrize("batch", range(3))
def test_fuzz_hadamard(orc, batch):
    """Block Hadamard rotation fused with MXFP4 and NVFP4 quantization on random shapes,
    block sizes and binades."""
    for k in range(4):
        r = np.random.default_rng(30000 + 10 * batch + k)
        n = int(r.choice([16, 32, 64, 128]))
        rows, cols = int(r.integers(1, 40)), 128 * int(r.integers(1, 6))
        x = inputs.f32_to_bf16_bits((r.laplace(size=(rows, cols)) * float(10.0 ** r.uniform(-20, 20)))
                                    .astype(np.float32))
        xd = G.bf16_dev(x)
        y = orc.hadamard_rotate(x, n)
        q, e8 = nv4.hadamard_mxfp4_quant(xd, n)
        rq, re8, _ = orc.mxfp4_quant(y)
        qn, scn, s2n, _ = nv4.hadamard_nvfp4_quant(xd, n)
        nq, nsc, ns2, _ = orc.rtn_quant(y, float(np.abs(y).max()))
        torch.cuda.synchronize()
        assert np.array_equal(G.host(e8), re8) and np.array_equal(G.host(q), rq), (k, n)
        assert s2n.item() == ns2 and np.array_equal(G.host(scn), nsc) and np.array_equal(G.host(qn), nq), (k, n)


@pytest.mark.parametrize("batch", range(3))
def test_fuzz_two_sided_hadamard(orc, batch):
    """Two-sided block Hadamard of weight tiles (n = 16, 32) fused with MXFP4 and NVFP4
    quantization on random shapes, dtypes, row pitches and binades: rotated values, codes
    and scales bit for bit."""
    for k in range(4):
        r = np.random.default_rng(40000 + 10 * batch + k)
        n = int(r.choice([16, 32]))
        rows, cols = n * int(r.integers(1, 8)), 32 * int(r.integers(1, 7))
        w = (r.standard_normal((rows, cols)) * float(10.0 ** r.uniform(-25, 25))).astype(np.float32)
        w[np.abs(w) < np.float32(1e-3) * np.abs(w).max()] = 0.0   # keeps every tile inside the FP64-exact span
        if r.random() < 0.5:
            w = inputs.f32_to_bf16_bits(w)
        pad = int(r.choice([0, 32]))
        dt = torch.float32 if w.dtype == np.float32 else torch.bfloat16
        full = torch.zeros((rows, cols + pad), dtype=dt, device=G.DEV)
        full[:, :cols] = G.f32_dev(w) if w.dtype == np.float32 else G.bf16_dev(w)
        wd = full[:, :cols]
        y = orc.hadamard2_rotate(w, n)
        got = nv4.hadamard2_rotate(wd, n)
        q, e8 = nv4.hadamard2_mxfp4_quant(wd, n)
        qn, scn, s2n, _ = nv4.hadamard2_nvfp4_quant(wd, n)
        torch.cuda.synchronize()
        assert np.array_equal(G.host(got).view(np.uint32), y.view(np.uint32)), (k, n)
        rq, re8, _ = orc.mxfp4_quant(y)
        assert np.array_equal(G.host(e8), re8) and np.array_equal(G.host(q), rq), (k, n)
        nq, nsc, ns2, _ = orc.rtn_quant(y, float(np.abs(y).max()))
        assert s2n.item() == ns2 and np.array_equal(G.host(scn), nsc) and np.array_equal(G.host(qn), nq), (k, n)


@pytest.mark.parametrize("batch", range(4))
def test_fuzz_sweep_conditioning(orc, batch):
    """Hessian columns of random conditioning: scaled Gershgorin ratio rho from -0.5 through
    0.95.  Whether the bounds are on is decided by the certified lambda_min (at least rho):
    columns without a bound go to the FP64 search, uncertified ones walk in FP32 with FP64
    re-searches of near and exact ties.  BF16 and FP32 weights; the plain parity rule, and
    the codes-only call equal to the full call."""
    r = np.random.default_rng(50000 + batch)
    rhos = r.uniform(-0.5, 0.95, 6)
    H = np.stack([_gershgorin_block(r, rho) for rho in rhos])
    w = (r.standard_normal((int(r.integers(40, 300)), 96)) * 0.02).astype(np.float32)
    w[:: int(r.integers(3, 9)), int(r.integers(0, 96))] *= 30.0
    if r.random() < 0.5:
        w = inputs.f32_to_bf16_bits(w)
    H32 = H.astype(np.float32)
    wd = G.f32_dev(w) if w.dtype == np.float32 else G.bf16_dev(w)
    d_amax = nv4.tensor_amax(wd)
    fl = G.flags_dev()
    codes, q, c1, c2 = nv4.scale_sweep(wd, G.f32_dev(H32), d_amax, d_flags=fl)
    co, qo, _, _ = nv4.scale_sweep(wd, G.f32_dev(H32), d_amax, with_costs=False, d_flags=fl)
    torch.cuda.synchronize()
    assert fl.item() == 0
    assert torch.equal(co, codes) and torch.equal(qo, q)
    ref = orc.scale_sweep(w, H32.astype(np.float64), orc.tensor_amax(w)[0])
    st = G.sweep_parity(G.host(codes), G.host(q), G.host(c1), ref, c2_gpu=G.host(c2))
    assert st["mismatch_frac"] < 1e-3, (rhos, st)


def _gershgorin_block(r, rho, tokens=4096):
    """D^1/2 (I + (1 - rho) S) D^1/2 with S symmetric, zero diagonal, random signs and largest
    absolute row sum 1: its scaled Gershgorin ratio is rho; positive definite for rho > 0,
    possibly indefinite below."""
    S = np.triu(r.standard_normal((16, 16)) * r.uniform(0.2, 1.0, (16, 16)), 1)
    S = S + S.T
    S /= np.abs(S).sum(1).max()
    d = tokens * 4.0 ** r.uniform(-1, 1, 16)
    return np.sqrt(d)[:, None] * (np.eye(16) + (1.0 - rho) * S) * np.sqrt(d)[None, :]
