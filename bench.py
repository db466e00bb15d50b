#!/usr/bin/env python
"""Throughput of the NVFP4 block-numerics hot path on B200.

One step is one pass of the whole hot path over one batch of synthetic input:

  act   -- the dynamic activation-quantization sweep: for each of the 15 shapes
           [T, C], C in {2048, 4096, 7168}, T in {1, 16, 256, 4096, 65536}:
           per-tensor amax -> NVFP4 quantize (E4M3 block scales, packed E2M1)
           -> dequantize to BF16;
  calib -- one Gemma-2B-like decoder layer's calibration: local Hessians of the
           layer input X [16384 x 2048] and of the down-projection input
           [16384 x 16384], the four weight amaxes, and the Hessian-weighted
           E4M3 scale sweep with NVFP4 pack of q_proj, gate, up and down (6.55 M
           blocks, one batched launch);
  moe   -- an MoE layer's expert calibration: local Hessians of the 64 experts'
           routed inputs X [2048 x 4096] and down-projection inputs [2048 x 1536]
           (128 Hessians, one batched launch), the 192 weight amaxes, and the
           Hessian-weighted sweep with pack of all 192 gate/up/down matrices
           (Student-t weights, 75.5 M blocks, one batched launch);
  cast  -- MXFP4 -> NVFP4 cast of 32 expert matrices 2880 x 2880 (one launch).

`value` is the first half of the metric, NVFP4 quant GB/s: algorithmic bytes of
the act part (amax 2 B, quantize 2.5625 B, dequantize 2.5625 B per element) over
its device time.  The second half, scale-sweep blocks/s against the FP32 pipe, is
reported in `sweep` (the dense layer) and `sweep_moe` (the expert stack); the FP32
peak is measured in the same run by an FMA microbenchmark (scalar and packed).  Each part runs as a CUDA graph; timing uses CUDA events on
the launching stream.  Every step touches ~5 GB, more than the 126 MB L2, so no
extra flush is inserted between steps.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       [--parts act,calib,moe,cast] (a subset, e.g. for profiling one kernel)
Under torchrun every rank runs its own replica of the step on its own GPU
(independent problems, no collective on the data path: weak scaling); times are
the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 quant GB/s (% HBM peak); scale-sweep blocks/s (% FP32 peak)"
# FP32 work of the sweep.  The algorithmic count (the roofline's) is the exhaustive search
# the method defines: 127 candidates per 16-element block, each a 136-entry symmetric
# quadratic form (272 FLOP) plus the 16 dequantize-subtracts (32), about 38 kFLOP per
# block.  The kernel proves most candidates irrelevant instead of evaluating them (same
# codes), so that figure reads above the FP32 peak; the work it does execute is counted on
# the device: candidate halves of 8 elements (w/S 8, e 16, bound 24 FLOP) and quadratic
# forms (272).  The second end of the rounding bracket and the conversions are not counted.
SWEEP_FLOP_PER_BLOCK = 127 * (272 + 32)   # algorithmic (exhaustive) count per block
SWEEP_FLOP_PER_HALF = 8 + 16 + 24         # executed: per visited candidate half
SWEEP_FLOP_PER_COST = 272                 # executed: per evaluated cost
ACT_BYTES = {"amax": 2.0, "act_quant": 2.5625, "dequant": 2.5625}
CAST_BYTES_PER_MX_BLOCK = 1 + 16 + 16 + 2  # read E8M0 + nibbles, write nibbles + 2 E4M3 scales
FP32_NOMINAL_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # SMs x FP32 lanes x FMA x max clock
N_EXPERTS = 64


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--parts", default="act,calib,moe,cast")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-rooflines", action="store_true",
                   help="skip the per-kernel micro-timings (for launch-list profiling of the step alone)")
    p.add_argument("--profile", default=None, choices=sorted(PROFILE_CASES),
                   help="run only one kernel, --profile-reps times, on a case sized for an ncu capture "
                        "(inputs above the L2, a few GB at most); prints nothing but a one-line summary")
    p.add_argument("--profile-reps", type=int, default=3)
    p.add_argument("--record-traffic", nargs="+", metavar="ROW=CSV", default=None,
                   help="write profiles/dram_traffic.json from ncu --csv logs of --profile runs")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def fp4_peak_tflops():
    """Dense NVFP4 tensor peak: the measured BF16 GEMM peak times the nominal FP4/BF16
    ratio (9 / 2.25 PFLOP/s), else the recipe's fallback 1.59 PFLOP/s BF16 times 4."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return 4.0 * float(json.load(f)["bf16_tflops"])
    except Exception:
        return 4.0 * 1590.0


# ---------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------- workload
def build_workload(parts, seed, dev):
    import torch

    from nvfp4_block_numerics_b200 import inputs

    def bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    W = {"host": {}}
    if "act" in parts:
        shapes = []
        for (T, C) in inputs.C2_SHAPES:
            xb = inputs.c2_shape(T, C, seed)
            shapes.append(dict(T=T, C=C, host=xb, x=bf16(xb),
                               q=torch.empty((T, C // 2), dtype=torch.uint8, device=dev),
                               sc=torch.empty((T, C // 16), dtype=torch.uint8, device=dev),
                               out=torch.empty((T, C), dtype=torch.bfloat16, device=dev)))
        W["act"] = shapes
        W["amax_act"] = torch.zeros(len(shapes), dtype=torch.float32, device=dev)
        W["s2_act"] = torch.zeros(len(shapes), dtype=torch.float32, device=dev)
    if "calib" in parts:
        d = inputs.c3_layer(seed)
        W["X"], W["Xd"] = bf16(d["X"]), bf16(d["X_down"])
        W["H"] = torch.zeros((2048 // 16, 16, 16), dtype=torch.float32, device=dev)
        W["Hd"] = torch.zeros((16384 // 16, 16, 16), dtype=torch.float32, device=dev)
        W["amax_w"] = torch.zeros(4, dtype=torch.float32, device=dev)
        W["weights"] = []
        for k, name in enumerate(("W_q", "W_gate", "W_up", "W_down")):
            w = bf16(d[name])
            rows, cols = w.shape
            W["weights"].append(dict(
                name=name, w=w, H=W["Hd"] if name == "W_down" else W["H"], d_amax_w=W["amax_w"][k:k + 1],
                codes=torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev),
                q=torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)))
        W["host"]["c3"] = d
    if "moe" in parts:
        from concurrent.futures import ThreadPoolExecutor

        def expert(e):
            d = inputs.c4_expert(e, seed)
            return {k: bf16(v) for k, v in d.items()}

        with ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
            experts = list(ex.map(expert, range(N_EXPERTS)))
        W["moe_X"] = [d["X"] for d in experts]
        W["moe_Xd"] = [d["X_down"] for d in experts]
        W["moe_H"] = torch.zeros((N_EXPERTS, 4096 // 16, 16, 16), dtype=torch.float32, device=dev)
        W["moe_Hd"] = torch.zeros((N_EXPERTS, 1536 // 16, 16, 16), dtype=torch.float32, device=dev)
        W["moe_amax"] = torch.zeros(3 * N_EXPERTS, dtype=torch.float32, device=dev)
        W["moe_weights"] = []
        for e, d in enumerate(experts):
            for k, name in enumerate(("W_gate", "W_up", "W_down")):
                w = d[name]
                rows, cols = w.shape
                i = 3 * e + k
                W["moe_weights"].append(dict(
                    name=f"e{e}/{name}", w=w, H=W["moe_Hd"][e] if name == "W_down" else W["moe_H"][e],
                    d_amax_w=W["moe_amax"][i:i + 1],
                    codes=torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev),
                    q=torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)))
        del experts
    if "cast" in parts:
        jobs = []
        for i in range(32):
            mq, e8 = inputs.c5_cast(i, seed)
            m = torch.from_numpy(mq).to(dev)
            jobs.append(dict(mx_q=m, e8m0=torch.from_numpy(e8).to(dev), nv_q=torch.empty_like(m),
                             nv_scales=torch.empty((mq.shape[0], mq.shape[1] // 8), dtype=torch.uint8, device=dev),
                             d_global_amax=torch.empty(1, dtype=torch.float32, device=dev),
                             d_s2=torch.empty(1, dtype=torch.float32, device=dev)))
        W["cast"] = jobs
        W["counts"] = torch.zeros(3, dtype=torch.int64, device=dev)
    W["flags"] = torch.zeros(1, dtype=torch.int32, device=dev)
    return W


def part_act(W):
    """The 15 shapes in three batched launches: amax of every tensor, then their NVFP4
    quantization (each with its own s2), then the dequantization round trip."""
    from nvfp4_block_numerics_b200 import binding as nv4

    W["amax_act"].zero_()
    n = len(W["act"])
    am = [W["amax_act"][i:i + 1] for i in range(n)]
    s2 = [W["s2_act"][i:i + 1] for i in range(n)]
    nv4.nv4_tensor_amax_batched([s["x"] for s in W["act"]], am, W["flags"])
    nv4.nv4_act_quant_batched([dict(x=s["x"], d_amax=am[i], q=s["q"], scales=s["sc"], d_s2=s2[i])
                               for i, s in enumerate(W["act"])], W["flags"])
    nv4.nv4_dequant_batched([dict(q=s["q"], scales=s["sc"], d_s2=s2[i], out=s["out"]) for i, s in enumerate(W["act"])])


def part_calib(W):
    from nvfp4_block_numerics_b200 import binding as nv4

    W["H"].zero_()
    W["Hd"].zero_()
    W["amax_w"].zero_()
    nv4.nv4_hessian_accum_batched([W["X"], W["Xd"]], [W["H"], W["Hd"]], W["flags"])
    nv4.nv4_tensor_amax_batched([j["w"] for j in W["weights"]], [j["d_amax_w"] for j in W["weights"]], W["flags"])
    # the production call: winning codes and packed E2M1 nibbles (no cost diagnostics)
    nv4.nv4_scale_sweep_batched([{k: j[k] for k in ("w", "H", "d_amax_w", "codes", "q")}
                                 for j in W["weights"]], W["flags"])


def part_moe(W):
    """The expert stack's calibration: 128 Hessians in one launch, 192 weight amaxes (two
    launches of at most 128 tensors), one sweep launch over all 192 matrices."""
    from nvfp4_block_numerics_b200 import binding as nv4

    W["moe_H"].zero_()
    W["moe_Hd"].zero_()
    W["moe_amax"].zero_()
    nv4.nv4_hessian_accum_batched(W["moe_X"] + W["moe_Xd"], list(W["moe_H"]) + list(W["moe_Hd"]), W["flags"])
    mw = W["moe_weights"]
    for k in range(0, len(mw), 128):
        nv4.nv4_tensor_amax_batched([j["w"] for j in mw[k:k + 128]], [j["d_amax_w"] for j in mw[k:k + 128]],
                                    W["flags"])
    nv4.nv4_scale_sweep_batched([{k: j[k] for k in ("w", "H", "d_amax_w", "codes", "q")} for j in mw], W["flags"])


def part_cast(W):
    from nvfp4_block_numerics_b200 import binding as nv4

    W["counts"].zero_()
    nv4.nv4_mxfp4_to_nvfp4_batched(W["cast"], W["counts"], W["flags"])


PARTS = {"act": part_act, "calib": part_calib, "moe": part_moe, "cast": part_cast}
LAUNCHES = {"act": 3, "calib": 3, "moe": 4, "cast": 2}   # launches of this library's kernels per part


def traffic_table():
    """DRAM bytes per unit for the rows recorded in profiles/dram_traffic.json, for kernels
    whose sources still hash to the values recorded with the capture (else the entry is
    dropped): {row: bytes per unit of the row's --profile case}."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            doc = json.load(f)
    except Exception:
        return {}
    out = {}
    for k, e in doc.get("kernels", {}).items():
        try:
            ok = _sources_sha([os.path.basename(f) for f in e["files"]]) == e.get("sources_sha256")
        except OSError:
            continue
        if ok and e.get("units"):
            out[k] = (e["dram_read_bytes"] + e["dram_write_bytes"]) / e["units"]
    return out


def time_launch(fn, reps=20, flush=None):
    """Average device duration of one call, events around the call only.

    The call is captured once in a CUDA graph (after one eager call, which does any
    first-use set-up) and replayed between the events, so the host-side argument
    marshalling of the binding stays outside the measured interval.

    flush = (w, r): before each replay, write w and then read r, two buffers larger
    than the L2.  The write evicts the call's data; the read then replaces the write's
    dirty lines with clean ones, so the timed call starts from a cold L2 without
    paying for the write-back of the flush buffer."""
    import torch

    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    s = torch.cuda.current_stream()
    tot = 0.0
    for _ in range(reps):
        if flush is not None:
            flush[0].fill_(1)
            flush[1].view(torch.int64).sum()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s)
        g.replay()
        b.record(s)
        b.synchronize()
        tot += a.elapsed_time(b)
    del g
    return tot / reps / 1e3


def fp32_peak(dev, reps=5):
    """The FP32 pipe's throughput on this GPU, measured: the library's FMA microbenchmark
    (16 independent chains per thread, 148 x 8 CTAs of 256 threads), scalar and packed
    two-lane FMAs, best of `reps` event-timed launches each."""
    import torch

    from nvfp4_block_numerics_b200 import binding as nv4

    blocks = torch.cuda.get_device_properties(dev).multi_processor_count * 8
    iters = 4096
    sink = torch.zeros(blocks, dtype=torch.float32, device=dev)
    out = {}
    for packed in (False, True):
        nv4.nv4_fp32_probe(packed, blocks, iters, sink)
        torch.cuda.synchronize()
        best = None
        s = torch.cuda.current_stream()
        for _ in range(reps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(s)
            nv4.nv4_fp32_probe(packed, blocks, iters, sink)
            b.record(s)
            b.synchronize()
            t = a.elapsed_time(b) / 1e3
            best = t if best is None else min(best, t)
        out["packed" if packed else "scalar"] = blocks * 256.0 * iters * 128 / best / 1e12
    out["measured"] = max(out["scalar"], out["packed"])
    out["nominal"] = FP32_NOMINAL_TFLOPS
    out["how"] = (f"nv4_fp32_probe: {blocks} CTAs x 256 threads x {iters} iterations x 128 FLOP of independent FMAs, "
                  f"scalar fma.rn.f32 and packed fma.rn.f32x2, best of {reps} event-timed launches each")
    return out


def sweep_row(nv4, jobs, flags, label, fp32):
    """Roofline row of one batched sweep launch (the production call, codes + nibbles):
    blocks/s, the algorithmic count against the measured FP32 peak, and the executed work
    from the kernel's device counters (one extra launch)."""
    import torch

    blocks = sum(j["codes"].numel() for j in jobs)
    work = torch.zeros(2, dtype=torch.int64, device=flags.device)
    nv4.nv4_scale_sweep_batched([dict(j, d_work=work) for j in jobs], flags)
    torch.cuda.synchronize()
    halves, costs = (int(x) for x in work.tolist())
    t = time_launch(lambda: nv4.nv4_scale_sweep_batched(jobs, flags), reps=5)
    executed = SWEEP_FLOP_PER_HALF * halves + SWEEP_FLOP_PER_COST * costs
    return {"bound": "alu", "flops": SWEEP_FLOP_PER_BLOCK * blocks, "blocks": blocks, "units": blocks, "s": t,
            "half_visits_per_block": halves / blocks, "costs_per_block": costs / blocks,
            "executed_tflops": executed / t / 1e12,
            "executed_frac": executed / t / 1e12 / fp32["measured"],
            "executed_frac_nominal": executed / t / 1e12 / fp32["nominal"],
            "launch": label}


def kernel_rooflines(W, hbm_peak, fp32):
    """Per-kernel achieved throughput on each kernel's largest launch of the step."""
    import torch

    from nvfp4_block_numerics_b200 import binding as nv4

    flush = (torch.empty(256 << 20, dtype=torch.uint8, device=W["flags"].device),
             torch.zeros(256 << 20, dtype=torch.uint8, device=W["flags"].device))
    out = {}
    if "act" in W:
        big = max(W["act"], key=lambda s: s["T"] * s["C"])
        n = big["T"] * big["C"]
        n_all = sum(s["T"] * s["C"] for s in W["act"])
        a = W["amax_act"][-1:]
        s2 = W["s2_act"][-1:]
        # the step's own launches: each kernel once over all 15 shapes
        ams = [W["amax_act"][i:i + 1] for i in range(len(W["act"]))]
        s2s = [W["s2_act"][i:i + 1] for i in range(len(W["act"]))]
        t = time_launch(lambda: nv4.nv4_tensor_amax_batched([s["x"] for s in W["act"]], ams, W["flags"]), flush=flush)
        out["tensor_amax"] = {"bound": "hbm", "bytes": ACT_BYTES["amax"] * n_all, "s": t}
        qj = [dict(x=s["x"], d_amax=ams[i], q=s["q"], scales=s["sc"], d_s2=s2s[i]) for i, s in enumerate(W["act"])]
        t = time_launch(lambda: nv4.nv4_act_quant_batched(qj, W["flags"]), flush=flush)
        out["act_quant"] = {"bound": "hbm", "bytes": ACT_BYTES["act_quant"] * n_all, "s": t}
        dj = [dict(q=s["q"], scales=s["sc"], d_s2=s2s[i], out=s["out"]) for i, s in enumerate(W["act"])]
        t = time_launch(lambda: nv4.nv4_dequant_batched(dj), flush=flush)
        out["dequant"] = {"bound": "hbm", "bytes": ACT_BYTES["dequant"] * n_all, "s": t}
        for k in ("tensor_amax", "act_quant", "dequant"):
            out[k]["launch"] = f"15 [T, C] bf16 shapes, {n_all / 1e6:.0f} M elements, one batched launch"
            out[k]["units"] = n_all
        # fused fake quantize-dequantize (a widening of the path; not part of the step)
        qdq = torch.empty_like(big["x"])
        t = time_launch(lambda: nv4.nv4_fake_qdq(big["x"], a, qdq, s2, W["flags"]), flush=flush)
        out["fake_qdq"] = {"bound": "hbm", "bytes": 4.0 * n, "s": t, "in_step": False}
        del qdq
        # format variants (widenings; not part of the step)
        mq = torch.empty((big["T"], big["C"] // 2), dtype=torch.uint8, device=big["x"].device)
        me = torch.empty((big["T"], big["C"] // 32), dtype=torch.uint8, device=big["x"].device)
        t = time_launch(lambda: nv4.nv4_mxfp4_quant(big["x"], mq, me, W["flags"]), flush=flush)
        out["mxfp4_quant"] = {"bound": "hbm", "bytes": (2 + 0.5 + 1 / 32) * n, "s": t, "in_step": False}
        del mq, me
        fq = torch.empty((big["T"], big["C"]), dtype=torch.uint8, device=big["x"].device)
        fs = torch.empty(1, dtype=torch.float32, device=big["x"].device)
        t = time_launch(lambda: nv4.nv4_fp8_quant(big["x"], a, fq, fs, W["flags"]), flush=flush)
        out["fp8_quant"] = {"bound": "hbm", "bytes": 3.0 * n, "s": t, "in_step": False}
        del fq
        # block Hadamard (n = 128) fused with MXFP4 quantization: one pass, 2 B in, 0.53 B out
        hq = torch.empty((big["T"], big["C"] // 2), dtype=torch.uint8, device=big["x"].device)
        he = torch.empty((big["T"], big["C"] // 32), dtype=torch.uint8, device=big["x"].device)
        t = time_launch(lambda: nv4.nv4_hadamard_mxfp4_quant(big["x"], 128, hq, he, W["flags"]), flush=flush)
        out["hadamard128_mxfp4_quant"] = {"bound": "hbm", "bytes": (2 + 0.5 + 1 / 32) * n, "s": t, "in_step": False}
        del hq, he
        for k in ("fake_qdq", "mxfp4_quant", "fp8_quant", "hadamard128_mxfp4_quant"):
            out[k]["launch"] = f"[{big['T']}, {big['C']}] bf16"
    if "weights" in W:
        # RTN weight quantization of the layer's four weights in one batched launch (a widening
        # of the path; not in the step)
        rjobs = [dict(w=j["w"], d_amax=j["d_amax_w"], q=torch.empty_like(j["q"]),
                      scales=torch.empty((j["w"].shape[0], j["w"].shape[1] // 16), dtype=torch.uint8,
                                         device=j["w"].device),
                      d_s2=torch.empty(1, dtype=torch.float32, device=j["w"].device)) for j in W["weights"]]
        t = time_launch(lambda: nv4.nv4_weight_quant_rtn_batched(rjobs, W["flags"]), flush=flush)
        out["weight_quant_rtn"] = {"bound": "hbm", "s": t, "in_step": False,
                                   "bytes": ACT_BYTES["act_quant"] * sum(j["w"].numel() for j in rjobs),
                                   "launch": " + ".join(f"{j['name']} {list(j['w'].shape)}" for j in W["weights"])
                                             + " bf16, one batched launch"}
        del rjobs
        X, Xd = W["X"], W["Xd"]
        t = time_launch(lambda: nv4.nv4_hessian_accum_batched([X, Xd], [W["H"], W["Hd"]], W["flags"]), reps=10,
                        flush=flush)
        out["hessian_accum"] = {"bound": "hbm", "bytes": 2.0 * (X.numel() + Xd.numel()), "s": t,
                                "units": X.numel() + Xd.numel(),
                                "launch": f"X [{X.shape[0]}, {X.shape[1]}] + X_down [{Xd.shape[0]}, {Xd.shape[1]}] bf16, "
                                          "one batched launch"}
        jobs = [{k: j[k] for k in ("w", "H", "d_amax_w", "codes", "q")} for j in W["weights"]]
        out["scale_sweep"] = sweep_row(nv4, jobs, W["flags"], "q_proj + gate + up + down, one batched launch", fp32)
    if "moe_weights" in W:
        Xs, Hs = W["moe_X"] + W["moe_Xd"], list(W["moe_H"]) + list(W["moe_Hd"])
        t = time_launch(lambda: nv4.nv4_hessian_accum_batched(Xs, Hs, W["flags"]), reps=10, flush=flush)
        out["hessian_accum_moe"] = {"bound": "hbm", "bytes": 2.0 * sum(x.numel() for x in Xs), "s": t,
                                    "launch": f"{len(W['moe_X'])} x [2048, 4096] + {len(W['moe_Xd'])} x [2048, 1536] "
                                              "bf16, one batched launch"}
        jobs = [{k: j[k] for k in ("w", "H", "d_amax_w", "codes", "q")} for j in W["moe_weights"]]
        out["scale_sweep_moe"] = sweep_row(nv4, jobs, W["flags"],
                                           f"{len(jobs)} expert matrices (gate/up [1536, 4096], down [4096, 1536]), "
                                           "one batched launch", fp32)
    if "calib" in W or "act" in W:
        # W4A4 GEMM (a widening of the path; not part of the step): a 16384-token batch
        # through the gate projection 2048 -> 16384 and a square 8192^3 product, random
        # NVFP4 operands (codes and scales resident in HBM, scales in the MMA layout)
        dev = W["flags"].device
        g = torch.Generator(device=dev).manual_seed(1)
        best = None
        for (M, N, K) in ((16384, 16384, 2048), (8192, 8192, 8192)):
            qa = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g)
            qb = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g)
            fa = nv4.mma_scales(torch.randint(0x30, 0x40, (M, K // 16), dtype=torch.uint8, device=dev, generator=g))
            fb = nv4.mma_scales(torch.randint(0x30, 0x40, (N, K // 16), dtype=torch.uint8, device=dev, generator=g))
            one = torch.ones(1, dtype=torch.float32, device=dev)
            o = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            t = time_launch(lambda: nv4.nv4_gemm_nvfp4(qa, fa, one, qb, fb, one, o, W["flags"]), reps=10)
            out[f"gemm_nvfp4_{M}x{N}x{K}"] = {"bound": "tensor", "flops": 2.0 * M * N * K, "s": t, "in_step": False,
                                              "launch": f"A [{M}, {K}] x B [{N}, {K}] NVFP4 -> BF16"}
            del qa, qb, fa, fb, o
    if "cast" in W:
        nmx = sum(j["e8m0"].numel() for j in W["cast"])
        t = time_launch(lambda: nv4.nv4_mxfp4_to_nvfp4_batched(W["cast"], W["counts"], W["flags"]), flush=flush)
        out["mxfp4_to_nvfp4"] = {"bound": "hbm", "bytes": CAST_BYTES_PER_MX_BLOCK * nmx, "s": t, "units": nmx,
                                 "launch": "32 x [2880, 2880], out of place"}
    for k, v in out.items():
        if v["bound"] == "hbm":
            v["achieved"] = v["bytes"] / v["s"] / 1e9
            v["peak"] = hbm_peak
            v["unit"] = "GB/s"
        elif v["bound"] == "tensor":
            v["achieved"] = v["flops"] / v["s"] / 1e12
            v["peak"] = fp4_peak_tflops()
            v["unit"] = "TFLOP/s"
        else:
            v["achieved"] = v["flops"] / v["s"] / 1e12
            v["peak"] = fp32["measured"]
            v["unit"] = "TFLOP/s"
            v["blocks_per_s"] = v["blocks"] / v["s"]
        v["frac"] = v["achieved"] / v["peak"]
        v["ms"] = v["s"] * 1e3
    traffic = traffic_table()
    for k, v in out.items():
        v["traffic"] = traffic[k] * v["units"] if k in traffic and v.get("units") else None
    return out


def e2e_act(W, steps):
    """The act part end to end through the public API: pinned host inputs copied in,
    amax -> quantize -> dequantize, packed codes, scales and BF16 output copied back.
    Copy-in, compute and copy-out run on three streams, ordered per shape by events,
    so the transfers of one shape overlap the kernels of its neighbours."""
    import torch

    from nvfp4_block_numerics_b200 import binding as nv4

    hx = [torch.from_numpy(s["host"].view(np.int16)).view(torch.bfloat16).pin_memory() for s in W["act"]]
    hq = [torch.empty(tuple(s["q"].shape), dtype=torch.uint8).pin_memory() for s in W["act"]]
    hs = [torch.empty(tuple(s["sc"].shape), dtype=torch.uint8).pin_memory() for s in W["act"]]
    ho = [torch.empty(tuple(s["out"].shape), dtype=torch.bfloat16).pin_memory() for s in W["act"]]
    h2d = sum(t.numel() * 2 for t in hx)
    d2h = sum(t.numel() for t in hq) + sum(t.numel() for t in hs) + sum(t.numel() * 2 for t in ho)
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    n = len(W["act"])
    done = [None] * n      # compute finished (x may be overwritten)
    drained = [None] * n   # copy-out finished (q, sc, out may be overwritten)

    def one():
        for i, s in enumerate(W["act"]):
            with torch.cuda.stream(s_in):
                if done[i] is not None:
                    s_in.wait_event(done[i])
                s["x"].copy_(hx[i], non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ready)
                if drained[i] is not None:
                    s_cmp.wait_event(drained[i])
                a, s2 = W["amax_act"][i:i + 1], W["s2_act"][i:i + 1]
                a.zero_()
                nv4.nv4_tensor_amax(s["x"], a, W["flags"], s_cmp)
                nv4.nv4_act_quant(s["x"], a, s["q"], s["sc"], s2, W["flags"], s_cmp)
                nv4.nv4_dequant(s["q"], s["sc"], s2, s["out"], s_cmp)
                done[i] = torch.cuda.Event()
                done[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[i])
                hq[i].copy_(s["q"], non_blocking=True)
                hs[i].copy_(s["sc"], non_blocking=True)
                ho[i].copy_(s["out"], non_blocking=True)
                drained[i] = torch.cuda.Event()
                drained[i].record(s_out)

    one()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for _ in range(steps):
        one()
    for ev in drained:
        s_out.wait_event(ev)
    b.record(s_out)
    b.synchronize()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / 1e3 / steps, h2d, d2h


def e2e_part(W, part, steps):
    """One part of the step end to end through the public API, from pinned host buffers:
    the part's inputs copied in, its launches, its outputs copied back, on one stream.
    calib: X, X_down and the four weights in; winning codes and packed nibbles out.
    moe: the 128 routed inputs and 192 weights in; codes and nibbles out.  cast: MXFP4
    nibbles and E8M0 scales in; NVFP4 nibbles, E4M3 scales, s2 and counts out."""
    import torch

    if part == "calib":
        ins = [W["X"], W["Xd"]] + [j["w"] for j in W["weights"]]
        outs = [t for j in W["weights"] for t in (j["codes"], j["q"])]
    elif part == "moe":
        ins = W["moe_X"] + W["moe_Xd"] + [j["w"] for j in W["moe_weights"]]
        outs = [t for j in W["moe_weights"] for t in (j["codes"], j["q"])]
    else:
        ins = [t for j in W["cast"] for t in (j["mx_q"], j["e8m0"])]
        outs = [t for j in W["cast"] for t in (j["nv_q"], j["nv_scales"], j["d_s2"])] + [W["counts"]]
    h_in = [t.cpu().pin_memory() for t in ins]
    h_out = [torch.empty(tuple(t.shape), dtype=t.dtype).pin_memory() for t in outs]
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = sum(t.numel() * t.element_size() for t in h_out)
    st = torch.cuda.Stream()

    def one():
        with torch.cuda.stream(st):
            for d, h in zip(ins, h_in):
                d.copy_(h, non_blocking=True)
            PARTS[part](W)
            for h, d in zip(h_out, outs):
                h.copy_(d, non_blocking=True)

    one()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(steps):
        one()
    b.record(st)
    b.synchronize()
    del h_in, h_out
    return a.elapsed_time(b) / 1e3 / steps, h2d, d2h


def act_bytes(W):
    n = sum(s["T"] * s["C"] for s in W["act"])
    return n * sum(ACT_BYTES.values()), n


# ---------------------------------------------------------------------- CPU baseline (oracle)
def cpu_baseline(seed, budget_s=20.0):
    """The oracle as it stands, on a bounded sample of the same workload, on this host's cores."""
    import oracle
    from nvfp4_block_numerics_b200 import inputs

    threads = oracle.default_threads()
    # act path: every shape, at most 256 rows of each (all rows of the small ones)
    xs = [inputs.c2_shape(min(T, 256), C, seed + 1000) for (T, C) in inputs.C2_SHAPES]
    nelem = sum(x.size for x in xs)
    reps = 0
    tt = time.perf_counter()
    while True:
        for x in xs:
            a, _ = oracle.tensor_amax(x, threads)
            q, sc, s2, _ = oracle.act_quant(x, a, threads=threads)
            oracle.dequant(q, sc, s2, "bf16", threads)
        reps += 1
        act_elapsed = time.perf_counter() - tt
        if act_elapsed > budget_s / 2 or reps >= 50:
            break
    act_gbs = reps * nelem * sum(ACT_BYTES.values()) / act_elapsed / 1e9
    # sweep: sampled rows of q_proj against an identity-free Hessian of a slice of X
    d = inputs.c3_layer(seed + 1000, tokens=1024, which=("X", "W_q"))
    H = oracle.hessian_accum(d["X"], threads=threads)
    amax, _ = oracle.tensor_amax(d["W_q"], threads)
    rows = np.arange(64)
    tt = time.perf_counter()
    n_blocks = 0
    while True:
        oracle.scale_sweep(d["W_q"], H, amax, rows=rows, threads=threads)
        n_blocks += len(rows) * (d["W_q"].shape[1] // 16)
        el = time.perf_counter() - tt
        if el > budget_s / 2:
            break
    sweep_bps = n_blocks / el
    moe_bps, moe_blocks = _oracle_moe_sweep(seed, threads, budget_s / 4)
    return {"value": act_gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"act path on min(T,256) rows of each of the 15 [T, C] shapes ({nelem} elements, "
                      f"{reps} reps); sweep on {len(rows)} rows x 128 blocks of q_proj, {n_blocks} blocks; "
                      f"expert sweep on 32 rows x 256 blocks of expert 0's gate projection, {moe_blocks} blocks",
            "sweep_blocks_per_s": sweep_bps, "sweep_moe_blocks_per_s": moe_bps}


def _oracle_moe_sweep(seed, threads, budget_s):
    """The oracle's sweep on 32 rows of one expert's gate projection (Student-t weights,
    its routed input's Hessian): blocks/s on this host."""
    import oracle
    from nvfp4_block_numerics_b200 import inputs

    d = inputs.c4_expert(0, seed + 1000, which=("X", "W_gate"))
    H = oracle.hessian_accum(d["X"], threads=threads)
    amax, _ = oracle.tensor_amax(d["W_gate"], threads)
    rows = np.arange(32)
    n = 0
    tt = time.perf_counter()
    while True:
        oracle.scale_sweep(d["W_gate"], H, amax, rows=rows, threads=threads)
        n += len(rows) * (d["W_gate"].shape[1] // 16)
        el = time.perf_counter() - tt
        if el > budget_s:
            break
    return n / el, n


# ---------------------------------------------------------------------- arms
def workload_config(parts, seed, ws):
    """The workload both arms report (the reference arm times a bounded sample of it)."""
    return {"workload": "NVFP4 hot path: activation quant sweep (15 [T,C] shapes, amax->quant->dequant) "
                        "+ Gemma-2B-like layer calibration (Hessians of X 16384x2048 and 16384x16384, "
                        "sweep of q/gate/up/down -> winning E4M3 codes + packed E2M1) + MoE expert stack "
                        "calibration (64 experts: 128 Hessians of 2048-token inputs, sweep of 192 gate/up/down "
                        "matrices, 75.5 M blocks) + MXFP4->NVFP4 cast of 32 x 2880x2880",
            "parts": list(parts), "seed": seed, "parallelism": f"replicas x{ws}",
            "l2": "no flush between steps: every step touches ~5 GB, above the 126 MB L2; per-kernel "
                  "rooflines: graph replay after writing then reading two 256 MB buffers"}


def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def run_reference(args):
    """The oracle (plain CPU code, FP64) as the reference arm: each step runs a bounded sample
    of the same workload on the host cores -- the activation path on <= 64 rows of every
    shape (the metric's GB/s half), and the Hessian-weighted sweep on 64 rows x 128 blocks of
    q_proj and on 32 rows x 256 blocks of one expert's gate projection (its blocks/s half)."""
    ws, rank, _ = dist_setup(args)
    if rank != 0:
        return
    import oracle
    from nvfp4_block_numerics_b200 import inputs

    threads = oracle.default_threads()
    xs = [inputs.c2_shape(min(T, 64), C, args.seed) for (T, C) in inputs.C2_SHAPES]
    nelem = sum(x.size for x in xs)
    d = inputs.c3_layer(args.seed, which=("X", "W_q"))
    H = oracle.hessian_accum(d["X"][:2048], threads=threads)
    wq = np.ascontiguousarray(d["W_q"][:64])
    amax_w = oracle.tensor_amax(d["W_q"], threads)[0]
    n_blocks = wq.size // 16
    e0 = inputs.c4_expert(0, args.seed, which=("X", "W_gate"))
    He = oracle.hessian_accum(e0["X"], threads=threads)
    we = np.ascontiguousarray(e0["W_gate"][:32])
    amax_e = oracle.tensor_amax(e0["W_gate"], threads)[0]
    n_blocks_e = we.size // 16
    t_act, t_sweep, t_moe = [0.0], [0.0], [0.0]

    def step():
        t0 = time.perf_counter()
        for x in xs:
            a, _ = oracle.tensor_amax(x, threads)
            q, sc, s2, _ = oracle.act_quant(x, a, threads=threads)
            oracle.dequant(q, sc, s2, "bf16", threads)
        t1 = time.perf_counter()
        oracle.scale_sweep(wq, H, amax_w, threads=threads)
        t2 = time.perf_counter()
        oracle.scale_sweep(we, He, amax_e, threads=threads)
        t3 = time.perf_counter()
        t_act[0] += t1 - t0
        t_sweep[0] += t2 - t1
        t_moe[0] += t3 - t2

    for _ in range(args.warmup):
        step()
    t_act[0] = t_sweep[0] = t_moe[0] = 0.0
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = (time.perf_counter() - t) / args.steps
    v = nelem * sum(ACT_BYTES.values()) / (t_act[0] / args.steps) / 1e9
    sweep_bps = n_blocks / (t_sweep[0] / args.steps)
    moe_bps = n_blocks_e / (t_moe[0] / args.steps)
    sample = (f"act path on min(T,64) rows of each of the 15 [T, C] shapes ({nelem} elements per step); "
              f"sweep on 64 rows x 128 blocks of q_proj ({n_blocks} blocks per step, H from 2048 tokens); "
              f"expert sweep on 32 rows x 256 blocks of expert 0's gate projection ({n_blocks_e} blocks per step)")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args.parts.split(","), args.seed, 1),
            "sweep": {"value": sweep_bps, "unit": "blocks/s"},
            "sweep_moe": {"value": moe_bps, "unit": "blocks/s"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch

    from nvfp4_block_numerics_b200 import dist

    ws, rank, local = dist.init(backend="nccl", timeout_s=300)
    parts = [p for p in args.parts.split(",") if p]
    if ws == 1:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    from nvfp4_block_numerics_b200 import binding as nv4

    nv4.lib()
    hbm_peak, peak_kind = peaks()
    W = build_workload(parts, args.seed + rank, dev)

    # eager warm-up (sets kernel attributes, encoders), then one CUDA graph per part
    for p in parts:
        PARTS[p](W)
    torch.cuda.synchronize()
    graphs = {}
    for p in parts:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            PARTS[p](W)
        graphs[p] = g
    for _ in range(max(args.warmup, 0)):
        for p in parts:
            graphs[p].replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(dev.index)
    dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    ev = {p: [] for p in parts}
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        torch.cuda.nvtx.range_push(f"step {i}")              # NVTX ranges: visible in an nsys/ncu timeline
        for p in parts:
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            torch.cuda.nvtx.range_push(p)
            a.record(stream)
            graphs[p].replay()
            b.record(stream)
            torch.cuda.nvtx.range_pop()
            ev[p].append((a, b))
        torch.cuda.nvtx.range_pop()
    end.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    total_s = start.elapsed_time(end) / 1e3
    part_s = {p: sum(a.elapsed_time(b) for a, b in ev[p]) / 1e3 for p in parts}
    t = dist.max_over_ranks([total_s] + [part_s[p] for p in parts])      # device times, max over ranks
    total_s = t[0]
    part_s = {p: t[i + 1] for i, p in enumerate(parts)}
    flags = int(W["flags"].item())
    cast_counts = [int(v) for v in W["counts"].tolist()] if "cast" in parts else None   # the last step's

    fp32 = None if args.no_rooflines else fp32_peak(dev)
    roof = {} if args.no_rooflines else kernel_rooflines(W, hbm_peak, fp32)
    e2e = None
    if "act" in parts and not args.no_e2e:
        e2e_s, h2d, d2h = e2e_act(W, max(1, min(args.steps, 3)))
        e2e_s = dist.max_over_ranks([e2e_s])[0]
        bytes_act, _ = act_bytes(W)
        e2e = {"value": ws * bytes_act / e2e_s / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_s * 1e3}
    if not args.no_e2e:
        # the other parts end to end from host buffers (one stream each, copies inside the
        # timed region), reported beside the act part's metric
        e2e_parts = {}
        for prt in ("calib", "moe", "cast"):
            if prt in parts:
                t_s, h2d_p, d2h_p = e2e_part(W, prt, 2)
                t_s = dist.max_over_ranks([t_s])[0]
                e2e_parts[prt] = {"ms_per_step": t_s * 1e3, "h2d_bytes_per_step": h2d_p,
                                  "d2h_bytes_per_step": d2h_p,
                                  "device_ms_per_step": part_s[prt] / args.steps * 1e3}
                if prt in ("calib", "moe"):
                    wts = W["weights"] if prt == "calib" else W["moe_weights"]
                    e2e_parts[prt]["blocks_per_s"] = ws * sum(j["codes"].numel() for j in wts) / t_s
        if e2e is None:
            e2e = {}
        e2e["parts"] = e2e_parts
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.seed)

    dist.finalize()
    if rank != 0:
        return

    value, unit = None, "GB/s"
    if "act" in parts:
        bytes_act, n_act = act_bytes(W)
        value = ws * bytes_act * args.steps / part_s["act"] / 1e9
    def sweep_summary(part, row, weights):
        blocks = sum(j["codes"].numel() for j in weights)
        sw = roof[row]
        return {"value": ws * blocks * args.steps / part_s[part], "unit": "blocks/s",
                "note": f"blocks over the whole {part} part (Hessians + amax + sweep)",
                "kernel_blocks_per_s": sw["blocks_per_s"],
                "algorithmic_tflops": sw["achieved"], "frac_fp32": sw["frac"],
                "fp32_peak_tflops": fp32["measured"], "fp32_nominal_tflops": fp32["nominal"],
                "executed_tflops": sw["executed_tflops"], "executed_frac_fp32": sw["executed_frac"],
                "executed_frac_fp32_nominal": sw["executed_frac_nominal"],
                "half_visits_per_block": sw["half_visits_per_block"], "costs_per_block": sw["costs_per_block"],
                "note_work": "algorithmic = blocks/s x the exhaustive 127 x 304 FLOP per block (above the FP32 "
                             "peak: an exact branch and bound proves most candidates irrelevant, same codes); "
                             "executed = the FLOPs actually done, from device counters (48 per candidate half "
                             "visited, 272 per cost evaluated); fractions of the measured FP32 peak, nominal beside"}

    sweep = sweep_summary("calib", "scale_sweep", W["weights"]) if "calib" in parts and "scale_sweep" in roof else None
    sweep_moe = (sweep_summary("moe", "scale_sweep_moe", W["moe_weights"])
                 if "moe" in parts and "scale_sweep_moe" in roof else None)
    # dominant kernel: the largest device time per step (every in-step row times the step's
    # own launch, which runs once per step)
    in_step = [k for k in roof if roof[k].get("in_step", True)]
    dom = max(in_step, key=lambda k: roof[k]["s"]) if in_step else None
    shares = {p: part_s[p] / total_s for p in parts}
    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_s / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(parts, args.seed, ws),
        "parts_ms_per_step": {p: part_s[p] / args.steps * 1e3 for p in parts},
        "parts_share": shares,
        "gpu_launches": args.steps * sum(LAUNCHES[p] for p in parts),
        "flags": flags,
        "clocks": clk,
        "fp32_peak": fp32,
    }
    if dom is not None:
        r = roof[dom]
        line["roofline"] = {"kernel": dom, "bound": r["bound"], "achieved": r["achieved"], "peak": r["peak"],
                            "unit": r["unit"], "frac": r["frac"], "traffic": r["traffic"],
                            "peak_kind": (peak_kind if r["bound"] == "hbm" else
                                          "measured (nv4_fp32_probe, this run)" if r["bound"] == "alu" else
                                          "4 x the measured BF16 GEMM peak")}
        if dom.startswith("scale_sweep"):
            line["roofline"]["executed"] = r["executed_tflops"]
            line["roofline"]["executed_frac"] = r["executed_frac"]
            line["roofline"]["executed_frac_nominal"] = r["executed_frac_nominal"]
            line["roofline"]["note"] = ("achieved counts the exhaustive 127-candidate search (38.6 kFLOP per block); "
                                        "the exact branch and bound skips provably irrelevant candidates, so it reads "
                                        "above the peak; executed counts the work done")
    line["rows"] = {k: {kk: v.get(kk) for kk in ("bound", "achieved", "peak", "unit", "frac", "ms", "launch", "traffic",
                                                  "in_step")}
                    for k, v in roof.items()}
    if sweep is not None:
        line["sweep"] = sweep
    if sweep_moe is not None:
        line["sweep_moe"] = sweep_moe
    if cast_counts is not None:
        n16 = cast_counts[0] + cast_counts[1]
        line["cast"] = {"in_window_blocks": cast_counts[0], "fallback_blocks": cast_counts[1],
                        "lossless_blocks": cast_counts[2], "lossless_fraction": cast_counts[2] / max(n16, 1),
                        "note": "16-element NVFP4 blocks of the 32 matrices; lossless = NVFP4 dequant equal to the "
                                "MXFP4 dequant bit for bit"}
    if e2e is not None:
        line["e2e"] = e2e
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------- single-kernel runs for ncu
def _prof_setup_gemm(dev, seed):
    import torch

    from nvfp4_block_numerics_b200 import binding as nv4

    M = N = K = 8192
    g = torch.Generator(device=dev).manual_seed(seed)
    r = lambda *sh, lo=0, hi=256: torch.randint(lo, hi, sh, dtype=torch.uint8, device=dev, generator=g)
    qa, qb = r(M, K // 2), r(N, K // 2)
    fa, fb = nv4.mma_scales(r(M, K // 16, lo=0x30, hi=0x40)), nv4.mma_scales(r(N, K // 16, lo=0x30, hi=0x40))
    one = torch.ones(1, dtype=torch.float32, device=dev)
    out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    return (lambda: nv4.nv4_gemm_nvfp4(qa, fa, one, qb, fb, one, out)), "gemm_nvfp4_kernel: 8192^3 NVFP4 -> BF16"


def _prof_setup_sweep(dev, seed):
    W = build_workload(["calib"], seed, dev)
    part_calib(W)
    from nvfp4_block_numerics_b200 import binding as nv4

    jobs = [{k: j[k] for k in ("w", "H", "d_amax_w", "codes", "q")} for j in W["weights"]]
    return (lambda: nv4.nv4_scale_sweep_batched(jobs, W["flags"])), "sweep_kernel: Gemma-like layer, 6.55 M blocks"


def _prof_setup_sweep_moe(dev, seed, experts=16):
    import torch

    from nvfp4_block_numerics_b200 import binding as nv4
    from nvfp4_block_numerics_b200 import inputs

    jobs = []
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    for e in range(experts):
        d = inputs.c4_expert(e, seed)
        b = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev) for k, v in d.items()}
        Hx = nv4.hessian_accum(b["X"])
        Hd = nv4.hessian_accum(b["X_down"])
        for name in ("W_gate", "W_up", "W_down"):
            w = b[name]
            jobs.append(dict(w=w, H=Hd if name == "W_down" else Hx, d_amax_w=nv4.tensor_amax(w),
                             codes=torch.empty((w.shape[0], w.shape[1] // 16), dtype=torch.uint8, device=dev),
                             q=torch.empty((w.shape[0], w.shape[1] // 2), dtype=torch.uint8, device=dev)))
    blocks = sum(j["codes"].numel() for j in jobs)
    return (lambda: nv4.nv4_scale_sweep_batched(jobs, flags)), \
        f"sweep_kernel: {experts} MoE experts ({3 * experts} matrices, {blocks / 1e6:.1f} M blocks)"


def _prof_setup_hessian(dev, seed):
    W = build_workload(["calib"], seed, dev)
    from nvfp4_block_numerics_b200 import binding as nv4

    return (lambda: nv4.nv4_hessian_accum_batched([W["X"], W["Xd"]], [W["H"], W["Hd"]], W["flags"])), \
        "hessian_kernel: X [16384, 2048] + X_down [16384, 16384] bf16"


def _prof_setup_act(kind):
    def setup(dev, seed):
        import torch

        from nvfp4_block_numerics_b200 import binding as nv4
        from nvfp4_block_numerics_b200 import inputs

        xb = inputs.c2_shape(65536, 7168, seed)
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
        a = nv4.tensor_amax(x)
        q, sc, s2 = nv4.act_quant(x, a)
        fn = {"amax": lambda: nv4.nv4_tensor_amax(x, a),
              "act_quant": lambda: nv4.nv4_act_quant(x, a, q, sc, s2),
              "dequant": lambda: nv4.nv4_dequant(q, sc, s2, torch.empty_like(x)),
              "fake_qdq": lambda: nv4.nv4_fake_qdq(x, a, torch.empty_like(x), s2),
              "rtn": lambda: nv4.nv4_weight_quant_rtn(x, a, q, sc, s2),
              "fp8": lambda: nv4.nv4_fp8_quant(x, a, torch.empty(x.shape, dtype=torch.uint8, device=dev), s2),
              "mxfp4": lambda: nv4.mxfp4_quant(x),
              "hadamard": lambda: nv4.hadamard_mxfp4_quant(x, 128)}[kind]
        return fn, f"{kind}: [65536, 7168] bf16"
    return setup


def _prof_setup_hadamard2(dev, seed):
    import torch

    from nvfp4_block_numerics_b200 import binding as nv4
    from nvfp4_block_numerics_b200 import inputs

    w = inputs.f32_to_bf16_bits(inputs.normal_weights(inputs.rng_for(seed, "prof", "h2"), 16384, 8192, 0.02))
    wd = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).to(dev)
    q = torch.empty((16384, 4096), dtype=torch.uint8, device=dev)
    e8 = torch.empty((16384, 256), dtype=torch.uint8, device=dev)
    return (lambda: nv4.nv4_hadamard2_mxfp4_quant(wd, 32, q, e8)), \
        "hadamard2_kernel: [16384, 8192] bf16 weights, 32 x 32 tiles, MXFP4"


def _prof_setup_cast(dev, seed):
    W = build_workload(["cast"], seed, dev)
    from nvfp4_block_numerics_b200 import binding as nv4

    return (lambda: nv4.nv4_mxfp4_to_nvfp4_batched(W["cast"], W["counts"], W["flags"])), \
        "cast kernels: 32 x [2880, 2880] MXFP4, out of place"


PROFILE_CASES = {"gemm": _prof_setup_gemm, "sweep": _prof_setup_sweep, "sweep_moe": _prof_setup_sweep_moe,
                 "hessian": _prof_setup_hessian, "cast": _prof_setup_cast, "hadamard2": _prof_setup_hadamard2,
                 **{k: _prof_setup_act(k) for k in ("amax", "act_quant", "dequant", "fake_qdq", "rtn", "fp8",
                                                    "mxfp4", "hadamard")}}


# Roofline rows whose DRAM traffic comes from an ncu capture of a --profile case: the
# case, the kernel-name pattern, the sources the figure is valid for, and the units the
# case processes (the bench scales the per-unit traffic to its own launch of the row).
TRAFFIC_ROWS = {
    "tensor_amax": ("amax", "amax_kernel", ["quant.cu", "nv4_common.cuh"], 65536 * 7168),
    "act_quant": ("act_quant", "act_quant_kernel", ["quant.cu", "nv4_common.cuh"], 65536 * 7168),
    "dequant": ("dequant", "dequant_kernel", ["quant.cu", "nv4_common.cuh"], 65536 * 7168),
    "hessian_accum": ("hessian", "hessian_kernel", ["hessian.cu", "nv4_async.cuh", "nv4_common.cuh"],
                      16384 * 2048 + 16384 * 16384),
    "scale_sweep": ("sweep", "sweep_kernel", ["sweep.cu", "nv4_common.cuh"], 6553600),
    "scale_sweep_moe": ("sweep_moe", "sweep_kernel", ["sweep.cu", "nv4_common.cuh"], 16 * 3 * 1536 * 4096 // 16),
    "mxfp4_to_nvfp4": ("cast", "cast_", ["cast.cu", "nv4_common.cuh"], 32 * 2880 * 90),
}


def _sources_sha(files):
    import hashlib

    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "nvfp4_block_numerics_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def record_traffic(pairs):
    """profiles/dram_traffic.json from ncu CSV logs (ROW=PATH): DRAM bytes per launch of the
    row's kernels in the row's --profile case (summed over the kernels one call launches,
    averaged over the captured calls), with the units the case processed and the hash of the
    sources they are valid for."""
    import csv

    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            doc = json.load(f)
    except Exception:
        doc = {}
    doc["about"] = ("DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of each row's kernels in one call "
                    "of its bench.py --profile case, from one ncu capture, with the units that case processes; "
                    "bench.py scales them to the units of its own launch of the row and reports null once the "
                    "kernel sources no longer hash to sources_sha256.  Written by bench.py --record-traffic.")
    kern = doc.setdefault("kernels", {})
    for pair in pairs:
        row, csv_path = pair.split("=", 1)
        case, pattern, files, units = TRAFFIC_ROWS[row]
        per_id = {}
        scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}
        with open(csv_path) as f:
            lines = [ln for ln in f if ln.startswith('"')]
        recs = list(csv.reader(lines))
        hdr = recs[0]
        if "Metric Name" in hdr:            # ncu --csv --metrics ... (one row per metric)
            for rec in (dict(zip(hdr, r)) for r in recs[1:]):
                name = rec.get("Metric Name")
                if pattern not in rec.get("Kernel Name", "") or name not in ("dram__bytes_read.sum",
                                                                           "dram__bytes_write.sum"):
                    continue
                val = float(rec["Metric Value"].replace(",", "")) * scale.get(rec.get("Metric Unit", "byte"), 1)
                d = per_id.setdefault(rec["ID"], {"read": 0.0, "write": 0.0})
                d["read" if name.endswith("read.sum") else "write"] += val
        else:                               # ncu -i REP --csv --page raw --metrics ... (one row per launch)
            units_row = dict(zip(hdr, recs[1]))
            for rec in (dict(zip(hdr, r)) for r in recs[2:]):
                if pattern not in rec.get("Kernel Name", ""):
                    continue
                d = per_id.setdefault(rec["ID"], {"read": 0.0, "write": 0.0})
                for key, col in (("read", "dram__bytes_read.sum"), ("write", "dram__bytes_write.sum")):
                    d[key] += float(rec[col].replace(",", "")) * scale.get(units_row.get(col, "byte"), 1)
        if not per_id:
            raise SystemExit(f"no {pattern} launches with DRAM counters in {csv_path}")
        # a call of the case launches one kernel (two for the cast): group captured launches per call
        per_call = 2 if row == "mxfp4_to_nvfp4" else 1
        ids = sorted(per_id, key=int)
        calls = max(1, len(ids) // per_call)
        rd = sum(per_id[i]["read"] for i in ids[:calls * per_call]) / calls
        wr = sum(per_id[i]["write"] for i in ids[:calls * per_call]) / calls
        kern[row] = {"files": [f"nvfp4_block_numerics_b200/csrc/{f}" for f in files], "case": f"--profile {case}",
                     "units": units, "dram_read_bytes": int(round(rd)), "dram_write_bytes": int(round(wr)),
                     "sources_sha256": _sources_sha(files)}
        print(row, kern[row]["dram_read_bytes"], kern[row]["dram_write_bytes"])
    with open(path, "w") as f:
        json.dump(doc, f, indent=1)


def run_profile(args):
    """One kernel's launch, args.profile_reps times in a row, for an ncu capture (-k, -s, -c
    select among them); the same call the bench times."""
    import torch

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    fn, what = PROFILE_CASES[args.profile](dev, args.seed)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.profile_reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    print(json.dumps({"profile": args.profile, "case": what, "reps": args.profile_reps,
                      "ms_per_rep": a.elapsed_time(b) / args.profile_reps}), flush=True)


def main():
    args = parse_args()
    if args.record_traffic is not None:
        record_traffic(args.record_traffic)
    elif args.profile is not None:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
