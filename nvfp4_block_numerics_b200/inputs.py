"""Seeded synthetic inputs shaped like the workloads on the NVFP4 pages.

This module draws random numbers and stores them in the element formats the
library consumes (BF16 bit patterns, FP32, packed E2M1 bytes, E8M0 codes).  It
holds none of the method's arithmetic, and both the CUDA path and the CPU oracle
consume what it returns.  Every tensor is keyed by (seed, workload, tensor name)
so that any one of them can be regenerated alone.

Distributions (stand-ins for data that is not available here):
  * activations: Laplace(b=1) -- the heavy-tailed shape of LLM weights and
    activations in "FP4 quantization overview" 2.1 -- with a few outlier channels
    scaled up, the structure that makes per-16 block scales and the local Hessian
    matter;
  * calibration sequences of 4096 tokens, as in the calibration method note
    (section 1) and the DSpark recipe (--calib_seq 4096);
  * weights: N(0, sigma^2), or Student-t(4) rescaled to the same std for MoE
    experts (heavier tails);
  * MXFP4 expert weights: uniform random E2M1 nibbles with E8M0 block exponents.
"""
from __future__ import annotations

import os
import zlib
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = [
    "rng_for", "f32_to_bf16_bits", "bf16_bits_to_f32", "laplace_bf16", "normal_weights",
    "student_t_weights", "mxfp4_matrix", "c1_tiny_linear", "c2_shape", "C2_SHAPES",
    "c3_layer", "c4_expert", "c5_cast",
]


def rng_for(seed: int, workload: str, name: str) -> np.random.Generator:
    """Independent generator per (seed, workload, tensor name)."""
    key = zlib.crc32(f"{workload}/{name}".encode())
    return np.random.default_rng(np.random.SeedSequence([seed, key]))


_CHUNK = 1 << 22          # elements per independently seeded chunk
_THREADS = max(1, min(32, (os.cpu_count() or 1)))


def _chunked(rng: np.random.Generator, rows: int, cols: int, fill, out: np.ndarray):
    """Fill out[rows, cols] chunk by chunk; chunk k draws from its own child generator
    (spawned from rng), so the result does not depend on the number of threads."""
    rows_per = max(1, _CHUNK // max(cols, 1))
    bounds = [(r, min(rows, r + rows_per)) for r in range(0, rows, rows_per)]
    children = rng.spawn(len(bounds)) if bounds else []

    def run(k):
        r0, r1 = bounds[k]
        out[r0:r1] = fill(children[k], r1 - r0, r0)

    if len(bounds) > 1 and _THREADS > 1:
        with ThreadPoolExecutor(_THREADS) as ex:
            list(ex.map(run, range(len(bounds))))
    else:
        for k in range(len(bounds)):
            run(k)
    return out


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Storage conversion of finite float32 samples to BF16 bit patterns (nearest, ties even)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def _laplace_f32(rng: np.random.Generator, shape, b: float) -> np.ndarray:
    mag = rng.standard_exponential(size=shape, dtype=np.float32)
    sign = rng.integers(0, 2, size=shape, dtype=np.int8)
    mag *= np.float32(b)
    return np.where(sign == 1, -mag, mag)


def laplace_bf16(rng: np.random.Generator, rows: int, cols: int, b: float = 1.0,
                 outlier_channels=(), outlier_scale: float = 1.0,
                 zero_block_frac: float = 0.0) -> np.ndarray:
    """BF16 bits [rows, cols]: Laplace(b) rows, listed channels scaled, and a fraction of
    (row, 16-element block) pairs set to +0.0."""
    oc = np.asarray(list(outlier_channels), dtype=np.int64)

    def fill(r, n, _r0):
        v = _laplace_f32(r, (n, cols), b)
        if oc.size:
            v[:, oc] *= np.float32(outlier_scale)
        if zero_block_frac > 0.0:
            nb = cols // 16
            z = r.random((n, nb)) < zero_block_frac
            v.reshape(n, nb, 16)[z] = 0.0
        return f32_to_bf16_bits(v)

    return _chunked(rng, rows, cols, fill, np.empty((rows, cols), np.uint16))


def normal_weights(rng: np.random.Generator, rows: int, cols: int, std: float) -> np.ndarray:
    def fill(r, n, _r0):
        return r.standard_normal((n, cols), dtype=np.float32) * np.float32(std)

    return _chunked(rng, rows, cols, fill, np.empty((rows, cols), np.float32))


def student_t_weights(rng: np.random.Generator, rows: int, cols: int, std: float) -> np.ndarray:
    """Student-t with 4 degrees of freedom scaled to the given standard deviation.
    t_4 = Z / sqrt(V/4) with V ~ chi-square(4) = 2*(E1 + E2), E exponential(1); Var(t_4) = 2."""
    def fill(r, n, _r0):
        z = r.standard_normal((n, cols), dtype=np.float32)
        e = r.standard_exponential((n, cols), dtype=np.float32)
        e += r.standard_exponential((n, cols), dtype=np.float32)
        return z * np.sqrt(np.float32(2.0) / e) * np.float32(std / np.sqrt(2.0))

    return _chunked(rng, rows, cols, fill, np.empty((rows, cols), np.float32))


def mxfp4_matrix(rng: np.random.Generator, rows: int, cols: int, mean_exp: float = -8.0,
                 std_exp: float = 2.0, fallback_frac: float = 0.001):
    """MXFP4 matrix: uniform random E2M1 nibbles (all 16 codes, two per byte) and one
    E8M0 code per 32 elements, code = 127 + round(N(mean_exp, std_exp)); a fraction of
    the blocks is forced 18..20 binades below the matrix's largest exponent."""
    q = rng.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)
    k = np.rint(rng.normal(mean_exp, std_exp, size=(rows, cols // 32))).astype(np.int64)
    codes = np.clip(127 + k, 0, 254)
    kmax = int(codes.max())
    n = codes.size
    nf = int(round(fallback_frac * n))
    if nf:
        pick = rng.choice(n, size=nf, replace=False)
        low = kmax - 18 - rng.integers(0, 3, size=nf)
        codes.reshape(-1)[pick] = np.clip(low, 0, 254)
    return q, codes.astype(np.uint8)


# ----------------------------------------------------------------- workloads
def c1_tiny_linear(seed: int = 0):
    """Tiny single Linear: W 128x256 FP32 N(0, 0.02^2) with input columns 3 and 77 x20;
    calibration X 256 tokens x 256 BF16 Laplace(1) with channels 5, 40, 130, 200 x30."""
    w = normal_weights(rng_for(seed, "c1", "W"), 128, 256, 0.02)
    w[:, [3, 77]] *= np.float32(20.0)
    x = laplace_bf16(rng_for(seed, "c1", "X"), 256, 256, outlier_channels=(5, 40, 130, 200),
                     outlier_scale=30.0)
    return {"W": np.ascontiguousarray(w), "X": x}


C2_SHAPES = [(t, c) for c in (2048, 4096, 7168) for t in (1, 16, 256, 4096, 65536)]


def c2_shape(T: int, C: int, seed: int = 0):
    """Dynamic activation quant input: BF16 [T, C] Laplace(1), round(0.005*C) outlier
    channels x50 (seeded choice), 1% of (row, block) pairs exactly +0.0."""
    r = rng_for(seed, "c2", f"X_{T}x{C}")
    n_out = int(round(0.005 * C))
    oc = np.sort(r.choice(C, size=n_out, replace=False))
    return laplace_bf16(r, T, C, outlier_channels=oc, outlier_scale=50.0, zero_block_frac=0.01)


def c3_layer(seed: int = 0, tokens: int = 16384, hidden: int = 2048, inter: int = 16384,
             which=("X", "X_down", "W_q", "W_gate", "W_up", "W_down")):
    """Gemma-2B-like decoder layer: X [4x4096 tokens, 2048] Laplace with 8 outlier channels
    x40 (input of q_proj, gate, up); X_down [tokens, 16384] with the same distribution;
    weights BF16 N(0, 0.02^2): q 2048x2048, gate/up 16384x2048, down 2048x16384."""
    out = {}
    for name in which:
        r = rng_for(seed, "c3", name)
        if name == "X":
            oc = r.choice(hidden, size=8, replace=False)
            out[name] = laplace_bf16(r, tokens, hidden, outlier_channels=oc, outlier_scale=40.0)
        elif name == "X_down":
            oc = r.choice(inter, size=8, replace=False)
            out[name] = laplace_bf16(r, tokens, inter, outlier_channels=oc, outlier_scale=40.0)
        else:
            shape = {"W_q": (hidden, hidden), "W_gate": (inter, hidden), "W_up": (inter, hidden),
                     "W_down": (hidden, inter)}[name]
            out[name] = f32_to_bf16_bits(normal_weights(r, shape[0], shape[1], 0.02))
    return out


def c4_expert(e: int, seed: int = 0, hidden: int = 4096, inter: int = 1536, tokens: int = 2048,
              which=("X", "X_down", "W_gate", "W_up", "W_down")):
    """One MoE expert: gate/up W [1536, 4096] and down W [4096, 1536], BF16 Student-t(4)
    with std 0.015; routed calibration X [2048, 4096] and X_down [2048, 1536] Laplace(1)."""
    out = {}
    for name in which:
        r = rng_for(seed, "c4", f"e{e}/{name}")
        if name == "X":
            out[name] = laplace_bf16(r, tokens, hidden)
        elif name == "X_down":
            out[name] = laplace_bf16(r, tokens, inter)
        else:
            shape = {"W_gate": (inter, hidden), "W_up": (inter, hidden), "W_down": (hidden, inter)}[name]
            out[name] = f32_to_bf16_bits(student_t_weights(r, shape[0], shape[1], 0.015))
    return out


def c5_cast(i: int, seed: int = 0, rows: int = 2880, cols: int = 2880):
    """MXFP4 expert matrix i of 32: 2880x2880 uniform nibbles, E8M0 k_j = 127 + round(N(-8, 2)),
    0.1% of blocks forced >= 18 below k_max."""
    return mxfp4_matrix(rng_for(seed, "c5", f"m{i}"), rows, cols)
