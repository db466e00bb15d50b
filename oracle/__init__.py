"""CPU oracle for the NVFP4 block-numerics hot path (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps the plain C99 library built from
the ``*.c`` files beside this file (FP64, exact comparisons) and shares nothing
with the CUDA library: no code, headers, tables or constants, and it never
imports the product package.

Rows (or Hessian blocks) are fanned out over a thread pool; the C calls release
the GIL, so the threads run in parallel.  Each function's definition and source
page is documented in the C file that implements it.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
_SOURCES = ["formats.c", "act.c", "hessian.c", "sweep.c", "cast.c", "variants.c"]
_LIB_PATH = os.path.join(_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

BF16, F32 = 0, 2
FLAG_NONFINITE, FLAG_E8M0_NAN, FLAG_OVERFLOW = 1, 2, 4


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (no FMA contraction, no fast-math)."""
    srcs = [os.path.join(_DIR, s) for s in _SOURCES]
    hdr = os.path.join(_DIR, "nv4_oracle.h")
    if not force and os.path.exists(_LIB_PATH):
        newest = max(os.path.getmtime(p) for p in srcs + [hdr])
        if os.path.getmtime(_LIB_PATH) >= newest:
            return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fPIC", "-shared",
           "-ffp-contract=off", "-fno-fast-math", *srcs, "-lm", "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = C.CDLL(_LIB_PATH)
            vp, i64, u32p = C.c_void_p, C.c_int64, C.POINTER(C.c_uint32)
            sig = {
                "orc_e2m1_value": (C.c_double, [C.c_uint]),
                "orc_e4m3_value": (C.c_double, [C.c_uint]),
                "orc_e8m0_value": (C.c_double, [C.c_uint]),
                "orc_e4m3_encode": (C.c_uint, [C.c_double, C.c_double]),
                "orc_e2m1_encode": (C.c_uint, [C.c_double, C.c_double]),
                "orc_s2_from_amax": (C.c_float, [C.c_float]),
                "orc_bf16_value": (C.c_double, [C.c_uint16]),
                "orc_f32_to_bf16": (C.c_uint16, [C.c_float]),
                "orc_f32_to_f16": (C.c_uint16, [C.c_float]),
                "orc_tensor_amax": (C.c_float, [vp, C.c_int, i64, u32p]),
                "orc_act_quant": (C.c_float, [vp, i64, i64, i64, C.c_float, i64, i64, vp, vp, u32p]),
                "orc_block_quant": (C.c_float, [vp, C.c_int, i64, i64, i64, C.c_float, i64, i64, vp, vp, u32p]),
                "orc_dequant": (None, [vp, vp, C.c_float, i64, i64, C.c_int, i64, i64, vp]),
                "orc_mxfp4_quant": (None, [vp, C.c_int, i64, i64, i64, i64, vp, vp, u32p]),
                "orc_mxfp4_dequant": (None, [vp, vp, i64, i64, i64, C.c_int, vp]),
                "orc_fp8_quant": (C.c_float, [vp, C.c_int, i64, i64, C.c_float, i64, i64, vp, u32p]),
                "orc_hessian_accum": (None, [vp, i64, i64, i64, i64, i64, vp]),
                "orc_scale_sweep": (None, [vp, C.c_int, i64, i64, i64, vp, C.c_float, i64, i64,
                                           vp, vp, vp, vp, u32p]),
                "orc_mx_kmax": (C.c_int, [vp, i64, u32p]),
                "orc_mxfp4_to_nvfp4": (None, [vp, vp, i64, i64, C.c_int, i64, i64, vp, vp, vp]),
                "orc_mx_global": (None, [C.c_int, C.POINTER(C.c_float), C.POINTER(C.c_float), u32p]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype, fn.argtypes = res, args
            _lib = lib
    return _lib


def default_threads() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _chunks(n: int, parts: int):
    parts = max(1, min(parts, n))
    step = -(-n // parts)
    return [(i, min(n, i + step)) for i in range(0, n, step)]


def _fanout(fn, n: int, threads: int | None):
    threads = threads or default_threads()
    ranges = _chunks(n, threads * 4)
    if threads == 1 or len(ranges) == 1:
        for r in ranges:
            fn(*r)
        return
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(lambda r: fn(*r), ranges))


# ---------------------------------------------------------------- formats
def e2m1_value(code: int) -> float:
    return _L().orc_e2m1_value(code)


def e4m3_value(code: int) -> float:
    return _L().orc_e4m3_value(code)


def e8m0_value(code: int) -> float:
    return _L().orc_e8m0_value(code)


def e4m3_encode(num: float, den: float) -> int:
    return _L().orc_e4m3_encode(num, den)


def e2m1_encode(x: float, S: float) -> int:
    return _L().orc_e2m1_encode(x, S)


def s2_from_amax(amax: float) -> float:
    return _L().orc_s2_from_amax(amax)


def f32_to_bf16(f: float) -> int:
    return _L().orc_f32_to_bf16(f)


def f32_to_f16(f: float) -> int:
    return _L().orc_f32_to_f16(f)


# ---------------------------------------------------------------- amax
def tensor_amax(x: np.ndarray, threads: int | None = None):
    """x: uint16 (bf16 bits) or float32, any shape (contiguous).  Returns (amax, flags)."""
    x = np.ascontiguousarray(x)
    dtype = F32 if x.dtype == np.float32 else BF16
    assert x.dtype in (np.float32, np.uint16)
    flat = x.reshape(-1)
    n = flat.size
    ranges = _chunks(n, (threads or default_threads()) * 4) if n else []
    res = [None] * len(ranges)

    def run(k):
        lo, hi = ranges[k]
        f = C.c_uint32(0)
        a = _L().orc_tensor_amax(_p(flat[lo:hi]), dtype, hi - lo, C.byref(f))
        res[k] = (a, f.value)

    if len(ranges) > 1 and (threads or default_threads()) > 1:
        with ThreadPoolExecutor(threads or default_threads()) as ex:
            list(ex.map(run, range(len(ranges))))
    else:
        for k in range(len(ranges)):
            run(k)
    amax = max([r[0] for r in res], default=0.0)
    flags = 0
    for r in res:
        flags |= r[1]
    return float(np.float32(amax)), flags


# ---------------------------------------------------------------- act quant / dequant
def act_quant(x: np.ndarray, amax: float, cols: int | None = None, threads: int | None = None):
    """x: uint16 bf16 bits [rows, ld].  Returns (q [rows, cols/2], scales [rows, cols/16], s2, flags)."""
    assert x.dtype == np.uint16 and x.ndim == 2 and x.flags.c_contiguous
    rows, ld = x.shape
    cols = ld if cols is None else cols
    assert cols % 16 == 0
    q = np.zeros((rows, cols // 2), np.uint8)
    sc = np.zeros((rows, cols // 16), np.uint8)
    flags = [0]
    s2 = [0.0]
    lk = threading.Lock()

    def run(r0, r1):
        f = C.c_uint32(0)
        s = _L().orc_act_quant(_p(x), rows, cols, ld, amax, r0, r1, _p(q), _p(sc), C.byref(f))
        with lk:
            flags[0] |= f.value
            s2[0] = s

    if rows == 0:
        f = C.c_uint32(0)
        s2[0] = _L().orc_act_quant(_p(x), 0, cols, ld, amax, 0, 0, _p(q), _p(sc), C.byref(f))
    else:
        _fanout(run, rows, threads)
    return q, sc, float(np.float32(s2[0])), flags[0]


def rtn_quant(w: np.ndarray, amax: float, cols: int | None = None, threads: int | None = None):
    """Round-to-nearest weight quantization with max-calibrated block scales.

    w: float32 or uint16 (bf16 bits) [rows, ld].  The activation quantizer's
    arithmetic ([FLOW] 3.4-3.5) applied to a weight tensor with its own amax.
    Returns (q [rows, cols/2], scales [rows, cols/16], s2, flags)."""
    assert w.ndim == 2 and w.flags.c_contiguous and w.dtype in (np.float32, np.uint16)
    dt = F32 if w.dtype == np.float32 else BF16
    rows, ld = w.shape
    cols = ld if cols is None else cols
    assert cols % 16 == 0
    q = np.zeros((rows, cols // 2), np.uint8)
    sc = np.zeros((rows, cols // 16), np.uint8)
    flags = [0]
    s2 = [float(np.float32(_L().orc_s2_from_amax(amax)))]
    lk = threading.Lock()

    def run(r0, r1):
        f = C.c_uint32(0)
        _L().orc_block_quant(_p(w), dt, rows, cols, ld, amax, r0, r1, _p(q), _p(sc), C.byref(f))
        with lk:
            flags[0] |= f.value

    if rows:
        _fanout(run, rows, threads)
    else:
        f = C.c_uint32(0)
        _L().orc_block_quant(_p(w), dt, 0, cols, ld, amax, 0, 0, _p(q), _p(sc), C.byref(f))
        flags[0] |= f.value
    return q, sc, s2[0], flags[0]


def fake_qdq(x: np.ndarray, amax: float, out_dtype: str = "bf16", threads: int | None = None):
    """Quantize then dequantize ([FLOW] 3.4: quantizer followed by DQ1/DQ2), the
    plain composition of act_quant and dequant.  Returns (out, s2, flags)."""
    q, sc, s2, flags = act_quant(x, amax, threads=threads)
    return dequant(q, sc, s2, out_dtype, threads=threads), s2, flags


def dequant(q: np.ndarray, scales: np.ndarray, s2: float, out_dtype: str = "bf16",
            threads: int | None = None) -> np.ndarray:
    """Returns uint16 bits (bf16/fp16) or float32 [rows, cols]."""
    rows = q.shape[0]
    cols = q.shape[1] * 2
    code = {"bf16": 0, "fp16": 1, "fp32": 2}[out_dtype]
    out = np.zeros((rows, cols), np.float32 if code == 2 else np.uint16)
    q = np.ascontiguousarray(q)
    scales = np.ascontiguousarray(scales)
    _fanout(lambda r0, r1: _L().orc_dequant(_p(q), _p(scales), s2, rows, cols, code, r0, r1, _p(out)),
            rows, threads)
    return out


# ---------------------------------------------------------------- Hessian
def hessian_accum(x: np.ndarray, H: np.ndarray | None = None, cols: int | None = None,
                  threads: int | None = None) -> np.ndarray:
    """x: uint16 bf16 bits [tokens, ld]; returns H (float64 [cols/16, 16, 16]) += X_b^T X_b."""
    assert x.dtype == np.uint16 and x.ndim == 2 and x.flags.c_contiguous
    tokens, ld = x.shape
    cols = ld if cols is None else cols
    nblk = cols // 16
    if H is None:
        H = np.zeros((nblk, 16, 16), np.float64)
    assert H.dtype == np.float64 and H.flags.c_contiguous and H.shape == (nblk, 16, 16)
    _fanout(lambda b0, b1: _L().orc_hessian_accum(_p(x), tokens, cols, ld, b0, b1, _p(H)), nblk, threads)
    return H


# ---------------------------------------------------------------- sweep
def scale_sweep(w: np.ndarray, H: np.ndarray, amax_w: float, rows=None, cols: int | None = None,
                threads: int | None = None):
    """w: float32 or uint16 (bf16 bits) [N, ld]; H: float64 [cols/16, 16, 16].

    ``rows``: None for all rows, or an iterable of row indices (a sample); outputs
    then hold the sampled rows in the given order.  Returns a dict with codes, q,
    cost1, cost2 and flags.
    """
    assert w.ndim == 2 and w.flags.c_contiguous
    dtype = F32 if w.dtype == np.float32 else BF16
    assert w.dtype in (np.float32, np.uint16)
    N, ld = w.shape
    cols = ld if cols is None else cols
    nblk = cols // 16
    H = np.ascontiguousarray(H, dtype=np.float64)
    assert H.shape == (nblk, 16, 16)
    idx = np.arange(N) if rows is None else np.asarray(list(rows), dtype=np.int64)
    n = len(idx)
    codes = np.zeros((n, nblk), np.uint8)
    q = np.zeros((n, cols // 2), np.uint8)
    c1 = np.zeros((n, nblk), np.float64)
    c2 = np.zeros((n, nblk), np.float64)
    flags = [0]
    lk = threading.Lock()
    es = w.itemsize

    def run(k0, k1):
        f = C.c_uint32(0)
        for k in range(k0, k1):
            r = int(idx[k])
            wp = C.c_void_p(w.ctypes.data + r * ld * es)
            _L().orc_scale_sweep(wp, dtype, 1, cols, ld, _p(H), amax_w, 0, 1,
                                 _p(codes[k]), _p(q[k]), _p(c1[k]), _p(c2[k]), C.byref(f))
        with lk:
            flags[0] |= f.value

    if n:
        _fanout(run, n, threads)
    return {"codes": codes, "q": q, "cost1": c1, "cost2": c2, "flags": flags[0], "rows": idx}


# ---------------------------------------------------------------- MXFP4 -> NVFP4
def _mx_check(mx_q, e8m0):
    mx_q = np.ascontiguousarray(mx_q)
    e8m0 = np.ascontiguousarray(e8m0)
    rows, half = mx_q.shape
    assert (2 * half) % 32 == 0 and e8m0.shape == (rows, 2 * half // 32)
    return mx_q, e8m0


def _mx_kmax(e8m0):
    f = C.c_uint32(0)
    kmax = _L().orc_mx_kmax(_p(e8m0), e8m0.size, C.byref(f))
    if f.value & FLAG_E8M0_NAN:
        raise ValueError("E8M0 NaN code 0xFF in the input")
    return kmax


def mxfp4_to_nvfp4(mx_q: np.ndarray, e8m0: np.ndarray, threads: int | None = None, k_max: int | None = None):
    """One matrix: mx_q uint8 [rows, cols/2], e8m0 uint8 [rows, cols/32].

    k_max: None for the matrix's own largest exponent ([CAST] section 2, per layer),
    or a shared one (a group of matrices with one scale_2, see mxfp4_to_nvfp4_group).
    Raises ValueError on an E8M0 NaN code.  Returns a dict with nv_q, nv_scales, s2,
    global_amax, k_max, counts (in-window, fallback, lossless 16-blocks) and flags.
    """
    mx_q, e8m0 = _mx_check(mx_q, e8m0)
    rows, half = mx_q.shape
    cols = 2 * half
    kmax = _mx_kmax(e8m0) if k_max is None else int(k_max)
    f = C.c_uint32(0)
    s2 = C.c_float(0)
    ga = C.c_float(0)
    _L().orc_mx_global(kmax, C.byref(s2), C.byref(ga), C.byref(f))
    nv_q = np.zeros_like(mx_q)
    nv_s = np.zeros((rows, cols // 16), np.uint8)
    parts = []
    lk = threading.Lock()

    def run(r0, r1):
        cnt = np.zeros(3, np.int64)
        _L().orc_mxfp4_to_nvfp4(_p(mx_q), _p(e8m0), rows, cols, kmax, r0, r1, _p(nv_q), _p(nv_s), _p(cnt))
        with lk:
            parts.append(cnt)

    _fanout(run, rows, threads)
    counts = np.sum(parts, axis=0) if parts else np.zeros(3, np.int64)
    return {"nv_q": nv_q, "nv_scales": nv_s, "s2": s2.value, "global_amax": ga.value,
            "k_max": kmax, "counts": counts, "flags": f.value}


def mxfp4_to_nvfp4_group(mats, threads: int | None = None):
    """Matrices that share one scale_2 ([CAST] section 3: DeepSeek V4 routed experts,
    w1 and w3 with one scale_2).  Reading: k_max is the largest exponent over the
    union of the group's E8M0 codes, and every member is cast against it (window and
    fallback relative to the shared k_max).  mats: list of (mx_q, e8m0)."""
    mats = [_mx_check(q, e) for q, e in mats]
    kmax = max(_mx_kmax(e) for _, e in mats)
    return [mxfp4_to_nvfp4(q, e, threads, k_max=kmax) for q, e in mats]


# ---------------------------------------------------------------- W4A4 GEMM (NVFP4 x NVFP4)
def _dequant_exact(q: np.ndarray, sc: np.ndarray, s2: float) -> np.ndarray:
    """Exact dequantized values e2m1(code) * e4m3(s_b) * s2 in FP64 (each factor has at
    most 24 significant bits and the product at most 31, so FP64 holds it exactly)."""
    e2m1 = np.array([e2m1_value(c) for c in range(16)], np.float64)
    e4m3 = np.array([e4m3_value(c) for c in range(256)], np.float64)
    q = np.ascontiguousarray(q)
    nib = np.stack([q & 15, q >> 4], axis=-1).reshape(q.shape[0], -1)
    s = np.repeat(e4m3[np.ascontiguousarray(sc)], 16, axis=1)
    return e2m1[nib] * s * float(s2)


def gemm_nvfp4(qa, sa, s2a: float, qb, sb, s2b: float):
    """NVFP4 x NVFP4 GEMM, D[m, n] = sum_k A[m, k] * B[n, k] with A and B the exact
    dequantized values of packed codes q [rows, K/2], E4M3 scales [rows, K/16] and FP32
    second-level scales ([FP4] section 4.1: block-scaled FP4 matrix multiply on tcgen05;
    [CAST] section 4: W4A4, activations and weights both NVFP4).

    Returns (D, Dabs): D in FP64 (the product of the exactly dequantized matrices, one
    library matmul), and Dabs = |A| |B|^T, the scale of the accumulation error bound."""
    A = _dequant_exact(qa, sa, s2a)
    B = _dequant_exact(qb, sb, s2b)
    return A @ B.T, np.abs(A) @ np.abs(B).T


def scales_to_mma_layout(sc: np.ndarray) -> np.ndarray:
    """Block-scale bytes [rows, kb] (kb = K/16) rearranged into the layout that the
    Blackwell block-scaled MMA reads ([FP4] section 4.1: scale factors reorganized for
    tcgen05.mma): 512-byte atoms of 128 rows x 4 scales, atom (r // 128, j // 4) at
    ((r // 128) * ceil(kb / 4) + j // 4) * 512, and inside an atom row r, scale j at
    (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4.  Rows and scale columns are padded
    with zeros to multiples of 128 and 4."""
    rows, kb = sc.shape
    rt, kt = -(-rows // 128), -(-kb // 4)
    out = np.zeros(rt * kt * 512, np.uint8)
    r = np.arange(rows)[:, None]
    j = np.arange(kb)[None, :]
    off = ((r // 128) * kt + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4
    out[off] = sc
    return out


# ---------------------------------------------------------------- format variants
def mxfp4_quant(x: np.ndarray, cols: int | None = None, threads: int | None = None):
    """MXFP4 round-to-nearest quantization ([FP4] sections 1.2 and 3.2): 32-element blocks,
    E8M0 shared exponent floor(log2 amax) - 2, E2M1 elements.  x: float32 or uint16
    (bf16 bits) [rows, ld].  Returns (q [rows, cols/2], e8m0 [rows, cols/32], flags)."""
    assert x.ndim == 2 and x.flags.c_contiguous and x.dtype in (np.float32, np.uint16)
    dt = F32 if x.dtype == np.float32 else BF16
    rows, ld = x.shape
    cols = ld if cols is None else cols
    assert cols % 32 == 0
    q = np.zeros((rows, cols // 2), np.uint8)
    e = np.zeros((rows, cols // 32), np.uint8)
    flags = [0]
    lk = threading.Lock()

    def run(r0, r1):
        f = C.c_uint32(0)
        _L().orc_mxfp4_quant(_p(x), dt, cols, ld, r0, r1, _p(q), _p(e), C.byref(f))
        with lk:
            flags[0] |= f.value

    if rows:
        _fanout(run, rows, threads)
    return q, e, flags[0]


def mxfp4_dequant(q: np.ndarray, e8m0: np.ndarray, out_dtype: str = "bf16", threads: int | None = None):
    """e2m1(code) * 2^(e8m0 - 127), rounded once to the output type."""
    rows, cols = q.shape[0], 2 * q.shape[1]
    code = {"bf16": 0, "fp16": 1, "fp32": 2}[out_dtype]
    out = np.zeros((rows, cols), np.float32 if code == 2 else np.uint16)
    q, e8m0 = np.ascontiguousarray(q), np.ascontiguousarray(e8m0)
    _fanout(lambda r0, r1: _L().orc_mxfp4_dequant(_p(q), _p(e8m0), cols, r0, r1, code, _p(out)), rows, threads)
    return out


def fp8_quant(x: np.ndarray, amax: float, cols: int | None = None, threads: int | None = None):
    """FP8 E4M3 with one static per-tensor scale ([CAL] layer table: W8A8 layers):
    s = RN32(amax / 448), code = sign | nearest E4M3 to |x| / s.  Returns (q, s, flags)."""
    assert x.ndim == 2 and x.flags.c_contiguous and x.dtype in (np.float32, np.uint16)
    dt = F32 if x.dtype == np.float32 else BF16
    rows, ld = x.shape
    cols = ld if cols is None else cols
    q = np.zeros((rows, cols), np.uint8)
    flags = [0]
    s = [float(np.float32(amax / 448.0))]
    lk = threading.Lock()

    def run(r0, r1):
        f = C.c_uint32(0)
        s[0] = _L().orc_fp8_quant(_p(x), dt, cols, ld, amax, r0, r1, _p(q), C.byref(f))
        with lk:
            flags[0] |= f.value

    if rows:
        _fanout(run, rows, threads)
    return q, float(np.float32(s[0])), flags[0]


def fp8_dequant(q: np.ndarray, s: float) -> np.ndarray:
    """Exact values e4m3(code) * s (FP64); the caller rounds to its output type."""
    tab = np.array([e4m3_value(c) for c in range(256)], np.float64)
    return tab[np.ascontiguousarray(q)] * float(s)


# ---------------------------------------------------------------- block Hadamard rotation
def _sylvester(n: int) -> np.ndarray:
    """H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]] (the natural-order Hadamard matrix)."""
    H = np.ones((1, 1), np.float64)
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def hadamard_rotate(x: np.ndarray, n: int) -> np.ndarray:
    """Block Hadamard rotation along each row ([FP4] section 3.1: blocks of 16..128 values
    rotated by H / sqrt(n) before FP4 quantization; section 4.1: block sizes 16/32/64/128).
    Reading: y = RN32(RN64(x_block @ H_n) * RN64(1 / sqrt(n))), the Hadamard sums in FP64
    (exact for BF16 inputs whose values in a block span fewer than ~38 binades).
    x: float32 or uint16 (bf16 bits) [rows, cols], cols % n == 0.  Returns float32."""
    assert n in (16, 32, 64, 128) and x.ndim == 2 and x.shape[1] % n == 0
    xf = (x.astype(np.uint32) << 16).view(np.float32) if x.dtype == np.uint16 else x
    rows, cols = xf.shape
    z = xf.astype(np.float64).reshape(rows, cols // n, n) @ _sylvester(n)     # H_n is symmetric
    c = float(np.float64(1.0) / np.sqrt(np.float64(n)))
    return (z * c).astype(np.float32).reshape(rows, cols)


def _rn32_of_int(N: int, k: int) -> float:
    """RN32(N * 2^k) for an integer N, ties to even, with FP32 subnormals and overflow to
    infinity; returned as a Python float (exactly representable)."""
    if N == 0:
        return 0.0
    sign = -1.0 if N < 0 else 1.0
    N = abs(N)
    e = N.bit_length() - 1 + k                  # exponent of the leading bit
    lsb = max(e - 23, -149)                     # exponent of the last bit FP32 keeps
    shift = lsb - k
    if shift > 0:
        q, r = divmod(N, 1 << shift)
        half = 1 << (shift - 1)
        if r > half or (r == half and q & 1):
            q += 1
    else:
        q = N << (-shift)
    v = float(q) * 2.0 ** lsb                   # q <= 2^24: exact
    return sign * v if v < 2.0 ** 128 else sign * float("inf")


def hadamard2_rotate(w: np.ndarray, n: int) -> np.ndarray:
    """Two-sided block Hadamard rotation of weight tiles ([FP4] section 3.1: the weight
    matrix is cut into n x n tiles, n = 16 or 32, and each tile B becomes
    (H / sqrt(n)) B (H / sqrt(n))^T = H B H^T / n, H the natural-order Hadamard matrix).
    Reading: y = RN32(exact(H B H^T) / n): 1/n is a power of two, so the final rounding to
    FP32 is the only one.  The tile's sums are formed in FP64 where that is exact (every
    value an integer multiple of the tile's smallest unit in the last place, and the sums,
    with their 2 log2(n) bits of growth, inside 53 bits), else in Python integers.
    w: float32 or uint16 (bf16 bits) [rows, cols], rows and cols multiples of n.
    Returns float32 [rows, cols]."""
    assert n in (16, 32) and w.ndim == 2 and w.shape[0] % n == 0 and w.shape[1] % n == 0
    wf = (w.astype(np.uint32) << 16).view(np.float32) if w.dtype == np.uint16 else w
    rows, cols = wf.shape
    H = _sylvester(n)
    growth = 2 * int(np.log2(n))
    out = np.empty((rows, cols), np.float32)
    for r0 in range(0, rows, n):
        for c0 in range(0, cols, n):
            B = wf[r0:r0 + n, c0:c0 + n].astype(np.float64)
            nz = np.abs(B[B != 0.0])
            if nz.size == 0:
                out[r0:r0 + n, c0:c0 + n] = 0.0
                continue
            hi = int(np.frexp(nz.max())[1])                      # 2^(hi-1) <= max < 2^hi
            ulp = int(np.frexp(nz)[1].min()) - 24                 # every FP32 value is a multiple of 2^ulp
            ulp = max(ulp, -149)
            if hi - ulp + growth <= 53:
                Y = H @ B @ H.T                                   # exact: integers times 2^ulp below 2^53
                out[r0:r0 + n, c0:c0 + n] = (Y / n).astype(np.float32)
            else:
                Bi = np.array([[int(v) for v in row] for row in np.ldexp(B, -ulp)], dtype=object)
                Hi = H.astype(np.int64).astype(object)
                Yi = Hi.dot(Bi).dot(Hi.T)
                lg = int(np.log2(n))
                for i in range(n):
                    for j in range(n):
                        out[r0 + i, c0 + j] = _rn32_of_int(int(Yi[i, j]), ulp - lg)
    return out
