"""Thin ctypes binding of libnv4.so (declared in include/nv4.h).

Argument marshalling only: torch tensors provide device memory and the current
CUDA stream; every step of the computation runs in the library's sm_100a
kernels.  The functions carry the C names.  A missing or unloadable library is
an error -- there is no fallback implementation.

Convenience wrappers at the end (``tensor_amax``, ``act_quant`` ...) allocate
their outputs with torch and call the same entry points.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

import torch

from .build import LIB_PATH

__all__ = [
    "NV4Error", "lib", "nv4_selftest_wait", "nv4_tensor_amax", "nv4_act_quant", "nv4_weight_quant_rtn", "nv4_fake_qdq",
    "nv4_dequant", "nv4_hessian_accum", "weight_quant_rtn", "fake_qdq", "nv4_mma_scale_bytes",
    "nv4_scales_to_mma_layout", "nv4_gemm_nvfp4", "mma_scales", "gemm_nvfp4", "nv4_mxfp4_quant",
    "nv4_mxfp4_dequant", "nv4_fp8_quant", "nv4_fp8_dequant", "mxfp4_quant", "fp8_quant", "nv4_hadamard_amax",
    "nv4_hadamard_mxfp4_quant", "nv4_hadamard_nvfp4_quant", "hadamard_mxfp4_quant", "hadamard_nvfp4_quant",
    "nv4_hessian_accum_batched", "nv4_scale_sweep", "nv4_scale_sweep_batched", "nv4_mxfp4_to_nvfp4",
    "nv4_mxfp4_to_nvfp4_batched", "nv4_selftest", "nv4_version", "FLAG_NONFINITE", "FLAG_E8M0_NAN",
    "FLAG_OVERFLOW", "FLAG_TIMEOUT", "tensor_amax", "act_quant", "dequant", "hessian_accum",
    "scale_sweep", "mxfp4_to_nvfp4", "HessianJob", "SweepJob", "CastJob", "AmaxJob", "ActJob", "DequantJob",
    "nv4_tensor_amax_batched", "nv4_act_quant_batched", "nv4_dequant_batched", "nv4_weight_quant_rtn_batched",
]

BF16, FP16, FP32 = 0, 1, 2
FLAG_NONFINITE, FLAG_E8M0_NAN, FLAG_OVERFLOW, FLAG_TIMEOUT = 1, 2, 4, 8
_DT = {torch.bfloat16: BF16, torch.float16: FP16, torch.float32: FP32}

_vp, _i64 = C.c_void_p, C.c_int64


class AmaxJob(C.Structure):
    _fields_ = [("x", _vp), ("n", _i64), ("d_amax", _vp)]


class ActJob(C.Structure):
    _fields_ = [("x", _vp), ("rows", _i64), ("cols", _i64), ("ld", _i64), ("d_amax", _vp), ("q", _vp),
                ("scales", _vp), ("d_s2", _vp)]


class DequantJob(C.Structure):
    _fields_ = [("q", _vp), ("scales", _vp), ("d_s2", _vp), ("rows", _i64), ("cols", _i64), ("out", _vp)]


class HessianJob(C.Structure):
    _fields_ = [("x", _vp), ("tokens", _i64), ("cols", _i64), ("ld", _i64), ("H", _vp)]


class SweepJob(C.Structure):
    _fields_ = [("w", _vp), ("rows", _i64), ("cols", _i64), ("ld", _i64), ("H", _vp), ("d_amax_w", _vp),
                ("codes", _vp), ("q", _vp), ("cost1", _vp), ("cost2", _vp), ("d_work", _vp)]


class CastJob(C.Structure):
    _fields_ = [("mx_q", _vp), ("e8m0", _vp), ("rows", _i64), ("cols", _i64), ("nv_q", _vp),
                ("nv_scales", _vp), ("d_global_amax", _vp), ("d_s2", _vp), ("group", C.c_int32)]


class NV4Error(RuntimeError):
    pass


_lock = threading.Lock()
_lib = None

_SIGS = {
    "nv4_status_str": (C.c_char_p, [C.c_int]),
    "nv4_version": (C.c_int, []),
    "nv4_tensor_amax": (C.c_int, [_vp, C.c_int, _i64, _vp, _vp, _vp]),
    "nv4_act_quant": (C.c_int, [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "nv4_tensor_amax_batched": (C.c_int, [C.POINTER(AmaxJob), C.c_int, C.c_int, _vp, _vp]),
    "nv4_act_quant_batched": (C.c_int, [C.POINTER(ActJob), C.c_int, _vp, _vp]),
    "nv4_weight_quant_rtn_batched": (C.c_int, [C.POINTER(ActJob), C.c_int, C.c_int, _vp, _vp]),
    "nv4_dequant_batched": (C.c_int, [C.POINTER(DequantJob), C.c_int, C.c_int, _vp]),
    "nv4_weight_quant_rtn": (C.c_int, [_vp, C.c_int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "nv4_fake_qdq": (C.c_int, [_vp, _i64, _i64, _i64, _vp, C.c_int, _vp, _i64, _vp, _vp, _vp]),
    "nv4_dequant": (C.c_int, [_vp, _vp, _vp, _i64, _i64, C.c_int, _vp, _vp]),
    "nv4_mma_scale_bytes": (C.c_size_t, [_i64, _i64]),
    "nv4_selftest_wait": (C.c_int, [_vp, C.c_uint64, _vp, _vp]),
    "nv4_mxfp4_quant": (C.c_int, [_vp, C.c_int, _i64, _i64, _i64, _vp, _vp, _vp, _vp]),
    "nv4_mxfp4_dequant": (C.c_int, [_vp, _vp, _i64, _i64, C.c_int, _vp, _vp]),
    "nv4_fp8_quant": (C.c_int, [_vp, C.c_int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp]),
    "nv4_fp8_dequant": (C.c_int, [_vp, _vp, _i64, _i64, C.c_int, _vp, _vp]),
    "nv4_hadamard_amax": (C.c_int, [_vp, _i64, _i64, _i64, C.c_int, _vp, _vp, _vp]),
    "nv4_hadamard_mxfp4_quant": (C.c_int, [_vp, _i64, _i64, _i64, C.c_int, _vp, _vp, _vp, _vp]),
    "nv4_hadamard_nvfp4_quant": (C.c_int, [_vp, _i64, _i64, _i64, C.c_int, _vp, _vp, _vp, _vp, _vp, _vp]),
    "nv4_scales_to_mma_layout": (C.c_int, [_vp, _i64, _i64, _vp, _vp]),
    "nv4_gemm_nvfp4": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, C.c_int, _vp, _i64, _vp, _vp]),
    "nv4_hessian_accum": (C.c_int, [_vp, _i64, _i64, _i64, _vp, _vp, _vp]),
    "nv4_hessian_accum_batched": (C.c_int, [C.POINTER(HessianJob), C.c_int, _vp, _vp]),
    "nv4_scale_sweep": (C.c_int, [_vp, C.c_int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "nv4_scale_sweep_batched": (C.c_int, [C.POINTER(SweepJob), C.c_int, C.c_int, _vp, _vp]),
    "nv4_mxfp4_to_nvfp4": (C.c_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "nv4_mxfp4_to_nvfp4_batched": (C.c_int, [C.POINTER(CastJob), C.c_int, _vp, _vp, _vp]),
    "nv4_selftest": (C.c_int, [_vp, _vp]),
    "nv4_fp32_probe": (C.c_int, [C.c_int, C.c_uint32, C.c_uint32, _vp, _vp]),
    "nv4_hadamard2_rotate": (C.c_int, [_vp, C.c_int, _i64, _i64, _i64, C.c_int, _vp, _vp, _vp]),
    "nv4_hadamard2_amax": (C.c_int, [_vp, C.c_int, _i64, _i64, _i64, C.c_int, _vp, _vp, _vp]),
    "nv4_hadamard2_mxfp4_quant": (C.c_int, [_vp, C.c_int, _i64, _i64, _i64, C.c_int, _vp, _vp, _vp, _vp]),
    "nv4_hadamard2_nvfp4_quant": (C.c_int, [_vp, C.c_int, _i64, _i64, _i64, C.c_int, _vp, _vp, _vp, _vp, _vp, _vp]),
}


def lib() -> C.CDLL:
    """Load libnv4.so (built in-tree by nvfp4_block_numerics_b200.build)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise NV4Error(f"{LIB_PATH} is missing: build it with nvfp4_block_numerics_b200.build.build_library()")
            L = C.CDLL(LIB_PATH)
            for name, (res, args) in _SIGS.items():
                fn = getattr(L, name)
                fn.restype, fn.argtypes = res, args
            _lib = L
    return _lib


def _check(status: int, what: str):
    if status != 0:
        raise NV4Error(f"{what}: {lib().nv4_status_str(status).decode()}")


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise NV4Error("tensor must live on a CUDA device")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _rowmajor(x: torch.Tensor, name: str):
    if x.dim() != 2 or x.stride(1) != 1:
        raise NV4Error(f"{name} must be a 2-D tensor with unit column stride")
    return x.shape[0], x.shape[1], x.stride(0)


def _scalar_f32(t: torch.Tensor, name: str):
    if t.dtype != torch.float32 or t.numel() < 1 or not t.is_cuda:
        raise NV4Error(f"{name} must be a float32 CUDA tensor")
    return t.data_ptr()


def nv4_version() -> int:
    return lib().nv4_version()


# ------------------------------------------------------------------ raw entry points
def nv4_tensor_amax(x: torch.Tensor, d_amax: torch.Tensor, d_flags: torch.Tensor | None = None, stream=None):
    if x.dtype not in (torch.bfloat16, torch.float32) or not x.is_contiguous():
        raise NV4Error("x must be a contiguous bf16 or float32 tensor")
    _check(lib().nv4_tensor_amax(_ptr(x), _DT[x.dtype], x.numel(), _scalar_f32(d_amax, "d_amax"),
                                 _ptr(d_flags), _stream(stream)), "nv4_tensor_amax")


def nv4_act_quant(x: torch.Tensor, d_amax: torch.Tensor, q: torch.Tensor, scales: torch.Tensor,
                  d_s2: torch.Tensor, d_flags: torch.Tensor | None = None, stream=None):
    if x.dtype != torch.bfloat16:
        raise NV4Error("x must be bf16")
    rows, cols, ld = _rowmajor(x, "x")
    if q.dtype != torch.uint8 or tuple(q.shape) != (rows, cols // 2) or not q.is_contiguous():
        raise NV4Error("q must be a contiguous uint8 tensor [rows, cols/2]")
    if scales.dtype != torch.uint8 or tuple(scales.shape) != (rows, cols // 16) or not scales.is_contiguous():
        raise NV4Error("scales must be a contiguous uint8 tensor [rows, cols/16]")
    _check(lib().nv4_act_quant(_ptr(x), rows, cols, ld, _scalar_f32(d_amax, "d_amax"), _ptr(q), _ptr(scales),
                               _scalar_f32(d_s2, "d_s2"), _ptr(d_flags), _stream(stream)), "nv4_act_quant")


def nv4_tensor_amax_batched(xs, d_amaxes, d_flags: torch.Tensor | None = None, stream=None):
    """The amax of every tensor of xs (one dtype, contiguous) into the matching d_amaxes entry,
    in one launch."""
    if len(xs) != len(d_amaxes):
        raise NV4Error("one d_amax per tensor")
    if not xs:
        return
    dt = xs[0].dtype
    if dt not in (torch.bfloat16, torch.float32) or any(x.dtype != dt or not x.is_contiguous() for x in xs):
        raise NV4Error("xs must be contiguous tensors of one dtype, bf16 or float32")
    arr = (AmaxJob * len(xs))(*[AmaxJob(_ptr(x), x.numel(), _scalar_f32(a, "d_amax")) for x, a in zip(xs, d_amaxes)])
    _check(lib().nv4_tensor_amax_batched(arr, len(xs), _DT[dt], _ptr(d_flags), _stream(stream)),
           "nv4_tensor_amax_batched")


def nv4_act_quant_batched(jobs: list[dict], d_flags: torch.Tensor | None = None, stream=None):
    """jobs: dicts with keys x (bf16 [rows, cols]), d_amax, q, scales, d_s2 -- nv4_act_quant per
    tensor, in one launch."""
    arr = (ActJob * len(jobs))()
    for i, j in enumerate(jobs):
        x = j["x"]
        if x.dtype != torch.bfloat16:
            raise NV4Error("x must be bf16")
        rows, cols, ld = _rowmajor(x, "x")
        q, sc = j["q"], j["scales"]
        if q.dtype != torch.uint8 or tuple(q.shape) != (rows, cols // 2) or not q.is_contiguous():
            raise NV4Error("q must be a contiguous uint8 tensor [rows, cols/2]")
        if sc.dtype != torch.uint8 or tuple(sc.shape) != (rows, cols // 16) or not sc.is_contiguous():
            raise NV4Error("scales must be a contiguous uint8 tensor [rows, cols/16]")
        arr[i] = ActJob(_ptr(x), rows, cols, ld, _scalar_f32(j["d_amax"], "d_amax"), _ptr(q), _ptr(sc),
                        _scalar_f32(j["d_s2"], "d_s2"))
    _check(lib().nv4_act_quant_batched(arr, len(jobs), _ptr(d_flags), _stream(stream)), "nv4_act_quant_batched")


def nv4_weight_quant_rtn_batched(jobs: list[dict], d_flags: torch.Tensor | None = None, stream=None):
    """jobs: dicts with keys w (bf16 or float32 [rows, cols], one dtype), d_amax, q, scales,
    d_s2 -- nv4_weight_quant_rtn per tensor, in one launch."""
    if not jobs:
        return
    dt = jobs[0]["w"].dtype
    if dt not in (torch.bfloat16, torch.float32):
        raise NV4Error("w must be bf16 or float32")
    arr = (ActJob * len(jobs))()
    for i, j in enumerate(jobs):
        w = j["w"]
        if w.dtype != dt:
            raise NV4Error("all weights of one call must share a dtype")
        rows, cols, ld = _rowmajor(w, "w")
        q, sc = j["q"], j["scales"]
        if q.dtype != torch.uint8 or tuple(q.shape) != (rows, cols // 2) or not q.is_contiguous():
            raise NV4Error("q must be a contiguous uint8 tensor [rows, cols/2]")
        if sc.dtype != torch.uint8 or tuple(sc.shape) != (rows, cols // 16) or not sc.is_contiguous():
            raise NV4Error("scales must be a contiguous uint8 tensor [rows, cols/16]")
        arr[i] = ActJob(_ptr(w), rows, cols, ld, _scalar_f32(j["d_amax"], "d_amax"), _ptr(q), _ptr(sc),
                        _scalar_f32(j["d_s2"], "d_s2"))
    _check(lib().nv4_weight_quant_rtn_batched(arr, len(jobs), _DT[dt], _ptr(d_flags), _stream(stream)),
           "nv4_weight_quant_rtn_batched")


def nv4_dequant_batched(jobs: list[dict], stream=None):
    """jobs: dicts with keys q, scales, d_s2, out (all outputs of one dtype) -- nv4_dequant per
    tensor, in one launch."""
    if not jobs:
        return
    dt = jobs[0]["out"].dtype
    arr = (DequantJob * len(jobs))()
    for i, j in enumerate(jobs):
        q, sc, out = j["q"], j["scales"], j["out"]
        if out.dtype != dt or out.dtype not in _DT or not out.is_contiguous() or out.dim() != 2:
            raise NV4Error("outs must be contiguous 2-D tensors of one dtype (bf16, fp16 or float32)")
        rows, cols = out.shape
        if tuple(q.shape) != (rows, cols // 2) or tuple(sc.shape) != (rows, cols // 16):
            raise NV4Error("q / scales shapes do not match out")
        if not (q.is_contiguous() and sc.is_contiguous()):
            raise NV4Error("q and scales must be contiguous")
        arr[i] = DequantJob(_ptr(q), _ptr(sc), _scalar_f32(j["d_s2"], "d_s2"), rows, cols, _ptr(out))
    _check(lib().nv4_dequant_batched(arr, len(jobs), _DT[dt], _stream(stream)), "nv4_dequant_batched")


def nv4_weight_quant_rtn(w: torch.Tensor, d_amax: torch.Tensor, q: torch.Tensor, scales: torch.Tensor,
                         d_s2: torch.Tensor, d_flags: torch.Tensor | None = None, stream=None):
    if w.dtype not in (torch.bfloat16, torch.float32):
        raise NV4Error("w must be bf16 or float32")
    rows, cols, ld = _rowmajor(w, "w")
    if q.dtype != torch.uint8 or tuple(q.shape) != (rows, cols // 2) or not q.is_contiguous():
        raise NV4Error("q must be a contiguous uint8 tensor [rows, cols/2]")
    if scales.dtype != torch.uint8 or tuple(scales.shape) != (rows, cols // 16) or not scales.is_contiguous():
        raise NV4Error("scales must be a contiguous uint8 tensor [rows, cols/16]")
    _check(lib().nv4_weight_quant_rtn(_ptr(w), _DT[w.dtype], rows, cols, ld, _scalar_f32(d_amax, "d_amax"), _ptr(q),
                                      _ptr(scales), _scalar_f32(d_s2, "d_s2"), _ptr(d_flags), _stream(stream)),
           "nv4_weight_quant_rtn")


def nv4_fake_qdq(x: torch.Tensor, d_amax: torch.Tensor, out: torch.Tensor, d_s2: torch.Tensor,
                 d_flags: torch.Tensor | None = None, stream=None):
    if x.dtype != torch.bfloat16:
        raise NV4Error("x must be bf16")
    if out.dtype not in _DT:
        raise NV4Error("out must be bf16, float16 or float32")
    rows, cols, ld = _rowmajor(x, "x")
    orows, ocols, ld_out = _rowmajor(out, "out")
    if (orows, ocols) != (rows, cols):
        raise NV4Error("out must have the shape of x")
    _check(lib().nv4_fake_qdq(_ptr(x), rows, cols, ld, _scalar_f32(d_amax, "d_amax"), _DT[out.dtype], _ptr(out),
                              ld_out, _scalar_f32(d_s2, "d_s2"), _ptr(d_flags), _stream(stream)), "nv4_fake_qdq")


def nv4_dequant(q: torch.Tensor, scales: torch.Tensor, d_s2: torch.Tensor, out: torch.Tensor, stream=None):
    rows, cols = out.shape
    if out.dtype not in _DT or not out.is_contiguous():
        raise NV4Error("out must be a contiguous bf16, fp16 or float32 tensor")
    if tuple(q.shape) != (rows, cols // 2) or tuple(scales.shape) != (rows, cols // 16):
        raise NV4Error("q / scales shapes do not match out")
    if not (q.is_contiguous() and scales.is_contiguous()):
        raise NV4Error("q and scales must be contiguous")
    _check(lib().nv4_dequant(_ptr(q), _ptr(scales), _scalar_f32(d_s2, "d_s2"), rows, cols, _DT[out.dtype],
                             _ptr(out), _stream(stream)), "nv4_dequant")


def _hjob(x: torch.Tensor, H: torch.Tensor) -> HessianJob:
    if x.dtype != torch.bfloat16:
        raise NV4Error("x must be bf16")
    tokens, cols, ld = _rowmajor(x, "x")
    if H.dtype != torch.float32 or not H.is_contiguous() or H.numel() != (cols // 16) * 256:
        raise NV4Error("H must be a contiguous float32 tensor [cols/16, 16, 16]")
    return HessianJob(_ptr(x), tokens, cols, ld, _ptr(H))


def nv4_hessian_accum(x: torch.Tensor, H: torch.Tensor, d_flags: torch.Tensor | None = None, stream=None):
    j = _hjob(x, H)
    _check(lib().nv4_hessian_accum(j.x, j.tokens, j.cols, j.ld, j.H, _ptr(d_flags), _stream(stream)),
           "nv4_hessian_accum")


def nv4_hessian_accum_batched(xs, Hs, d_flags: torch.Tensor | None = None, stream=None):
    jobs = (HessianJob * len(xs))(*[_hjob(x, H) for x, H in zip(xs, Hs)])
    _check(lib().nv4_hessian_accum_batched(jobs, len(xs), _ptr(d_flags), _stream(stream)),
           "nv4_hessian_accum_batched")


def _sjob(w, H, d_amax_w, codes, q=None, cost1=None, cost2=None, d_work=None) -> SweepJob:
    rows, cols, ld = _rowmajor(w, "w")
    nblk = cols // 16
    if H.dtype != torch.float32 or not H.is_contiguous() or H.numel() != nblk * 256:
        raise NV4Error("H must be a contiguous float32 tensor [cols/16, 16, 16]")
    if codes.dtype != torch.uint8 or tuple(codes.shape) != (rows, nblk) or not codes.is_contiguous():
        raise NV4Error("codes must be a contiguous uint8 tensor [rows, cols/16]")
    if q is not None and (q.dtype != torch.uint8 or tuple(q.shape) != (rows, cols // 2) or not q.is_contiguous()):
        raise NV4Error("q must be a contiguous uint8 tensor [rows, cols/2]")
    for c in (cost1, cost2):
        if c is not None and (c.dtype != torch.float32 or tuple(c.shape) != (rows, nblk) or not c.is_contiguous()):
            raise NV4Error("cost1/cost2 must be contiguous float32 tensors [rows, cols/16]")
    if d_work is not None and (d_work.dtype != torch.int64 or d_work.numel() < 2 or not d_work.is_contiguous()):
        raise NV4Error("d_work must be a contiguous int64 tensor of at least 2 elements")
    return SweepJob(_ptr(w), rows, cols, ld, _ptr(H), _scalar_f32(d_amax_w, "d_amax_w"), _ptr(codes), _ptr(q),
                    _ptr(cost1), _ptr(cost2), _ptr(d_work))


def nv4_scale_sweep(w, H, d_amax_w, codes, q=None, cost1=None, cost2=None, d_flags=None, stream=None):
    if w.dtype not in (torch.bfloat16, torch.float32):
        raise NV4Error("w must be bf16 or float32")
    j = _sjob(w, H, d_amax_w, codes, q, cost1, cost2)
    _check(lib().nv4_scale_sweep(j.w, _DT[w.dtype], j.rows, j.cols, j.ld, j.H, j.d_amax_w, j.codes, j.q, j.cost1,
                                 j.cost2, _ptr(d_flags), _stream(stream)), "nv4_scale_sweep")


def nv4_scale_sweep_batched(jobs: list[dict], d_flags=None, stream=None):
    """jobs: dicts with keys w, H, d_amax_w, codes and optional q, cost1, cost2, d_work (one dtype)."""
    dts = {j["w"].dtype for j in jobs}
    if len(dts) != 1 or next(iter(dts)) not in (torch.bfloat16, torch.float32):
        raise NV4Error("all w must share one dtype, bf16 or float32")
    arr = (SweepJob * len(jobs))(*[_sjob(**j) for j in jobs])
    _check(lib().nv4_scale_sweep_batched(arr, len(jobs), _DT[next(iter(dts))], _ptr(d_flags), _stream(stream)),
           "nv4_scale_sweep_batched")


def _cjob(mx_q, e8m0, nv_q, nv_scales, d_global_amax, d_s2, group: int = -1) -> CastJob:
    rows, half = mx_q.shape
    cols = 2 * half
    for t, shape, name in ((mx_q, (rows, half), "mx_q"), (e8m0, (rows, cols // 32), "e8m0"),
                           (nv_q, (rows, half), "nv_q"), (nv_scales, (rows, cols // 16), "nv_scales")):
        if t.dtype != torch.uint8 or tuple(t.shape) != shape or not t.is_contiguous():
            raise NV4Error(f"{name} must be a contiguous uint8 tensor {shape}")
    return CastJob(_ptr(mx_q), _ptr(e8m0), rows, cols, _ptr(nv_q), _ptr(nv_scales),
                   _scalar_f32(d_global_amax, "d_global_amax"), _scalar_f32(d_s2, "d_s2"), int(group))


def nv4_mxfp4_to_nvfp4(mx_q, e8m0, nv_q, nv_scales, d_global_amax, d_s2, d_counts=None, d_flags=None, stream=None):
    j = _cjob(mx_q, e8m0, nv_q, nv_scales, d_global_amax, d_s2)
    _check(lib().nv4_mxfp4_to_nvfp4(j.mx_q, j.e8m0, j.rows, j.cols, j.nv_q, j.nv_scales, j.d_global_amax, j.d_s2,
                                    _ptr(d_counts), _ptr(d_flags), _stream(stream)), "nv4_mxfp4_to_nvfp4")


def nv4_mxfp4_to_nvfp4_batched(jobs: list[dict], d_counts=None, d_flags=None, stream=None):
    """jobs: dicts with keys mx_q, e8m0, nv_q, nv_scales, d_global_amax, d_s2 and optional group
    (jobs with the same group id >= 0 share one scale_2)."""
    arr = (CastJob * len(jobs))(*[_cjob(**j) for j in jobs])
    _check(lib().nv4_mxfp4_to_nvfp4_batched(arr, len(jobs), _ptr(d_counts), _ptr(d_flags), _stream(stream)),
           "nv4_mxfp4_to_nvfp4_batched")


def nv4_selftest_wait(flag: torch.Tensor, limit_ns: int, status: torch.Tensor, stream=None):
    if flag.dtype != torch.int32 or status.dtype != torch.int32 or status.numel() < 2:
        raise NV4Error("flag and status must be int32 CUDA tensors (status of at least 2 elements)")
    _check(lib().nv4_selftest_wait(_ptr(flag), int(limit_ns), _ptr(status), _stream(stream)), "nv4_selftest_wait")


def _w_rows(w, name="w"):
    if w.dtype not in (torch.bfloat16, torch.float32):
        raise NV4Error(f"{name} must be bf16 or float32")
    return _rowmajor(w, name)


def nv4_hadamard2_rotate(w: torch.Tensor, n: int, out: torch.Tensor, d_flags=None, stream=None):
    rows, cols, ld = _w_rows(w)
    if out.dtype != torch.float32 or tuple(out.shape) != (rows, cols) or not out.is_contiguous():
        raise NV4Error("out must be a contiguous float32 tensor [rows, cols]")
    _check(lib().nv4_hadamard2_rotate(_ptr(w), _DT[w.dtype], rows, cols, ld, n, _ptr(out), _ptr(d_flags),
                                      _stream(stream)), "nv4_hadamard2_rotate")


def nv4_hadamard2_amax(w: torch.Tensor, n: int, d_amax: torch.Tensor, d_flags=None, stream=None):
    rows, cols, ld = _w_rows(w)
    _check(lib().nv4_hadamard2_amax(_ptr(w), _DT[w.dtype], rows, cols, ld, n, _scalar_f32(d_amax, "d_amax"),
                                    _ptr(d_flags), _stream(stream)), "nv4_hadamard2_amax")


def nv4_hadamard2_mxfp4_quant(w: torch.Tensor, n: int, q: torch.Tensor, e8m0: torch.Tensor, d_flags=None,
                              stream=None):
    rows, cols, ld = _w_rows(w)
    _u8(q, (rows, cols // 2), "q")
    _u8(e8m0, (rows, cols // 32), "e8m0")
    _check(lib().nv4_hadamard2_mxfp4_quant(_ptr(w), _DT[w.dtype], rows, cols, ld, n, _ptr(q), _ptr(e8m0),
                                           _ptr(d_flags), _stream(stream)), "nv4_hadamard2_mxfp4_quant")


def nv4_hadamard2_nvfp4_quant(w: torch.Tensor, n: int, d_amax: torch.Tensor, q: torch.Tensor, scales: torch.Tensor,
                              d_s2: torch.Tensor, d_flags=None, stream=None):
    rows, cols, ld = _w_rows(w)
    _u8(q, (rows, cols // 2), "q")
    _u8(scales, (rows, cols // 16), "scales")
    _check(lib().nv4_hadamard2_nvfp4_quant(_ptr(w), _DT[w.dtype], rows, cols, ld, n, _scalar_f32(d_amax, "d_amax"),
                                           _ptr(q), _ptr(scales), _scalar_f32(d_s2, "d_s2"), _ptr(d_flags),
                                           _stream(stream)), "nv4_hadamard2_nvfp4_quant")


def hadamard2_rotate(w: torch.Tensor, n: int, d_flags=None, stream=None) -> torch.Tensor:
    out = torch.empty(tuple(w.shape), dtype=torch.float32, device=w.device)
    nv4_hadamard2_rotate(w, n, out, d_flags, stream)
    return out


def hadamard2_mxfp4_quant(w: torch.Tensor, n: int, d_flags=None, stream=None):
    rows, cols = w.shape
    q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=w.device)
    e8 = torch.empty((rows, cols // 32), dtype=torch.uint8, device=w.device)
    nv4_hadamard2_mxfp4_quant(w, n, q, e8, d_flags, stream)
    return q, e8


def hadamard2_nvfp4_quant(w: torch.Tensor, n: int, d_flags=None, stream=None):
    """Two passes: the amax of the rotated tensor, then the NVFP4 quantization."""
    rows, cols = w.shape
    amax = torch.zeros(1, dtype=torch.float32, device=w.device)
    nv4_hadamard2_amax(w, n, amax, d_flags, stream)
    q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=w.device)
    sc = torch.empty((rows, cols // 16), dtype=torch.uint8, device=w.device)
    s2 = torch.empty(1, dtype=torch.float32, device=w.device)
    nv4_hadamard2_nvfp4_quant(w, n, amax, q, sc, s2, d_flags, stream)
    return q, sc, s2, amax


def nv4_fp32_probe(packed: bool, blocks: int, iters: int, sink: torch.Tensor, stream=None):
    """FP32 pipe microbenchmark: blocks * 256 * iters * 128 FLOP of independent FMAs."""
    if sink.dtype != torch.float32 or sink.numel() < blocks:
        raise NV4Error("sink must be a float32 CUDA tensor with one element per block")
    _check(lib().nv4_fp32_probe(1 if packed else 0, blocks, iters, _ptr(sink), _stream(stream)), "nv4_fp32_probe")


def nv4_selftest(out: torch.Tensor, stream=None):
    if out.dtype != torch.int32 or out.numel() < 64:
        raise NV4Error("out must be an int32 CUDA tensor of at least 64 elements")
    _check(lib().nv4_selftest(_ptr(out), _stream(stream)), "nv4_selftest")


# ------------------------------------------------------------------ allocating helpers
def _zeros(shape, dtype, device):
    return torch.zeros(shape, dtype=dtype, device=device)


def tensor_amax(x: torch.Tensor, d_amax: torch.Tensor | None = None, d_flags=None, stream=None) -> torch.Tensor:
    d_amax = _zeros((1,), torch.float32, x.device) if d_amax is None else d_amax
    nv4_tensor_amax(x, d_amax, d_flags, stream)
    return d_amax


def act_quant(x: torch.Tensor, d_amax: torch.Tensor, d_flags=None, stream=None):
    rows, cols = x.shape
    q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    sc = torch.empty((rows, cols // 16), dtype=torch.uint8, device=x.device)
    s2 = torch.empty((1,), dtype=torch.float32, device=x.device)
    nv4_act_quant(x, d_amax, q, sc, s2, d_flags, stream)
    return q, sc, s2


def weight_quant_rtn(w: torch.Tensor, d_amax: torch.Tensor, d_flags=None, stream=None):
    rows, cols = w.shape
    q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=w.device)
    sc = torch.empty((rows, cols // 16), dtype=torch.uint8, device=w.device)
    s2 = torch.empty((1,), dtype=torch.float32, device=w.device)
    nv4_weight_quant_rtn(w, d_amax, q, sc, s2, d_flags, stream)
    return q, sc, s2


def fake_qdq(x: torch.Tensor, d_amax: torch.Tensor, dtype=torch.bfloat16, d_flags=None, stream=None):
    out = torch.empty(tuple(x.shape), dtype=dtype, device=x.device)
    s2 = torch.empty((1,), dtype=torch.float32, device=x.device)
    nv4_fake_qdq(x, d_amax, out, s2, d_flags, stream)
    return out, s2


def _u8(t, shape, name):
    if t.dtype != torch.uint8 or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise NV4Error(f"{name} must be a contiguous uint8 tensor {tuple(shape)}")


def nv4_mxfp4_quant(x: torch.Tensor, q: torch.Tensor, e8m0: torch.Tensor, d_flags=None, stream=None):
    if x.dtype not in (torch.bfloat16, torch.float32):
        raise NV4Error("x must be bf16 or float32")
    rows, cols, ld = _rowmajor(x, "x")
    _u8(q, (rows, cols // 2), "q")
    _u8(e8m0, (rows, cols // 32), "e8m0")
    _check(lib().nv4_mxfp4_quant(_ptr(x), _DT[x.dtype], rows, cols, ld, _ptr(q), _ptr(e8m0), _ptr(d_flags),
                                 _stream(stream)), "nv4_mxfp4_quant")


def nv4_mxfp4_dequant(q: torch.Tensor, e8m0: torch.Tensor, out: torch.Tensor, stream=None):
    rows, cols = out.shape
    _u8(q, (rows, cols // 2), "q")
    _u8(e8m0, (rows, cols // 32), "e8m0")
    if out.dtype not in _DT or not out.is_contiguous():
        raise NV4Error("out must be a contiguous bf16, float16 or float32 tensor")
    _check(lib().nv4_mxfp4_dequant(_ptr(q), _ptr(e8m0), rows, cols, _DT[out.dtype], _ptr(out), _stream(stream)),
           "nv4_mxfp4_dequant")


def nv4_fp8_quant(x: torch.Tensor, d_amax: torch.Tensor, q: torch.Tensor, d_scale: torch.Tensor, d_flags=None,
                  stream=None):
    if x.dtype not in (torch.bfloat16, torch.float32):
        raise NV4Error("x must be bf16 or float32")
    rows, cols, ld = _rowmajor(x, "x")
    _u8(q, (rows, cols), "q")
    _check(lib().nv4_fp8_quant(_ptr(x), _DT[x.dtype], rows, cols, ld, _scalar_f32(d_amax, "d_amax"), _ptr(q),
                               _scalar_f32(d_scale, "d_scale"), _ptr(d_flags), _stream(stream)), "nv4_fp8_quant")


def nv4_fp8_dequant(q: torch.Tensor, d_scale: torch.Tensor, out: torch.Tensor, stream=None):
    rows, cols = out.shape
    _u8(q, (rows, cols), "q")
    if out.dtype not in _DT or not out.is_contiguous():
        raise NV4Error("out must be a contiguous bf16, float16 or float32 tensor")
    _check(lib().nv4_fp8_dequant(_ptr(q), _scalar_f32(d_scale, "d_scale"), rows, cols, _DT[out.dtype], _ptr(out),
                                 _stream(stream)), "nv4_fp8_dequant")


def _bf16_rows(x, name="x"):
    if x.dtype != torch.bfloat16:
        raise NV4Error(f"{name} must be bf16")
    return _rowmajor(x, name)


def nv4_hadamard_amax(x: torch.Tensor, n: int, d_amax: torch.Tensor, d_flags=None, stream=None):
    rows, cols, ld = _bf16_rows(x)
    _check(lib().nv4_hadamard_amax(_ptr(x), rows, cols, ld, n, _scalar_f32(d_amax, "d_amax"), _ptr(d_flags),
                                   _stream(stream)), "nv4_hadamard_amax")


def nv4_hadamard_mxfp4_quant(x: torch.Tensor, n: int, q: torch.Tensor, e8m0: torch.Tensor, d_flags=None,
                             stream=None):
    rows, cols, ld = _bf16_rows(x)
    _u8(q, (rows, cols // 2), "q")
    _u8(e8m0, (rows, cols // 32), "e8m0")
    _check(lib().nv4_hadamard_mxfp4_quant(_ptr(x), rows, cols, ld, n, _ptr(q), _ptr(e8m0), _ptr(d_flags),
                                          _stream(stream)), "nv4_hadamard_mxfp4_quant")


def nv4_hadamard_nvfp4_quant(x: torch.Tensor, n: int, d_amax: torch.Tensor, q: torch.Tensor, scales: torch.Tensor,
                             d_s2: torch.Tensor, d_flags=None, stream=None):
    rows, cols, ld = _bf16_rows(x)
    _u8(q, (rows, cols // 2), "q")
    _u8(scales, (rows, cols // 16), "scales")
    _check(lib().nv4_hadamard_nvfp4_quant(_ptr(x), rows, cols, ld, n, _scalar_f32(d_amax, "d_amax"), _ptr(q),
                                          _ptr(scales), _scalar_f32(d_s2, "d_s2"), _ptr(d_flags), _stream(stream)),
           "nv4_hadamard_nvfp4_quant")


def hadamard_mxfp4_quant(x: torch.Tensor, n: int, d_flags=None, stream=None):
    rows, cols = x.shape
    q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    e8 = torch.empty((rows, cols // 32), dtype=torch.uint8, device=x.device)
    nv4_hadamard_mxfp4_quant(x, n, q, e8, d_flags, stream)
    return q, e8


def hadamard_nvfp4_quant(x: torch.Tensor, n: int, d_flags=None, stream=None):
    """Two passes: the amax of the rotated tensor, then the NVFP4 quantization."""
    rows, cols = x.shape
    amax = torch.zeros(1, dtype=torch.float32, device=x.device)
    nv4_hadamard_amax(x, n, amax, d_flags, stream)
    q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    sc = torch.empty((rows, cols // 16), dtype=torch.uint8, device=x.device)
    s2 = torch.empty(1, dtype=torch.float32, device=x.device)
    nv4_hadamard_nvfp4_quant(x, n, amax, q, sc, s2, d_flags, stream)
    return q, sc, s2, amax


def mxfp4_quant(x: torch.Tensor, d_flags=None, stream=None):
    rows, cols = x.shape
    q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    e8 = torch.empty((rows, cols // 32), dtype=torch.uint8, device=x.device)
    nv4_mxfp4_quant(x, q, e8, d_flags, stream)
    return q, e8


def fp8_quant(x: torch.Tensor, d_amax: torch.Tensor, d_flags=None, stream=None):
    q = torch.empty(tuple(x.shape), dtype=torch.uint8, device=x.device)
    sc = torch.empty(1, dtype=torch.float32, device=x.device)
    nv4_fp8_quant(x, d_amax, q, sc, d_flags, stream)
    return q, sc


def nv4_mma_scale_bytes(rows: int, cols: int) -> int:
    return int(lib().nv4_mma_scale_bytes(rows, cols))


def nv4_scales_to_mma_layout(scales: torch.Tensor, out: torch.Tensor, stream=None):
    """scales: contiguous uint8 [rows, cols/16]; out: uint8, nv4_mma_scale_bytes(rows, cols) bytes."""
    if scales.dtype != torch.uint8 or scales.dim() != 2 or not scales.is_contiguous():
        raise NV4Error("scales must be a contiguous uint8 tensor [rows, cols/16]")
    rows, kb = scales.shape
    need = nv4_mma_scale_bytes(rows, 16 * kb)
    if out.dtype != torch.uint8 or out.numel() < need or not out.is_contiguous():
        raise NV4Error(f"out must be a contiguous uint8 tensor of at least {need} bytes")
    _check(lib().nv4_scales_to_mma_layout(_ptr(scales), rows, 16 * kb, _ptr(out), _stream(stream)),
           "nv4_scales_to_mma_layout")


def nv4_gemm_nvfp4(qa, sfa_mma, d_s2a, qb, sfb_mma, d_s2b, out, d_flags=None, stream=None):
    """out[M, N] = s2a * s2b * A @ B^T for NVFP4 operands (codes [rows, K/2], MMA-layout scales)."""
    M, half = qa.shape
    N = qb.shape[0]
    K = 2 * half
    for t, shape, name in ((qa, (M, half), "qa"), (qb, (N, half), "qb")):
        if t.dtype != torch.uint8 or tuple(t.shape) != shape or not t.is_contiguous():
            raise NV4Error(f"{name} must be a contiguous uint8 tensor {shape}")
    for t, rows, name in ((sfa_mma, M, "sfa_mma"), (sfb_mma, N, "sfb_mma")):
        if t.dtype != torch.uint8 or t.numel() < nv4_mma_scale_bytes(rows, K):
            raise NV4Error(f"{name} must hold nv4_mma_scale_bytes({rows}, {K}) bytes")
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise NV4Error("out must be bf16 or float32")
    orows, ocols, ldd = _rowmajor(out, "out")
    if (orows, ocols) != (M, N):
        raise NV4Error("out must be [M, N]")
    _check(lib().nv4_gemm_nvfp4(_ptr(qa), _ptr(sfa_mma), _scalar_f32(d_s2a, "d_s2a"), _ptr(qb), _ptr(sfb_mma),
                                _scalar_f32(d_s2b, "d_s2b"), M, N, K, _DT[out.dtype], _ptr(out), ldd, _ptr(d_flags),
                                _stream(stream)), "nv4_gemm_nvfp4")


def mma_scales(scales: torch.Tensor, stream=None) -> torch.Tensor:
    rows, kb = scales.shape
    out = torch.empty(nv4_mma_scale_bytes(rows, 16 * kb), dtype=torch.uint8, device=scales.device)
    nv4_scales_to_mma_layout(scales, out, stream)
    return out


def gemm_nvfp4(qa, sa, d_s2a, qb, sb, d_s2b, dtype=torch.bfloat16, d_flags=None, stream=None):
    out = torch.empty((qa.shape[0], qb.shape[0]), dtype=dtype, device=qa.device)
    nv4_gemm_nvfp4(qa, mma_scales(sa, stream), d_s2a, qb, mma_scales(sb, stream), d_s2b, out, d_flags, stream)
    return out


def dequant(q, scales, d_s2, dtype=torch.bfloat16, stream=None):
    out = torch.empty((q.shape[0], q.shape[1] * 2), dtype=dtype, device=q.device)
    nv4_dequant(q, scales, d_s2, out, stream)
    return out


def hessian_accum(x: torch.Tensor, H: torch.Tensor | None = None, d_flags=None, stream=None):
    H = _zeros((x.shape[1] // 16, 16, 16), torch.float32, x.device) if H is None else H
    nv4_hessian_accum(x, H, d_flags, stream)
    return H


def scale_sweep(w, H, d_amax_w, with_costs=True, d_flags=None, stream=None):
    rows, cols = w.shape
    dev = w.device
    codes = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    c1 = torch.empty((rows, cols // 16), dtype=torch.float32, device=dev) if with_costs else None
    c2 = torch.empty((rows, cols // 16), dtype=torch.float32, device=dev) if with_costs else None
    nv4_scale_sweep(w, H, d_amax_w, codes, q, c1, c2, d_flags, stream)
    return codes, q, c1, c2


def mxfp4_to_nvfp4(mx_q, e8m0, in_place=False, d_counts=None, d_flags=None, stream=None):
    dev = mx_q.device
    nv_q = mx_q if in_place else torch.empty_like(mx_q)
    nv_s = torch.empty((mx_q.shape[0], mx_q.shape[1] // 8), dtype=torch.uint8, device=dev)
    ga = torch.empty((1,), dtype=torch.float32, device=dev)
    s2 = torch.empty((1,), dtype=torch.float32, device=dev)
    nv4_mxfp4_to_nvfp4(mx_q, e8m0, nv_q, nv_s, ga, s2, d_counts, d_flags, stream)
    return nv_q, nv_s, ga, s2
