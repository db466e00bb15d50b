"""CPU-only checks of the C-ABI library: it loads, exports every entry point that
include/nv4.h declares, and rejects bad arguments before touching the GPU."""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def nv4lib():
    from nvfp4_block_numerics_b200.build import build_library
    from nvfp4_block_numerics_b200 import binding

    build_library()
    return binding.lib()


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "nv4.h")).read()
    return sorted(set(re.findall(r"^NV4_API\s+[\w\s\*]+?\b(nv4_\w+)\(", txt, flags=re.M)))


def test_header_declares_the_hot_path():
    names = declared_symbols()
    for n in ("nv4_tensor_amax", "nv4_act_quant", "nv4_dequant", "nv4_hessian_accum", "nv4_scale_sweep",
              "nv4_mxfp4_to_nvfp4", "nv4_weight_quant_rtn", "nv4_fake_qdq", "nv4_gemm_nvfp4",
              "nv4_scales_to_mma_layout", "nv4_mma_scale_bytes", "nv4_mxfp4_quant", "nv4_mxfp4_dequant",
              "nv4_fp8_quant", "nv4_fp8_dequant", "nv4_hadamard_amax", "nv4_hadamard_mxfp4_quant",
              "nv4_hadamard_nvfp4_quant", "nv4_selftest_wait", "nv4_tensor_amax_batched", "nv4_act_quant_batched",
              "nv4_dequant_batched", "nv4_weight_quant_rtn_batched"):
        assert n in names


def test_library_exports_every_declared_symbol(nv4lib):
    from nvfp4_block_numerics_b200.build import LIB_PATH

    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)$", out, flags=re.M))
    for n in declared_symbols():
        assert n in exported, n
        assert getattr(nv4lib, n) is not None
    # nothing else leaks out of the library
    assert {e for e in exported if not e.startswith("nv4_")} <= {"_init", "_fini"}


def test_status_strings_and_version(nv4lib):
    assert nv4lib.nv4_version() == 100
    for s in range(7):
        assert nv4lib.nv4_status_str(s).startswith(b"NV4_")


def test_validation_rejects_before_any_launch(nv4lib):
    L = nv4lib
    fake = 0x1000  # never dereferenced: every call below fails validation first
    assert L.nv4_act_quant(fake, 4, 24, 24, fake, fake, fake, fake, None, None) == 2      # cols % 16
    assert L.nv4_act_quant(fake, 4, 32, 16, fake, fake, fake, fake, None, None) == 2      # ld < cols
    assert L.nv4_act_quant(fake + 2, 4, 32, 32, fake, fake, fake, fake, None, None) == 3  # misaligned x
    assert L.nv4_act_quant(fake, 4, 32, 36, fake, fake, fake, fake, None, None) == 3      # ld*2 % 16
    assert L.nv4_act_quant(None, 4, 32, 32, fake, fake, fake, fake, None, None) == 1
    assert L.nv4_tensor_amax(fake, 1, 16, fake, None, None) == 4                           # fp16 unsupported
    assert L.nv4_tensor_amax(fake, 0, -1, fake, None, None) == 2
    assert L.nv4_tensor_amax(fake, 0, 0, fake, None, None) == 0                            # no-op
    assert L.nv4_dequant(fake, fake, fake, 2, 32, 7, fake, None) == 4
    # RTN weight quantization: dtype, shape, alignment (FP32 rows need ld % 4), nulls
    assert L.nv4_weight_quant_rtn(fake, 1, 4, 32, 32, fake, fake, fake, fake, None, None) == 4    # fp16 w
    assert L.nv4_weight_quant_rtn(fake, 2, 4, 40, 40, fake, fake, fake, fake, None, None) == 2    # cols % 16
    assert L.nv4_weight_quant_rtn(fake, 2, 4, 32, 34, fake, fake, fake, fake, None, None) == 3    # ld*4 % 16
    assert L.nv4_weight_quant_rtn(fake, 0, 4, 32, 36, fake, fake, fake, fake, None, None) == 3    # ld*2 % 16
    assert L.nv4_weight_quant_rtn(fake, 2, 4, 32, 32, fake, None, fake, fake, None, None) == 1
    # empty: passes validation with NULL tensors, then launches the kernel that writes s2
    # (NV4_ERR_CUDA here, where no GPU is present)
    assert L.nv4_weight_quant_rtn(fake, 2, 0, 32, 32, fake, None, None, fake, None, None) in (0, 5)
    # fused fake quantize-dequantize
    assert L.nv4_fake_qdq(fake, 4, 32, 32, fake, 5, fake, 32, fake, None, None) == 4              # out dtype
    assert L.nv4_fake_qdq(fake, 4, 32, 32, fake, 0, fake, 16, fake, None, None) == 2              # ld_out < cols
    assert L.nv4_fake_qdq(fake, 4, 32, 32, fake, 2, fake, 34, fake, None, None) == 3              # fp32 ld_out
    assert L.nv4_fake_qdq(fake, 4, 32, 32, fake, 0, fake + 8, 32, fake, None, None) == 3          # misaligned out
    assert L.nv4_fake_qdq(fake, 4, 32, 32, None, 0, fake, 32, fake, None, None) == 1
    # W4A4 GEMM: shape multiples (M, N of 128; K of 256), dtype, alignment, nulls
    g = lambda M, N, K, dt=0, ldd=None, out=fake, qa=fake: L.nv4_gemm_nvfp4(
        qa, fake, fake, fake, fake, fake, M, N, K, dt, out, N if ldd is None else ldd, None, None)
    assert g(128, 128, 256, dt=1) == 4                     # fp16 out unsupported
    assert g(100, 128, 256) == 2 and g(128, 120, 256) == 2 and g(128, 128, 200) == 2
    assert g(128, 128, 256, ldd=64) == 2                   # ldd < N
    assert g(128, 128, 256, ldd=132) == 3                  # bf16 row pitch not 16-byte
    assert g(128, 128, 256, out=fake + 4) == 3
    assert g(128, 128, 256, qa=None) == 1
    assert g(0, 128, 256) == 0                             # empty
    assert L.nv4_mma_scale_bytes(200, 144) == 256 * 12 and L.nv4_mma_scale_bytes(1, 16) == 512
    assert L.nv4_mma_scale_bytes(5, 20) == 0
    assert L.nv4_scales_to_mma_layout(fake, 4, 20, fake, None) == 2
    assert L.nv4_scales_to_mma_layout(fake, 4, 32, fake + 8, None) == 3
    # format variants
    assert L.nv4_mxfp4_quant(fake, 1, 4, 32, 32, fake, fake, None, None) == 4        # fp16 input
    assert L.nv4_mxfp4_quant(fake, 0, 4, 48, 48, fake, fake, None, None) == 2        # cols % 32
    assert L.nv4_mxfp4_quant(fake, 2, 4, 32, 34, fake, fake, None, None) == 3        # fp32 row pitch
    assert L.nv4_mxfp4_quant(None, 0, 4, 32, 32, fake, fake, None, None) == 1
    assert L.nv4_mxfp4_dequant(fake, fake, 4, 48, 0, fake, None) == 2
    assert L.nv4_fp8_quant(fake, 0, 4, 24, 24, fake, fake, fake, None, None) == 2    # cols % 16
    assert L.nv4_fp8_quant(fake, 0, 4, 32, 32, None, fake, fake, None, None) == 1    # amax
    assert L.nv4_fp8_quant(fake, 0, 4, 32, 32, fake, fake + 4, fake, None, None) == 3
    assert L.nv4_fp8_dequant(fake, fake, 4, 32, 9, fake, None) == 4
    assert L.nv4_selftest_wait(fake, 3_000_000_000, fake, None) == 6                 # above the kernels' 2 s limit
    assert L.nv4_selftest_wait(None, 1000, fake, None) == 1
    # block Hadamard + FP4
    assert L.nv4_hadamard_mxfp4_quant(fake, 4, 128, 128, 8, fake, fake, None, None) == 2    # n not in 16..128
    assert L.nv4_hadamard_mxfp4_quant(fake, 4, 96, 96, 32, fake, fake, None, None) == 2     # cols % 128
    assert L.nv4_hadamard_mxfp4_quant(fake, 4, 128, 132, 32, fake, fake, None, None) == 3   # ld % 8
    assert L.nv4_hadamard_amax(fake, 4, 128, 128, 64, None, None, None) == 1
    assert L.nv4_hadamard_nvfp4_quant(fake, 4, 128, 128, 128, fake, None, fake, fake, None, None) == 1
    assert L.nv4_hadamard_mxfp4_quant(fake, 1 << 26, 1024, 1024, 128, fake, fake, None, None) == 6  # 2^31 chunks
    # two-sided block Hadamard of weight tiles: n, tile and strip shapes, dtype, alignment, nulls
    assert L.nv4_hadamard2_rotate(fake, 0, 32, 64, 64, 64, fake, None, None) == 2          # n not 16 or 32
    assert L.nv4_hadamard2_rotate(fake, 0, 40, 64, 64, 32, fake, None, None) == 2          # rows % n
    assert L.nv4_hadamard2_rotate(fake, 0, 32, 48, 48, 16, fake, None, None) == 2          # cols % 32
    assert L.nv4_hadamard2_rotate(fake, 1, 32, 64, 64, 32, fake, None, None) == 4          # fp16 w
    assert L.nv4_hadamard2_rotate(fake, 2, 32, 64, 66, 32, fake, None, None) == 3          # fp32 row pitch
    assert L.nv4_hadamard2_rotate(fake, 0, 32, 64, 64, 32, fake + 8, None, None) == 3      # misaligned out
    assert L.nv4_hadamard2_mxfp4_quant(fake, 0, 32, 64, 64, 32, None, fake, None, None) == 1
    assert L.nv4_hadamard2_nvfp4_quant(fake, 0, 32, 64, 64, 32, None, fake, fake, fake, None, None) == 1
    assert L.nv4_hadamard2_amax(fake, 0, 0, 64, 64, 32, fake, None, None) == 0             # empty: no-op
    assert L.nv4_fp32_probe(0, 0, 16, fake, None) == 6 and L.nv4_fp32_probe(0, 8, 16, None, None) == 1
    assert L.nv4_hessian_accum(fake, 10, 40, 40, fake, None, None) == 2
    assert L.nv4_hessian_accum(fake, 10, 32, 36, fake, None, None) == 3
    assert L.nv4_scale_sweep(fake, 2, 4, 32, 34, fake, fake, fake, None, None, None, None, None) == 3  # fp32 ld*4
    assert L.nv4_scale_sweep(fake, 1, 4, 32, 32, fake, fake, fake, None, None, None, None, None) == 4  # fp16 w
    assert L.nv4_mxfp4_to_nvfp4(fake, fake, 4, 48, fake, fake, fake, fake, None, None, None) == 2     # cols % 32
    # overlapping but not identical nibble buffers are rejected
    assert L.nv4_mxfp4_to_nvfp4(fake, fake, 4, 64, fake + 16, fake, fake, fake, None, None, None) == 2
    from nvfp4_block_numerics_b200 import binding as b

    jobs = (b.HessianJob * 129)()
    assert L.nv4_hessian_accum_batched(jobs, 129, None, None) == 6                         # > 128 jobs


def test_batched_act_path_validation(nv4lib):
    """The batched amax / act quant / dequant entries apply the single-tensor rules to
    every job and reject the call before any launch."""
    from nvfp4_block_numerics_b200 import binding as b

    L, fake = nv4lib, 0x1000
    am = (b.AmaxJob * 2)(b.AmaxJob(fake, 64, fake), b.AmaxJob(fake + 4, 64, fake))
    assert L.nv4_tensor_amax_batched(am, 2, 0, None, None) == 3          # second x misaligned
    assert L.nv4_tensor_amax_batched(am, 1, 1, None, None) == 4          # fp16
    assert L.nv4_tensor_amax_batched(am, -1, 0, None, None) == 2
    assert L.nv4_tensor_amax_batched(None, 2, 0, None, None) == 1
    assert L.nv4_tensor_amax_batched(None, 0, 0, None, None) == 0        # no-op
    big = (b.AmaxJob * 129)()
    assert L.nv4_tensor_amax_batched(big, 129, 0, None, None) == 6       # > 128 jobs
    am2 = (b.AmaxJob * 1)(b.AmaxJob(fake, 1 << 37, fake))
    assert L.nv4_tensor_amax_batched(am2, 1, 0, None, None) == 6         # n >= 2^37
    aj = (b.ActJob * 2)(b.ActJob(fake, 4, 32, 32, fake, fake, fake, fake), b.ActJob(fake, 4, 24, 24, fake, fake, fake, fake))
    assert L.nv4_act_quant_batched(aj, 2, None, None) == 2               # second: cols % 16
    aj[1] = b.ActJob(fake, 4, 32, 36, fake, fake, fake, fake)
    assert L.nv4_act_quant_batched(aj, 2, None, None) == 3               # second: ld*2 % 16
    aj[1] = b.ActJob(fake, 4, 32, 32, None, fake, fake, fake)
    assert L.nv4_act_quant_batched(aj, 2, None, None) == 1               # second: amax
    assert L.nv4_act_quant_batched((b.ActJob * 129)(), 129, None, None) == 6
    rj = (b.ActJob * 2)(b.ActJob(fake, 4, 32, 36, fake, fake, fake, fake), b.ActJob(fake, 4, 32, 34, fake, fake, fake, fake))
    assert L.nv4_weight_quant_rtn_batched((b.ActJob * 129)(), 129, 2, None, None) == 6
    assert L.nv4_weight_quant_rtn_batched(rj, 2, 2, None, None) == 3     # second: FP32 row pitch 34
    assert L.nv4_weight_quant_rtn_batched(rj, 2, 0, None, None) == 3     # BF16 needs a pitch of 8
    assert L.nv4_weight_quant_rtn_batched(rj, 2, 1, None, None) == 4     # fp16 weights
    dj = (b.DequantJob * 2)(b.DequantJob(fake, fake, fake, 4, 32, fake), b.DequantJob(fake, fake, fake, 4, 32, fake + 8))
    assert L.nv4_dequant_batched(dj, 2, 0, None) == 3                    # second out misaligned
    assert L.nv4_dequant_batched(dj, 1, 7, None) == 4                    # out dtype
    dj[1] = b.DequantJob(fake, fake, None, 4, 32, fake)
    assert L.nv4_dequant_batched(dj, 2, 0, None) == 1


def fastdiv_params(d):
    s = 0
    while (1 << s) < d:
        s += 1
    m = ((1 << 32) * ((1 << s) - d)) // d + 1
    return m & 0xFFFFFFFF, s


@pytest.mark.parametrize("d", [1, 2, 3, 7, 16, 90, 128, 256, 448, 1000, 4097, 65535, 123457, 2 ** 31 - 1])
def test_fastdiv_formula(d):
    """The device's n / d = (mulhi(n, m) + n) >> s (Granlund-Montgomery), mirrored here."""
    m, s = fastdiv_params(d)
    rng = np.random.default_rng(d)
    ns = np.concatenate([rng.integers(0, 2 ** 32, 20000, dtype=np.uint64),
                         np.array([0, 1, d - 1, d, d + 1, 2 ** 32 - 1, (2 ** 32 - 1) // d * d], dtype=np.uint64)])
    for n in ns.tolist():
        q = (((n * m) >> 32) + n) >> s
        assert q == n // d, (n, d)
