"""Exact rational reference arithmetic used to pin the oracle (test-only).

Nothing here calls the oracle: values come from the golden fixtures (the pages'
printed numbers) and from torch's own float8 decoders; rounding is done on
``fractions.Fraction`` by brute force over the candidate values.
"""
from __future__ import annotations

import os
from fractions import Fraction as Fr

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden_lines(name: str) -> list[str]:
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def golden_kv(name: str) -> dict[str, str]:
    return dict(ln.split(None, 1) for ln in golden_lines(name))


GRID = [Fr(s) for s in golden_lines("e2m1_grid.txt")]          # magnitudes 0..6
E4M3 = [Fr(float(v)) for v in torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).float()]


def nearest_index(values: list[Fr], y: Fr) -> int:
    """Index of the value nearest to y; on an exact tie the even index wins."""
    best, bd = 0, abs(values[0] - y)
    for k in range(1, len(values)):
        d = abs(values[k] - y)
        if d < bd or (d == bd and k % 2 == 0):
            best, bd = k, d
    return best


def floor_log2(a: Fr) -> int:
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fr(2) ** e > a:
        e -= 1
    elif Fr(2) ** (e + 1) <= a:
        e += 1
    return e


def rn_format(x: Fr, p: int, emin: int, maxv: Fr) -> Fr | float:
    """Nearest value of a binary format with p significand bits, min normal exponent emin,
    ties to even; +-inf beyond the overflow threshold."""
    if x == 0:
        return Fr(0)
    s = -1 if x < 0 else 1
    a = abs(x)
    lead = max(floor_log2(a), emin)
    quantum = Fr(2) ** (lead - p + 1)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fr(1, 2) or (rem == Fr(1, 2) and fl % 2 == 1):
        fl += 1
    r = fl * quantum
    if r > maxv:
        return s * float("inf")
    return s * r


FLT_MAX = (2 - Fr(1, 2 ** 23)) * Fr(2) ** 127


def rn32(x: Fr):
    return rn_format(x, 24, -126, FLT_MAX)


def e4m3_code(num: Fr, den: Fr) -> int:
    if den == 0:
        return 0
    return nearest_index(E4M3, num / den)


def e2m1_code(x: float, S: Fr) -> int:
    sign = 8 if np.signbit(x) else 0
    if S == 0:
        return sign
    return sign | nearest_index(GRID, abs(Fr(float(x))) / S)


def e2m1_signed_value(code: int) -> Fr:
    v = GRID[code & 7]
    return -v if code & 8 else v


def f32(x) -> float:
    return float(np.float32(x))


def act_quant_block(xs: list[float], s2: Fr):
    """Block scale code, FP32 block scale S and E2M1 codes of one 16-block (exact)."""
    a = max(abs(Fr(float(v))) for v in xs)
    code = e4m3_code(a, 6 * s2)
    S = rn32(E4M3[code] * s2)
    return code, S, [e2m1_code(v, S) for v in xs]
