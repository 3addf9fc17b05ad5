"""Helpers shared by the tests: bit conversions and exact reference arithmetic.

Nothing here calls the CUDA path; nothing here restates the oracle's code.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# E2M1 magnitudes by code, from the format definition: 2 exponent bits (bias 1),
# 1 mantissa bit; exponent 0 is subnormal (0 and 0.5).
E2M1_MAG = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    return (np.asarray(b).astype(np.uint32) << 16).view(np.float32)


def fraction_to_bf16(fr: Fraction) -> Fraction:
    """Exact value of the bf16 nearest to fr (ties to even)."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 7)  # 8 significant bits
    q = a / ulp
    n = math.floor(q)
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * ulp


def e2m1_value(code: int) -> float:
    m = E2M1_MAG[code & 7]
    return -m if code & 8 else m


def e2m1_values(codes: np.ndarray) -> np.ndarray:
    mag = np.asarray(E2M1_MAG, dtype=np.float64)[codes & 7]
    return np.where(codes & 8, -mag, mag)


def e4m3_values(codes: np.ndarray) -> np.ndarray:
    """E4M3 bytes to float64 through torch's float8_e4m3fn (a library decoder)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """[..., n/2] bytes -> [..., n] codes; element 2i sits in the low nibble."""
    lo = packed & 15
    hi = packed >> 4
    return np.stack([lo, hi], axis=-1).reshape(packed.shape[:-1] + (packed.shape[-1] * 2,))


def dequant_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Contraction-domain values val(code) * dec(scale) of blocks along the last axis."""
    c = unpack_codes(codes)
    s = np.repeat(e4m3_values(scales), 16, axis=-1)
    return e2m1_values(c) * s


def load_golden(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def golden_tensors(g: dict):
    """(q, k, v) bf16 bit arrays of a golden case (all listed values are bf16-exact)."""
    s = g["shape"]
    B, H, Hkv, N, D = s["B"], s["H"], s["Hkv"], s["N"], s["D"]
    q = np.zeros((B, H, N, D), np.float32)
    k = np.zeros((B, Hkv, N, D), np.float32)
    v = np.zeros((B, Hkv, N, D), np.float32)
    for arr, key in ((q, "q"), (k, "k"), (v, "v")):
        for b, h, n, d, val in g[key]:
            arr[b, h, n, d] = val
    for arr in (q, k, v):
        assert np.array_equal(bf16_bits_to_f32(f32_to_bf16_bits(arr)), arr)
    return f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v)


def bits_to_float(bits: str) -> float:
    return float(np.array([int(bits, 16)], np.uint32).view(np.float32)[0])
