"""Pins of the oracle's number formats (E2M1 values, E4M3 block scales).

The pages name the formats (block-scaled E2M1 with E4M3 scales, NVFP4:
TetraJet-v2 abstract and Minima summary; EFQ-Softmax abstract) but print no
table, so the pins come from the format definitions, a brute-force nearest
search and torch's float8_e4m3fn conversion.
"""
import math

import numpy as np
import pytest
import torch

from _util import E2M1_MAG, e4m3_values


def e2m1_from_fields(code: int) -> float:
    """E2M1 by its bit fields: sign, 2-bit exponent (bias 1), 1-bit mantissa."""
    s = -1.0 if code & 8 else 1.0
    e, m = (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
    return math.copysign(mag, s)


def brute_nearest(a: float, mags) -> int:
    """Index of the magnitude nearest to a; ties to the even index; beyond
    the largest magnitude, the largest (saturation)."""
    if a >= mags[-1]:
        return len(mags) - 1
    best, bd = 0, math.inf
    for c, m in enumerate(mags):
        d = abs(a - m)
        if d < bd or (d == bd and c % 2 == 0):
            best, bd = c, d
    return best


def test_e2m1_decode_matches_bit_fields(ora):
    for c in range(16):
        got, want = ora.e2m1_decode(c), e2m1_from_fields(c)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), c
    assert [e2m1_from_fields(c) for c in range(8)] == E2M1_MAG


def _e2m1_inputs():
    rng = np.random.default_rng(1)
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    xs = list(E2M1_MAG) + mids
    for m in mids + list(E2M1_MAG):
        m32 = np.float32(m)
        xs += [float(np.nextafter(m32, np.float32(0))), float(np.nextafter(m32, np.float32(10)))]
    xs += list(rng.uniform(-8, 8, 20000).astype(np.float32))
    xs += [1e-30, 1e30, 6.0001, 7.0, 1e-45]
    xs += [-x for x in xs]
    return [float(np.float32(x)) for x in xs]


def test_e2m1_encode_is_nearest_even_saturating(ora):
    for x in _e2m1_inputs():
        code = ora.e2m1_encode(x)
        want = brute_nearest(abs(x), E2M1_MAG) | (8 if math.copysign(1, x) < 0 else 0)
        assert code == want, (x, code, want)


def test_e2m1_midpoints_by_hand(ora):
    # ties go to the even code: 0.25->0, 0.75->1.0, 1.25->1.0, 1.75->2, 2.5->2, 3.5->4, 5->4
    assert [ora.e2m1_encode(x) for x in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)] == \
        [0, 2, 2, 4, 4, 6, 6]
    assert ora.e2m1_encode(float("inf")) == 7 and ora.e2m1_encode(-float("inf")) == 15
    assert ora.e2m1_encode(-0.0) == 8 and ora.e2m1_encode(-0.1) == 8


def e4m3_from_fields(code: int) -> float:
    """OCP FP8 E4M3: bias 7, S.1111.111 is NaN, no infinities."""
    s = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 15, code & 7
    if e == 15 and m == 7:
        return math.nan
    mag = (m / 8) * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
    return math.copysign(mag, s)


def test_e4m3_decode_matches_definition_and_torch(ora):
    lib = e4m3_values(np.arange(256, dtype=np.uint8))
    for c in range(256):
        got, want = ora.e4m3_decode(c), e4m3_from_fields(c)
        if math.isnan(want):
            assert math.isnan(got) and math.isnan(lib[c])
        else:
            assert got == want == lib[c], c
    assert ora.e4m3_decode(0x7E) == 448.0 and ora.e4m3_decode(1) == 2.0 ** -9


def _e4m3_inputs():
    rng = np.random.default_rng(2)
    mags = [e4m3_from_fields(c) for c in range(127)]
    xs = list(mags)
    for a, b in zip(mags[:-1], mags[1:]):
        mid = np.float32((a + b) / 2)  # exact: adjacent E4M3 values differ in few bits
        xs += [float(mid), float(np.nextafter(mid, np.float32(0))),
               float(np.nextafter(mid, np.float32(1e9)))]
    xs += list(np.exp(rng.uniform(np.log(1e-4), np.log(460), 20000)).astype(np.float32))
    xs += [1e-30, 2.0 ** -10, 3 * 2.0 ** -11]
    xs += [-x for x in xs]
    return np.asarray(xs, dtype=np.float32)


def test_e4m3_encode_matches_torch_within_range(ora):
    xs = _e4m3_inputs()
    xs = xs[np.abs(xs) <= 448]
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([ora.e4m3_encode(float(x)) for x in xs], dtype=np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(xs[i]), int(got[i]), int(ref[i])) for i in bad[:5]]


def test_e4m3_encode_brute_force_and_saturation(ora):
    mags = [e4m3_from_fields(c) for c in range(127)]
    rng = np.random.default_rng(3)
    for x in list(rng.uniform(0, 500, 3000).astype(np.float32)) + [448.0, 449.0, 464.0, 465.0,
                                                                    1e30, float("inf")]:
        want = brute_nearest(float(x), mags)
        assert ora.e4m3_encode(float(x)) == want, x
        assert ora.e4m3_encode(-float(x)) == (want | 0x80 if want else 0x80), x


@pytest.mark.parametrize("start", [0x00000000, 0x3E7FFF00, 0x40BFFF80, 0xBF3FFFC0, 0x7F7FFFF0])
def test_encode_range_matches_scalar(ora, start):
    n = 4096
    bits = (np.arange(n, dtype=np.uint64) + start).astype(np.uint32)
    xs = bits.view(np.float32)
    e2 = ora.e2m1_encode_range(start, n)
    e4 = ora.e4m3_encode_range(start, n)
    for i in range(0, n, 7):
        if np.isnan(xs[i]):
            assert e2[i] == 0xFF and e4[i] == 0xFF
        else:
            assert e2[i] == ora.e2m1_encode(float(xs[i]))
            assert e4[i] == ora.e4m3_encode(float(xs[i]))
