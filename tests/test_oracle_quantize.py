"""Pins of the oracle's NVFP4 quantiser (tensor scale, 16-element blocks, layouts).

Reading pinned here (the pages name "block-scaled E2M1" / NVFP4 without a
recipe; EFQ-Softmax abstract, TetraJet-v2 abstract): the two-level NVFP4 recipe
s_enc = 2688 / amax, block scale E4M3(a_b / 6 * s_enc), codes E2M1(x * s_enc /
dec(scale)).
"""
import math

import numpy as np
import pytest

from _util import (E2M1_MAG, bf16_bits_to_f32, dequant_rows, e2m1_values, e4m3_values,
                   f32_to_bf16_bits, unpack_codes)


def test_tensor_scale_cases(ora):
    assert ora.tensor_scale(0.0) == (1.0, 1.0)
    assert ora.tensor_scale(2688.0) == (1.0, 1.0)
    assert ora.tensor_scale(10.5) == (256.0, 2.0 ** -8)
    s, d = ora.tensor_scale(1.0)
    assert s == 2688.0 and d == float(np.float32(1) / np.float32(2688))
    s, _ = ora.tensor_scale(1e-45)  # quotient overflows fp32
    assert s == float(np.finfo(np.float32).max)


def test_block_probability_example(ora):
    # p-block {1, 1/2, 1/4, 1/12} with s_enc = 2688 (a-priori amax 1):
    # scale E4M3(fl(fl(1/6) * 2688)) = E4M3(448) = 0x7E, r = 2688/448 = 6,
    # 6p = {6, 3, 1.5, 0.5} -> codes {7, 5, 3, 1}
    x = np.array([1.0, 0.5, 0.25, np.float32(1) / np.float32(12)], np.float32)
    codes, e = ora.quantize_block(x, 2688.0)
    assert e == 0x7E and list(codes) == [7, 5, 3, 1]


def test_block_all_zero_and_signed_zero(ora):
    codes, e = ora.quantize_block(np.zeros(16, np.float32), 2688.0)
    assert e == 0 and not codes.any()
    codes, e = ora.quantize_block(-np.zeros(16, np.float32), 2688.0)
    assert e == 0 and (codes == 8).all()  # sign of zero is kept (r = 0 -> x * 0 = -0)


def test_block_scale_underflow_gives_zero_codes(ora):
    # a_b * s_enc / 6 below half the smallest E4M3 subnormal (2^-10): scale 0, r = 0
    x = np.array([1e-4, -2e-4, 3e-4], np.float32)
    codes, e = ora.quantize_block(x, 1.0)
    assert e == 0 and list(codes) == [0, 8, 0]


@pytest.mark.parametrize("s_enc", [1.0, 256.0, 2.0 ** -3])
def test_exact_round_trip_every_scale(ora, s_enc):
    """Values val(c) * dec(e) / s_enc with a block maximum of 6 dec(e) / s_enc
    re-quantise to the same codes and scale, for every finite nonzero scale e."""
    rng = np.random.default_rng(4)
    for e in range(1, 127):
        de = float(e4m3_values(np.array([e], np.uint8))[0])
        for _ in range(4):
            codes = rng.integers(0, 16, 16).astype(np.uint8)
            codes[rng.integers(0, 16)] = rng.choice([7, 15])
            x = (e2m1_values(codes) * de / s_enc).astype(np.float32)
            assert np.array_equal(x.astype(np.float64), e2m1_values(codes) * de / s_enc)
            got, ge = ora.quantize_block(x, s_enc)
            want = np.where(e2m1_values(codes) == 0, codes & 8, codes)  # +-0 both decode to 0
            assert ge == e, (e, ge)
            assert np.array_equal(got, want), (e, got, codes)


def test_single_nonzero_block_gives_code_six(ora):
    """One nonzero x0 per block: the code is +-6 (index 7) and dec(scale) is the
    E4M3 value nearest |x0| s_enc / 6 (within the two fp32 roundings)."""
    rng = np.random.default_rng(5)
    s_enc = 2688.0 / 5.0
    mags = e4m3_values(np.arange(127, dtype=np.uint8))
    for _ in range(500):
        x0 = np.float32(rng.uniform(0.01, 5.0) * rng.choice([-1, 1]))
        x = np.zeros(16, np.float32)
        pos = rng.integers(0, 16)
        x[pos] = x0
        codes, e = ora.quantize_block(x, s_enc)
        target = abs(float(x0)) * s_enc / 6
        nearest = int(np.argmin(np.abs(mags - target)))
        assert abs(e - nearest) <= 1 and abs(mags[e] - target) <= abs(mags[nearest] - target) * (1 + 1e-6) + 1e-12
        assert codes[pos] == (7 if x0 > 0 else 15)
        assert not np.delete(codes, pos).any()


def test_dequantisation_error_bound(ora, syn):
    """|x~ - x| <= (17/16) a_b / 6 per element for blocks with normal E4M3 scales
    (E2M1 half-step times the scale, with the scale's own 2^-4 rounding)."""
    x = syn.normal_bf16(64 * 128, seed=11).reshape(64, 128)
    amax = ora.amax_bf16(x)
    s_enc, d = ora.tensor_scale(amax)
    codes, scales = ora.quantize_rows(x, s_enc)
    xt = dequant_rows(codes, scales) * d
    xf = bf16_bits_to_f32(x).astype(np.float64)
    ab = np.repeat(np.abs(xf).reshape(64, 8, 16).max(-1), 16, axis=-1)
    normal = np.repeat(scales >= 8, 16, axis=-1)
    err = np.abs(xt - xf)
    assert (err[normal] <= ab[normal] * 17 / 96 * (1 + 1e-6)).all()
    assert np.abs(xt).max() <= amax * (1 + 1e-6)


def test_quantize_rows_layout(ora, syn):
    """quantize_rows = quantize_block on each 16-block, element 2i in the low nibble."""
    x = syn.normal_bf16(7 * 64, seed=12, scale=3.0).reshape(7, 64)
    s_enc, _ = ora.tensor_scale(ora.amax_bf16(x))
    codes, scales = ora.quantize_rows(x, s_enc)
    xf = bf16_bits_to_f32(x)
    for r in range(7):
        for b in range(4):
            c, e = ora.quantize_block(xf[r, b * 16:(b + 1) * 16], s_enc)
            assert scales[r, b] == e
            assert np.array_equal(unpack_codes(codes[r, b * 8:(b + 1) * 8]), c)


@pytest.mark.parametrize("N", [37, 128, 1])
def test_quantize_tokens_T_is_padded_transpose(ora, syn, N):
    """V's blocks run along tokens: quantize_tokens_T(V) equals quantize_rows of
    V^T zero-padded to a multiple of 16 tokens."""
    D = 32
    v = syn.normal_bf16(N * D, seed=13).reshape(N, D)
    s_enc, _ = ora.tensor_scale(ora.amax_bf16(v))
    npad = (N + 15) // 16 * 16
    codes, scales = ora.quantize_tokens_T(v, s_enc)
    vt = np.zeros((D, npad), np.uint16)
    vt[:, :N] = v.T
    c2, s2 = ora.quantize_rows(vt, s_enc)
    assert np.array_equal(codes, c2) and np.array_equal(scales, s2)
    # larger padding adds only zero codes and zero scales
    codes3, scales3 = ora.quantize_tokens_T(v, s_enc, npad=npad + 32)
    assert np.array_equal(codes3[:, :npad // 2], codes) and not codes3[:, npad // 2:].any()
    assert not scales3[:, npad // 16:].any()


def test_amax_matches_numpy(ora, syn):
    x = syn.normal_bf16(100003, seed=14, scale=2.5)
    assert ora.amax_bf16(x) == float(np.abs(bf16_bits_to_f32(x)).max())
