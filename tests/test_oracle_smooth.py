"""Pins of the oracle's Q/K smoothing (oracle flags 32 and 64).

SageAttention2 abstract (searcharxiv.com author page "Pengle Zhang"): Q is
smoothed to make the low-bit QK^T more accurate. Reading (in the oracle's
source, at channel_mean): per (batch, head) and channel the mean over the
head's tokens on a fixed-point grid 2^-(44 - E) (2^(E-1) <= amax < 2^E, each
element truncated toward zero, the integers summed exactly), x' = fl32(x - mean),
quantised as usual; K's correction is a per-row constant the softmax cancels;
Q's is delta_j = mean_Q . k'_j (an fp32 fma chain), taken to the contraction's
units, beta = fl32(delta fl32(s_Q s_K)), split into two tf32 parts hi + lo
(mantissas truncated to 10 bits), and added to the scores before their
rounding: x_ij = fl32(fl32(S'_ij + hi_j + lo_j) c).

Pins: the mean's grid, truncation direction and power-of-two edge by hand; the
mean within one grid step of the fp64 mean; the smoothed quantiser against the
pinned block quantiser on numpy fp32 differences; delta against an exact
rational fma chain; the tf32 split by hand; K-offset invariance of the whole
forward, bit for bit;
closed forms where Q's rows are all equal (Q' = 0, the scores are exactly the
correction), grouped heads included; smoothing lowering the error against
exact attention when Q and K carry channel offsets.
"""
from fractions import Fraction

import numpy as np
import pytest

from _util import bf16_bits_to_f32, f32_to_bf16_bits

LOG2E = np.float32(1.44269504088896340736)


def bf(a):
    return f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def fraction_to_f32(fr: Fraction) -> np.float32:
    """The fp32 nearest to fr, ties to even (exact comparison of the two
    fp32 neighbours of the double nearest to fr)."""
    d = np.float32(float(fr))
    lo = np.nextafter(d, np.float32(-np.inf), dtype=np.float32)
    hi = np.nextafter(d, np.float32(np.inf), dtype=np.float32)
    best = d
    for c in (lo, hi):
        dc, db = abs(Fraction(float(c)) - fr), abs(Fraction(float(best)) - fr)
        if dc < db or (dc == db and (int(np.array(c).view(np.uint32)) & 1) == 0):
            best = c
    return best


def test_mean_hand_cases(ora):
    # amax 1.0 = 0.5 * 2^1: E = 1, grid 2^-43
    x = bf([[1.0, 0.0], [0.5, 0.0], [-0.25, 0.0], [2.0 ** -50, 3.0 * 2.0 ** -44]])
    m = ora.channel_mean(x, 1.0)
    # 2^43 + 2^42 - 2^41 + trunc(2^-7) = 5 * 2^41 -> 5/16; channel 1: trunc(1.5) = 1 -> 2^-43 / 4
    assert m[0] == np.float32(0.3125) and m[1] == np.float32(2.0 ** -45)
    # amax 1024 = 0.5 * 2^11: E = 11, grid 2^-33; 1.5 and -1.5 grid steps truncate toward zero
    x = bf([[3.0 * 2.0 ** -34, -3.0 * 2.0 ** -34, 2.0 ** -40], [0.0, 0.0, 0.0]])
    m = ora.channel_mean(x, 1024.0)
    assert list(m) == [np.float32(2.0 ** -34), np.float32(-(2.0 ** -34)), 0.0]
    # amax just below a power of two: 1.9921875 < 2^1, same E = 1 as 1.0
    x = bf([[1.9921875], [2.0 ** -43]])
    assert ora.channel_mean(x, 1.9921875)[0] == np.float32((1.9921875 + 2.0 ** -43) / 2)
    assert (ora.channel_mean(bf(np.zeros((5, 16))), 0.0) == 0).all()


@pytest.mark.parametrize("N,D,scale", [(1000, 64, 1.0), (4096, 128, 30.0), (7, 16, 1e-3)])
def test_mean_within_one_grid_step(ora, syn, N, D, scale):
    x = syn.normal_bf16(N * D, seed=N + D, scale=scale).reshape(N, D)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    amax = float(np.abs(xf).max())
    E = int(np.frexp(amax)[1])
    step = 2.0 ** (E - 44)
    m = ora.channel_mean(x, amax)
    exact = xf.mean(axis=0)
    assert (np.abs(m.astype(np.float64) - exact) <= step + np.abs(exact) * 2.0 ** -23).all()
    # on the grid (N a power of two), the mean is the fp32 rounding of the exact mean
    g = bf16_bits_to_f32(syn.normal_bf16(256 * D, seed=9)).astype(np.float64).reshape(256, D)
    x2 = bf(np.round(g * 64) / 64)
    x2f = bf16_bits_to_f32(x2).astype(np.float64)
    m2 = ora.channel_mean(x2, float(np.abs(x2f).max()))
    np.testing.assert_array_equal(m2, x2f.mean(axis=0).astype(np.float32))


def test_smoothed_quantiser_and_amax(ora, syn):
    N, D = 300, 128
    x = syn.normal_bf16(N * D, seed=31, scale=2.0).reshape(N, D)
    xf = bf16_bits_to_f32(x)
    xf_off = xf + np.linspace(-6, 6, D, dtype=np.float32)[None, :]
    x = bf(xf_off)
    xf = bf16_bits_to_f32(x)
    mean = ora.channel_mean(x, float(np.abs(xf).max()))
    sm = (xf - mean[None, :]).astype(np.float32)  # fl32(x - mean)
    assert ora.smoothed_amax(x[None], mean[None]) == np.float32(np.abs(sm).max())
    s_enc, _ = ora.tensor_scale(float(np.abs(sm).max()))
    codes, scales = ora.quantize_rows_smoothed(x, s_enc, mean)
    for r in (0, 17, 299):
        for b in range(D // 16):
            c, e = ora.quantize_block(sm[r, 16 * b:16 * b + 16], s_enc)
            assert scales[r, b] == e
            packed = (c[0::2] | (c[1::2] << 4)).astype(np.uint8)
            np.testing.assert_array_equal(codes[r, 8 * b:8 * b + 8], packed)


@pytest.mark.parametrize("smooth_k", [False, True])
def test_score_bias_is_an_fp32_fma_chain(ora, syn, smooth_k):
    N, D = 9, 32
    k = syn.normal_bf16(N * D, seed=41, scale=3.0).reshape(N, D)
    qmean = bf16_bits_to_f32(syn.normal_bf16(D, seed=42)) * np.float32(1.3)
    kmean = (bf16_bits_to_f32(syn.normal_bf16(D, seed=43)) * np.float32(0.7)) if smooth_k else None
    got = ora.score_bias(qmean, k, kmean)
    kf = bf16_bits_to_f32(k)
    for j in range(N):
        kp = (kf[j] - kmean).astype(np.float32) if smooth_k else kf[j]
        delta = np.float32(0.0)
        for d in range(D):
            delta = fraction_to_f32(Fraction(float(qmean[d])) * Fraction(float(kp[d])) +
                                    Fraction(float(delta)))
        assert got[j] == delta, (j, got[j], delta)


def test_bias_split_by_hand(ora):
    # beta = 1 + 2^-12 + 2^-20: tf32 keeps 10 mantissa bits, hi = 1, lo = 2^-12 (1 + 2^-8)
    hi, lo = ora.bias_split(1.0 + 2.0 ** -12 + 2.0 ** -20, 1.0)
    assert (hi, lo) == (1.0, 2.0 ** -12 + 2.0 ** -20)
    # beta = 3 (1 + 2^-23): the last bits go; hi = 3, lo = tf32(3 2^-23) = 3 2^-23
    b = float(np.float32(3.0 * (1 + 2.0 ** -23)))
    hi, lo = ora.bias_split(b, 1.0)
    assert hi == 3.0 and lo == b - 3.0
    # negative values truncate toward zero; fl32(delta sqsk) first: -5 * 0.75
    hi, lo = ora.bias_split(-5.0, 0.75)
    assert (hi, lo) == (-3.75, 0.0)
    # a 24-bit mantissa: hi + lo keeps 11 + 11 bits, the rest is dropped (toward zero)
    m = float(np.float32(1.0 + sum(2.0 ** -i for i in range(1, 24))))  # 2 - 2^-23
    hi, lo = ora.bias_split(m, 1.0)
    assert hi == 2.0 - 2.0 ** -10 and lo == float(np.float32(2.0 ** -10 - 2.0 ** -21))
    assert 0 < m - (hi + lo) < 2.0 ** -20


def _unit_cs_scale():
    """A softmax scale s with fl32(s * log2 e) == 1 exactly, so the scores'
    correction is delta_j itself."""
    s = np.float32(1.0) / LOG2E
    for _ in range(8):
        if np.float32(s * LOG2E) == np.float32(1.0):
            return float(s)
        s = np.nextafter(s, np.float32(1.0), dtype=np.float32)
    raise AssertionError("no fp32 scale maps to 1")


@pytest.mark.parametrize("flags_extra", [0, 32])
def test_equal_query_rows_closed_form(ora, flags_extra):
    """Every row of a query head equals q0 = e_c (channel c = the head): the
    means are q0 exactly, Q' = 0 (s_Q = 1), S' = 0, and the scores are the
    correction alone: x_j = fl32(beta'_j c), beta' = delta_j s_K, c = d_K (the
    unit scale): x_j = k'_jc. K's maximum 5.25 = 2688 / 512 makes s_K = 512
    and every step exact. With k_jc in {0, -1, -2} (+ a constant under K
    smoothing, which cancels; there s_K is not a power of two and the result
    is exact to 2^-18), p = 2^(k_jc - max) in {1, 1/2, 1/4} and V in
    {0, +-1, 1/2} are exact in NVFP4, so out = sum_j p_j v_j / sum_j p_j
    (grouped heads: query head h reads key/value head h / 2)."""
    B, H, Hkv, N, D = 1, 4, 2, 64, 32  # N = 64: the means of integers are exact, so is k - mean
    rng = np.random.default_rng(5)
    q = np.zeros((B, H, N, D), np.float32)
    for h in range(H):
        q[0, h, :, h] = 1.0
    k = np.clip(rng.normal(size=(B, Hkv, N, D)), -4, 4).astype(np.float32)
    for h in range(H):
        k[0, h // 2, :, h] = rng.integers(-2, 1, size=N)
    k[0, 0, 0, D - 1] = 5.25  # max |K| = 2688 / 512
    v = rng.choice([0.0, 1.0, -1.0, 0.5], size=(B, Hkv, N, D)).astype(np.float32)
    v[0, :, 0, 0] = 1.0  # amax(V) = 1
    qb, kb, vb = bf(q), bf(k), bf(v)
    kb_f = bf16_bits_to_f32(kb)
    scale = _unit_cs_scale()
    res = ora.attn_fwd(qb, kb, vb, causal=False, softmax_scale=scale, want_f64=True,
                       flags=ora.FLAG_SMOOTH_Q | flags_extra)
    for h in range(H):
        x = kb_f[0, h // 2, :, h].astype(np.float64)
        p = [Fraction(2) ** int(xi - x.max()) for xi in x]
        for d in range(D):
            exact = sum(pj * Fraction(float(v[0, h // 2, j, d])) for j, pj in enumerate(p)) / sum(p)
            got = res["f64"][0, h, 0, d]
            tol = Fraction(1, 2 ** 21) if not flags_extra else Fraction(1, 2 ** 18)
            assert abs(Fraction(got) - exact) <= abs(exact) * tol + \
                Fraction(1, 2 ** 60), (h, d, got, float(exact))
        # every query row of the head is the same row
        np.testing.assert_array_equal(res["f64"][0, h], np.broadcast_to(res["f64"][0, h, 0], (N, D)))
    # without the correction the scores would all be 0: the plain mean of v, not this
    plain = ora.attn_fwd(qb - qb, kb, vb, causal=False, softmax_scale=scale, want_f64=True)
    assert np.abs(plain["f64"] - res["f64"]).max() > 0.05


@pytest.mark.parametrize("flags", [32, 32 | 64])
@pytest.mark.parametrize("causal", [False, True])
def test_k_offset_invariance(ora, flags, causal):
    """K2 = K + b (one offset per channel for every token): with K smoothed,
    K' is the same bit for bit (values and offsets on a grid where every step
    is exact), so the whole forward is unchanged, bit for bit; unsmoothed it is
    not."""
    B, H, N, D = 1, 2, 200, 64
    rng = np.random.default_rng(7)
    q = bf(rng.normal(size=(B, H, N, D)))
    k = rng.integers(-32, 33, size=(B, H, N, D)) / 8.0        # multiples of 1/8 in [-4, 4]
    b = rng.integers(-8, 9, size=(B, H, 1, D)).astype(np.float64)
    v = bf(rng.normal(size=(B, H, N, D)))
    k1, k2 = bf(k), bf(k + b)
    assert (bf16_bits_to_f32(k2) == (k + b).astype(np.float32)).all()  # exact in bf16
    r1 = ora.attn_fwd(q, k1, v, causal=causal, flags=flags)["bf16"]
    r2 = ora.attn_fwd(q, k2, v, causal=causal, flags=flags)["bf16"]
    np.testing.assert_array_equal(r1, r2)
    u1 = ora.attn_fwd(q, k1, v, causal=causal)["bf16"]
    u2 = ora.attn_fwd(q, k2, v, causal=causal)["bf16"]
    assert (u1 != u2).any()


def test_smoothing_reduces_error_on_channel_offsets(ora, syn):
    """Q and K with large per-channel offsets: smoothing both brings the NVFP4
    forward closer to exact attention of the bf16 inputs."""
    B, H, N, D = 1, 2, 256, 64
    rng = np.random.default_rng(11)
    off_q = rng.normal(scale=6.0, size=(1, H, 1, D))
    off_k = rng.normal(scale=6.0, size=(1, H, 1, D))
    q = bf(rng.normal(size=(B, H, N, D)) + off_q)
    k = bf(rng.normal(size=(B, H, N, D)) + off_k)
    v = bf(rng.normal(size=(B, H, N, D)))
    qf, kf, vf = (bf16_bits_to_f32(t).astype(np.float64) for t in (q, k, v))
    s = np.einsum("bhnd,bhmd->bhnm", qf, kf) / np.sqrt(D)
    p = np.exp(s - s.max(-1, keepdims=True))
    exact = np.einsum("bhnm,bhmd->bhnd", p / p.sum(-1, keepdims=True), vf)
    plain = ora.attn_fwd(q, k, v, causal=False, want_f64=True)["f64"]
    smooth = ora.attn_fwd(q, k, v, causal=False, want_f64=True,
                          flags=ora.FLAG_SMOOTH_Q | ora.FLAG_SMOOTH_K)["f64"]
    e_plain, e_smooth = np.abs(plain - exact).mean(), np.abs(smooth - exact).mean()
    assert e_smooth < 0.7 * e_plain, (e_plain, e_smooth)
