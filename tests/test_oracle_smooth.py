"""Pins of the oracle's Q/K smoothing (oracle flags 32 and 64).

SageAttention2 abstract (searcharxiv.com author page "Pengle Zhang"): Q is
smoothed to make the low-bit QK^T more accurate. Reading (in the oracle's
source, at channel_mean): per (batch, head) and channel the mean over the
head's tokens on a fixed-point grid 2^-(44 - E) (2^(E-1) <= amax < 2^E, each
element truncated toward zero, the integers summed exactly), x' = fl32(x - mean),
quantised as usual; K's correction is a per-row constant the softmax cancels;
Q's is the dot product delta_j = mean_Q . k'_j, taken to the contraction's
units, beta_j = delta_j s_Q s_K, and added to the scores before their one
rounding: x_ij = fl32(fl32(S'_ij + beta_j) c).

Pins: the mean's grid, truncation direction and power-of-two edge by hand; the
mean within one grid step of the fp64 mean; the smoothed quantiser against the
pinned block quantiser on numpy fp32 differences; delta against the exact
rational dot product; smoothing Q leaving the forward unchanged, bit for bit,
on inputs every step represents exactly (so S' + beta equals the unsmoothed
score); K-offset invariance of the whole forward, bit for bit; closed forms
where Q's rows are all equal (Q' = 0, the scores are exactly the correction),
grouped heads included; smoothing lowering the error against exact attention
when Q and K carry channel offsets.
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
def test_score_bias_is_the_dot_product(ora, syn, smooth_k):
    """delta_j and sum_d |mean_d k'_jd| against exact rational arithmetic: a
    double sum of exact products, within D 2^-53 of the magnitude sum."""
    N, D = 9, 32
    k = syn.normal_bf16(N * D, seed=41, scale=3.0).reshape(N, D)
    qmean = bf16_bits_to_f32(syn.normal_bf16(D, seed=42)) * np.float32(1.3)
    qmean[3] = np.float32(2.0 ** 12 + 1.0)   # a wide exponent spread: the sum needs
    qmean[5] = np.float32(2.0 ** -14)         # more than fp32's 24 bits
    kmean = (bf16_bits_to_f32(syn.normal_bf16(D, seed=43)) * np.float32(0.7)) if smooth_k else None
    got, mag = ora.score_bias(qmean, k, kmean, want_absum=True)
    kf = bf16_bits_to_f32(k)
    for j in range(N):
        kp = (kf[j] - kmean).astype(np.float32) if smooth_k else kf[j]
        prods = [Fraction(float(qmean[d])) * Fraction(float(kp[d])) for d in range(D)]
        exact, absum = sum(prods), sum(abs(t) for t in prods)
        assert abs(Fraction(got[j]) - exact) <= absum * Fraction(D, 2 ** 53), (j, got[j])
        assert abs(Fraction(mag[j]) - absum) <= absum * Fraction(D, 2 ** 53), (j, mag[j])
        # not representable in fp32: the oracle keeps the bits an fp32 sum loses
        assert Fraction(float(np.float32(got[j]))) != exact


def _exact_q_for_smoothing(rng, H, N, D):
    """Q [1, H, N, D] with channel means m (5.25 on channels 16..31, else 0) such
    that Q and Q' = Q - m are both exactly representable in NVFP4 with
    power-of-two tensor scales: every 16-block of a Q' row holds +-5.25 and
    multiples 0.875 g of E2M1 values g; rows come in pairs q' and -q' (the
    channel means of Q' are 0), and channels 16..31 of Q' hold only
    0.875 {0, +-2, +-6} with both +-6 in each row, so Q = Q' + 5.25 there takes
    0.875 {0, 4, 8, 12}: max |Q| = 10.5 = 2688 / 256, max |Q'| = 5.25 = 2688 / 512."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    q = np.zeros((1, H, N, D))
    for h in range(H):
        for i in range(0, N, 2):
            row = np.zeros(D)
            g0 = rng.choice(grid, size=16) * rng.choice([-1, 1], size=16)
            g0[rng.integers(16)] = 6 * rng.choice([-1, 1])
            row[:16] = g0
            g1 = rng.choice([0, 2, 6], size=16) * rng.choice([-1, 1], size=16)
            a, b = rng.choice(16, size=2, replace=False)
            g1[a], g1[b] = 6, -6
            row[16:32] = g1
            q[0, h, i], q[0, h, i + 1] = 0.875 * row, -0.875 * row
    mean = np.zeros(D)
    mean[16:32] = 5.25
    return q + mean


@pytest.mark.parametrize("causal", [False, True])
def test_q_smoothing_is_exact_on_representable_inputs(ora, syn, causal):
    """When Q, Q' = Q - mean_Q and K are exactly representable in NVFP4 with
    power-of-two tensor scales, S'_ij + beta_j is the unsmoothed score in the
    smoothed units (q'_i . k_j + mean_Q . k_j = q_i . k_j), and the two c differ
    by that same power of two: flag 64 must give the unsmoothed forward bit for
    bit. A dropped or mis-signed correction, the wrong key, or a missing
    s_Q s_K factor changes the scores."""
    H, Hkv, N, D = 2, 1, 64, 32
    rng = np.random.default_rng(13)
    q = bf(_exact_q_for_smoothing(rng, H, N, D))
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    k = np.zeros((1, Hkv, N, D))
    for j in range(N):
        for b0 in (0, 16):
            g = rng.choice(grid, size=16) * rng.choice([-1, 1], size=16)
            g[rng.integers(16)] = 6.0
            k[0, 0, j, b0:b0 + 16] = 0.875 * g * 2.0 ** -int(rng.integers(0, 3))
    k[0, 0, 0, :16] = 0.875 * np.where(np.arange(16) == 0, 6.0, 0.0)  # max |K| = 5.25
    kb = bf(k)
    v = syn.normal_bf16(Hkv * N * D, seed=17).reshape(1, Hkv, N, D)
    qf = bf16_bits_to_f32(q).astype(np.float64)
    assert np.abs(qf).max() == 10.5 and (bf16_bits_to_f32(kb) == k).all()
    mean = ora.channel_mean(q[0, 0], float(np.abs(qf).max()))
    assert (mean[16:] == 5.25).all() and (mean[:16] == 0).all()
    plain = ora.attn_fwd(q, kb, v, causal=causal, want_f64=True)
    smooth = ora.attn_fwd(q, kb, v, causal=causal, want_f64=True, flags=ora.FLAG_SMOOTH_Q)
    np.testing.assert_array_equal(smooth["f64"], plain["f64"])
    np.testing.assert_array_equal(smooth["bf16"], plain["bf16"])
    # the correction is needed: Q' alone (the same codes, no beta) is different
    qp = bf(qf - np.concatenate([np.zeros(16), np.full(16, 5.25)]))
    alone = ora.attn_fwd(qp, kb, v, causal=causal, want_f64=True)
    assert np.abs(alone["f64"] - plain["f64"]).max() > 1e-3


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
