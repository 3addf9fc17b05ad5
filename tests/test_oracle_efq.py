"""Pins of the oracle's EFQ-Softmax P generation (oracle flag 8).

EFQ-Softmax abstract (scholarbro.com page "AVQ Attention: Adaptive
Vector-Quantized Attention"): per microscaling block an exponent-only scale
from the local maximum, the shifted scores mapped to a normalised residual
domain, E2M1 codes from a single affine rule, and the same operand in the
numerator (P~V) and the denominator (P~1); row-maximum update, rescaling,
accumulation and normalisation unchanged. The reading (in the oracle's source):
E = floor(max z) - 2, code = clamp(rne(2 (z - E) + 2), 0, 7), p~ = val(code) 2^E,
stored with P's tensor scale 2^-10.

Pins: block codes listed by hand (ties, clamp, the E4M3 power-of-two scale byte,
its subnormal end and underflow); invariants any block must satisfy (the maximum
lands on code 6 or 7; p~ / 2^z lies in the band the affine rule allows; keys
more than 2.75 binades below the block scale are dropped); the hand-worked
golden attention cases (tests/golden/, "expected_efq"); closed forms (uniform
scores, constant V, one key); the flip bound against perturbed evaluations.
"""
from fractions import Fraction

import numpy as np
import pytest

from _util import (bf16_bits_to_f32, bits_to_float, e2m1_values, e4m3_values, f32_to_bf16_bits,
                   fraction_to_bf16, golden_tensors, load_golden, unpack_codes)

NEG = -np.inf


def _block(ora, z):
    codes, e, E = ora.efq_block(np.array(z, dtype=np.float64))
    return list(codes), e, E


def test_block_hand_cases(ora):
    # max z = 0 -> E = -2, 2 (z - E) + 2 = 2 z + 6; scale byte 2^(E + 10) = 2^8 = 0x78
    codes, e, E = _block(ora, [0, -0.5, -1, -1.25, -2, -3, -2.75, -2.25, -2.5, NEG])
    assert E == -2 and e == 0x78
    # 2z+6: 6, 5, 4, 3.5 (tie -> even 4), 2, 0, 0.5 (tie -> even 0), 1.5 (tie -> 2), 1, masked
    assert codes == [6, 5, 4, 4, 2, 0, 0, 2, 1, 0]
    # max z = -0.1 -> floor -1, E = -3, 2 z + 8: -0.3 -> 7.4 -> 7, -0.1 -> 7.8 -> 8 clamped to 7
    codes, e, E = _block(ora, [-0.3, -0.1, -1.1, -4.2])
    assert E == -3 and e == 0x70  # 2^7
    # -1.1 -> 5.8 -> 6; -4.2 -> -0.4 -> 0
    assert codes == [7, 7, 6, 0]
    # max z = -5.5 -> floor -6, E = -8, scale 2^2 = 0x48; 2 (z + 8) + 2 = 2z + 18
    codes, e, E = _block(ora, [-5.5, -6.0, -7.75, -8.25])
    assert E == -8 and e == 0x48
    # 7, 6, 2.5 (tie -> 2), 1.5 (tie -> 2)
    assert codes == [7, 6, 2, 2]
    # E + 10 = -9: the smallest E4M3 power of two, the subnormal 2^-9 (byte 0x01)
    codes, e, E = _block(ora, [-16.5, -17.0])
    assert (E, e, codes) == (-19, 0x01, [7, 6])
    # E + 10 = -10: no E4M3 byte, the block is zero
    codes, e, E = _block(ora, [-17.2, -17.5])
    assert (E, e, codes) == (-20, 0, [0, 0])
    codes, e, E = _block(ora, [NEG, NEG])
    assert (E, e, codes) == (None, 0, [0, 0])


def test_block_invariants(ora):
    rng = np.random.default_rng(7)
    e2m1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    for trial in range(400):
        n = int(rng.integers(1, 17))
        top = -float(rng.uniform(0, 14))
        z = top - rng.exponential(1.5, n)
        z[int(rng.integers(0, n))] = top
        if trial % 5 == 0:
            z[rng.random(n) < 0.3] = NEG
            z[0] = top
        codes, e, E = ora.efq_block(z)
        assert E == int(np.floor(top)) - 2
        assert e4m3_values(np.array([e]))[0] == 2.0 ** (E + 10)
        live = np.isfinite(z)
        assert codes[np.argmax(np.where(live, z, NEG))] in (6, 7)
        order = np.argsort(np.where(live, z, -1e9))
        assert (np.diff(codes[order].astype(int)) >= 0).all()  # monotone in z
        pt = e2m1[codes] * 2.0 ** E
        r = z - E
        kept = codes > 0
        ratio = pt[kept] / 2.0 ** z[kept]
        # |2r + 2 - code| <= 1/2 bounds val(code) / 2^r by [0.59, 1.27]; the clamp at
        # code 7 for r in [2.75, 3) by [0.75, 0.9]
        assert ((ratio > 0.59) & (ratio < 1.27)).all(), (z, codes)
        assert (r[live & ~kept] < -0.75 + 1e-12).all()  # dropped keys lie below the code-1 band
        assert (r[live & kept] >= -0.75 - 1e-12).all()


@pytest.mark.parametrize("name", ["attn_4x4.json", "attn_2x2_gqa.json"])
@pytest.mark.parametrize("mode", ["noncausal", "causal"])
def test_golden_hand_worked(ora, name, mode):
    g = load_golden(name)
    q, k, v = golden_tensors(g)
    scale = bits_to_float(g["softmax_scale_bits"])
    res = ora.attn_fwd(q, k, v, causal=(mode == "causal"), softmax_scale=scale, want_ml=True,
                       want_f64=True, flags=ora.FLAG_EFQ)
    H, Hkv = g["shape"]["H"], g["shape"]["Hkv"]
    vf = bf16_bits_to_f32(v).astype(np.float64)
    for row in g["expected_efq"][mode]:
        b, h, i = row["row"]
        m, l = res["ml"][b, h, i][:2]
        assert m == max(row["x"])
        pt = [Fraction(p) for p in row["p_tilde"]]
        assert Fraction(l) == Fraction(row["l"]) == sum(pt)
        hk = h // (H // Hkv)
        for d in range(g["shape"]["D"]):
            exact = sum(pt[j] * Fraction(float(vf[b, hk, j, d])) for j in range(len(pt))) / sum(pt)
            got = Fraction(float(bf16_bits_to_f32(res["bf16"][b, h, i, d])))
            assert got == fraction_to_bf16(exact), (name, mode, row["row"], d, got, exact)


def _dequant_v(ora, v_head, s_enc):
    N, D = v_head.shape
    codes, scales = ora.quantize_tokens_T(v_head, s_enc)
    vals = e2m1_values(unpack_codes(codes)) * np.repeat(e4m3_values(scales), 16, axis=-1)
    return vals[:, :N].T * float(np.float32(1) / np.float32(s_enc))


def test_uniform_scores_give_mean_v(ora, syn):
    """Q = 0: every z is 0, every code 6, p~ equal: out = mean_j v~_j."""
    B, H, N, D = 1, 2, 300, 64
    q = np.zeros((B, H, N, D), np.uint16)
    k = syn.normal_bf16(B * H * N * D, seed=61).reshape(B, H, N, D)
    v = syn.normal_bf16(B * H * N * D, seed=62).reshape(B, H, N, D)
    s_v, _ = ora.tensor_scale(ora.amax_bf16(v))
    for causal in (False, True):
        res = ora.attn_fwd(q, k, v, causal=causal, want_f64=True, flags=ora.FLAG_EFQ)
        for h in range(H):
            vt = _dequant_v(ora, v[0, h], s_v)
            if causal:
                want = np.cumsum(vt, axis=0) / np.arange(1, N + 1)[:, None]
            else:
                want = np.broadcast_to(vt.mean(0), (N, D))
            np.testing.assert_allclose(res["f64"][0, h], want, rtol=1e-6, atol=1e-7)


def test_constant_v_and_single_key(ora, syn):
    """The same p~ weights the numerator and the denominator: constant V gives
    out = 1 exactly; one key gives v~_0."""
    B, H, N, D = 1, 2, 200, 32
    q = syn.normal_bf16(B * H * N * D, seed=63, scale=2.0).reshape(B, H, N, D)
    k = syn.normal_bf16(B * H * N * D, seed=64, scale=2.0).reshape(B, H, N, D)
    v = f32_to_bf16_bits(np.ones((B, H, N, D), np.float32))
    for causal in (False, True):
        res = ora.attn_fwd(q, k, v, causal=causal, want_f64=True, flags=ora.FLAG_EFQ)
        assert (bf16_bits_to_f32(res["bf16"]) == 1.0).all()
        np.testing.assert_allclose(res["f64"], 1.0, rtol=1e-6)  # fl32(d_P d_V) rounds
    q1 = syn.normal_bf16(D, seed=65).reshape(1, 1, 1, D)
    k1 = syn.normal_bf16(D, seed=66).reshape(1, 1, 1, D)
    v1 = syn.normal_bf16(D, seed=67).reshape(1, 1, 1, D)
    res = ora.attn_fwd(q1, k1, v1, causal=False, want_f64=True, flags=ora.FLAG_EFQ)
    s_v, _ = ora.tensor_scale(ora.amax_bf16(v1))
    np.testing.assert_allclose(res["f64"][0, 0, 0], _dequant_v(ora, v1[0, 0], s_v)[0], rtol=1e-12)


def test_differs_from_exp_then_quantize(ora, syn):
    """EFQ is another P: on random inputs its outputs differ from the
    exp-then-quantize path (and stay a weighted mean of v~: within max |v~|)."""
    B, H, N, D = 1, 2, 256, 64
    q = syn.normal_bf16(B * H * N * D, seed=68, scale=2.0).reshape(B, H, N, D)
    k = syn.normal_bf16(B * H * N * D, seed=69, scale=2.0).reshape(B, H, N, D)
    v = syn.normal_bf16(B * H * N * D, seed=70).reshape(B, H, N, D)
    a = ora.attn_fwd(q, k, v, causal=False, want_f64=True)["f64"]
    e = ora.attn_fwd(q, k, v, causal=False, want_f64=True, flags=ora.FLAG_EFQ)["f64"]
    assert np.abs(a - e).max() > 1e-3
    assert np.abs(e).max() <= np.abs(bf16_bits_to_f32(v)).max() * 1.0001


def test_flip_bound_covers_perturbed_evaluations(ora, syn):
    B, H, N, D = 1, 4, 600, 64
    q = syn.normal_bf16(B * H * N * D, seed=71, scale=3.0).reshape(B, H, N, D)
    k = syn.normal_bf16(B * H * N * D, seed=72, scale=3.0).reshape(B, H, N, D)
    v = syn.normal_bf16(B * H * N * D, seed=73).reshape(B, H, N, D)
    vmax = float(np.abs(bf16_bits_to_f32(v)).max())
    flipped = 0
    for causal in (False, True):
        base = ora.attn_fwd(q, k, v, causal=causal, want_f64=True, want_flip=True,
                            flags=ora.FLAG_EFQ)
        pert = ora.attn_fwd(q, k, v, causal=causal, want_f64=True,
                            flags=ora.FLAG_EFQ | ora.FLAG_PERTURB_P)
        diff = np.abs(pert["f64"] - base["f64"])
        slack = 1e-9 * vmax
        assert (diff <= base["flip"] + slack).all()
        flipped += int((diff > slack).sum())
    assert flipped > 0  # the perturbation crosses rounding points: the check is not vacuous
    zero = ora.attn_fwd(np.zeros_like(q), k, v, causal=False, want_flip=True, want_f64=True,
                        flags=ora.FLAG_EFQ)
    assert (zero["flip"] == 0).all()  # every t is exactly 6, max z exactly 0
