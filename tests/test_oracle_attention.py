"""Pins of the oracle's tiled NVFP4 attention forward.

Steps pinned (EFQ-Softmax abstract: exp-then-quantize P, FlashAttention
row-maximum update, historical rescaling, high-precision accumulation, final
normalisation; HiFA4 summary: QK^T and PV both as 4-bit GEMMs with the softmax
state in higher precision):
  * hand-worked 4x4 and 2x2 (grouped heads) examples, tests/golden/;
  * closed forms: uniform scores give mean(v~); one key gives v~_0; causal row
    0 gives v~_0; constant V gives exactly 1 with the p~ denominator;
  * the unscaled scores equal an fp64 matmul of the dequantised operands;
  * tiling: with integer log2-scores the whole forward is exact, so any key
    tile (and the ragged last tile) must equal an untiled exact evaluation;
  * random inputs: brute-force fp64 attention on the dequantised operands with
    unquantised P lies within the a-posteriori FP4 bound of the oracle.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from _util import (bf16_bits_to_f32, bits_to_float, dequant_rows, e2m1_values, e4m3_values,
                   f32_to_bf16_bits, fraction_to_bf16, golden_tensors, load_golden, unpack_codes)


def _dequant_v(ora, v_head, s_enc):
    """[N, D] bf16 -> v~ in real units [N, D] (float64) via the oracle's pinned
    token-block quantiser; s_enc is the whole tensor's scale."""
    N, D = v_head.shape
    codes, scales = ora.quantize_tokens_T(v_head, s_enc)
    vals = e2m1_values(unpack_codes(codes)) * np.repeat(e4m3_values(scales), 16, axis=-1)
    d = float(np.float32(1) / np.float32(s_enc))
    return vals[:, :N].T * d


@pytest.mark.parametrize("name", ["attn_4x4.json", "attn_2x2_gqa.json"])
@pytest.mark.parametrize("mode", ["noncausal", "causal"])
def test_golden_hand_worked(ora, name, mode):
    g = load_golden(name)
    q, k, v = golden_tensors(g)
    scale = bits_to_float(g["softmax_scale_bits"])
    res = ora.attn_fwd(q, k, v, causal=(mode == "causal"), softmax_scale=scale, want_ml=True,
                       want_f64=True)
    H, Hkv = g["shape"]["H"], g["shape"]["Hkv"]
    vf = bf16_bits_to_f32(v).astype(np.float64)
    for row in g["expected"][mode]:
        b, h, i = row["row"]
        m, l = res["ml"][b, h, i][:2]
        assert m == max(row["x"])
        assert Fraction(l) == Fraction(row["l"])
        assert sum(Fraction(p) for p in row["p"]) == Fraction(row["l"])
        pt = [Fraction(p) for p in row["p_tilde"]]
        hk = h // (H // Hkv)
        for d in range(g["shape"]["D"]):
            exact = sum(pt[j] * Fraction(float(vf[b, hk, j, d])) for j in range(len(pt))) / \
                Fraction(row["l"])
            got = Fraction(float(bf16_bits_to_f32(res["bf16"][b, h, i, d])))
            assert got == fraction_to_bf16(exact), (name, mode, row["row"], d, got, exact)
            assert abs(res["f64"][b, h, i, d] - float(exact)) <= 1e-6 * max(1.0, abs(float(exact)))


def test_uniform_scores_give_mean_v(ora, syn):
    """Q = 0: every score is 0, p = 1, p~ = 1 exactly, out = mean_j v~_j."""
    B, H, N, D = 1, 2, 300, 64
    q = np.zeros((B, H, N, D), np.uint16)
    k = syn.normal_bf16(B * H * N * D, seed=21).reshape(B, H, N, D)
    v = syn.normal_bf16(B * H * N * D, seed=22).reshape(B, H, N, D)
    for causal in (False, True):
        res = ora.attn_fwd(q, k, v, causal=causal, want_f64=True)
        s_v, _ = ora.tensor_scale(ora.amax_bf16(v))
        for h in range(H):
            vt = _dequant_v(ora, v[0, h], s_v)
            if causal:
                want = np.cumsum(vt, axis=0) / np.arange(1, N + 1)[:, None]
            else:
                want = np.broadcast_to(vt.mean(0), (N, D))
            np.testing.assert_allclose(res["f64"][0, h], want, rtol=1e-6, atol=1e-7)


def test_single_key_and_causal_row0(ora, syn):
    B, H, D = 1, 1, 32
    for N, causal in ((1, False), (77, True)):
        q = syn.normal_bf16(N * D, seed=23).reshape(B, H, N, D)
        k = syn.normal_bf16(N * D, seed=24).reshape(B, H, N, D)
        v = syn.normal_bf16(N * D, seed=25).reshape(B, H, N, D)
        res = ora.attn_fwd(q, k, v, causal=causal, want_f64=True)
        s_v, _ = ora.tensor_scale(ora.amax_bf16(v))
        vt = _dequant_v(ora, v[0, 0], s_v)
        np.testing.assert_allclose(res["f64"][0, 0, 0], vt[0], rtol=1e-6, atol=1e-7)


def test_constant_v_with_quantized_denominator(ora, syn):
    """V = 1 quantises exactly (scale 448, code 6); with l summing p~ the
    weights sum to one exactly, so out = 1 in every row; with l summing the
    fp32 p the error stays inside the P-quantisation bound."""
    B, H, N, D = 1, 2, 200, 32
    q = syn.normal_bf16(B * H * N * D, seed=26, scale=2.0).reshape(B, H, N, D)
    k = syn.normal_bf16(B * H * N * D, seed=27, scale=2.0).reshape(B, H, N, D)
    v = f32_to_bf16_bits(np.ones((B, H, N, D), np.float32))
    res = ora.attn_fwd(q, k, v, causal=False, flags=ora.FLAG_QP_DENOMINATOR, want_f64=True)
    assert (bf16_bits_to_f32(res["bf16"]) == 1.0).all()
    np.testing.assert_allclose(res["f64"], 1.0, rtol=1e-6)
    res2 = ora.attn_fwd(q, k, v, causal=False, want_f64=True)
    assert np.abs(res2["f64"] - 1.0).max() <= 17 / 96 * 1.0001


def test_scores_match_dequantised_matmul(ora, syn):
    B, H, Hkv, N, D = 1, 4, 2, 96, 64
    q = syn.normal_bf16(B * H * N * D, seed=28).reshape(B, H, N, D)
    k = syn.normal_bf16(B * Hkv * N * D, seed=29, scale=1.7).reshape(B, Hkv, N, D)
    sq, _ = ora.tensor_scale(ora.amax_bf16(q))
    sk, _ = ora.tensor_scale(ora.amax_bf16(k))
    for h in (0, 3):
        S = ora.scores_head(q, k, 0, h)
        qd = dequant_rows(*ora.quantize_rows(q[0, h], sq))
        kd = dequant_rows(*ora.quantize_rows(k[0, h // 2], sk))
        want = (qd @ kd.T).astype(np.float32)
        assert np.array_equal(S, want)


def _dyadic_case(rng, B, H, Hkv, N, D, xmax):
    """Q on the E2M1 grid with a carrier 6 in channel 14, K on 0.25 x grid with
    a carrier 1.5 in channel 15 (so every first block has a power-of-two scale
    and quantises exactly), tensor maxima 10.5 in the second block (Q channel
    16, K channel 17): d_Q = d_K = 2^-8 and, with softmax_scale 0x3F317218,
    the log2 scores x = q . k are integers (channels 0..3 only)."""
    assert D == 32
    q = np.zeros((B, H, N, D), np.float32)
    k = np.zeros((B, Hkv, N, D), np.float32)
    q[..., 14] = 6.0
    k[..., 15] = 1.5
    q[..., :4] = rng.choice([0.0, 4.0], size=(B, H, N, 4))
    k[..., :4] = rng.choice([0.0, 0.25, 0.5, 0.75], size=(B, Hkv, N, 4))
    q[0, 0, 0, 16] = 10.5
    k[0, 0, 0, 17] = 10.5
    x = np.einsum("bhnd,bhmd->bhnm", q[..., :4], np.repeat(k[..., :4], H // Hkv, axis=1))
    assert x.max() <= xmax and np.all(x == np.round(x))
    v = rng.standard_normal((B, Hkv, N, D)).astype(np.float32)
    return f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v), x


# P codes for p = 2^-n relative to the block maximum: 6 * 2^-n is 6, 3, 1.5,
# then 0.75 (tie -> 1), 0.375 (-> 0.5), <= 0.1875 (-> 0); p~ / a_b in sixths.
P_TILDE_BY_SHIFT = {0: Fraction(1), 1: Fraction(1, 2), 2: Fraction(1, 4), 3: Fraction(1, 6),
                    4: Fraction(1, 12)}


def _exact_untiled(x_row, vt, causal_i=None):
    """Untiled, exact evaluation with the global row maximum."""
    n = len(x_row) if causal_i is None else causal_i + 1
    xs = [int(x_row[j]) for j in range(n)]
    M = max(xs)
    p = [Fraction(2) ** (xj - M) for xj in xs]
    l = sum(p)
    num = [Fraction(0)] * vt.shape[1]
    for b0 in range(0, n, 16):
        blk = range(b0, min(b0 + 16, n))
        top = max(xs[j] for j in blk)
        for j in blk:
            pt = Fraction(2) ** (top - M) * P_TILDE_BY_SHIFT.get(top - xs[j], Fraction(0))
            if pt:
                for d in range(vt.shape[1]):
                    num[d] += pt * Fraction(float(vt[j, d]))
    return [nd / l for nd in num]


@pytest.mark.parametrize("Bc", [128, 64, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_tiling_is_exact_on_integer_scores(ora, Bc, causal):
    rng = np.random.default_rng(30)
    B, H, Hkv, N, D = 1, 2, 1, 300, 32
    q, k, v, x = _dyadic_case(rng, B, H, Hkv, N, D, xmax=12)
    scale = bits_to_float("0x3F317218")
    rows = np.array([(0, h, i) for h in range(H) for i in (0, 1, 127, 128, 200, 299)], np.int64)
    res = ora.attn_fwd(q, k, v, causal=causal, softmax_scale=scale, rows=rows, Bc=Bc,
                       want_f64=True)
    s_v, _ = ora.tensor_scale(ora.amax_bf16(v))
    vt = _dequant_v(ora, v[0, 0], s_v)
    for r, (b, h, i) in enumerate(rows):
        want = _exact_untiled(x[b, h, i], vt, i if causal else None)
        np.testing.assert_allclose(res["f64"][r], [float(w) for w in want], rtol=2e-7, atol=1e-9)


def test_bruteforce_fp64_attention_within_fp4_bound(ora, syn):
    """Softmax attention in fp64 on the dequantised q~, k~, v~ with unquantised
    P differs from the oracle only by P's quantisation:
      |out - ref| <= sum_j (17/96) A_b(j) |v~_j| / L  (+ rounding slack)
    with A_b(j) the largest exp2(x - max x) of key j's 16-block."""
    B, H, Hkv, N, D = 1, 2, 1, 200, 64
    q = syn.normal_bf16(B * H * N * D, seed=31).reshape(B, H, N, D)
    k = syn.normal_bf16(B * Hkv * N * D, seed=32).reshape(B, Hkv, N, D)
    v = syn.normal_bf16(B * Hkv * N * D, seed=33).reshape(B, Hkv, N, D)
    for causal in (False, True):
        res = ora.attn_fwd(q, k, v, causal=causal, want_f64=True)
        sq, dq = ora.tensor_scale(ora.amax_bf16(q))
        sk, dk = ora.tensor_scale(ora.amax_bf16(k))
        sv, _ = ora.tensor_scale(ora.amax_bf16(v))
        kd = dequant_rows(*ora.quantize_rows(k[0, 0], sk)) * dk
        vt = _dequant_v(ora, v[0, 0], sv)
        worst = 0.0
        for h in range(H):
            qd = dequant_rows(*ora.quantize_rows(q[0, h], sq)) * dq
            z = (qd @ kd.T) / math.sqrt(D) * math.log2(math.e)
            for i in range(N):
                n = i + 1 if causal else N
                zi = z[i, :n]
                p = np.exp2(zi - zi.max())
                ref = p @ vt[:n] / p.sum()
                A = np.zeros(n)
                for b0 in range(0, n, 16):
                    A[b0:b0 + 16] = p[b0:b0 + 16].max()
                bound = (17 / 96) * (A[:, None] * np.abs(vt[:n])).sum(0) / p.sum()
                err = np.abs(res["f64"][0, h, i] - ref)
                assert (err <= bound * 1.001 + 1e-5).all(), (h, i)
                worst = max(worst, float((err / (bound + 1e-12)).max()))
        assert worst < 1.0


def test_flip_bound_covers_perturbed_evaluations(ora, syn):
    """The flip bound (how far another correct fp32 evaluation can move an
    output through P codes or block scales near a rounding boundary) covers an
    evaluation whose p values are perturbed within the stated uncertainty, and
    is zero where no decision is near a boundary (Q = 0: every 6p is exactly 6)."""
    B, H, N, D = 1, 4, 600, 64
    q = syn.normal_bf16(B * H * N * D, seed=41, scale=3.0).reshape(B, H, N, D)
    k = syn.normal_bf16(B * H * N * D, seed=42, scale=3.0).reshape(B, H, N, D)
    v = syn.normal_bf16(B * H * N * D, seed=43).reshape(B, H, N, D)
    vmax = float(np.abs(bf16_bits_to_f32(v)).max())
    flipped = 0
    for causal in (False, True):
        base = ora.attn_fwd(q, k, v, causal=causal, want_f64=True, want_flip=True, want_ml=True)
        pert = ora.attn_fwd(q, k, v, causal=causal, want_f64=True, flags=ora.FLAG_PERTURB_P)
        diff = np.abs(pert["f64"] - base["f64"])
        slack = 1e-9 * vmax  # rounding of the outputs themselves
        assert (diff <= base["flip"] + slack).all()
        # beyond the continuous change of l (eps |out|) only a flipped decision moves out
        cont = base["ml"][..., 2:3] * np.abs(base["f64"])
        flipped += int((diff > cont + slack).sum())
    assert flipped > 0  # the perturbation does cross boundaries: the check is not vacuous
    zero = ora.attn_fwd(np.zeros_like(q), k, v, causal=False, want_flip=True, want_f64=True)
    assert (zero["flip"] <= 1e-5 * np.abs(zero["f64"])).all()  # only the continuous term
