"""Pins of the oracle's FP8 P and V path (oracle flag 16).

SageAttention2 abstract (searcharxiv.com author page "Pengle Zhang"): P~ and V
quantised to FP8 for the PV product. Reading (in the oracle's source): V with
one fp32 scale s8 = 448 / amax, codes E4M3(fl(v s8)); P~ = E4M3(fl(256 p)) / 256;
l sums the unquantised p. Pins: the FP8 V quantiser against torch's
float8_e4m3fn cast and its layout; the hand-worked golden case
(tests/golden/attn_4x4_fp8.json); closed forms (uniform scores, constant V with
the p~ denominator); the E4M3 error bound of P~; the flip bound against
perturbed evaluations."""
from fractions import Fraction

import numpy as np
import pytest

from _util import (bf16_bits_to_f32, bits_to_float, f32_to_bf16_bits, fraction_to_bf16,
                   golden_tensors, load_golden)


def test_fp8_v_quantiser_matches_torch(ora, syn):
    import torch
    N, D = 77, 64
    x = syn.normal_bf16(N * D, seed=81, scale=3.0).reshape(N, D)
    x[5, 7] = f32_to_bf16_bits(np.array([-40.0], np.float32))[0]
    amax = ora.amax_bf16(x)
    s8, d8 = ora.fp8_tensor_scale(amax)
    assert s8 == np.float32(448.0) / np.float32(amax) and d8 == np.float32(1.0) / np.float32(s8)
    codes = ora.quantize_fp8_tokens_T(x, s8, npad=128)
    assert codes.shape == (D, 128) and not codes[:, N:].any()
    prod = (bf16_bits_to_f32(x).astype(np.float32) * np.float32(s8)).astype(np.float32)
    want = torch.from_numpy(prod).to(torch.float8_e4m3fn).view(torch.uint8).numpy().T
    np.testing.assert_array_equal(codes[:, :N], want)
    assert ora.fp8_tensor_scale(0.0) == (1.0, 1.0)


@pytest.mark.parametrize("mode", ["noncausal", "causal"])
def test_golden_hand_worked(ora, mode):
    g = load_golden("attn_4x4_fp8.json")
    q, k, v = golden_tensors(g)
    scale = bits_to_float(g["softmax_scale_bits"])
    res = ora.attn_fwd(q, k, v, causal=(mode == "causal"), softmax_scale=scale, want_ml=True,
                       want_f64=True, flags=ora.FLAG_FP8PV)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    for row in g["expected"][mode]:
        b, h, i = row["row"]
        m, l = res["ml"][b, h, i][:2]
        assert m == max(row["x"])
        assert Fraction(l) == Fraction(row["l"])
        pt = [Fraction(p) for p in row["p_tilde"]]
        for d in range(g["shape"]["D"]):
            exact = sum(pt[j] * Fraction(float(vf[b, 0, j, d])) for j in range(len(pt))) / \
                Fraction(row["l"])
            got = Fraction(float(bf16_bits_to_f32(res["bf16"][b, h, i, d])))
            assert got == fraction_to_bf16(exact), (mode, row["row"], d, got, exact)


def test_uniform_scores_and_constant_v(ora, syn):
    B, H, N, D = 1, 2, 300, 64
    q = np.zeros((B, H, N, D), np.uint16)
    k = syn.normal_bf16(B * H * N * D, seed=82).reshape(B, H, N, D)
    v = syn.normal_bf16(B * H * N * D, seed=83).reshape(B, H, N, D)
    s8, d8 = ora.fp8_tensor_scale(ora.amax_bf16(v))
    res = ora.attn_fwd(q, k, v, causal=False, want_f64=True, flags=ora.FLAG_FP8PV)
    for h in range(H):
        from_codes = ora.quantize_fp8_tokens_T(v[0, h], s8)
        import torch
        vt = torch.from_numpy(from_codes).view(torch.float8_e4m3fn).float().numpy().T * d8
        np.testing.assert_allclose(res["f64"][0, h], np.broadcast_to(vt.mean(0), (N, D)),
                                   rtol=1e-6, atol=1e-7)
    ones = f32_to_bf16_bits(np.ones((B, H, N, D), np.float32))
    qn = syn.normal_bf16(B * H * N * D, seed=84, scale=2.0).reshape(B, H, N, D)
    res = ora.attn_fwd(qn, k, ones, causal=True, want_f64=True,
                       flags=ora.FLAG_FP8PV | ora.FLAG_QP_DENOMINATOR)
    assert (bf16_bits_to_f32(res["bf16"]) == 1.0).all()


def test_p_quantisation_error_bound(ora, syn):
    """E4M3 keeps 3 fraction bits: p~ = p (1 + d) with |d| <= 2^-4 (256 p normal;
    below that the absolute error is under 2^-18), and l sums the unquantised p,
    so out is within 2^-4 max|v~| of fp64 softmax attention on the same
    dequantised scores and V (computed here from the pinned score and
    quantiser routines)."""
    import torch
    B, H, N, D = 1, 2, 256, 64
    q = syn.normal_bf16(B * H * N * D, seed=85, scale=1.5).reshape(B, H, N, D)
    k = syn.normal_bf16(B * H * N * D, seed=86, scale=1.5).reshape(B, H, N, D)
    v = syn.normal_bf16(B * H * N * D, seed=87).reshape(B, H, N, D)
    got = ora.attn_fwd(q, k, v, causal=False, want_f64=True, flags=ora.FLAG_FP8PV)["f64"]
    sq, dq = ora.tensor_scale(ora.amax_bf16(q))
    sk, dk = ora.tensor_scale(ora.amax_bf16(k))
    s8, d8 = ora.fp8_tensor_scale(ora.amax_bf16(v))
    c = np.float32(np.float32(np.float32(dq) * np.float32(dk)) * np.float32(1.0 / 8.0)) * \
        np.float32(1.4426950408889634)
    for h in range(H):
        x = ora.scores_head(q, k, 0, h).astype(np.float64) * float(c)
        w = np.exp2(x - x.max(1, keepdims=True))
        w /= w.sum(1, keepdims=True)
        vt = torch.from_numpy(ora.quantize_fp8_tokens_T(v[0, h], s8)).view(
            torch.float8_e4m3fn).double().numpy().T * d8
        exact = w @ vt
        assert np.abs(got[0, h] - exact).max() <= 2.0 ** -4 * np.abs(vt).max() * 1.001


def test_flip_bound_covers_perturbed_evaluations(ora, syn):
    B, H, N, D = 1, 4, 600, 64
    q = syn.normal_bf16(B * H * N * D, seed=88, scale=3.0).reshape(B, H, N, D)
    k = syn.normal_bf16(B * H * N * D, seed=89, scale=3.0).reshape(B, H, N, D)
    v = syn.normal_bf16(B * H * N * D, seed=90).reshape(B, H, N, D)
    vmax = float(np.abs(bf16_bits_to_f32(v)).max())
    flipped = 0
    for causal in (False, True):
        base = ora.attn_fwd(q, k, v, causal=causal, want_f64=True, want_flip=True, want_ml=True,
                            flags=ora.FLAG_FP8PV)
        pert = ora.attn_fwd(q, k, v, causal=causal, want_f64=True,
                            flags=ora.FLAG_FP8PV | ora.FLAG_PERTURB_P)
        diff = np.abs(pert["f64"] - base["f64"])
        slack = 1e-9 * vmax
        assert (diff <= base["flip"] + slack).all()
        cont = base["ml"][..., 2:3] * np.abs(base["f64"])
        flipped += int((diff > cont + slack).sum())
    assert flipped > 0
