"""Pins of the oracle's FP4 attention backward (ora_attn_bwd).

Attn-QAT abstract (arxiv listing "Attn-QAT: 4-Bit Attention With
Quantization-Aware Training"): the backward recomputes the scores in the
forward's low precision, and FlashAttention's D = dO . O carries an implicit
precision assumption. Reading (in the oracle's source, at bwd_row): scores from
the forward's dequantised NVFP4 operands, P their exact softmax (the forward's
probabilities before quantisation), D_i = sum_j P_ij dP_ij from that P and
v~, straight-through quantisers.

Pins: torch autograd in fp64 of softmax(q~ k~^T scale) v~ (a library routine:
the gradient of attention over the dequantised operands, grouped heads by
repeating k~, v~); D against dO . (P v~) and not dO . O of the FP4 forward;
sampled rows against the full computation; the uniform-attention closed form.
"""
import numpy as np
import pytest

from _util import bf16_bits_to_f32

CASES = [  # B, H, Hkv, N, D, causal
    (1, 2, 1, 70, 32, False),
    (1, 2, 1, 70, 32, True),
    (2, 4, 2, 33, 16, True),
    (1, 1, 1, 1, 16, False),
]


def _inputs(syn, B, H, Hkv, N, D, seed):
    q = syn.normal_bf16(B * H * N * D, seed=seed, stream=1, scale=1.5).reshape(B, H, N, D)
    k = syn.normal_bf16(B * Hkv * N * D, seed=seed, stream=2, scale=1.5).reshape(B, Hkv, N, D)
    v = syn.normal_bf16(B * Hkv * N * D, seed=seed, stream=3).reshape(B, Hkv, N, D)
    do = syn.normal_bf16(B * H * N * D, seed=seed, stream=4).reshape(B, H, N, D)
    return q, k, v, do


def _torch_grads(ora, q, k, v, do, causal, scale):
    import torch
    B, H, N, D = q.shape
    G = H // k.shape[1]
    qt = torch.tensor(ora.dequantized(q, "rows"), dtype=torch.float64, requires_grad=True)
    kt = torch.tensor(ora.dequantized(k, "rows"), dtype=torch.float64, requires_grad=True)
    vt = torch.tensor(ora.dequantized(v, "tokens"), dtype=torch.float64, requires_grad=True)
    kr, vr = kt.repeat_interleave(G, dim=1), vt.repeat_interleave(G, dim=1)
    s = torch.einsum("bhnd,bhmd->bhnm", qt, kr) * scale
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    p = torch.softmax(s, dim=-1)
    out = torch.einsum("bhnm,bhmd->bhnd", p, vr)
    dot = torch.tensor(bf16_bits_to_f32(do), dtype=torch.float64)
    (out * dot).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy(), p.detach().numpy(), vr.detach()


@pytest.mark.parametrize("case", CASES)
def test_against_torch_autograd(ora, syn, case):
    B, H, Hkv, N, D, causal = case
    q, k, v, do = _inputs(syn, B, H, Hkv, N, D, 300 + N + D)
    scale = 0.125
    res = ora.attn_bwd(q, k, v, do, causal, softmax_scale=scale, want_D=True)
    gq, gk, gv, p, vr = _torch_grads(ora, q, k, v, do, causal, scale)
    for name, got, want in (("dq", res["dq"], gq), ("dk", res["dk"], gk), ("dv", res["dv"], gv)):
        np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-12 * max(1.0, np.abs(want).max()),
                                   err_msg=name)
    # D = dO . (P v~): the backward's own O, in its own precision
    o_hp = np.einsum("bhnm,bhmd->bhnd", p, vr.numpy())
    np.testing.assert_allclose(res["D"], (bf16_bits_to_f32(do) * o_hp).sum(-1), rtol=1e-9,
                               atol=1e-12)


def test_D_is_not_taken_from_the_fp4_output(ora, syn):
    """The FP4 forward's output uses quantised P~ over the unquantised sum:
    dO . O_fp4 differs from sum_j P_ij dP_ij, which the oracle uses."""
    B, H, N, D = 1, 2, 256, 64
    q, k, v, do = _inputs(syn, B, H, H, N, D, 311)
    res = ora.attn_bwd(q, k, v, do, False, want_D=True, kv_rows=np.zeros((0, 3), np.int64))
    o_fp4 = ora.attn_fwd(q, k, v, causal=False, want_f64=True)["f64"]
    d_fp4 = (bf16_bits_to_f32(do) * o_fp4).sum(-1)
    assert np.abs(res["D"] - d_fp4).max() > 1e-3 * np.abs(res["D"]).max()


def test_sampled_rows_match_the_full_computation(ora, syn):
    B, H, Hkv, N, D = 2, 4, 2, 90, 32
    q, k, v, do = _inputs(syn, B, H, Hkv, N, D, 321)
    full = ora.attn_bwd(q, k, v, do, True)
    qr = np.array([[0, 0, 0], [1, 3, 89], [0, 2, 45], [1, 1, 7]], np.int64)
    kr = np.array([[0, 1, 0], [1, 0, 89], [1, 1, 30]], np.int64)
    part = ora.attn_bwd(q, k, v, do, True, q_rows=qr, kv_rows=kr)
    np.testing.assert_array_equal(part["dq"], full["dq"][qr[:, 0], qr[:, 1], qr[:, 2]])
    np.testing.assert_array_equal(part["dk"], full["dk"][kr[:, 0], kr[:, 1], kr[:, 2]])
    np.testing.assert_array_equal(part["dv"], full["dv"][kr[:, 0], kr[:, 1], kr[:, 2]])


def test_uniform_attention_closed_form(ora, syn):
    """Q = 0: P = 1/N for every key (non-causal), so dv_j = sum over the
    group's heads of mean_i dO_i, and dk = 0 (every dS row is multiplied by
    q~ = 0)."""
    B, H, Hkv, N, D = 1, 4, 2, 50, 32
    _, k, v, do = _inputs(syn, B, H, Hkv, N, D, 331)
    q = np.zeros((B, H, N, D), np.uint16)
    res = ora.attn_bwd(q, k, v, do, False)
    dof = bf16_bits_to_f32(do).astype(np.float64)
    want_dv = dof.mean(axis=2).reshape(B, Hkv, 2, D).sum(axis=2)
    for j in range(N):
        np.testing.assert_allclose(res["dv"][:, :, j], want_dv, rtol=1e-12, atol=1e-14)
    assert (res["dk"] == 0).all()
