"""FP4 attention backward parity: fp4_attn_fwd_lse and fp4_attn_bwd (through
the C ABI) against the oracle (ora_attn_bwd, pinned in tests/test_oracle_bwd.py).

Bar. The oracle computes in fp64; the CUDA path recomputes the same scores
from the same FP4 operands (bit-identical quantisation), forms P in fp32 with
ex2.approx, rounds P and dS to bf16 for the tensor-core contractions (fp32
accumulation) and writes bf16 gradients. Each of those roundings is 2^-9
relative; the sums over keys or queries do not grow it. The tolerance per
gradient tensor: |g - o| <= 1e-2 * max|o| per element, and per head a cosine
similarity >= 0.9995 between the GPU and the oracle gradients.
"""
import numpy as np
import pytest

import bit_attention_transformers_b200 as fa
from _util import bf16_bits_to_f32, f32_to_bf16_bits
from gpu_util import from_dev, to_dev

pytestmark = pytest.mark.gpu

ATOL_REL = 1e-2
COS_MIN = 0.9995

CASES = [  # B, H, Hkv, N, D, causal
    (1, 2, 1, 300, 128, False),
    (1, 2, 1, 300, 128, True),
    (2, 4, 2, 130, 64, True),
    (1, 1, 1, 1, 128, False),
    (1, 1, 1, 1, 64, True),
    (1, 3, 1, 513, 128, False),
    (1, 2, 2, 1000, 64, True),
    (1, 2, 2, 129, 128, False),
    (2, 2, 1, 64, 128, True),
]


def _inputs(syn, B, H, Hkv, N, D, seed):
    q = syn.normal_bf16(B * H * N * D, seed=seed, stream=1, scale=1.5).reshape(B, H, N, D)
    k = syn.normal_bf16(B * Hkv * N * D, seed=seed, stream=2, scale=1.5).reshape(B, Hkv, N, D)
    v = syn.normal_bf16(B * Hkv * N * D, seed=seed, stream=3).reshape(B, Hkv, N, D)
    do = syn.normal_bf16(B * H * N * D, seed=seed, stream=4).reshape(B, H, N, D)
    return q, k, v, do


def run_gpu(q, k, v, do, causal, softmax_scale=0.0):
    import torch
    dq_, dk_, dv_, ddo = (to_dev(t) for t in (q, k, v, do))
    out, lse = fa.fp4_attn_fwd_lse(dq_, dk_, dv_, causal=causal, softmax_scale=softmax_scale or None)
    gq, gk, gv = fa.fp4_attn_bwd(dq_, dk_, dv_, out, ddo, lse, causal=causal,
                                 softmax_scale=softmax_scale or None)
    torch.cuda.synchronize()
    fa.fp4_status()
    return (from_dev(out), lse.cpu().numpy(), bf16_bits_to_f32(from_dev(gq)),
            bf16_bits_to_f32(from_dev(gk)), bf16_bits_to_f32(from_dev(gv)))


def check(got, want, heads, label):
    """got, want: [rows, D]; heads: [rows] head id of each row."""
    got = got.astype(np.float64)
    # a gradient that is exactly 0 (one key: dS = P (dP - D) = 0) comes out of
    # fp32 arithmetic as rounding noise: an absolute floor of 1e-4 (the inputs
    # and dO are O(1))
    scale = max(np.abs(want).max(), 1e-4)
    err = np.abs(got - want)
    assert np.isfinite(got).all(), label
    assert err.max() <= ATOL_REL * scale + 1e-30, \
        f"{label}: max err {err.max():.3e} > {ATOL_REL} * {scale:.3e}"
    for h in np.unique(heads):
        a, b = got[heads == h].ravel(), want[heads == h].ravel()
        na, nb = np.linalg.norm(a), np.linalg.norm(b)
        if nb < 1e-12:
            assert na <= 1e-5 * max(1.0, np.sqrt(a.size)), label
            continue
        cos = a @ b / (na * nb)
        assert cos >= COS_MIN, f"{label} head {h}: cosine {cos:.6f}"


def test_forward_lse_matches_the_oracle(ora, syn):
    B, H, Hkv, N, D = 1, 4, 2, 700, 128
    q, k, v, do = _inputs(syn, B, H, Hkv, N, D, 41)
    import torch
    for causal in (False, True):
        out, lse, *_ = run_gpu(q, k, v, do, causal)
        plain = from_dev(fa.fp4_attn_fwd(to_dev(q), to_dev(k), to_dev(v), causal=causal))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out, plain)  # the same forward, plus lse
        ml = ora.attn_fwd(q, k, v, causal=causal, want_ml=True)["ml"]
        want = ml[..., 0] + np.log2(ml[..., 1])
        np.testing.assert_allclose(lse, want, rtol=0, atol=2e-5 * max(1.0, np.abs(want).max()))


@pytest.mark.parametrize("case", CASES)
def test_backward_small(ora, syn, case):
    B, H, Hkv, N, D, causal = case
    q, k, v, do = _inputs(syn, B, H, Hkv, N, D, 100 + N + D + H)
    _, _, gq, gk, gv = run_gpu(q, k, v, do, causal)
    want = ora.attn_bwd(q, k, v, do, causal)
    label = f"B{B} H{H} Hkv{Hkv} N{N} D{D} causal={causal}"
    check(gq.reshape(-1, D), want["dq"].reshape(-1, D), np.repeat(np.arange(B * H), N), "dq " + label)
    check(gk.reshape(-1, D), want["dk"].reshape(-1, D), np.repeat(np.arange(B * Hkv), N),
          "dk " + label)
    check(gv.reshape(-1, D), want["dv"].reshape(-1, D), np.repeat(np.arange(B * Hkv), N),
          "dv " + label)


def test_backward_softmax_scale_and_peaked(ora, syn):
    B, H, N, D = 1, 2, 256, 64
    q, k, v, do = _inputs(syn, B, H, H, N, D, 55)
    _, _, gq, gk, gv = run_gpu(q, k, v, do, False, softmax_scale=0.6)
    want = ora.attn_bwd(q, k, v, do, False, softmax_scale=0.6)
    heads = np.repeat(np.arange(B * H), N)
    for name, g in (("dq", gq), ("dk", gk), ("dv", gv)):
        check(g.reshape(-1, D), want[name].reshape(-1, D), heads, name + " peaked")


@pytest.mark.parametrize("name", ["tiny", "heavy_tailed", "llm_prefill", "video_dit"])
def test_backward_workloads(ora, syn, name):
    wl = syn.WORKLOADS[name]
    q, k, v = syn.workload_inputs(wl)
    do = syn.normal_bf16(q.size, seed=wl.seed + 17, stream=5).reshape(q.shape)
    _, _, gq, gk, gv = run_gpu(q, k, v, do, wl.causal)
    D = wl.D
    if name in ("tiny", "heavy_tailed"):
        want = ora.attn_bwd(q, k, v, do, wl.causal)
        check(gq.reshape(-1, D), want["dq"].reshape(-1, D), np.repeat(np.arange(wl.B * wl.H), wl.N),
              "dq " + name)
        kvh = np.repeat(np.arange(wl.B * wl.Hkv), wl.N)
        check(gk.reshape(-1, D), want["dk"].reshape(-1, D), kvh, "dk " + name)
        check(gv.reshape(-1, D), want["dv"].reshape(-1, D), kvh, "dv " + name)
        return
    # large: seeded sampled dq rows of every head; dk / dv rows of the first
    # key/value head (their oracle cost grows with N^2)
    rows = syn.sample_rows(wl, 8)
    want = ora.attn_bwd(q, k, v, do, wl.causal, q_rows=rows, kv_rows=np.zeros((0, 3), np.int64))
    got = gq[rows[:, 0], rows[:, 1], rows[:, 2]]
    check(got, want["dq"], rows[:, 0] * wl.H + rows[:, 1], "dq " + name)
    if name == "llm_prefill":
        kr = np.stack([np.zeros(16, np.int64), np.zeros(16, np.int64),
                       np.sort(syn.distinct(16, wl.N, seed=wl.seed + 3))], axis=1)
        want = ora.attn_bwd(q, k, v, do, wl.causal, q_rows=np.zeros((0, 3), np.int64), kv_rows=kr)
        check(gk[kr[:, 0], kr[:, 1], kr[:, 2]], want["dk"], np.zeros(16), "dk " + name)
        check(gv[kr[:, 0], kr[:, 1], kr[:, 2]], want["dv"], np.zeros(16), "dv " + name)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_offset_v_and_peaked_rows(ora, syn, causal):
    """V with a large common offset per channel (dP_ij = dO_i . v_j then shares
    a large term across the keys of a row) and sharp scores (most rows' P sits
    on a few keys): the cases where dQ = scale d_K (A - (D - c) B), formed in
    one pass, could cancel large terms. The bar is the usual one."""
    B, H, Hkv, N, D = 1, 2, 1, 300, 128
    q, k, v, do = _inputs(syn, B, H, Hkv, N, D, 321)
    qf = bf16_bits_to_f32(q) * 3.0
    kf = bf16_bits_to_f32(k) * 3.0
    offs = (np.arange(D, dtype=np.float32) % 7 - 3.0) * 4.0  # per-channel offsets up to 12
    vf = bf16_bits_to_f32(v) + offs
    q, k, v = (f32_to_bf16_bits(x) for x in (qf, kf, vf))
    _, _, gq, gk, gv = run_gpu(q, k, v, do, causal)
    want = ora.attn_bwd(q, k, v, do, causal)
    label = f"offset V, peaked, causal={causal}"
    check(gq.reshape(-1, D), want["dq"].reshape(-1, D), np.repeat(np.arange(B * H), N), "dq " + label)
    check(gk.reshape(-1, D), want["dk"].reshape(-1, D), np.repeat(np.arange(B * Hkv), N),
          "dk " + label)
    check(gv.reshape(-1, D), want["dv"].reshape(-1, D), np.repeat(np.arange(B * Hkv), N),
          "dv " + label)
