"""FP8 P and V parity: the CUDA forward with P~ and V in E4M3
(fp4_attn_fwd_fp8pv, through the C ABI) against the oracle with flag 16, and
the FP8 V quantiser (fp4_quantize_fp8) bit-exact against the oracle's.

Same bar and allowances as the exp-then-quantize path
(tests/test_gpu_attention.py): |O_gpu - O_oracle| <= 2e-3 * max|V| per element
plus half a bf16 step of the output plus the oracle's flip bound (keys whose
256 p lies within the fp32 arithmetic's uncertainty of an E4M3 rounding
midpoint; pinned in tests/test_oracle_fp8pv.py), and per-head cosine
>= 0.9999.
"""
import numpy as np
import pytest

import bit_attention_transformers_b200 as fa
from _util import bf16_bits_to_f32, bits_to_float, f32_to_bf16_bits, golden_tensors, load_golden
from gpu_util import from_dev, to_dev
from test_gpu_attention import SMALL, _rows_per_head, compare

pytestmark = pytest.mark.gpu


def run_gpu(q, k, v, causal, softmax_scale=0.0):
    import torch
    out = fa.fp4_attn_fwd(to_dev(q), to_dev(k), to_dev(v), causal=causal,
                          softmax_scale=softmax_scale or None, fp8pv=True)
    torch.cuda.synchronize()
    fa.fp4_status()
    return from_dev(out)


def run_full(ora, q, k, v, causal, label, softmax_scale=0.0):
    B, H, N, D = q.shape
    got = run_gpu(q, k, v, causal, softmax_scale)
    want = ora.attn_fwd(q, k, v, causal=causal, softmax_scale=softmax_scale, want_f64=True,
                        want_flip=True, want_ml=True, flags=ora.FLAG_FP8PV)
    heads = np.repeat(np.arange(B * H), N)
    vmax = float(np.abs(bf16_bits_to_f32(v)).max())
    compare(got.reshape(-1, D), {k2: a.reshape(-1, a.shape[-1]) for k2, a in want.items()}, heads, vmax,
            "FP8PV " + label)


@pytest.mark.parametrize("G,N,D", [(1, 1, 64), (2, 37, 128), (3, 300, 64), (2, 1000, 128)])
def test_fp8_v_quantiser_bit_exact(ora, syn, G, N, D):
    import torch
    x = syn.normal_bf16(G * N * D, seed=900 + N + D, scale=2.0).reshape(G, N, D)
    x[0, 0, 0] = f32_to_bf16_bits(np.array([-30.5], np.float32))[0]  # the maximum, negative
    t = fa.fp4_quantize_fp8(to_dev(x))
    torch.cuda.synchronize()
    fa.fp4_status()
    assert t.scales is None and t.axis == fa.FP8_TOKENS_T
    a = ora.amax_bf16(x)
    assert float(t.amax[0].item()) == a
    s8, _ = ora.fp8_tensor_scale(a)
    npad = (N + 127) // 128 * 128
    codes = t.codes.cpu().numpy().reshape(G, D, npad)
    for g in range(G):
        np.testing.assert_array_equal(codes[g], ora.quantize_fp8_tokens_T(x[g], s8, npad=npad))
    # with the maximum given (the sharded path): the same codes
    t2 = fa.fp4_quantize_fp8(to_dev(x), amax=t.amax)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(t2.codes.cpu().numpy().reshape(G, D, npad), codes)


@pytest.mark.parametrize("B,H,Hkv,N,D,causal", SMALL)
def test_fp8pv_small(ora, syn, B, H, Hkv, N, D, causal):
    s = 6000 + N * 7 + D + 3 * H + int(causal)
    q = syn.normal_bf16(B * H * N * D, seed=s, stream=1, scale=1.5).reshape(B, H, N, D)
    k = syn.normal_bf16(B * Hkv * N * D, seed=s, stream=2, scale=1.5).reshape(B, Hkv, N, D)
    v = syn.normal_bf16(B * Hkv * N * D, seed=s, stream=3).reshape(B, Hkv, N, D)
    run_full(ora, q, k, v, causal, f"B{B} H{H} Hkv{Hkv} N{N} D{D} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_fp8pv_golden(ora, causal):
    """The hand-worked FP8 case (tests/golden/attn_4x4_fp8.json, D = 32),
    zero-padded to D = 64 (zero channels change no dot product, maximum or
    output channel)."""
    g = load_golden("attn_4x4_fp8.json")
    q, k, v = (np.concatenate([t, np.zeros_like(t)], axis=-1) for t in golden_tensors(g))
    run_full(ora, q, k, v, causal, f"golden causal={causal}",
             softmax_scale=bits_to_float(g["softmax_scale_bits"]))
    got = run_gpu(q, k, v, causal, bits_to_float(g["softmax_scale_bits"]))
    want = ora.attn_fwd(q, k, v, causal=causal,
                        softmax_scale=bits_to_float(g["softmax_scale_bits"]),
                        flags=ora.FLAG_FP8PV)["bf16"]
    np.testing.assert_array_equal(got[..., 32:], 0)
    # the hand-worked rows are exact in bf16: the kernel agrees to a bf16 step
    diff = np.abs(bf16_bits_to_f32(got[..., :32]) - bf16_bits_to_f32(want[..., :32]))
    assert diff.max() <= 2.0 ** -7 * np.abs(bf16_bits_to_f32(want)).max() + 1e-30


def test_fp8pv_uniform_and_peaked(ora, syn):
    B, H, N, D = 1, 2, 400, 128
    v = syn.normal_bf16(B * H * N * D, seed=277).reshape(B, H, N, D)
    k = syn.normal_bf16(B * H * N * D, seed=278, scale=4.0).reshape(B, H, N, D)
    run_full(ora, np.zeros_like(v), k, v, False, "Q=0")
    q = syn.normal_bf16(B * H * N * D, seed=279, scale=4.0).reshape(B, H, N, D)
    run_full(ora, q, k, v, True, "peaked causal")


def test_fp8pv_constant_v(ora, syn):
    """V = c: every output is c~ (l sums p, P~ rounds each p to E4M3: the
    output is c~ sum p~ / sum p, within E4M3's half step 2^-4 of c~)."""
    B, H, N, D = 1, 2, 333, 64
    q = syn.normal_bf16(B * H * N * D, seed=280, scale=2.0).reshape(B, H, N, D)
    k = syn.normal_bf16(B * H * N * D, seed=281, scale=2.0).reshape(B, H, N, D)
    v = f32_to_bf16_bits(np.full((B, H, N, D), 0.75, np.float32))
    for causal in (False, True):
        run_full(ora, q, k, v, causal, f"constant V causal={causal}")
        got = bf16_bits_to_f32(run_gpu(q, k, v, causal))
        assert np.abs(got - 0.75).max() <= 0.75 * 2.0 ** -4


@pytest.mark.parametrize("name", ["tiny", "heavy_tailed", "llm_prefill", "video_dit",
                                  "long_context"])
def test_fp8pv_workloads(ora, syn, name):
    wl = syn.WORKLOADS[name]
    q, k, v = syn.workload_inputs(wl)
    got = run_gpu(q, k, v, wl.causal)
    vmax = float(np.abs(bf16_bits_to_f32(v)).max())
    per_head = _rows_per_head(wl)
    if per_head == 0:
        want = ora.attn_fwd(q, k, v, causal=wl.causal, want_f64=True, want_flip=True, want_ml=True,
                            flags=ora.FLAG_FP8PV)
        heads = np.repeat(np.arange(wl.B * wl.H), wl.N)
        compare(got.reshape(-1, wl.D), {k2: a.reshape(-1, a.shape[-1]) for k2, a in want.items()},
                heads, vmax, "FP8PV " + name)
        return
    rows = syn.sample_rows(wl, per_head)
    want = ora.attn_fwd(q, k, v, causal=wl.causal, rows=rows, want_f64=True, want_flip=True, want_ml=True,
                        flags=ora.FLAG_FP8PV)
    got_rows = got[rows[:, 0], rows[:, 1], rows[:, 2]]
    compare(got_rows, want, rows[:, 0] * wl.H + rows[:, 1], vmax,
            f"FP8PV {name} ({per_head} rows/head)")


def test_fp8pv_quantized_entry_matches(syn):
    """fp4_attn_fwd_quantized_fp8pv on fp4_quantize / fp4_quantize_fp8 outputs
    is the same computation as fp4_attn_fwd_fp8pv: bit-identical outputs."""
    import torch
    B, H, Hkv, N, D = 2, 4, 2, 700, 128
    q = to_dev(syn.normal_bf16(B * H * N * D, seed=290).reshape(B, H, N, D))
    k = to_dev(syn.normal_bf16(B * Hkv * N * D, seed=291).reshape(B, Hkv, N, D))
    v = to_dev(syn.normal_bf16(B * Hkv * N * D, seed=292).reshape(B, Hkv, N, D))
    for causal in (False, True):
        a = fa.fp4_attn_fwd(q, k, v, causal=causal, fp8pv=True)
        qq = fa.fp4_quantize(q, fa.FP4_BLOCK_ALONG_D)
        kq = fa.fp4_quantize(k, fa.FP4_BLOCK_ALONG_D)
        vq = fa.fp4_quantize_fp8(v)
        b = fa.fp4_attn_fwd_quantized(qq, kq, vq, B, H, Hkv, causal=causal, fp8pv=True)
        torch.cuda.synchronize()
        fa.fp4_status()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    with pytest.raises(ValueError):
        fa.fp4_attn_fwd_quantized(qq, kq, vq, B, H, Hkv)  # FP8 V without fp8pv
