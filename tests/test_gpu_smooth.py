"""Q/K smoothing parity: the CUDA steps (channel means, smoothed maximum,
smoothed NVFP4 codes and scales) bit-exact against the oracle's, Q's score
correction within its stated error bound of the oracle's exact value, and the
whole smoothed forward (fp4_attn_fwd_smooth, through the C
ABI) against the oracle with flags 32 (K) and 64 (Q), with the same bar and
allowances as the main path (tests/test_gpu_attention.py)."""
import numpy as np
import pytest

import bit_attention_transformers_b200 as fa
from _util import bf16_bits_to_f32, f32_to_bf16_bits
from gpu_util import from_dev, scales_rows_logical, to_dev
from test_gpu_attention import SMALL, _rows_per_head, compare

pytestmark = pytest.mark.gpu

SMOOTH = [fa.FP4_SMOOTH_K, fa.FP4_SMOOTH_Q, fa.FP4_SMOOTH_K | fa.FP4_SMOOTH_Q]


def _flags(ora, smooth):
    return (ora.FLAG_SMOOTH_K if smooth & fa.FP4_SMOOTH_K else 0) | \
        (ora.FLAG_SMOOTH_Q if smooth & fa.FP4_SMOOTH_Q else 0)


def _with_offsets(syn, shape, seed, scale=1.0, offset=4.0):
    """bf16 N(0, scale^2) plus a seeded offset per (head, channel), the same
    for every token: the channel outliers smoothing removes."""
    B, H, N, D = shape
    x = bf16_bits_to_f32(syn.normal_bf16(B * H * N * D, seed=seed, scale=scale)).reshape(shape)
    off = bf16_bits_to_f32(syn.normal_bf16(B * H * D, seed=seed, stream=9, scale=offset))
    return f32_to_bf16_bits(x + off.reshape(B, H, 1, D))


@pytest.mark.parametrize("G,N,D", [(1, 1, 64), (2, 37, 128), (3, 300, 64), (2, 1000, 128),
                                   (1, 4096, 128)])
def test_smoothing_steps_bit_exact(ora, syn, G, N, D):
    import torch
    x = _with_offsets(syn, (1, G, N, D), seed=700 + N + D, scale=2.0)[0]
    xd = to_dev(x)
    amax = fa.fp4_amax(xd)
    mean = fa.fp4_channel_mean(xd, amax)
    am_s = fa.fp4_amax_smoothed(xd, mean)
    t = fa.fp4_quantize_smoothed(xd, mean, am_s)
    torch.cuda.synchronize()
    fa.fp4_status()
    a = ora.amax_bf16(x)
    assert float(amax[0].item()) == a
    want_mean = np.stack([ora.channel_mean(x[g], a) for g in range(G)])
    got_mean = mean.cpu().numpy()
    np.testing.assert_array_equal(got_mean.view(np.uint32), want_mean.view(np.uint32))
    a_s = ora.smoothed_amax(x, want_mean)
    assert float(am_s[0].item()) == a_s
    s_enc, _ = ora.tensor_scale(a_s)
    npad = (N + 127) // 128 * 128
    codes = t.codes.cpu().numpy().reshape(G, npad, D // 2)
    scales = scales_rows_logical(t.scales.cpu().numpy(), G, N, D)
    for g in range(G):
        oc, os_ = ora.quantize_rows_smoothed(x[g], s_enc, want_mean[g])
        np.testing.assert_array_equal(codes[g, :N], oc)
        assert not codes[g, N:].any()
        np.testing.assert_array_equal(scales[g], os_)


@pytest.mark.parametrize("B,H,Hkv,N,D", [(1, 2, 2, 300, 64), (2, 4, 2, 130, 128),
                                         (1, 8, 2, 1000, 128)])
@pytest.mark.parametrize("smooth_k", [False, True])
def test_score_bias_within_bound(ora, syn, B, H, Hkv, N, D, smooth_k):
    """The kernel's correction: delta as an fp32 dot product, times fl32(s_Q s_K),
    carried as two parts (hi, lo) of 11 significant bits each (the operands of
    the rank-1 tensor-core product that adds it to S). Against the oracle's
    beta = delta s_Q s_K (exact dot product): |hi + lo - beta| <=
    (D + 4) 2^-24 s_Q s_K sum_d |mean_d k'_d| + 2^-20 |beta|, the distance the
    oracle's flip bound allows for another evaluation of beta."""
    import torch
    k = _with_offsets(syn, (B, Hkv, N, D), seed=800 + N, scale=1.5)
    qmean = bf16_bits_to_f32(syn.normal_bf16(B * H * D, seed=801, scale=3.0)).reshape(B * H, D)
    kmean = (bf16_bits_to_f32(syn.normal_bf16(B * Hkv * D, seed=802, scale=2.0))
             .reshape(B * Hkv, D) if smooth_k else None)
    amax_q, amax_k = np.float32(7.3125), np.float32(11.5)  # the quantised Q', K maxima
    got = fa.fp4_score_bias(torch.from_numpy(qmean).cuda(), to_dev(k),
                            None if kmean is None else torch.from_numpy(kmean).cuda(), H,
                            torch.tensor([amax_q], device="cuda"), torch.tensor([amax_k], device="cuda"))
    torch.cuda.synchronize()
    fa.fp4_status()
    got = got.cpu().numpy()
    sqsk = float(ora.tensor_scale(amax_q)[0]) * float(ora.tensor_scale(amax_k)[0])
    G = H // Hkv
    worst = 0.0
    for b in range(B):
        for h in range(H):
            gk = b * Hkv + h // G
            delta, absum = ora.score_bias(qmean[b * H + h], k[b, h // G],
                                          None if kmean is None else kmean[gk], want_absum=True)
            beta = delta * sqsk
            bound = (D + 4) * 2.0 ** -24 * sqsk * absum + 2.0 ** -20 * np.abs(beta)
            row = got[b * H + h]
            hi, lo = row[:N, 0].astype(np.float64), row[:N, 1].astype(np.float64)
            # two parts of 11 significant bits: the low 13 mantissa bits are clear
            assert not (row[:N, :2].view(np.uint32) & 0x1FFF).any()
            err = np.abs(hi + lo - beta)
            assert (err <= bound).all(), (b, h, float((err / np.maximum(bound, 1e-300)).max()))
            worst = max(worst, float((err / np.maximum(bound, 1e-300)).max()))
            assert not row[:N, 2:].any() and not row[N:].any()
    print(f"score correction: worst |hi + lo - beta| / bound = {worst:.3g}")


def run_smooth(ora, q, k, v, causal, smooth, label, rows=None):
    import torch
    B, H, N, D = q.shape
    out = fa.fp4_attn_fwd_smooth(to_dev(q), to_dev(k), to_dev(v), smooth=smooth, causal=causal)
    torch.cuda.synchronize()
    fa.fp4_status()
    got = from_dev(out)
    vmax = float(np.abs(bf16_bits_to_f32(v)).max())
    if rows is None:
        want = ora.attn_fwd(q, k, v, causal=causal, want_f64=True, want_flip=True, want_ml=True,
                            flags=_flags(ora, smooth))
        heads = np.repeat(np.arange(B * H), N)
        compare(got.reshape(-1, D), {k2: a.reshape(-1, a.shape[-1]) for k2, a in want.items()}, heads, vmax,
                label)
    else:
        want = ora.attn_fwd(q, k, v, causal=causal, rows=rows, want_f64=True, want_flip=True, want_ml=True,
                            flags=_flags(ora, smooth))
        compare(got[rows[:, 0], rows[:, 1], rows[:, 2]], want, rows[:, 0] * H + rows[:, 1], vmax,
                label)
    return got


@pytest.mark.parametrize("B,H,Hkv,N,D,causal", SMALL)
@pytest.mark.parametrize("smooth", SMOOTH)
def test_smooth_small(ora, syn, B, H, Hkv, N, D, causal, smooth):
    s = 9000 + N * 7 + D + 3 * H + int(causal)
    q = _with_offsets(syn, (B, H, N, D), seed=s, scale=1.5)
    k = _with_offsets(syn, (B, Hkv, N, D), seed=s + 1, scale=1.5)
    v = syn.normal_bf16(B * Hkv * N * D, seed=s, stream=3).reshape(B, Hkv, N, D)
    run_smooth(ora, q, k, v, causal, smooth,
               f"smooth={smooth} B{B} H{H} Hkv{Hkv} N{N} D{D} causal={causal}")


def test_smooth_zero_is_the_plain_forward(syn):
    import torch
    B, H, Hkv, N, D = 1, 4, 2, 700, 128
    q = to_dev(_with_offsets(syn, (B, H, N, D), seed=31))
    k = to_dev(_with_offsets(syn, (B, Hkv, N, D), seed=32))
    v = to_dev(syn.normal_bf16(B * Hkv * N * D, seed=33).reshape(B, Hkv, N, D))
    for causal in (False, True):
        a = fa.fp4_attn_fwd_smooth(q, k, v, smooth=0, causal=causal)
        b = fa.fp4_attn_fwd(q, k, v, causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_steps_compose_to_the_fused_call(syn):
    """amax -> means -> smoothed maxima -> smoothed codes -> score correction ->
    fp4_attn_fwd_quantized_bias, through the C ABI step by step, is bit-identical
    to fp4_attn_fwd_smooth."""
    import torch
    B, H, Hkv, N, D = 2, 4, 2, 333, 128
    q = to_dev(_with_offsets(syn, (B, H, N, D), seed=41))
    k = to_dev(_with_offsets(syn, (B, Hkv, N, D), seed=42))
    v = to_dev(syn.normal_bf16(B * Hkv * N * D, seed=43).reshape(B, Hkv, N, D))
    for causal in (False, True):
        want = fa.fp4_attn_fwd_smooth(q, k, v, causal=causal)
        kmean = fa.fp4_channel_mean(k, fa.fp4_amax(k))
        qmean = fa.fp4_channel_mean(q, fa.fp4_amax(q))
        kq = fa.fp4_quantize_smoothed(k, kmean, fa.fp4_amax_smoothed(k, kmean))
        qq = fa.fp4_quantize_smoothed(q, qmean, fa.fp4_amax_smoothed(q, qmean))
        vq = fa.fp4_quantize(v, fa.FP4_BLOCK_ALONG_N_T)
        bias = fa.fp4_score_bias(qmean, k, kmean, H, qq.amax, kq.amax)
        got = fa.fp4_attn_fwd_quantized_bias(qq, kq, vq, bias, B, H, Hkv, causal=causal)
        torch.cuda.synchronize()
        fa.fp4_status()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))


@pytest.mark.parametrize("name", ["tiny", "heavy_tailed", "llm_prefill", "video_dit"])
def test_smooth_workloads(ora, syn, name):
    wl = syn.WORKLOADS[name]
    q, k, v = syn.workload_inputs(wl)
    smooth = fa.FP4_SMOOTH_K | fa.FP4_SMOOTH_Q
    per_head = _rows_per_head(wl)
    rows = syn.sample_rows(wl, per_head) if per_head else None
    run_smooth(ora, q, k, v, wl.causal, smooth, f"smooth {name}", rows=rows)


def test_smoothing_helps_with_channel_offsets(ora, syn):
    """On Q and K with per-channel offsets the smoothed GPU forward is closer
    to exact attention than the plain one."""
    import torch
    B, H, N, D = 1, 4, 1024, 128
    q = _with_offsets(syn, (B, H, N, D), seed=51, offset=6.0)
    k = _with_offsets(syn, (B, H, N, D), seed=52, offset=6.0)
    v = syn.normal_bf16(B * H * N * D, seed=53).reshape(B, H, N, D)
    qf, kf, vf = (bf16_bits_to_f32(t).astype(np.float64) for t in (q, k, v))
    s = np.einsum("bhnd,bhmd->bhnm", qf, kf) / np.sqrt(D)
    p = np.exp(s - s.max(-1, keepdims=True))
    exact = np.einsum("bhnm,bhmd->bhnd", p / p.sum(-1, keepdims=True), vf)
    plain = bf16_bits_to_f32(from_dev(fa.fp4_attn_fwd(to_dev(q), to_dev(k), to_dev(v))))
    smooth = bf16_bits_to_f32(from_dev(fa.fp4_attn_fwd_smooth(to_dev(q), to_dev(k), to_dev(v))))
    torch.cuda.synchronize()
    assert np.abs(smooth - exact).mean() < 0.7 * np.abs(plain - exact).mean()
