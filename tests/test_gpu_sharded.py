"""The head-sharded forward on one GPU, through the C ABI.

fp4_amax / fp4_quantize_scaled split fp4_quantize in two; with one rank the
sharded call must equal fp4_attn_fwd bit for bit. 2- and 3-way shardings are
emulated on the one GPU: every shard's maxima come from fp4_amax, they are
combined by max (what the all-reduce computes across ranks), and each shard
is quantised with them and run alone. Its codes, scales and output heads must
equal the corresponding slabs of the unsharded run exactly."""
import numpy as np
import pytest

import bit_attention_transformers_b200 as fa
from gpu_util import from_dev, to_dev

pytestmark = pytest.mark.gpu

CASES = [  # B, H, Hkv, N, D, causal
    (1, 4, 4, 300, 128, False),
    (2, 8, 2, 1000, 64, True),
    (1, 6, 3, 257, 128, True),
]


def _inputs(syn, B, H, Hkv, N, D, seed):
    q = syn.normal_bf16(B * H * N * D, seed, 1).reshape(B, H, N, D)
    k = syn.normal_bf16(B * Hkv * N * D, seed, 2, scale=2.0).reshape(B, Hkv, N, D)
    v = syn.normal_bf16(B * Hkv * N * D, seed, 3).reshape(B, Hkv, N, D)
    return to_dev(q), to_dev(k), to_dev(v), (q, k, v)


def test_amax_and_scaled_quantize(ora, syn):
    import torch
    for n, (G, N, D) in enumerate([(3, 300, 128), (2, 77, 64), (1, 1, 128)]):
        x = syn.normal_bf16(G * N * D, 40 + n, 0, scale=10.0 ** (n - 1)).reshape(G, N, D)
        dx = to_dev(x)
        a = fa.fp4_amax(dx)
        assert float(a.item()) == ora.amax_bf16(x)
        for axis in (fa.FP4_BLOCK_ALONG_D, fa.FP4_BLOCK_ALONG_N_T):
            whole = fa.fp4_quantize(dx, axis)
            split = fa.fp4_quantize(dx, axis, amax=a)
            torch.cuda.synchronize()
            assert torch.equal(whole.codes, split.codes)
            assert torch.equal(whole.scales, split.scales)
    fa.fp4_status()


@pytest.mark.parametrize("case", CASES)
def test_one_rank_equals_unsharded(syn, case):
    import torch
    B, H, Hkv, N, D, causal = case
    q, k, v, _ = _inputs(syn, B, H, Hkv, N, D, 500)
    ref = fa.fp4_attn_fwd(q, k, v, causal=causal)
    got = fa.fp4_attn_fwd_sharded(q.view(B * H, N, D), k.view(B * Hkv, N, D),
                                  v.view(B * Hkv, N, D), causal=causal)
    torch.cuda.synchronize()
    fa.fp4_status()
    assert torch.equal(ref.view(-1), got.view(-1))


def _slab(t, G, i0, i1):
    per = t.numel() // G
    return t[i0 * per:i1 * per]


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("case", CASES)
def test_emulated_shards_equal_unsharded(syn, case, world):
    import torch
    B, H, Hkv, N, D, causal = case
    q, k, v, _ = _inputs(syn, B, H, Hkv, N, D, 600 + world)
    ref = fa.fp4_attn_fwd(q, k, v, causal=causal)
    whole = [fa.fp4_quantize(q, fa.FP4_BLOCK_ALONG_D), fa.fp4_quantize(k, fa.FP4_BLOCK_ALONG_D),
             fa.fp4_quantize(v, fa.FP4_BLOCK_ALONG_N_T)]
    qf, kf, vf = q.view(B * H, N, D), k.view(B * Hkv, N, D), v.view(B * Hkv, N, D)
    shards = [fa.shard_rows(B, H, Hkv, world, r) for r in range(world)]
    amax = torch.zeros(3, dtype=torch.float32, device="cuda")
    for sq, skv in shards:  # each rank's maxima, combined as the all-reduce (MAX) does
        if skv.stop > skv.start:
            part = torch.stack([fa.fp4_amax(qf[sq]), fa.fp4_amax(kf[skv]),
                                fa.fp4_amax(vf[skv])]).view(3)
            amax = torch.maximum(amax, part)
    for t, w in zip(amax, whole):
        assert float(t) == float(w.amax[0])
    out = torch.empty_like(qf)
    for sq, skv in shards:
        if skv.stop == skv.start:
            continue
        qs = fa.fp4_quantize(qf[sq], fa.FP4_BLOCK_ALONG_D, amax=amax[0:1])
        ks = fa.fp4_quantize(kf[skv], fa.FP4_BLOCK_ALONG_D, amax=amax[1:2])
        vs = fa.fp4_quantize(vf[skv], fa.FP4_BLOCK_ALONG_N_T, amax=amax[2:3])
        for part, w, (i0, i1), G in ((qs, whole[0], (sq.start, sq.stop), B * H),
                                     (ks, whole[1], (skv.start, skv.stop), B * Hkv),
                                     (vs, whole[2], (skv.start, skv.stop), B * Hkv)):
            assert torch.equal(part.codes, _slab(w.codes, G, i0, i1))
            assert torch.equal(part.scales, _slab(w.scales, G, i0, i1))
        fa.fp4_attn_fwd_quantized(qs, ks, vs, 1, sq.stop - sq.start, skv.stop - skv.start,
                                  causal=causal, out=out[sq])
    torch.cuda.synchronize()
    fa.fp4_status()
    assert np.array_equal(from_dev(out).reshape(-1), from_dev(ref).reshape(-1))


@pytest.mark.parametrize("case", CASES)
def test_one_rank_smooth_equals_unsharded(syn, case):
    import torch
    B, H, Hkv, N, D, causal = case
    q, k, v, _ = _inputs(syn, B, H, Hkv, N, D, 700)
    for smooth in (fa.FP4_SMOOTH_K, fa.FP4_SMOOTH_Q, fa.FP4_SMOOTH_K | fa.FP4_SMOOTH_Q):
        ref = fa.fp4_attn_fwd_smooth(q, k, v, smooth=smooth, causal=causal)
        got = fa.fp4_attn_fwd_sharded(q.view(B * H, N, D), k.view(B * Hkv, N, D),
                                      v.view(B * Hkv, N, D), causal=causal, smooth=smooth)
        torch.cuda.synchronize()
        fa.fp4_status()
        assert torch.equal(ref.view(-1), got.view(-1))


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("case", CASES)
def test_emulated_smoothed_shards_equal_unsharded(syn, case, world):
    """Smoothing sharded by head: each shard's means come from the global raw
    maxima; the smoothed maxima are combined by max (the second all-reduce);
    each shard's output equals its slab of the unsharded smoothed run."""
    import torch
    B, H, Hkv, N, D, causal = case
    q, k, v, _ = _inputs(syn, B, H, Hkv, N, D, 800 + world)
    ref = fa.fp4_attn_fwd_smooth(q, k, v, causal=causal)
    qf, kf, vf = q.view(B * H, N, D), k.view(B * Hkv, N, D), v.view(B * Hkv, N, D)
    shards = [fa.shard_rows(B, H, Hkv, world, r) for r in range(world)
              if fa.shard_rows(B, H, Hkv, world, r)[1].stop > fa.shard_rows(B, H, Hkv, world, r)[1].start]
    amax = torch.zeros(3, dtype=torch.float32, device="cuda")
    for sq, skv in shards:
        part = torch.stack([fa.fp4_amax(qf[sq]), fa.fp4_amax(kf[skv]), fa.fp4_amax(vf[skv])]).view(3)
        amax = torch.maximum(amax, part)
    means = [(fa.fp4_channel_mean(qf[sq], amax[0:1]), fa.fp4_channel_mean(kf[skv], amax[1:2]))
             for sq, skv in shards]
    sm = torch.zeros(2, dtype=torch.float32, device="cuda")
    for (sq, skv), (qm, km) in zip(shards, means):
        part = torch.stack([fa.fp4_amax_smoothed(qf[sq], qm), fa.fp4_amax_smoothed(kf[skv], km)])
        sm = torch.maximum(sm, part.view(2))
    out = torch.empty_like(qf)
    for (sq, skv), (qm, km) in zip(shards, means):
        gq, gk = sq.stop - sq.start, skv.stop - skv.start
        qs = fa.fp4_quantize_smoothed(qf[sq], qm, sm[0:1])
        ks = fa.fp4_quantize_smoothed(kf[skv], km, sm[1:2])
        vs = fa.fp4_quantize(vf[skv], fa.FP4_BLOCK_ALONG_N_T, amax=amax[2:3])
        bias = fa.fp4_score_bias(qm, kf[skv].view(1, gk, N, D), km, gq, sm[0:1], sm[1:2])
        fa.fp4_attn_fwd_quantized_bias(qs, ks, vs, bias, 1, gq, gk, causal=causal, out=out[sq])
    torch.cuda.synchronize()
    fa.fp4_status()
    assert np.array_equal(from_dev(out).reshape(-1), from_dev(ref).reshape(-1))


@pytest.mark.parametrize("case", CASES)
def test_training_pass_one_rank_equals_unsharded(syn, case):
    """fp4_attn_fwd_sharded with lse and fp4_attn_bwd_sharded on one rank:
    the same outputs, lse and gradients as fp4_attn_fwd_lse / fp4_attn_bwd."""
    import torch
    B, H, Hkv, N, D, causal = case
    q, k, v, _ = _inputs(syn, B, H, Hkv, N, D, 900)
    do = to_dev(syn.normal_bf16(B * H * N * D, 901, 4).reshape(B, H, N, D))
    out, lse = fa.fp4_attn_fwd_lse(q, k, v, causal=causal)
    grads = fa.fp4_attn_bwd(q, k, v, out, do, lse, causal=causal)
    lse_s = torch.empty(B * H * N, dtype=torch.float32, device="cuda")
    out_s = fa.fp4_attn_fwd_sharded(q.view(B * H, N, D), k.view(B * Hkv, N, D),
                                    v.view(B * Hkv, N, D), causal=causal, lse=lse_s)
    grads_s = fa.fp4_attn_bwd_sharded(q.view(B * H, N, D), k.view(B * Hkv, N, D),
                                      v.view(B * Hkv, N, D), out_s.view(B * H, N, D),
                                      do.view(B * H, N, D), lse_s, causal=causal)
    torch.cuda.synchronize()
    fa.fp4_status()
    assert torch.equal(out.view(-1), out_s.view(-1))
    assert torch.equal(lse.view(-1), lse_s)
    for a, b in zip(grads, grads_s):
        assert torch.equal(a.view(-1), b.view(-1))


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("case", CASES)
def test_emulated_training_shards_equal_unsharded(syn, case, world):
    """The training pass sharded by head, emulated on one GPU: every shard's
    output, lse and gradients equal its slab of the unsharded pass, bit for
    bit (the maxima combined by max, as the all-reduce does)."""
    import torch
    B, H, Hkv, N, D, causal = case
    q, k, v, _ = _inputs(syn, B, H, Hkv, N, D, 910 + world)
    do = to_dev(syn.normal_bf16(B * H * N * D, 911, 4).reshape(B, H, N, D))
    out, lse = fa.fp4_attn_fwd_lse(q, k, v, causal=causal)
    gq_, gk_, gv_ = fa.fp4_attn_bwd(q, k, v, out, do, lse, causal=causal)
    qf, kf, vf, dof = (t.view(-1, N, D) for t in (q, k, v, do))
    shards = [fa.shard_rows(B, H, Hkv, world, r) for r in range(world)]
    shards = [(sq, skv) for sq, skv in shards if skv.stop > skv.start]
    amax = torch.zeros(3, dtype=torch.float32, device="cuda")
    for sq, skv in shards:
        part = torch.stack([fa.fp4_amax(qf[sq]), fa.fp4_amax(kf[skv]), fa.fp4_amax(vf[skv])]).view(3)
        amax = torch.maximum(amax, part)
    for sq, skv in shards:
        g1, g2 = sq.stop - sq.start, skv.stop - skv.start
        qs = fa.fp4_quantize(qf[sq], fa.FP4_BLOCK_ALONG_D, amax=amax[0:1])
        ks = fa.fp4_quantize(kf[skv], fa.FP4_BLOCK_ALONG_D, amax=amax[1:2])
        vs = fa.fp4_quantize(vf[skv], fa.FP4_BLOCK_ALONG_N_T, amax=amax[2:3])
        lse_s = torch.empty(g1 * N, dtype=torch.float32, device="cuda")
        out_s = fa.fp4_attn_fwd_quantized(qs, ks, vs, 1, g1, g2, causal=causal, lse=lse_s)
        as4 = lambda t: t.contiguous().view(1, -1, N, D)
        d = fa.fp4_attn_bwd(as4(qf[sq]), as4(kf[skv]), as4(vf[skv]), as4(out_s),
                            as4(dof[sq]), lse_s.view(1, g1, N), causal=causal, amax=amax)
        torch.cuda.synchronize()
        fa.fp4_status()
        assert torch.equal(out_s.view(-1), out.view(-1, N, D)[sq].reshape(-1))
        assert torch.equal(lse_s, lse.view(-1, N)[sq].reshape(-1))
        assert torch.equal(d[0].view(-1), gq_.view(-1, N, D)[sq].reshape(-1))
        assert torch.equal(d[1].view(-1), gk_.view(-1, N, D)[skv].reshape(-1))
        assert torch.equal(d[2].view(-1), gv_.view(-1, N, D)[skv].reshape(-1))
