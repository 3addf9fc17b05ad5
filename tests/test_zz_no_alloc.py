"""fp4_attn_fwd_noalloc: the attention forward for callers that cannot
allocate device memory (their device memory belongs to a host framework that
gives them no allocator, or they must avoid cudaMalloc's implicit device
synchronisation). It uses the library's built-in scratch array instead of a
workspace. Checked through the C ABI against fp4_attn_fwd on two calls in a
row, with different shapes, so the second call runs on the first call's
leftover scratch contents. Collected last on purpose."""
import ctypes

import numpy as np
import pytest

import bit_attention_transformers_b200 as fa
from _util import bf16_bits_to_f32
from gpu_util import from_dev, to_dev

ATOL_REL = 2e-3
COS_MIN = 0.9999


def _case(syn, B, H, Hkv, N, D, seed):
    q = syn.normal_bf16(B * H * N * D, seed=seed, stream=1).reshape(B, H, N, D)
    k = syn.normal_bf16(B * Hkv * N * D, seed=seed, stream=2).reshape(B, Hkv, N, D)
    v = syn.normal_bf16(B * Hkv * N * D, seed=seed, stream=3).reshape(B, Hkv, N, D)
    return q, k, v


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point(syn):
    import torch
    fa.build()
    L = fa.lib()
    vp = ctypes.c_void_p
    for (B, H, Hkv, N, D, causal, seed) in ((1, 4, 2, 1000, 128, False, 901),
                                            (2, 2, 2, 333, 64, True, 902)):
        q, k, v = _case(syn, B, H, Hkv, N, D, seed)
        dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
        ref = fa.fp4_attn_fwd(dq, dk, dv, causal=causal)
        out = torch.empty_like(dq)
        stream = torch.cuda.current_stream().cuda_stream
        rc = L.fp4_attn_fwd_noalloc(vp(dq.data_ptr()), vp(dk.data_ptr()), vp(dv.data_ptr()),
                                    vp(out.data_ptr()), B, H, Hkv, N, D, int(causal), 0.0,
                                    vp(stream))
        assert rc == fa.FP4_OK, L.fp4_last_error()
        fa.fp4_status()
        g = bf16_bits_to_f32(from_dev(out)).astype(np.float64)
        r = bf16_bits_to_f32(from_dev(ref)).astype(np.float64)
        vmax = float(np.abs(bf16_bits_to_f32(v)).max())
        assert np.abs(g - r).max() <= ATOL_REL * vmax
        for h in range(B * H):
            a, b = g.reshape(B * H, -1)[h], r.reshape(B * H, -1)[h]
            assert a @ b / (np.linalg.norm(a) * np.linalg.norm(b)) >= COS_MIN


@pytest.mark.gpu
def test_noalloc_rejects_problems_beyond_its_scratch():
    fa.build()
    L = fa.lib()
    vp = ctypes.c_void_p
    # 32 heads x 65536 tokens x 128 channels needs ~ 455 MB of scratch
    rc = L.fp4_attn_fwd_noalloc(vp(16), vp(16), vp(16), vp(16), 1, 32, 32, 65536, 128, 0, 0.0,
                                vp(0))
    assert rc == fa.FP4_ERR_WORKSPACE
    assert b"scratch" in L.fp4_last_error()
