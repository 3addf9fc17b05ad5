"""fp4_attn_fwd_noalloc: the attention forward for callers that cannot
allocate device memory (their device memory belongs to a host framework that
gives them no allocator, or they must avoid cudaMalloc's implicit device
synchronisation). It uses the library's built-in scratch array instead of a
workspace. Checked through the C ABI against fp4_attn_fwd on two calls in a
row, with different shapes, so the second call runs on the first call's
leftover scratch contents. Both run the same deterministic kernels on the same
inputs, so the outputs must be identical bit for bit: any difference would be
leftover scratch (stale padding, a stale maximum) leaking into the result.
Collected last on purpose."""
import ctypes

import pytest

import bit_attention_transformers_b200 as fa
from gpu_util import to_dev


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
        assert torch.equal(out, ref), (B, H, Hkv, N, D, causal)


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
