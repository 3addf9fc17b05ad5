"""The end-to-end host APIs: fp4_attn_fwd_host (one batch) and
fp4_attn_fwd_host_many (a stream of batches with copies overlapped with
compute) give, for every batch, the same output as fp4_attn_fwd on device
copies of its inputs, bit for bit."""
import pytest

import bit_attention_transformers_b200 as fa
from gpu_util import to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("efq", [False, True])
def test_host_apis_match_the_device_call(syn, efq):
    import torch
    B, H, Hkv, N, D = 1, 4, 2, 700, 128
    batches, want = [], []
    for i in range(5):
        t = [syn.normal_bf16(B * h * N * D, 300 + i, s).reshape(B, h, N, D)
             for s, h in ((1, H), (2, Hkv), (3, Hkv))]
        dev = [to_dev(x) for x in t]
        want.append(fa.fp4_attn_fwd(*dev, causal=bool(i % 2), efq=efq).cpu())
        batches.append(tuple(x.cpu().pin_memory() for x in dev))
    one = fa.fp4_attn_fwd_host(*batches[1], causal=True, efq=efq)
    assert torch.equal(one, want[1])
    outs = [torch.empty_like(w).pin_memory() for w in want]
    # causal alternates per batch in `want`; run the stream twice, once per mode
    for causal in (False, True):
        idx = [i for i in range(5) if bool(i % 2) == causal]
        got, ms = fa.fp4_attn_fwd_host_many([batches[i] for i in idx], [outs[i] for i in idx],
                                            causal=causal, efq=efq, return_ms=True)
        assert ms > 0
        for i in idx:
            assert torch.equal(outs[i], want[i]), (i, causal)
    fa.fp4_status()
