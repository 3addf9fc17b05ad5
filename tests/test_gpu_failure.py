"""Failure detection on the GPU without a fault: a bounded wait that nothing
ends (the attention kernel's own wait routine, with a 20 ms limit) expires,
sets the device error word and returns; fp4_status reports FP4_ERR_TIMEOUT once
and clears it, and the context keeps working (an attention call afterwards
matches one made before)."""
import time

import numpy as np
import pytest

import bit_attention_transformers_b200 as fa
from gpu_util import to_dev

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_context_survives(syn):
    import torch
    B, H, N, D = 1, 2, 300, 128
    q, k, v = (to_dev(syn.normal_bf16(B * H * N * D, 90, s).reshape(B, H, N, D)) for s in (1, 2, 3))
    before = fa.fp4_attn_fwd(q, k, v).clone()
    fa.fp4_status()  # nothing pending
    t0 = time.perf_counter()
    ok = fa.fp4_test_wait_timeout(20_000_000)
    with pytest.raises(fa.Fp4Error) as err:
        fa.fp4_status()
    elapsed = time.perf_counter() - t0
    assert err.value.code == fa.FP4_ERR_TIMEOUT
    assert int(ok.item()) == 0
    assert 0.015 < elapsed < 2.0  # the 20 ms limit, not a hang
    fa.fp4_status()  # the report was cleared
    after = fa.fp4_attn_fwd(q, k, v)
    torch.cuda.synchronize()
    fa.fp4_status()
    assert torch.equal(before, after)
