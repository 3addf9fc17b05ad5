"""The FP4_DEBUG build (libfp4attn_debug.so, the bounds checker that stands in
for compute-sanitizer): every guarded global access of the kernels (bulk
copies, TMA coordinates and the 16-byte rule for their x, epilogue stores,
quantizer writes) is checked against the extent of its buffer, and a failed
check is reported by fp4_status as FP4_ERR_BOUNDS instead of trapping.

On shapes with ragged tails, causal masks, GQA and D = 64, the forward (every
P generation and the smoothed path), the quantizers and the backward run in
the debug build with no failed check and give the release build's outputs
bit for bit. The reporting path is exercised by a check that fails by
construction and addresses no memory."""
import os

import pytest

import bit_attention_transformers_b200 as fa
from gpu_util import to_dev

pytestmark = pytest.mark.gpu

CASES = [  # B, H, Hkv, N, D, causal
    (1, 2, 1, 300, 128, False),
    (2, 4, 2, 130, 64, True),
    (1, 3, 1, 513, 128, True),
    (1, 1, 1, 1, 64, False),
]


@pytest.fixture(scope="module")
def libs():
    if not os.path.exists(fa._DEBUG_LIB_PATH):
        pytest.fail(f"{fa._DEBUG_LIB_PATH} is missing: run bit_attention_transformers_b200.build()")
    yield
    fa.load(debug=False)


def _run_all(q, k, v, do, causal):
    import torch
    res = {}
    res["fwd"] = fa.fp4_attn_fwd(q, k, v, causal=causal)
    res["efq"] = fa.fp4_attn_fwd(q, k, v, causal=causal, efq=True)
    res["fp8pv"] = fa.fp4_attn_fwd(q, k, v, causal=causal, fp8pv=True)
    res["smooth"] = fa.fp4_attn_fwd_smooth(q, k, v, causal=causal)
    qq = fa.fp4_quantize(q)
    vq = fa.fp4_quantize(v, fa.FP4_BLOCK_ALONG_N_T)
    res["q_codes"], res["q_scales"] = qq.codes, qq.scales
    res["v_codes"], res["v_scales"] = vq.codes, vq.scales
    out, lse = fa.fp4_attn_fwd_lse(q, k, v, causal=causal)
    res["out"], res["lse"] = out, lse
    res["dq"], res["dk"], res["dv"] = fa.fp4_attn_bwd(q, k, v, out, do, lse, causal=causal)
    torch.cuda.synchronize()
    fa.fp4_status()  # raises FP4_ERR_BOUNDS if any check failed
    return {name: t.clone() for name, t in res.items()}


@pytest.mark.parametrize("case", CASES)
def test_debug_build_checks_pass_and_match_release(syn, libs, case):
    import torch
    B, H, Hkv, N, D, causal = case
    seed = 700 + N + D
    q = to_dev(syn.normal_bf16(B * H * N * D, seed=seed, stream=1, scale=1.5).reshape(B, H, N, D))
    k = to_dev(syn.normal_bf16(B * Hkv * N * D, seed=seed, stream=2, scale=1.5)
               .reshape(B, Hkv, N, D))
    v = to_dev(syn.normal_bf16(B * Hkv * N * D, seed=seed, stream=3).reshape(B, Hkv, N, D))
    do = to_dev(syn.normal_bf16(B * H * N * D, seed=seed, stream=4).reshape(B, H, N, D))
    fa.load(debug=False)
    assert not fa.fp4_debug_build()
    want = _run_all(q, k, v, do, causal)
    fa.load(debug=True)
    assert fa.fp4_debug_build()
    got = _run_all(q, k, v, do, causal)
    for name in want:
        assert torch.equal(got[name], want[name]), name


def test_failed_check_is_reported_not_trapped(libs):
    import torch
    fa.load(debug=False)
    with pytest.raises(fa.Fp4Error) as e:
        fa.fp4_debug_selftest(7)
    assert e.value.code == fa.FP4_ERR_UNSUPPORTED
    fa.load(debug=True)
    fa.fp4_status()  # nothing pending
    fa.fp4_debug_selftest(42)
    with pytest.raises(fa.Fp4Error) as e:
        fa.fp4_status()
    assert e.value.code == fa.FP4_ERR_BOUNDS and "site 42" in str(e.value)
    fa.fp4_status()  # the report was cleared; the context still works
    x = torch.ones(4, dtype=torch.float32, device="cuda")
    assert float((x * 2).sum()) == 8.0
