"""EFQ-Softmax parity: the CUDA forward with EFQ P generation (fp4_attn_fwd_efq,
through the C ABI) against the oracle with flag 8.

Same bar and allowances as the exp-then-quantize path (tests/test_gpu_attention.py):
|O_gpu - O_oracle| <= 2e-3 * max|V| per element plus half a bf16 step of the
output plus the oracle's EFQ flip bound (codes whose affine argument, or blocks
whose max shifted score, lie within the fp32 arithmetic's uncertainty of a
rounding point; pinned in tests/test_oracle_efq.py), and per-head cosine
>= 0.9999. Every row of the small cases and the hand-worked golden cases; the
workloads on every row (tiny, heavy-tailed) or on seeded sampled rows.
"""
import numpy as np
import pytest

from _util import bf16_bits_to_f32, bits_to_float, golden_tensors, load_golden
from gpu_util import run_attn
from test_gpu_attention import SMALL, _rows_per_head, compare

pytestmark = pytest.mark.gpu


def run_full(ora, q, k, v, causal, label, softmax_scale=0.0):
    B, H, N, D = q.shape
    got = run_attn(q, k, v, causal, softmax_scale, efq=True)
    want = ora.attn_fwd(q, k, v, causal=causal, softmax_scale=softmax_scale, want_f64=True,
                        want_flip=True, want_ml=True, flags=ora.FLAG_EFQ)
    heads = np.repeat(np.arange(B * H), N)
    vmax = float(np.abs(bf16_bits_to_f32(v)).max())
    compare(got.reshape(-1, D), {k2: a.reshape(-1, a.shape[-1]) for k2, a in want.items()}, heads, vmax,
            "EFQ " + label)


@pytest.mark.parametrize("B,H,Hkv,N,D,causal", SMALL)
def test_efq_small(ora, syn, B, H, Hkv, N, D, causal):
    s = 5000 + N * 7 + D + 3 * H + int(causal)
    q = syn.normal_bf16(B * H * N * D, seed=s, stream=1, scale=1.5).reshape(B, H, N, D)
    k = syn.normal_bf16(B * Hkv * N * D, seed=s, stream=2, scale=1.5).reshape(B, Hkv, N, D)
    v = syn.normal_bf16(B * Hkv * N * D, seed=s, stream=3).reshape(B, Hkv, N, D)
    run_full(ora, q, k, v, causal, f"B{B} H{H} Hkv{Hkv} N{N} D{D} causal={causal}")


@pytest.mark.parametrize("name", ["attn_4x4.json", "attn_2x2_gqa.json"])
@pytest.mark.parametrize("causal", [False, True])
def test_efq_golden(ora, name, causal):
    """The hand-worked cases (their EFQ rows in tests/golden/), zero-padded to D = 64."""
    g = load_golden(name)
    q, k, v = (np.concatenate([t, np.zeros_like(t)], axis=-1) for t in golden_tensors(g))
    run_full(ora, q, k, v, causal, f"{name} causal={causal}",
             softmax_scale=bits_to_float(g["softmax_scale_bits"]))


def test_efq_uniform_and_peaked(ora, syn):
    B, H, N, D = 1, 2, 400, 128
    v = syn.normal_bf16(B * H * N * D, seed=177).reshape(B, H, N, D)
    k = syn.normal_bf16(B * H * N * D, seed=178, scale=4.0).reshape(B, H, N, D)
    run_full(ora, np.zeros_like(v), k, v, False, "Q=0")
    q = syn.normal_bf16(B * H * N * D, seed=179, scale=4.0).reshape(B, H, N, D)
    run_full(ora, q, k, v, True, "peaked causal")


@pytest.mark.parametrize("name", ["tiny", "heavy_tailed", "llm_prefill", "video_dit",
                                  "long_context"])
def test_efq_workloads(ora, syn, name):
    wl = syn.WORKLOADS[name]
    q, k, v = syn.workload_inputs(wl)
    got = run_attn(q, k, v, wl.causal, efq=True)
    vmax = float(np.abs(bf16_bits_to_f32(v)).max())
    per_head = _rows_per_head(wl)
    if per_head == 0:
        want = ora.attn_fwd(q, k, v, causal=wl.causal, want_f64=True, want_flip=True, want_ml=True,
                            flags=ora.FLAG_EFQ)
        heads = np.repeat(np.arange(wl.B * wl.H), wl.N)
        compare(got.reshape(-1, wl.D), {k2: a.reshape(-1, a.shape[-1]) for k2, a in want.items()},
                heads, vmax, "EFQ " + name)
        return
    rows = syn.sample_rows(wl, per_head)
    want = ora.attn_fwd(q, k, v, causal=wl.causal, rows=rows, want_f64=True, want_flip=True, want_ml=True,
                        flags=ora.FLAG_EFQ)
    got_rows = got[rows[:, 0], rows[:, 1], rows[:, 2]]
    compare(got_rows, want, rows[:, 0] * wl.H + rows[:, 1], vmax,
            f"EFQ {name} ({per_head} rows/head)")
