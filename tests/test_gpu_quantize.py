"""Quantiser parity: the CUDA quantiser's E2M1 codes, E4M3 block scales and
tensor maximum are bit-exact against the oracle, on edge cases and on the
full tensors of all five workloads."""
import numpy as np
import pytest

import bit_attention_transformers_b200 as fa
from _util import f32_to_bf16_bits
from gpu_util import scales_rows_logical, scales_tokens_logical, to_dev


def _gpu_quant(x_u16, axis):
    import torch
    G, N, D = x_u16.shape
    t = fa.fp4_quantize(to_dev(x_u16), axis)
    canon = fa.fp4_scales_to_canonical(t)  # the C ABI's logical view of the scales
    torch.cuda.synchronize()
    fa.fp4_status()
    return t.codes.cpu().numpy(), t.scales.cpu().numpy(), float(t.amax[0].item()), \
        canon.cpu().numpy()


def check_rows(ora, x):
    """x: uint16 [G, N, D]; blocks along D."""
    G, N, D = x.shape
    Npad = (N + 127) // 128 * 128
    codes, scales, amax, canon = _gpu_quant(x, fa.FP4_BLOCK_ALONG_D)
    a = ora.amax_bf16(x)
    assert amax == a
    s_enc, _ = ora.tensor_scale(a)
    oc, os_ = ora.quantize_rows(x.reshape(G * N, D), s_enc)
    codes = codes.reshape(G, Npad, D // 2)
    np.testing.assert_array_equal(codes[:, :N], oc.reshape(G, N, D // 2))
    assert not codes[:, N:].any()
    np.testing.assert_array_equal(scales_rows_logical(scales, G, N, D), os_.reshape(G, N, D // 16))
    np.testing.assert_array_equal(canon, os_.reshape(G, N, D // 16))


def check_tokens(ora, x):
    """x: uint16 [G, N, D]; blocks along tokens, transposed."""
    G, N, D = x.shape
    Npad = (N + 127) // 128 * 128
    n16 = (N + 15) // 16 * 16
    codes, scales, amax, canon = _gpu_quant(x, fa.FP4_BLOCK_ALONG_N_T)
    a = ora.amax_bf16(x)
    assert amax == a
    s_enc, _ = ora.tensor_scale(a)
    codes = codes.reshape(G, D, Npad // 2)
    sc, pad = scales_tokens_logical(scales, G, N, D)
    assert not pad.any()
    for g in range(G):
        oc, os_ = ora.quantize_tokens_T(x[g], s_enc)
        np.testing.assert_array_equal(codes[g, :, :n16 // 2], oc)
        assert not codes[g, :, n16 // 2:].any()
        np.testing.assert_array_equal(sc[g, :, :n16 // 16], os_)
        assert not sc[g, :, n16 // 16:].any()
        np.testing.assert_array_equal(canon[g], sc[g])


CASES = [(1, 1, 64), (2, 37, 128), (3, 300, 64), (1, 128, 128), (2, 1000, 128), (5, 257, 64)]


@pytest.mark.gpu
@pytest.mark.parametrize("G,N,D", CASES)
def test_quantize_random_shapes(ora, syn, G, N, D):
    x = syn.normal_bf16(G * N * D, seed=100 + N, scale=1.5).reshape(G, N, D)
    check_rows(ora, x)
    check_tokens(ora, x)


@pytest.mark.gpu
def test_quantize_edge_values(ora, syn):
    G, N, D = 2, 70, 128
    rng = np.random.default_rng(7)
    # zeros, negative zeros, a huge outlier (tiny and subnormal block scales),
    # exact E2M1 multiples, saturation boundaries
    x = rng.standard_normal((G, N, D)).astype(np.float32)
    x[0, :5] = 0.0
    x[0, 5:9] = -0.0
    x[1, 3, 7] = 3.0e4
    x[1, 10:20] *= 1e-3
    x[1, 20:22] = np.array([6, 3, 1.5, 0.5, -6, -4, 2, 1] * 32, np.float32).reshape(2, D)
    xb = f32_to_bf16_bits(x)
    check_rows(ora, xb)
    check_tokens(ora, xb)
    zero = np.zeros((1, 33, 64), np.uint16)
    check_rows(ora, zero)
    check_tokens(ora, zero)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny", "heavy_tailed", "llm_prefill", "video_dit",
                                  "long_context"])
def test_quantize_workloads_bit_exact(ora, syn, name):
    wl = syn.WORKLOADS[name]
    q, k, v = syn.workload_inputs(wl)
    check_rows(ora, q.reshape(wl.B * wl.H, wl.N, wl.D))
    check_rows(ora, k.reshape(wl.B * wl.Hkv, wl.N, wl.D))
    check_tokens(ora, v.reshape(wl.B * wl.Hkv, wl.N, wl.D))
