"""The C-ABI library: builds for sm_100a, loads, exports every symbol the header
declares, and rejects bad arguments on the host before launching anything.
No test here needs a GPU or launches a kernel."""
import ctypes
import os
import re

import pytest

import bit_attention_transformers_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    fa.build()
    return fa.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "fp4attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b(fp4_\w+)\s*\(", src))


def test_header_and_binding_agree():
    assert _declared() == set(fa.EXPORTS)


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_debug_build_exports_every_symbol(L):
    """The FP4_DEBUG build has the release build's entry points and says which
    it is (host-only calls: no GPU needed)."""
    import ctypes
    D = ctypes.CDLL(fa._DEBUG_LIB_PATH)
    for name in _declared():
        assert hasattr(D, name), name
    D.fp4_debug_build.restype = ctypes.c_int
    L.fp4_debug_build.restype = ctypes.c_int
    assert D.fp4_debug_build() == 1 and L.fp4_debug_build() == 0
    # an out-of-range site is rejected before anything is launched
    D.fp4_debug_selftest.argtypes = [ctypes.c_uint, ctypes.c_void_p]
    assert D.fp4_debug_selftest(0, None) == fa.FP4_ERR_INVALID_ARG


def test_sizes(L):
    # Npad = 384 for N = 300; codes 4 bits per element, scales 1 byte per 16
    assert fa.fp4_codes_bytes(3, 300, 128, fa.FP4_BLOCK_ALONG_D) == 3 * 384 * 64
    assert fa.fp4_scales_bytes(3, 300, 128, fa.FP4_BLOCK_ALONG_D) == 3 * 384 * 8
    assert fa.fp4_scales_bytes(3, 300, 64, fa.FP4_BLOCK_ALONG_N_T) == 3 * 6 * 512
    ws = fa.fp4_attn_workspace_bytes(2, 8, 2, 1000, 128)
    assert ws >= 2 * 8 * 1024 * 64 + 2 * 2 * 1024 * 64 * 2
    assert fa.fp4_attn_workspace_bytes(1, 3, 2, 10, 128) == 0  # H % Hkv != 0
    assert fa.fp4_attn_workspace_bytes(1, 1, 1, 10, 96) == 0   # unsupported D
    # FP8 V: one byte per element, channel-major over Npad tokens, no scales
    assert fa.fp4_fp8_codes_bytes(3, 300, 64) == 3 * 64 * 384
    assert fa.fp4_fp8_codes_bytes(0, 300, 64) == 0
    ws8 = fa.fp4_attn_workspace_bytes_fp8pv(2, 8, 2, 1000, 128)
    assert ws8 >= 2 * 8 * 1024 * 64 + 2 * 1024 * 64 * 2 + 2 * 2 * 128 * 1024
    assert ws8 > ws  # V codes twice as large, V block scales dropped
    assert fa.fp4_attn_workspace_bytes_fp8pv(1, 3, 2, 10, 128) == 0


def _call_fwd(L, q=16, k=16, v=16, out=16, B=1, H=1, Hkv=1, N=8, D=128, ws=1 << 20,
              wsz=1 << 30):
    vp = ctypes.c_void_p
    return L.fp4_attn_fwd(vp(q), vp(k), vp(v), vp(out), B, H, Hkv, N, D, 0, 0.0, vp(0), vp(ws),
                          wsz)


def test_argument_errors_launch_nothing(L):
    # fake, never dereferenced addresses: validation fails before any CUDA call
    assert _call_fwd(L, D=96) == fa.FP4_ERR_UNSUPPORTED
    assert _call_fwd(L, H=3, Hkv=2) == fa.FP4_ERR_INVALID_ARG
    assert _call_fwd(L, N=0) == fa.FP4_ERR_INVALID_ARG
    assert _call_fwd(L, q=0) == fa.FP4_ERR_INVALID_ARG
    assert _call_fwd(L, k=24) == fa.FP4_ERR_INVALID_ARG  # misaligned
    assert _call_fwd(L, wsz=100) == fa.FP4_ERR_WORKSPACE
    assert b"workspace" in L.fp4_last_error()
    vp = ctypes.c_void_p
    assert L.fp4_quantize(vp(16), 1, 8, 128, 7, vp(16), vp(16), vp(16), vp(0)) == \
        fa.FP4_ERR_INVALID_ARG
    assert L.fp4_quantize(vp(16), 1, 8, 128, 0, vp(0), vp(16), vp(16), vp(0)) == \
        fa.FP4_ERR_INVALID_ARG
    assert L.fp4_amax(vp(16), 1, 8, 96, vp(16), vp(0)) == fa.FP4_ERR_UNSUPPORTED
    assert L.fp4_amax(vp(16), 1, 8, 128, vp(0), vp(0)) == fa.FP4_ERR_INVALID_ARG
    assert L.fp4_amax(vp(24), 1, 8, 128, vp(16), vp(0)) == fa.FP4_ERR_INVALID_ARG  # misaligned x
    assert L.fp4_amax(vp(16), 1, 8, 128, vp(18), vp(0)) == fa.FP4_ERR_INVALID_ARG  # misaligned amax
    assert L.fp4_quantize_scaled(vp(16), 1, 8, 128, 2, vp(16), vp(16), vp(16), vp(0)) == \
        fa.FP4_ERR_INVALID_ARG
    assert L.fp4_quantize_scaled(vp(16), 1, 8, 128, 1, vp(0), vp(16), vp(16), vp(0)) == \
        fa.FP4_ERR_INVALID_ARG
    assert L.fp4_quantize_scaled(vp(16), 0, 8, 128, 1, vp(4), vp(16), vp(16), vp(0)) == \
        fa.FP4_ERR_INVALID_ARG
    assert L.fp4_probe_cvt(0xFFFFFFF0, 64, 0, vp(16), vp(0)) == fa.FP4_ERR_INVALID_ARG
    assert L.fp4_scales_to_canonical(vp(16), 1, 8, 128, 5, vp(16), vp(0)) == fa.FP4_ERR_INVALID_ARG
    assert L.fp4_scales_to_canonical(vp(0), 1, 8, 128, 0, vp(16), vp(0)) == fa.FP4_ERR_INVALID_ARG
    assert L.fp4_scales_to_canonical(vp(16), 1, 8, 96, 0, vp(16), vp(0)) == fa.FP4_ERR_UNSUPPORTED
    assert L.fp4_test_wait_timeout(0, vp(16), vp(0)) == fa.FP4_ERR_INVALID_ARG
    assert L.fp4_test_wait_timeout(6_000_000_000, vp(16), vp(0)) == fa.FP4_ERR_INVALID_ARG
    assert L.fp4_test_wait_timeout(1000, vp(0), vp(0)) == fa.FP4_ERR_INVALID_ARG
    assert L.fp4_probe_cvt(0, 16, 3, vp(16), vp(0)) == fa.FP4_ERR_INVALID_ARG
    # the FP8 P/V entries: same checks, before any launch
    assert L.fp4_attn_fwd_fp8pv(vp(16), vp(16), vp(16), vp(16), 1, 1, 1, 8, 96, 0, 0.0, vp(0),
                                vp(16), 1 << 30) == fa.FP4_ERR_UNSUPPORTED
    need = fa.fp4_attn_workspace_bytes_fp8pv(1, 1, 1, 8, 128)
    assert L.fp4_attn_fwd_fp8pv(vp(16), vp(16), vp(16), vp(16), 1, 1, 1, 8, 128, 0, 0.0, vp(0),
                                vp(16), need - 1) == fa.FP4_ERR_WORKSPACE
    assert L.fp4_quantize_fp8(vp(16), 1, 8, 128, vp(0), vp(16), vp(0)) == fa.FP4_ERR_INVALID_ARG
    assert L.fp4_quantize_fp8(vp(16), 1, 8, 128, vp(24), vp(16), vp(0)) == fa.FP4_ERR_INVALID_ARG
    assert L.fp4_quantize_fp8(vp(16), 1, 8, 96, vp(16), vp(16), vp(0)) == fa.FP4_ERR_UNSUPPORTED
    assert L.fp4_quantize_fp8_scaled(vp(16), 1, 8, 128, vp(18), vp(16), vp(0)) == \
        fa.FP4_ERR_INVALID_ARG
    assert L.fp4_quantize_fp8_scaled(vp(16), 1, 0, 128, vp(16), vp(16), vp(0)) == \
        fa.FP4_ERR_INVALID_ARG
    t = fa._Tensor(16, 16, 16)
    t0 = fa._Tensor(16, 0, 16)  # FP8 V: scales not read, may be NULL
    assert L.fp4_attn_fwd_quantized_fp8pv(ctypes.byref(t), ctypes.byref(t), ctypes.byref(t0),
                                          vp(16), 1, 3, 2, 8, 128, 0, 0.0, vp(0)) == \
        fa.FP4_ERR_INVALID_ARG  # H % Hkv
    assert L.fp4_attn_fwd_quantized_fp8pv(ctypes.byref(t0), ctypes.byref(t), ctypes.byref(t0),
                                          vp(16), 1, 1, 1, 8, 128, 0, 0.0, vp(0)) == \
        fa.FP4_ERR_INVALID_ARG  # Q without scales
    assert L.fp4_attn_fwd_quantized(ctypes.byref(t), ctypes.byref(t), ctypes.byref(t0),
                                    vp(16), 1, 1, 1, 8, 128, 0, 0.0, vp(0)) == \
        fa.FP4_ERR_INVALID_ARG  # NVFP4 V without scales
    # smoothing: unknown flags, N beyond the exact sums' range, workspace, misaligned maxima
    need = fa.fp4_attn_workspace_bytes_smooth(1, 1, 1, 8, 128)
    assert need > fa.fp4_attn_workspace_bytes(1, 1, 1, 8, 128)
    assert fa.fp4_attn_workspace_bytes_smooth(1, 1, 1, (1 << 19) + 1, 64) == 0
    smooth = lambda fl, N=8, wsz=1 << 30: L.fp4_attn_fwd_smooth(
        vp(16), vp(16), vp(16), vp(16), 1, 1, 1, N, 128, 0, 0.0, fl, vp(0), vp(16), wsz)
    assert smooth(4) == fa.FP4_ERR_INVALID_ARG
    assert smooth(3, N=(1 << 19) + 1) == fa.FP4_ERR_INVALID_ARG
    assert smooth(3, wsz=need - 1) == fa.FP4_ERR_WORKSPACE
    assert L.fp4_channel_mean(vp(16), 1, 8, 128, vp(16), vp(16), vp(0), vp(0)) == \
        fa.FP4_ERR_INVALID_ARG
    assert L.fp4_score_bias(vp(16), vp(16), vp(0), 1, 1, 1, 8, 128, vp(18), vp(16), vp(16),
                            vp(0)) == fa.FP4_ERR_INVALID_ARG
    assert L.fp4_attn_fwd_quantized_bias(ctypes.byref(t), ctypes.byref(t), ctypes.byref(t),
                                         vp(0), vp(16), 1, 1, 1, 8, 128, 0, 0.0, vp(0)) == \
        fa.FP4_ERR_INVALID_ARG
    # backward: workspace size, null lse, null out, misaligned output, too small a workspace
    wb = fa.lib().fp4_attn_bwd_workspace_bytes(1, 2, 1, 300, 128)
    assert wb >= 2 * 384 * 128 * 2 * 4  # Q^, Q^T, dO, dO^T at least
    assert fa.lib().fp4_attn_bwd_workspace_bytes(1, 3, 2, 300, 128) == 0
    bwd = lambda lse=16, dq=16, o=16, wsz=1 << 34: L.fp4_attn_bwd(
        vp(16), vp(16), vp(16), vp(o), vp(16), vp(lse), vp(dq), vp(16), vp(16), 1, 2, 1, 300,
        128, 0, 0.0, vp(0), vp(16), wsz)
    assert bwd(lse=0) == fa.FP4_ERR_INVALID_ARG
    assert bwd(o=0) == fa.FP4_ERR_INVALID_ARG
    assert bwd(o=40) == fa.FP4_ERR_INVALID_ARG
    assert bwd(dq=24) == fa.FP4_ERR_INVALID_ARG
    assert bwd(wsz=wb - 1) == fa.FP4_ERR_WORKSPACE
    assert L.fp4_attn_fwd_lse(vp(16), vp(16), vp(16), vp(16), vp(0), 1, 1, 1, 8, 128, 0, 0.0,
                              vp(0), vp(16), 1 << 30) == fa.FP4_ERR_INVALID_ARG
    assert L.fp4_attn_bwd_scaled(vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), vp(0), vp(16),
                                 vp(16), vp(16), 1, 2, 1, 300, 128, 0, 0.0, vp(0), vp(16),
                                 1 << 34) == \
        fa.FP4_ERR_INVALID_ARG  # no maxima
    assert L.fp4_attn_fwd_quantized_lse(ctypes.byref(t), ctypes.byref(t), ctypes.byref(t), vp(16),
                                        vp(0), 1, 1, 1, 8, 128, 0, 0.0, vp(0)) == \
        fa.FP4_ERR_INVALID_ARG  # no lse
    assert L.fp4_attn_fwd_quantized_lse(ctypes.byref(t), ctypes.byref(t), ctypes.byref(t), vp(16),
                                        vp(18), 1, 1, 1, 8, 128, 0, 0.0, vp(0)) == \
        fa.FP4_ERR_INVALID_ARG  # misaligned lse


def test_product_path_does_not_touch_the_oracle():
    """The package, its sources and bench's GPU leg never import the oracle."""
    pkg = os.path.join(ROOT, "bit_attention_transformers_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c", ".cpp")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in txt.lower(), f
