"""NVFP4 (4-bit) FlashAttention for B200: Python binding of libfp4attn.

A thin ctypes layer over the C ABI in include/fp4attn.h: it marshals torch
tensors (device memory and streams only) into the library's calls and raises
on error. Every step of the computation runs in the library's CUDA kernels;
there is no fallback path. The names are the C ABI's.

Forward: fp4_attn_fwd (P generation: exp-then-quantize, efq=True for
EFQ-Softmax, fp8pv=True for P and V in FP8; smooth= for Q/K smoothing), the
steps fp4_quantize / fp4_amax / fp4_quantize_scaled / fp4_attn_fwd_quantized,
fp4_attn_fwd_host(_many) from host buffers. Training: fp4_attn_fwd_lse and
fp4_attn_bwd. Several GPUs: fp4_attn_fwd_sharded, fp4_attn_bwd_sharded.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_HERE)
_SRC_DIR = os.path.join(_HERE, "csrc")
_RELEASE_LIB_PATH = os.path.join(_HERE, "libfp4attn.so")
_DEBUG_LIB_PATH = os.path.join(_HERE, "libfp4attn_debug.so")  # built with -DFP4_DEBUG
# FP4ATTN_DEBUG=1 in the environment loads the debug build (same entry points)
_LIB_PATH = _DEBUG_LIB_PATH if os.environ.get("FP4ATTN_DEBUG") == "1" else _RELEASE_LIB_PATH
_HEADER = os.path.join(_ROOT, "include", "fp4attn.h")

FP4_OK = 0
FP4_ERR_INVALID_ARG = 1
FP4_ERR_UNSUPPORTED = 2
FP4_ERR_WORKSPACE = 3
FP4_ERR_CUDA = 4
FP4_ERR_TIMEOUT = 5
FP4_ERR_BOUNDS = 6
FP4_BLOCK_ALONG_D = 0
FP4_BLOCK_ALONG_N_T = 1
FP8_TOKENS_T = -1  # Fp4Tensor.axis of E4M3 V codes [G][D][Npad] (no block scales)
FP4_SMOOTH_K = 1
FP4_SMOOTH_Q = 2

# Every symbol include/fp4attn.h declares.
EXPORTS = ("fp4_codes_bytes", "fp4_scales_bytes", "fp4_attn_workspace_bytes", "fp4_quantize",
           "fp4_amax", "fp4_quantize_scaled", "fp4_scales_to_canonical", "fp4_attn_fwd",
           "fp4_attn_fwd_quantized",
           "fp4_attn_fwd_efq", "fp4_attn_fwd_quantized_efq", "fp4_fp8_codes_bytes",
           "fp4_quantize_fp8", "fp4_quantize_fp8_scaled", "fp4_attn_workspace_bytes_fp8pv",
           "fp4_attn_fwd_fp8pv", "fp4_attn_fwd_quantized_fp8pv", "fp4_attn_workspace_bytes_smooth",
           "fp4_attn_fwd_smooth", "fp4_channel_mean", "fp4_amax_smoothed", "fp4_quantize_smoothed",
           "fp4_score_bias", "fp4_attn_fwd_quantized_bias", "fp4_attn_fwd_lse",
           "fp4_attn_bwd_workspace_bytes", "fp4_attn_bwd", "fp4_attn_bwd_scaled",
           "fp4_attn_fwd_quantized_lse", "fp4_attn_fwd_noalloc",
           "fp4_attn_host_workspace_bytes", "fp4_attn_fwd_host",
           "fp4_status", "fp4_last_error", "fp4_probe_cvt", "fp4_test_wait_timeout",
           "fp4_debug_build", "fp4_debug_selftest")
FP4_NOALLOC_SCRATCH_BYTES = 64 << 20

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


class Fp4Error(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"fp4attn error {code}: {msg}")
        self.code = code


def _sources():
    return [os.path.join(_SRC_DIR, f) for f in sorted(os.listdir(_SRC_DIR))
            if f.endswith((".cu", ".cuh"))] + [_HEADER]


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Compile libfp4attn.so in-tree for sm_100a (nvcc; no GPU needed), and
    with `debug` also libfp4attn_debug.so (-DFP4_DEBUG: the bounds-checking
    build). Returns the path of the library `lib()` loads."""
    newest = max(os.path.getmtime(s) for s in _sources())
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    for path, extra in ((_RELEASE_LIB_PATH, []), (_DEBUG_LIB_PATH, ["-DFP4_DEBUG"])):
        if extra and not debug:
            continue
        if force or not os.path.exists(path) or os.path.getmtime(path) < newest:
            tmp = path + f".tmp{os.getpid()}"
            cmd = [nvcc, *NVCC_FLAGS, *extra, "-o", tmp, os.path.join(_SRC_DIR, "fp4attn.cu")]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            subprocess.check_call(cmd)
            os.replace(tmp, path)
    return _LIB_PATH


def load(debug: bool = False) -> ctypes.CDLL:
    """Select the release (default) or the debug build for `lib()` and load
    it; the next calls of every entry point go to that library."""
    global _lib, _LIB_PATH
    path = _DEBUG_LIB_PATH if debug else _RELEASE_LIB_PATH
    if path != _LIB_PATH:
        _LIB_PATH, _lib = path, None
    return lib()


_lib = None


def lib():
    """The loaded library. Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: run bit_attention_transformers_b200.build()")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, i64, u32, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                      ctypes.c_uint32, ctypes.c_float, ctypes.c_size_t)
        L.fp4_codes_bytes.argtypes = [i32, i32, i32, i32]
        L.fp4_codes_bytes.restype = sz
        L.fp4_scales_bytes.argtypes = [i32, i32, i32, i32]
        L.fp4_scales_bytes.restype = sz
        L.fp4_attn_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
        L.fp4_attn_workspace_bytes.restype = sz
        L.fp4_quantize.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
        L.fp4_quantize.restype = i32
        L.fp4_amax.argtypes = [vp, i32, i32, i32, vp, vp]
        L.fp4_amax.restype = i32
        L.fp4_quantize_scaled.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
        L.fp4_quantize_scaled.restype = i32
        L.fp4_scales_to_canonical.argtypes = [vp, i32, i32, i32, i32, vp, vp]
        L.fp4_scales_to_canonical.restype = i32
        L.fp4_attn_fwd.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, vp, sz]
        L.fp4_attn_fwd.restype = i32
        L.fp4_attn_host_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
        L.fp4_attn_host_workspace_bytes.restype = sz
        L.fp4_attn_fwd_host.argtypes = L.fp4_attn_fwd.argtypes
        L.fp4_attn_fwd_host.restype = i32
        L.fp4_attn_fwd_quantized.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp]
        L.fp4_attn_fwd_quantized.restype = i32
        L.fp4_attn_fwd_efq.argtypes = L.fp4_attn_fwd.argtypes
        L.fp4_attn_fwd_efq.restype = i32
        L.fp4_attn_fwd_quantized_efq.argtypes = L.fp4_attn_fwd_quantized.argtypes
        L.fp4_attn_fwd_quantized_efq.restype = i32
        L.fp4_fp8_codes_bytes.argtypes = [i32, i32, i32]
        L.fp4_fp8_codes_bytes.restype = sz
        L.fp4_quantize_fp8.argtypes = [vp, i32, i32, i32, vp, vp, vp]
        L.fp4_quantize_fp8.restype = i32
        L.fp4_quantize_fp8_scaled.argtypes = [vp, i32, i32, i32, vp, vp, vp]
        L.fp4_quantize_fp8_scaled.restype = i32
        L.fp4_attn_workspace_bytes_fp8pv.argtypes = [i32, i32, i32, i32, i32]
        L.fp4_attn_workspace_bytes_fp8pv.restype = sz
        L.fp4_attn_fwd_fp8pv.argtypes = L.fp4_attn_fwd.argtypes
        L.fp4_attn_fwd_fp8pv.restype = i32
        L.fp4_attn_fwd_quantized_fp8pv.argtypes = L.fp4_attn_fwd_quantized.argtypes
        L.fp4_attn_fwd_quantized_fp8pv.restype = i32
        L.fp4_attn_workspace_bytes_smooth.argtypes = [i32, i32, i32, i32, i32]
        L.fp4_attn_workspace_bytes_smooth.restype = sz
        L.fp4_attn_fwd_smooth.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32,
                                          vp, vp, sz]
        L.fp4_attn_fwd_smooth.restype = i32
        L.fp4_channel_mean.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp]
        L.fp4_channel_mean.restype = i32
        L.fp4_amax_smoothed.argtypes = [vp, i32, i32, i32, vp, vp, vp]
        L.fp4_amax_smoothed.restype = i32
        L.fp4_quantize_smoothed.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp]
        L.fp4_quantize_smoothed.restype = i32
        L.fp4_score_bias.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp]
        L.fp4_score_bias.restype = i32
        L.fp4_attn_fwd_quantized_bias.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                                  f32, vp]
        L.fp4_attn_fwd_quantized_bias.restype = i32
        L.fp4_attn_fwd_lse.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp,
                                       vp, sz]
        L.fp4_attn_fwd_lse.restype = i32
        L.fp4_attn_bwd_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
        L.fp4_attn_bwd_workspace_bytes.restype = sz
        L.fp4_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                   i32, f32, vp, vp, sz]
        L.fp4_attn_bwd.restype = i32
        L.fp4_attn_bwd_scaled.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                          i32, i32, i32, f32, vp, vp, sz]
        L.fp4_attn_bwd_scaled.restype = i32
        L.fp4_attn_fwd_quantized_lse.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                                 f32, vp]
        L.fp4_attn_fwd_quantized_lse.restype = i32
        L.fp4_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp]
        L.fp4_attn_fwd_noalloc.restype = i32
        L.fp4_status.argtypes = [vp]
        L.fp4_status.restype = i32
        L.fp4_last_error.argtypes = []
        L.fp4_last_error.restype = ctypes.c_char_p
        L.fp4_probe_cvt.argtypes = [u32, i64, i32, vp, vp]
        L.fp4_probe_cvt.restype = i32
        L.fp4_test_wait_timeout.argtypes = [ctypes.c_uint64, vp, vp]
        L.fp4_test_wait_timeout.restype = i32
        L.fp4_debug_build.argtypes = []
        L.fp4_debug_build.restype = i32
        L.fp4_debug_selftest.argtypes = [ctypes.c_uint, vp]
        L.fp4_debug_selftest.restype = i32
        _lib = L
    return _lib


class _Tensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("amax", ctypes.c_void_p)]


def _check(rc: int):
    if rc != FP4_OK:
        raise Fp4Error(rc, lib().fp4_last_error().decode())


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


# ------------------------------------------------------------------ sizes ----
def fp4_codes_bytes(G: int, N: int, D: int, axis: int) -> int:
    return lib().fp4_codes_bytes(G, N, D, axis)


def fp4_scales_bytes(G: int, N: int, D: int, axis: int) -> int:
    return lib().fp4_scales_bytes(G, N, D, axis)


def fp4_attn_workspace_bytes(B: int, H: int, Hkv: int, N: int, D: int) -> int:
    return lib().fp4_attn_workspace_bytes(B, H, Hkv, N, D)


# --------------------------------------------------------------- quantise ----
@dataclass
class Fp4Tensor:
    """A quantised tensor on the device (layouts in include/fp4attn.h)."""
    codes: "object"
    scales: "object"
    amax: "object"
    G: int
    N: int
    D: int
    axis: int


def _gnd(x):
    import torch
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous()
    N, D = x.shape[-2], x.shape[-1]
    return x.numel() // (N * D), N, D


def fp4_quantize(x, axis: int = FP4_BLOCK_ALONG_D, stream=None, amax=None) -> Fp4Tensor:
    """x: bf16 CUDA tensor [..., N, D] (the leading dims form the groups G).
    With `amax` (a float32 CUDA tensor whose first element is the tensor
    maximum, e.g. combined over shards) the tensor scale comes from it
    (fp4_quantize_scaled); otherwise max |x| is computed first."""
    import torch
    G, N, D = _gnd(x)
    codes = torch.empty(fp4_codes_bytes(G, N, D, axis), dtype=torch.uint8, device=x.device)
    scales = torch.empty(fp4_scales_bytes(G, N, D, axis), dtype=torch.uint8, device=x.device)
    if amax is None:
        amax = torch.empty(4, dtype=torch.float32, device=x.device)
        _check(lib().fp4_quantize(_ptr(x), G, N, D, axis, _ptr(codes), _ptr(scales), _ptr(amax),
                                  _stream(stream)))
    else:
        assert amax.is_cuda and amax.dtype == torch.float32
        _check(lib().fp4_quantize_scaled(_ptr(x), G, N, D, axis, _ptr(amax), _ptr(codes),
                                         _ptr(scales), _stream(stream)))
    return Fp4Tensor(codes, scales, amax, G, N, D, axis)


def fp4_fp8_codes_bytes(G: int, N: int, D: int) -> int:
    return lib().fp4_fp8_codes_bytes(G, N, D)


def fp4_attn_workspace_bytes_fp8pv(B: int, H: int, Hkv: int, N: int, D: int) -> int:
    return lib().fp4_attn_workspace_bytes_fp8pv(B, H, Hkv, N, D)


def fp4_quantize_fp8(x, stream=None, amax=None) -> Fp4Tensor:
    """E4M3 quantisation of V for the FP8 P/V variant: x bf16 CUDA [..., N, D]
    -> codes [G][D][Npad] (one byte each), no block scales (scales is None,
    axis FP8_TOKENS_T). With `amax` (float32 CUDA, first element the tensor
    maximum) fp4_quantize_fp8_scaled runs; otherwise max |x| is computed first."""
    import torch
    G, N, D = _gnd(x)
    codes = torch.empty(fp4_fp8_codes_bytes(G, N, D), dtype=torch.uint8, device=x.device)
    if amax is None:
        amax = torch.empty(4, dtype=torch.float32, device=x.device)
        _check(lib().fp4_quantize_fp8(_ptr(x), G, N, D, _ptr(codes), _ptr(amax), _stream(stream)))
    else:
        assert amax.is_cuda and amax.dtype == torch.float32
        _check(lib().fp4_quantize_fp8_scaled(_ptr(x), G, N, D, _ptr(amax), _ptr(codes),
                                             _stream(stream)))
    return Fp4Tensor(codes, None, amax, G, N, D, FP8_TOKENS_T)


def fp4_scales_to_canonical(t: Fp4Tensor, stream=None):
    """t's block scales in their logical layout: [G][N][D/16] (blocks along D)
    or [G][D][Npad/16] (blocks along tokens), a uint8 CUDA tensor."""
    import torch
    npad = (t.N + 127) // 128 * 128
    shape = (t.G, t.N, t.D // 16) if t.axis == FP4_BLOCK_ALONG_D else (t.G, t.D, npad // 16)
    out = torch.empty(shape, dtype=torch.uint8, device=t.scales.device)
    _check(lib().fp4_scales_to_canonical(_ptr(t.scales), t.G, t.N, t.D, t.axis, _ptr(out),
                                         _stream(stream)))
    return out


def fp4_amax(x, out=None, stream=None):
    """max |x| of a bf16 CUDA tensor [..., N, D] into out[0] (float32 CUDA)."""
    import torch
    G, N, D = _gnd(x)
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(lib().fp4_amax(_ptr(x), G, N, D, _ptr(out), _stream(stream)))
    return out


# -------------------------------------------------------------- attention ----
# Cached workspaces, one per (device, stream, kind). Calls on one stream run in
# order, so they can share one; calls on two streams may overlap on the GPU and
# must not, so each stream gets its own. A caller that passes `ws` itself owns
# that rule: one workspace must not serve two calls that can overlap.
_ws_cache: dict = {}


def _stream_handle(stream) -> int:
    return _stream(stream).value or 0


def workspace(B, H, Hkv, N, D, device, fp8pv: bool = False, smooth: int = 0, stream=None):
    """A cached device workspace large enough for fp4_attn_fwd (or, with
    fp8pv, fp4_attn_fwd_fp8pv; with smooth, fp4_attn_fwd_smooth) on this shape,
    private to `stream` (default: the current stream) on `device`."""
    import torch
    fn = (fp4_attn_workspace_bytes_smooth if smooth else
          fp4_attn_workspace_bytes_fp8pv if fp8pv else fp4_attn_workspace_bytes)
    need = fn(B, H, Hkv, N, D)
    with torch.cuda.device(device):
        key = ("fwd", str(device), _stream_handle(stream))
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def _attn_fn(efq: bool, fp8pv: bool, quantized: bool):
    if efq and fp8pv:
        raise ValueError("efq and fp8pv are two different P generations; pick one")
    name = "fp4_attn_fwd_quantized" if quantized else "fp4_attn_fwd"
    return getattr(lib(), name + ("_efq" if efq else "_fp8pv" if fp8pv else ""))


def fp4_attn_fwd(q, k, v, causal: bool = False, softmax_scale: float | None = None, out=None,
                 stream=None, ws=None, efq: bool = False, fp8pv: bool = False, smooth: int = 0):
    """NVFP4 attention forward. q [B,H,N,D], k/v [B,Hkv,N,D]: contiguous bf16
    CUDA tensors. Returns out [B,H,N,D] bf16. efq=True calls fp4_attn_fwd_efq
    (P from EFQ-Softmax instead of exp-then-quantize); fp8pv=True calls
    fp4_attn_fwd_fp8pv (P and V in E4M3); smooth (FP4_SMOOTH_K | FP4_SMOOTH_Q)
    calls fp4_attn_fwd_smooth."""
    if smooth:
        if efq or fp8pv:
            raise ValueError("smoothing is built for the exp-then-quantize NVFP4 path")
        return fp4_attn_fwd_smooth(q, k, v, smooth, causal, softmax_scale, out=out, stream=stream,
                                   ws=ws)
    import torch
    B, H, N, D = q.shape
    Hkv = k.shape[1]
    for t in (q, k, v):
        assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
    assert k.shape == (B, Hkv, N, D) and v.shape == (B, Hkv, N, D)
    if out is None:
        out = torch.empty_like(q)
    fn = _attn_fn(efq, fp8pv, False)
    if ws is None:
        ws = workspace(B, H, Hkv, N, D, q.device, fp8pv, stream=stream)
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Hkv, N, D, int(bool(causal)),
              float(softmax_scale or 0.0), _stream(stream), _ptr(ws), ws.numel()))
    return out


def fp4_attn_fwd_lse(q, k, v, causal: bool = False, softmax_scale: float | None = None,
                     out=None, lse=None, stream=None, ws=None):
    """fp4_attn_fwd that also returns lse [B, H, N] fp32 (log2 units) for the
    backward. Returns (out, lse)."""
    import torch
    B, H, N, D = q.shape
    Hkv = k.shape[1]
    for t in (q, k, v):
        assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
    assert k.shape == (B, Hkv, N, D) and v.shape == (B, Hkv, N, D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(B, H, Hkv, N, D, q.device, stream=stream)
    _check(lib().fp4_attn_fwd_lse(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv, N, D,
                                  int(bool(causal)), float(softmax_scale or 0.0), _stream(stream),
                                  _ptr(ws), ws.numel()))
    return out, lse


def fp4_attn_bwd(q, k, v, out, dout, lse, causal: bool = False,
                 softmax_scale: float | None = None, dq=None, dk=None, dv=None, stream=None,
                 ws=None, amax=None):
    """The FP4 attention backward (reading in include/fp4attn.h): q, out, dout
    [B,H,N,D], k, v [B,Hkv,N,D] bf16 CUDA; out and lse [B,H,N] from
    fp4_attn_fwd_lse. With `amax` (float32 CUDA [3]: the maxima of Q, K, V,
    e.g. combined over shards) fp4_attn_bwd_scaled quantises with them.
    Returns (dq, dk, dv) bf16."""
    import torch
    B, H, N, D = q.shape
    Hkv = k.shape[1]
    for t in (q, k, v, out, dout):
        assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
    assert k.shape == (B, Hkv, N, D) and v.shape == k.shape
    assert dout.shape == q.shape and out.shape == q.shape
    assert lse.dtype == torch.float32 and lse.is_contiguous() and lse.numel() == B * H * N
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if ws is None:
        need = lib().fp4_attn_bwd_workspace_bytes(B, H, Hkv, N, D)
        with torch.cuda.device(q.device):
            key = ("bwd", str(q.device), _stream_handle(stream))
        ws = _ws_cache.get(key)
        if ws is None or ws.numel() < need:
            ws = torch.empty(need, dtype=torch.uint8, device=q.device)
            _ws_cache[key] = ws
    if amax is not None:
        assert amax.is_cuda and amax.dtype == torch.float32 and amax.numel() >= 3
        _check(lib().fp4_attn_bwd_scaled(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout),
                                         _ptr(lse), _ptr(amax), _ptr(dq), _ptr(dk), _ptr(dv), B, H,
                                         Hkv, N, D, int(bool(causal)),
                                         float(softmax_scale or 0.0), _stream(stream), _ptr(ws),
                                         ws.numel()))
        return dq, dk, dv
    _check(lib().fp4_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                              _ptr(dq), _ptr(dk), _ptr(dv), B, H, Hkv, N, D, int(bool(causal)),
                              float(softmax_scale or 0.0), _stream(stream), _ptr(ws), ws.numel()))
    return dq, dk, dv


def fp4_attn_workspace_bytes_smooth(B: int, H: int, Hkv: int, N: int, D: int) -> int:
    return lib().fp4_attn_workspace_bytes_smooth(B, H, Hkv, N, D)


def fp4_attn_fwd_smooth(q, k, v, smooth: int = FP4_SMOOTH_K | FP4_SMOOTH_Q, causal: bool = False,
                        softmax_scale: float | None = None, out=None, stream=None, ws=None):
    """NVFP4 attention forward with Q and/or K smoothed before quantisation
    (smooth = FP4_SMOOTH_K | FP4_SMOOTH_Q; the reading in include/fp4attn.h).
    Same tensors as fp4_attn_fwd."""
    import torch
    B, H, N, D = q.shape
    Hkv = k.shape[1]
    for t in (q, k, v):
        assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
    assert k.shape == (B, Hkv, N, D) and v.shape == (B, Hkv, N, D)
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        need = fp4_attn_workspace_bytes_smooth(B, H, Hkv, N, D)
        with torch.cuda.device(q.device):
            key = ("smooth", str(q.device), _stream_handle(stream))
        ws = _ws_cache.get(key)
        if ws is None or ws.numel() < need:
            ws = torch.empty(need, dtype=torch.uint8, device=q.device)
            _ws_cache[key] = ws
    _check(lib().fp4_attn_fwd_smooth(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Hkv, N, D,
                                     int(bool(causal)), float(softmax_scale or 0.0), int(smooth),
                                     _stream(stream), _ptr(ws), ws.numel()))
    return out


def fp4_channel_mean(x, amax, stream=None):
    """Smoothing means [G, D] fp32 of x [..., N, D] (bf16 CUDA) on the grid of
    amax (float32 CUDA tensor, first element the raw tensor's maximum)."""
    import torch
    G, N, D = _gnd(x)
    mean = torch.empty((G, D), dtype=torch.float32, device=x.device)
    sums = torch.empty((G, D), dtype=torch.int64, device=x.device)
    _check(lib().fp4_channel_mean(_ptr(x), G, N, D, _ptr(amax), _ptr(mean), _ptr(sums),
                                  _stream(stream)))
    return mean


def fp4_amax_smoothed(x, mean, stream=None):
    """max |fl32(x - mean)| (float32 CUDA tensor of one element)."""
    import torch
    G, N, D = _gnd(x)
    out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(lib().fp4_amax_smoothed(_ptr(x), G, N, D, _ptr(mean), _ptr(out), _stream(stream)))
    return out


def fp4_quantize_smoothed(x, mean, amax, stream=None) -> Fp4Tensor:
    """NVFP4 (blocks along D) of fl32(x - mean) with the smoothed tensor's
    maximum amax (float32 CUDA)."""
    import torch
    G, N, D = _gnd(x)
    codes = torch.empty(fp4_codes_bytes(G, N, D, FP4_BLOCK_ALONG_D), dtype=torch.uint8,
                        device=x.device)
    scales = torch.empty(fp4_scales_bytes(G, N, D, FP4_BLOCK_ALONG_D), dtype=torch.uint8,
                         device=x.device)
    _check(lib().fp4_quantize_smoothed(_ptr(x), G, N, D, _ptr(mean), _ptr(amax), _ptr(codes),
                                       _ptr(scales), _stream(stream)))
    return Fp4Tensor(codes, scales, amax, G, N, D, FP4_BLOCK_ALONG_D)


def fp4_score_bias(qmean, k, kmean, H: int, q_amax, k_amax, stream=None):
    """Smoothed Q's score correction [B*H, Npad, 8] fp32 (hi, lo, 0...): qmean
    [B*H, D], k [B, Hkv, N, D] bf16, kmean [B*Hkv, D] or None, q_amax / k_amax
    the maxima (float32 CUDA, first element) the quantised Q' and K use."""
    import torch
    B, Hkv, N, D = k.shape
    npad = (N + 127) // 128 * 128
    bias = torch.empty((B * H, npad, 8), dtype=torch.float32, device=k.device)
    _check(lib().fp4_score_bias(_ptr(qmean), _ptr(k), None if kmean is None else _ptr(kmean), B, H,
                                Hkv, N, D, _ptr(q_amax), _ptr(k_amax), _ptr(bias),
                                _stream(stream)))
    return bias


def fp4_attn_fwd_quantized_bias(qq: Fp4Tensor, kq: Fp4Tensor, vq: Fp4Tensor, bias, B: int, H: int,
                                Hkv: int, causal: bool = False,
                                softmax_scale: float | None = None, out=None, stream=None):
    """The fused forward on quantised tensors with the per-key score
    correction bias [B*H, Npad, 8] from fp4_score_bias (exp-then-quantize P)."""
    import torch
    N, D = qq.N, qq.D
    if out is None:
        out = torch.empty((B, H, N, D), dtype=torch.bfloat16, device=qq.codes.device)
    ts = [_Tensor(t.codes.data_ptr(), t.scales.data_ptr(), t.amax.data_ptr()) for t in (qq, kq, vq)]
    _check(lib().fp4_attn_fwd_quantized_bias(ctypes.byref(ts[0]), ctypes.byref(ts[1]),
                                             ctypes.byref(ts[2]), _ptr(bias), _ptr(out), B, H, Hkv,
                                             N, D, int(bool(causal)), float(softmax_scale or 0.0),
                                             _stream(stream)))
    return out


def fp4_attn_fwd_noalloc(q, k, v, causal: bool = False, softmax_scale: float | None = None,
                         out=None, stream=None):
    """fp4_attn_fwd for callers that cannot allocate device memory: the
    scratch is the library's built-in FP4_NOALLOC_SCRATCH_BYTES array, shared
    by every call on a device (calls that overlap on the GPU race on it), and
    larger problems are rejected. `out` must be given to avoid any allocation
    here (it is created only as a convenience when omitted)."""
    import torch
    B, H, N, D = q.shape
    Hkv = k.shape[1]
    for t in (q, k, v):
        assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
    if out is None:
        out = torch.empty_like(q)
    _check(lib().fp4_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Hkv, N, D,
                                      int(bool(causal)), float(softmax_scale or 0.0),
                                      _stream(stream)))
    return out


def fp4_attn_fwd_quantized(qq: Fp4Tensor, kq: Fp4Tensor, vq: Fp4Tensor, B: int, H: int,
                           Hkv: int, causal: bool = False, softmax_scale: float | None = None,
                           out=None, stream=None, efq: bool = False, fp8pv: bool = False,
                           lse=None):
    """The fused forward alone on tensors fp4_quantize() produced
    (fp4_attn_fwd_quantized_efq with efq=True; fp4_attn_fwd_quantized_fp8pv
    with fp8pv=True, vq from fp4_quantize_fp8; fp4_attn_fwd_quantized_lse,
    writing lse [B, H, N] fp32, when lse is given)."""
    import torch
    N, D = qq.N, qq.D
    if out is None:
        out = torch.empty((B, H, N, D), dtype=torch.bfloat16, device=qq.codes.device)
    fn = _attn_fn(efq, fp8pv, True)
    if (vq.axis == FP8_TOKENS_T) != bool(fp8pv):
        raise ValueError("vq must come from fp4_quantize_fp8 exactly when fp8pv is set")
    ts = [_Tensor(t.codes.data_ptr(), 0 if t.scales is None else t.scales.data_ptr(),
                  t.amax.data_ptr()) for t in (qq, kq, vq)]
    if lse is not None:
        if efq or fp8pv:
            raise ValueError("lse is written by the exp-then-quantize forward")
        assert lse.dtype == torch.float32 and lse.is_contiguous()
        _check(lib().fp4_attn_fwd_quantized_lse(ctypes.byref(ts[0]), ctypes.byref(ts[1]),
                                                ctypes.byref(ts[2]), _ptr(out), _ptr(lse), B, H,
                                                Hkv, N, D, int(bool(causal)),
                                                float(softmax_scale or 0.0), _stream(stream)))
        return out
    _check(fn(ctypes.byref(ts[0]), ctypes.byref(ts[1]), ctypes.byref(ts[2]), _ptr(out), B, H,
              Hkv, N, D, int(bool(causal)), float(softmax_scale or 0.0), _stream(stream)))
    return out


def fp4_attn_fwd_host(q, k, v, causal: bool = False, softmax_scale: float | None = None,
                      out=None, device="cuda", stream=None, efq: bool = False,
                      fp8pv: bool = False, smooth: int = 0):
    """End-to-end call on host buffers: q, k, v pinned CPU bf16 tensors in,
    `out` (a pinned CPU tensor, allocated if None) back, returned once it holds
    the result. The default path is one call of the C entry fp4_attn_fwd_host
    (copies in, the forward, the copy out, all on `stream`); the variants
    (efq, fp8pv, smooth) copy with torch on the same stream and call their
    device entry."""
    import torch
    dev = torch.device(device)
    for t in (q, k, v):
        assert not t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
    B, H, N, D = q.shape
    Hkv = k.shape[1]
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    assert not out.is_cuda and out.shape == q.shape and out.dtype == q.dtype and out.is_contiguous()
    with torch.cuda.device(dev):
        s = torch.cuda.current_stream() if stream is None else stream
        if not (efq or fp8pv or smooth):
            need = lib().fp4_attn_host_workspace_bytes(B, H, Hkv, N, D)
            key = ("host", str(dev), _stream_handle(s))
            ws = _ws_cache.get(key)
            if ws is None or ws.numel() < need:
                ws = torch.empty(need, dtype=torch.uint8, device=dev)
                _ws_cache[key] = ws
            _check(lib().fp4_attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Hkv, N, D,
                                           int(bool(causal)), float(softmax_scale or 0.0),
                                           _stream(s), _ptr(ws), ws.numel()))
            return out
        with torch.cuda.stream(s):
            dq, dk, dv = (t.to(dev, non_blocking=True) for t in (q, k, v))
            o = fp4_attn_fwd(dq, dk, dv, causal, softmax_scale, stream=s, efq=efq, fp8pv=fp8pv,
                             smooth=smooth)
            out.copy_(o, non_blocking=True)
        s.synchronize()
    return out


def fp4_attn_fwd_host_many(batches, outs, causal: bool = False,
                           softmax_scale: float | None = None, device="cuda", efq: bool = False,
                           return_ms: bool = False, fp8pv: bool = False, smooth: int = 0):
    """End-to-end over a sequence of host batches: batches = [(q, k, v), ...]
    pinned CPU bf16 tensors of one shape, outs = pinned CPU tensors for the
    outputs. Two sets of device buffers and three streams (copies in, compute,
    copies out) let batch i+1's host-to-device copies and batch i-1's
    device-to-host copy run while batch i is computed. Returns outs (and the
    device time in ms from the first copy in to the last copy out, measured
    with CUDA events, when return_ms) once everything has finished."""
    import torch
    if not batches:
        return (outs, 0.0) if return_ms else outs
    q0, k0, _ = batches[0]
    B, H, N, D = q0.shape
    Hkv = k0.shape[1]
    dev = torch.device(device)
    s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    bufs = [tuple(torch.empty(t.shape, dtype=torch.bfloat16, device=dev) for t in (q0, k0, k0, q0))
            for _ in range(2)]
    ws = workspace(B, H, Hkv, N, D, dev, fp8pv, smooth)
    free = [None, None]  # event: slot's last device-to-host copy done
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i, (hq, hk, hv) in enumerate(batches):
        slot = i % 2
        dq, dk, dv, do = bufs[slot]
        with torch.cuda.stream(s_in):
            if free[slot] is not None:
                s_in.wait_event(free[slot])
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            loaded = torch.cuda.Event()
            loaded.record(s_in)
        s_run.wait_event(loaded)
        fp4_attn_fwd(dq, dk, dv, causal, softmax_scale, out=do, stream=s_run, ws=ws, efq=efq,
                     fp8pv=fp8pv, smooth=smooth)
        done = torch.cuda.Event()
        done.record(s_run)
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            outs[i].copy_(do, non_blocking=True)
            free[slot] = torch.cuda.Event()
            free[slot].record(s_out)
    end.record(s_out)
    end.synchronize()  # every stream is done with the device buffers
    if return_ms:
        return outs, start.elapsed_time(end)
    return outs


def fp4_status(stream=None):
    """Synchronise and raise if a kernel reported an expired wait or (debug
    build) a failed bounds check."""
    _check(lib().fp4_status(_stream(stream)))


def fp4_debug_build() -> bool:
    """Whether the loaded library is the FP4_DEBUG (bounds-checking) build."""
    return bool(lib().fp4_debug_build())


def fp4_debug_selftest(site: int, stream=None):
    """Debug build only: one check that fails by construction (no memory is
    addressed); the next fp4_status raises FP4_ERR_BOUNDS naming `site`."""
    _check(lib().fp4_debug_selftest(int(site), _stream(stream)))


def fp4_test_wait_timeout(limit_ns: int, stream=None):
    """Test support: a bounded wait that nothing ends; returns the device int
    that receives 0 once the wait has expired (the next fp4_status raises
    FP4_ERR_TIMEOUT)."""
    import torch
    ok = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    _check(lib().fp4_test_wait_timeout(int(limit_ns), _ptr(ok), _stream(stream)))
    return ok


def fp4_probe_cvt(start: int, count: int, kind: int, out=None, stream=None):
    import torch
    if out is None:
        out = torch.empty(count, dtype=torch.uint8, device="cuda")
    _check(lib().fp4_probe_cvt(start, count, kind, _ptr(out), _stream(stream)))
    return out


from .sharded import (allreduce_max_, fp4_attn_bwd_sharded, fp4_attn_fwd_sharded,  # noqa: E402
                      shard_rows, shard_units)
