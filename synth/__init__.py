"""Seeded synthetic workloads for the NVFP4 attention forward.

Only random numbers live here: no quantisation and no attention arithmetic.
The CPU oracle and the CUDA path both consume these arrays unchanged.

The five workloads restate, as synthetic data, the settings the source pages
evaluate 4-bit attention on: a small Gaussian case, heavy-tailed keys (Attn-QAT
abstract: "attention's heavy-tailed activations"), LLM prefill with grouped
query heads (Qwen3-8B in the EFQ-Softmax abstract), a video-DiT latent grid
(WAN2.2 in the EFQ-Softmax and SQuad abstracts) and long context (16K-128K in
the EFQ-Softmax abstract). The generator recipes are documented in synth.c.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so beside it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, i64, i32 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int
        vp = ctypes.c_void_p
        lib.synth_normal_bf16.argtypes = [u64, u64, i64, ctypes.c_float, vp, i32]
        lib.synth_normal_bf16.restype = None
        lib.synth_uniform_int.argtypes = [u64, u64, i64, i64, vp]
        lib.synth_uniform_int.restype = None
        lib.synth_distinct.argtypes = [u64, u64, i64, i64, vp]
        lib.synth_distinct.restype = None
        lib.synth_config_tensor.argtypes = [i32, i32, i32, i32, i32, i32, vp, u64, vp, i32]
        lib.synth_config_tensor.restype = i32
        lib.synth_outlier_tokens.argtypes = [u64, i32, vp]
        lib.synth_outlier_tokens.restype = i64
        _lib = lib
    return _lib


def _threads() -> int:
    return max(1, os.cpu_count() or 1)


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    H: int
    Hkv: int
    N: int
    D: int
    causal: bool
    recipe: int
    grid: tuple = field(default=())
    oracle_rows_per_head: int = 0  # 0: the oracle checks every row

    @property
    def seed(self) -> int:
        return 0x5EED0000 + self.index

    @property
    def flops(self) -> float:
        """4*B*H*N^2*D, halved when causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.D
        return f / 2 if self.causal else f

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "Hkv": self.Hkv,
                "N": self.N, "D": self.D, "causal": self.causal}


WORKLOADS = {
    "tiny": Workload(1, "tiny", 1, 2, 2, 256, 64, False, 1),
    "heavy_tailed": Workload(2, "heavy_tailed", 1, 8, 8, 2048, 128, False, 2),
    "llm_prefill": Workload(3, "llm_prefill", 4, 32, 8, 8192, 128, True, 3,
                            oracle_rows_per_head=16),
    "video_dit": Workload(4, "video_dit", 1, 24, 24, 32760, 128, False, 4, (21, 39, 40),
                          oracle_rows_per_head=16),
    "long_context": Workload(5, "long_context", 1, 32, 8, 131072, 128, True, 5,
                             oracle_rows_per_head=256),
}


def tensor(recipe: int, which: str, B: int, Hx: int, N: int, D: int, seed: int,
           grid: tuple = (), out: np.ndarray | None = None) -> np.ndarray:
    """One bf16 tensor [B, Hx, N, D] (as uint16 bit patterns) of a recipe.

    which: "q", "k" or "v". out: optional preallocated uint16 array (e.g. the
    numpy view of pinned host memory)."""
    lib = _load()
    w = {"q": 0, "k": 1, "v": 2}[which]
    if out is None:
        out = np.empty((B, Hx, N, D), dtype=np.uint16)
    assert out.dtype == np.uint16 and out.size == B * Hx * N * D and out.flags.c_contiguous
    g = (ctypes.c_int * 3)(*(grid if grid else (0, 0, 0)))
    rc = lib.synth_config_tensor(recipe, w, B, Hx, N, D, g, seed,
                                 out.ctypes.data, _threads())
    if rc != 0:
        raise ValueError(f"synth: bad arguments for recipe {recipe}")
    return out


def workload_inputs(wl: Workload, seed: int | None = None, outs=None):
    """(q, k, v) uint16 bf16 bit arrays of a workload."""
    s = wl.seed if seed is None else seed
    o = outs or (None, None, None)
    q = tensor(wl.recipe, "q", wl.B, wl.H, wl.N, wl.D, s, wl.grid, o[0])
    k = tensor(wl.recipe, "k", wl.B, wl.Hkv, wl.N, wl.D, s, wl.grid, o[1])
    v = tensor(wl.recipe, "v", wl.B, wl.Hkv, wl.N, wl.D, s, wl.grid, o[2])
    return q, k, v


def normal_bf16(n: int, seed: int, stream: int = 0, scale: float = 1.0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    _load().synth_normal_bf16(seed, stream, n, scale, out.ctypes.data, _threads())
    return out


def uniform_int(n: int, m: int, seed: int, stream: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.int64)
    _load().synth_uniform_int(seed, stream, n, m, out.ctypes.data)
    return out


def distinct(k: int, m: int, seed: int, stream: int = 0) -> np.ndarray:
    out = np.empty(k, dtype=np.int64)
    _load().synth_distinct(seed, stream, k, m, out.ctypes.data)
    return out


def sample_rows(wl: Workload, per_head: int, seed: int | None = None) -> np.ndarray:
    """Seeded query rows to check, as int64 triples (b, h, i): `per_head`
    distinct rows of every head, drawn uniformly without replacement."""
    s = (wl.seed if seed is None else seed) ^ 0xA11
    rows = []
    for b in range(wl.B):
        for h in range(wl.H):
            idx = distinct(min(per_head, wl.N), wl.N, s, stream=b * wl.H + h + 1)
            rows.extend((b, h, int(i)) for i in idx)
    return np.asarray(rows, dtype=np.int64).reshape(-1, 3)


def outlier_tokens(wl: Workload, seed: int | None = None) -> np.ndarray:
    out = np.empty(max(1, round(0.01 * wl.N)), dtype=np.int64)
    n = _load().synth_outlier_tokens(wl.seed if seed is None else seed, wl.N, out.ctypes.data)
    return out[:n]


def bf16_bits_to_f32(x: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (x.astype(np.uint32) << 16).view(np.float32)
