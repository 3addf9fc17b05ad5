"""GPU-side helpers for the parity tests: run the CUDA path through the C ABI
and bring quantised tensors back in the oracle's logical layouts."""
from __future__ import annotations

import numpy as np

import bit_attention_transformers_b200 as fa


def to_dev(x_u16: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x_u16).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev(t) -> np.ndarray:
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def scales_rows_logical(native: np.ndarray, G: int, N: int, D: int) -> np.ndarray:
    """Block-scale atoms (blocks along D) -> [G][N][D/16].
    Atom (g, tile, chunk) holds byte (r % 32) * 16 + (r // 32) * 4 + k for row
    tile*128 + r and block chunk*4 + k."""
    Npad = (N + 127) // 128 * 128
    a = native.reshape(G, Npad // 128, D // 64, 32, 4, 4)   # g, tile, chunk, r%32, r//32, k
    a = a.transpose(0, 1, 4, 3, 2, 5).reshape(G, Npad, D // 16)
    return a[:, :N]


def scales_tokens_logical(native: np.ndarray, G: int, N: int, D: int):
    """Block-scale atoms (blocks along tokens, rows = channels) -> [G][D][Npad/16],
    plus the padding channels' bytes [G][128-D][Npad/16] (must be zero)."""
    Npad = (N + 127) // 128 * 128
    a = native.reshape(G, Npad // 64, 32, 4, 4)             # g, atom, d%32, d//32, k
    full = a.transpose(0, 3, 2, 1, 4).reshape(G, 128, Npad // 16)
    return full[:, :D, :], full[:, D:, :]


def run_attn(q, k, v, causal: bool, softmax_scale: float = 0.0, efq: bool = False) -> np.ndarray:
    import torch
    out = fa.fp4_attn_fwd(to_dev(q), to_dev(k), to_dev(v), causal=causal,
                          softmax_scale=softmax_scale or None, efq=efq)
    torch.cuda.synchronize()
    fa.fp4_status()
    return from_dev(out)
