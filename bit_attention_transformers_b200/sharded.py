"""Head-sharded NVFP4 attention forward across ranks (one process per GPU).

Every (batch, key/value head) unit of attention, with its G = H / Hkv query
heads, is independent of every other unit. The one quantity that couples them
is the NVFP4 tensor scale, which the recipe forms from max |x| over the whole
tensor (one fp32 scale per tensor: TetraJet-v2 abstract, NVFP4). So a tensor
held in shards is quantised exactly as the whole tensor would be: every rank
takes its shard's maxima of Q, K and V, one all-reduce (MAX) of those three
floats makes them global, and every rank then quantises its own shard with
them and runs the fused forward on it. Codes, scales and outputs are then the
same, bit for bit, as one GPU's run over the whole tensors; the outputs stay
sharded by head and nothing else crosses between ranks.

The units are the B * Hkv (batch, key/value head) pairs in memory order,
split into contiguous ranges, so that a rank's share of q viewed as
[B * H, N, D] and of k, v viewed as [B * Hkv, N, D] is one contiguous slab.
"""
from __future__ import annotations


def shard_units(B: int, Hkv: int, world: int, rank: int) -> tuple[int, int]:
    """[u0, u1): the (batch, key/value head) units of `rank`, unit u = b * Hkv + kv_head.

    Ranges are contiguous and in rank order, their sizes differ by at most one,
    and ranks beyond the number of units get an empty range."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if B < 0 or Hkv < 1:
        raise ValueError(f"B={B}, Hkv={Hkv}")
    base, extra = divmod(B * Hkv, world)
    u0 = rank * base + min(rank, extra)
    return u0, u0 + base + (1 if rank < extra else 0)


def shard_rows(B: int, H: int, Hkv: int, world: int, rank: int) -> tuple[slice, slice]:
    """Slices of the leading dim of q viewed as [B * H, N, D] and of k, v viewed
    as [B * Hkv, N, D] that `rank` owns (query head h of a batch reads key/value
    head h / G, so the query rows of unit u are u * G .. u * G + G - 1)."""
    if H % Hkv:
        raise ValueError(f"H ({H}) must be a multiple of Hkv ({Hkv})")
    g = H // Hkv
    u0, u1 = shard_units(B, Hkv, world, rank)
    return slice(u0 * g, u1 * g), slice(u0, u1)


def allreduce_max_(t, group=None):
    """In place: t = elementwise max of t over the ranks of `group`.

    A no-op unless torch.distributed has a process group with more than one
    rank (NCCL for CUDA tensors; any backend that supports MAX for others)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return t


def fp4_attn_fwd_sharded(q, k, v, causal: bool = False, softmax_scale: float | None = None,
                         group=None, out=None, stream=None, efq: bool = False,
                         fp8pv: bool = False, smooth: int = 0, lse=None):
    """This rank's part of a head-sharded NVFP4 attention forward.

    q: this rank's query heads, a contiguous bf16 CUDA tensor [..., N, D] whose
    leading dims hold Gq = U * G heads in unit order; k, v: its U key/value
    heads, [..., N, D]. Every rank of `group` calls this with the same N, D,
    G, causal and softmax_scale, an empty shard (U = 0) included: it still
    takes part in the all-reduce. Returns `out` (like q) with this rank's
    output heads. efq selects the EFQ-Softmax P generation, fp8pv the FP8 P
    and V variant, smooth (FP4_SMOOTH_K | FP4_SMOOTH_Q) Q/K smoothing: the
    means are per head, so local; their grid comes from the global raw
    maxima, and a second all-reduce (MAX) makes the smoothed maxima global.
    lse (float32, this rank's Gq * N values): the training forward also
    writes the rows' lse for fp4_attn_bwd_sharded."""
    import torch
    from . import (FP4_BLOCK_ALONG_D, FP4_BLOCK_ALONG_N_T, FP4_SMOOTH_K, FP4_SMOOTH_Q,
                   fp4_amax, fp4_amax_smoothed, fp4_attn_fwd_quantized,
                   fp4_attn_fwd_quantized_bias, fp4_channel_mean, fp4_quantize, fp4_quantize_fp8,
                   fp4_quantize_smoothed, fp4_score_bias)
    if smooth and (efq or fp8pv):
        raise ValueError("smoothing is built for the exp-then-quantize NVFP4 path")
    if lse is not None and (smooth or efq or fp8pv):
        raise ValueError("lse is written by the plain exp-then-quantize forward")
    N, D = q.shape[-2], q.shape[-1]
    if k.shape[-2:] != (N, D) or v.shape != k.shape:
        raise ValueError("q, k, v must share N and D, and k and v their shape")
    gq, gkv = q.numel() // (N * D), k.numel() // (N * D)
    if (gkv == 0) != (gq == 0) or (gkv and gq % gkv):
        raise ValueError(f"{gq} query heads for {gkv} key/value heads")
    amax = torch.zeros(3, dtype=torch.float32, device=q.device)
    if gkv:
        fp4_amax(q, amax[0:1], stream)
        fp4_amax(k, amax[1:2], stream)
        fp4_amax(v, amax[2:3], stream)
    allreduce_max_(amax, group)
    if out is None:
        out = torch.empty_like(q)
    if smooth:
        # means with the global raw maxima; then the smoothed maxima, made global
        sm = torch.zeros(2, dtype=torch.float32, device=q.device)
        qmean = kmean = None
        if gkv and smooth & FP4_SMOOTH_K:
            kmean = fp4_channel_mean(k, amax[1:2], stream)
            sm[1:2] = fp4_amax_smoothed(k, kmean, stream)
        if gkv and smooth & FP4_SMOOTH_Q:
            qmean = fp4_channel_mean(q, amax[0:1], stream)
            sm[0:1] = fp4_amax_smoothed(q, qmean, stream)
        allreduce_max_(sm, group)
        if gkv == 0:
            return out
        qq = (fp4_quantize_smoothed(q, qmean, sm[0:1], stream) if qmean is not None else
              fp4_quantize(q, FP4_BLOCK_ALONG_D, stream, amax=amax[0:1]))
        kq = (fp4_quantize_smoothed(k, kmean, sm[1:2], stream) if kmean is not None else
              fp4_quantize(k, FP4_BLOCK_ALONG_D, stream, amax=amax[1:2]))
        vq = fp4_quantize(v, FP4_BLOCK_ALONG_N_T, stream, amax=amax[2:3])
        if qmean is not None:
            bias = fp4_score_bias(qmean, k.view(1, gkv, N, D), kmean, gq, sm[0:1],
                                  sm[1:2] if kmean is not None else amax[1:2], stream)
            fp4_attn_fwd_quantized_bias(qq, kq, vq, bias, 1, gq, gkv, causal, softmax_scale,
                                        out=out, stream=stream)
        else:
            fp4_attn_fwd_quantized(qq, kq, vq, 1, gq, gkv, causal, softmax_scale, out=out,
                                   stream=stream)
        return out
    if gkv == 0:
        return out
    qq = fp4_quantize(q, FP4_BLOCK_ALONG_D, stream, amax=amax[0:1])
    kq = fp4_quantize(k, FP4_BLOCK_ALONG_D, stream, amax=amax[1:2])
    if fp8pv:
        vq = fp4_quantize_fp8(v, stream, amax=amax[2:3])
    else:
        vq = fp4_quantize(v, FP4_BLOCK_ALONG_N_T, stream, amax=amax[2:3])
    fp4_attn_fwd_quantized(qq, kq, vq, 1, gq, gkv, causal, softmax_scale, out=out, stream=stream,
                           efq=efq, fp8pv=fp8pv, lse=lse)
    return out


def fp4_attn_bwd_sharded(q, k, v, out, dout, lse, causal: bool = False,
                         softmax_scale: float | None = None, group=None, dq=None, dk=None,
                         dv=None, stream=None):
    """This rank's part of the head-sharded FP4 attention backward: the same
    units as fp4_attn_fwd_sharded (q, out, dout, lse: this rank's query heads;
    k, v: its key/value heads; out the forward's output), one all-reduce (MAX) of the three maxima so that
    the operands are quantised as the whole tensors' are, then fp4_attn_bwd
    on the shard. Every rank of `group` calls it, an empty shard included.
    Returns (dq, dk, dv) for the shard."""
    import torch
    from . import fp4_amax, fp4_attn_bwd
    N, D = q.shape[-2], q.shape[-1]
    gq, gkv = q.numel() // (N * D), k.numel() // (N * D)
    if (gkv == 0) != (gq == 0) or (gkv and gq % gkv):
        raise ValueError(f"{gq} query heads for {gkv} key/value heads")
    amax = torch.zeros(3, dtype=torch.float32, device=q.device)
    if gkv:
        fp4_amax(q, amax[0:1], stream)
        fp4_amax(k, amax[1:2], stream)
        fp4_amax(v, amax[2:3], stream)
    allreduce_max_(amax, group)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if gkv == 0:
        return dq, dk, dv
    as4 = lambda t: t.view(1, -1, N, D)
    fp4_attn_bwd(as4(q), as4(k), as4(v), as4(out), as4(dout), lse.reshape(1, gq, N), causal,
                 softmax_scale, dq=as4(dq), dk=as4(dk), dv=as4(dv), stream=stream, amax=amax)
    return dq, dk, dv
