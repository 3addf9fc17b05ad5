"""Host side of the head-sharded multi-GPU forward, on the CPU: the partition
of (batch, key/value head) units over ranks, and the one exchange the path has
(an all-reduce MAX of the three tensor maxima), run as 2 and 3 gloo ranks.

With the maxima combined, quantising each rank's shard must give exactly the
codes and scales of quantising the whole tensors; the quantisation here is the
oracle's (this checks the sharding and the exchange, not the kernels, which
tests/test_gpu_sharded.py checks on the GPU against the unsharded path)."""
import os
import socket

import numpy as np
import pytest

import bit_attention_transformers_b200.sharded as sh


@pytest.mark.parametrize("B,Hkv", [(1, 1), (1, 24), (2, 8), (4, 8), (3, 5), (1, 2)])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_units_partition(B, Hkv, world):
    ranges = [sh.shard_units(B, Hkv, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == B * Hkv
    for (a0, a1), (b0, _) in zip(ranges, ranges[1:]):
        assert a1 == b0  # contiguous, in rank order
    sizes = [u1 - u0 for u0, u1 in ranges]
    assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1
    assert sum(sizes) == B * Hkv


def test_rows_follow_kv_heads():
    B, H, Hkv, world = 2, 12, 4, 3
    G = H // Hkv
    owner_q, owner_kv = {}, {}
    for r in range(world):
        sq, skv = sh.shard_rows(B, H, Hkv, world, r)
        for i in range(sq.start, sq.stop):
            owner_q[i] = r
        for u in range(skv.start, skv.stop):
            owner_kv[u] = r
    assert sorted(owner_q) == list(range(B * H)) and sorted(owner_kv) == list(range(B * Hkv))
    for row in range(B * H):  # flattened query head b*H + h reads kv head b*Hkv + h // G
        b, h = divmod(row, H)
        assert owner_q[row] == owner_kv[b * Hkv + h // G]


def test_bad_arguments():
    with pytest.raises(ValueError):
        sh.shard_units(1, 4, 2, 2)
    with pytest.raises(ValueError):
        sh.shard_rows(1, 6, 4, 2, 0)


def test_allreduce_without_process_group_is_identity():
    import torch
    t = torch.tensor([1.0, 2.0, 3.0])
    assert sh.allreduce_max_(t) is t and t.tolist() == [1.0, 2.0, 3.0]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, shapes, arrays, out_dir):
    import torch
    import torch.distributed as dist
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, H, Hkv, N, D = shapes
        q, k, v = arrays
        sq, skv = sh.shard_rows(B, H, Hkv, world, rank)
        qs = q.reshape(B * H, N, D)[sq]
        ks = k.reshape(B * Hkv, N, D)[skv]
        vs = v.reshape(B * Hkv, N, D)[skv]
        amax = torch.tensor([oracle.amax_bf16(t) if t.size else 0.0 for t in (qs, ks, vs)],
                            dtype=torch.float32)
        sh.allreduce_max_(amax)
        res = {"amax": amax.numpy()}
        for name, t, axis in (("q", qs, "d"), ("k", ks, "d"), ("v", vs, "t")):
            s_enc, _ = oracle.tensor_scale(float(res["amax"]["qkv".index(name)]))
            if axis == "d":
                res[name] = oracle.quantize_rows(t, s_enc, threads=1)
            else:
                res[name] = [oracle.quantize_tokens_T(t[u], s_enc) for u in range(t.shape[0])]
        np.save(os.path.join(out_dir, f"rank{rank}.npy"), np.array(res, dtype=object),
                allow_pickle=True)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,B,H,Hkv", [(2, 2, 4, 2), (3, 1, 6, 3), (3, 1, 4, 2)])
def test_gloo_sharded_quantisation_matches_whole(ora, syn, tmp_path, world, B, H, Hkv):
    """world ranks over gloo; (3, 1, 4, 2) leaves rank 2 without units: it still
    joins the all-reduce, with maxima of 0."""
    import torch.multiprocessing as mp
    N, D = 40, 64
    q = syn.normal_bf16(B * H * N * D, 11, 0).reshape(B, H, N, D)
    k = syn.normal_bf16(B * Hkv * N * D, 11, 1, scale=3.0).reshape(B, Hkv, N, D)
    v = syn.normal_bf16(B * Hkv * N * D, 11, 2, scale=0.5).reshape(B, Hkv, N, D)
    mp.start_processes(_rank_main, args=(world, _free_port(), (B, H, Hkv, N, D), (q, k, v),
                                         str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    whole_amax = [ora.amax_bf16(t) for t in (q, k, v)]
    s_enc = [ora.tensor_scale(a)[0] for a in whole_amax]
    wq = ora.quantize_rows(q.reshape(B * H, N, D), s_enc[0])
    wk = ora.quantize_rows(k.reshape(B * Hkv, N, D), s_enc[1])
    wv = [ora.quantize_tokens_T(v.reshape(B * Hkv, N, D)[u], s_enc[2]) for u in range(B * Hkv)]
    for r in range(world):
        res = np.load(tmp_path / f"rank{r}.npy", allow_pickle=True).item()
        assert list(res["amax"]) == whole_amax  # every rank holds the global maxima
        sq, skv = sh.shard_rows(B, H, Hkv, world, r)
        for got, want in zip(res["q"], wq):
            assert np.array_equal(got, want[sq])
        for got, want in zip(res["k"], wk):
            assert np.array_equal(got, want[skv])
        for u, (c, s) in zip(range(skv.start, skv.stop), res["v"]):
            assert np.array_equal(c, wv[u][0]) and np.array_equal(s, wv[u][1])


def _rank_smooth_main(rank, world, port, shapes, arrays, out_dir):
    """The smoothed sharded path's exchanges: the raw maxima (MAX), the
    per-head means on the global raw maxima's grid, the smoothed maxima (a
    second MAX), then the shard's smoothed codes and Q's correction."""
    import torch
    import torch.distributed as dist
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, H, Hkv, N, D = shapes
        q, k = arrays
        sq, skv = sh.shard_rows(B, H, Hkv, world, rank)
        qs, ks = q.reshape(B * H, N, D)[sq], k.reshape(B * Hkv, N, D)[skv]
        amax = torch.tensor([oracle.amax_bf16(t) if t.size else 0.0 for t in (qs, ks)],
                            dtype=torch.float32)
        sh.allreduce_max_(amax)
        qm = np.stack([oracle.channel_mean(x, float(amax[0])) for x in qs]) if qs.size else \
            np.zeros((0, D), np.float32)
        km = np.stack([oracle.channel_mean(x, float(amax[1])) for x in ks]) if ks.size else \
            np.zeros((0, D), np.float32)
        sm = torch.tensor([oracle.smoothed_amax(qs, qm) if qs.size else 0.0,
                           oracle.smoothed_amax(ks, km) if ks.size else 0.0], dtype=torch.float32)
        sh.allreduce_max_(sm)
        s_q, s_k = oracle.tensor_scale(float(sm[0]))[0], oracle.tensor_scale(float(sm[1]))[0]
        res = {"sm": sm.numpy(), "q": [], "k": [], "bias": []}
        for x, m in zip(qs, qm):
            res["q"].append(oracle.quantize_rows_smoothed(x, s_q, m))
        for x, m in zip(ks, km):
            res["k"].append(oracle.quantize_rows_smoothed(x, s_k, m))
        G = H // Hkv
        sqsk = float(s_q) * float(s_k)
        for i in range(sq.stop - sq.start):
            u = i // G  # the shard's key/value head of this query head
            res["bias"].append(oracle.score_bias(qm[i], ks[u], km[u]) * sqsk)
        np.save(os.path.join(out_dir, f"rank{rank}.npy"), np.array(res, dtype=object),
                allow_pickle=True)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,B,H,Hkv", [(2, 2, 4, 2), (3, 1, 4, 2)])
def test_gloo_smoothed_sharding_matches_whole(ora, syn, tmp_path, world, B, H, Hkv):
    """Smoothing sharded by head: every rank's smoothed codes and Q correction
    equal the whole tensors' slabs, with two MAX all-reduces (raw maxima for the
    means' grid, smoothed maxima for the tensor scales)."""
    import torch.multiprocessing as mp
    N, D = 40, 32
    rng = np.random.default_rng(5)
    q = syn.normal_bf16(B * H * N * D, 21, 0).reshape(B, H, N, D)
    k = syn.normal_bf16(B * Hkv * N * D, 21, 1, scale=2.0).reshape(B, Hkv, N, D)
    from _util import bf16_bits_to_f32, f32_to_bf16_bits
    q = f32_to_bf16_bits(bf16_bits_to_f32(q) + rng.normal(scale=4, size=(B, H, 1, D)).astype(np.float32))
    k = f32_to_bf16_bits(bf16_bits_to_f32(k) + rng.normal(scale=4, size=(B, Hkv, 1, D)).astype(np.float32))
    mp.start_processes(_rank_smooth_main, args=(world, _free_port(), (B, H, Hkv, N, D), (q, k),
                                                str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    qf, kf = q.reshape(B * H, N, D), k.reshape(B * Hkv, N, D)
    aq, ak = ora.amax_bf16(q), ora.amax_bf16(k)
    qm = np.stack([ora.channel_mean(x, aq) for x in qf])
    km = np.stack([ora.channel_mean(x, ak) for x in kf])
    sm = [ora.smoothed_amax(qf, qm), ora.smoothed_amax(kf, km)]
    s_q, s_k = ora.tensor_scale(sm[0])[0], ora.tensor_scale(sm[1])[0]
    sqsk = float(s_q) * float(s_k)
    G = H // Hkv
    for r in range(world):
        res = np.load(tmp_path / f"rank{r}.npy", allow_pickle=True).item()
        assert list(res["sm"]) == sm  # the second all-reduce: global smoothed maxima
        sq, skv = sh.shard_rows(B, H, Hkv, world, r)
        for i, got in zip(range(sq.start, sq.stop), res["q"]):
            want = ora.quantize_rows_smoothed(qf[i], s_q, qm[i])
            assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])
            delta = ora.score_bias(qm[i], kf[(i // H) * Hkv + (i % H) // G], km[(i // H) * Hkv + (i % H) // G])
            wb = delta * sqsk
            assert np.array_equal(res["bias"][i - sq.start], wb)
        for u, got in zip(range(skv.start, skv.stop), res["k"]):
            want = ora.quantize_rows_smoothed(kf[u], s_k, km[u])
            assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])
