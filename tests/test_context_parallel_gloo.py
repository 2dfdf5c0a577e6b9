"""Context-parallel decode plumbing on CPU: two gloo ranks each hold a token
shard, compute their part's output and softmax state, and all-gather them with
context_parallel.gather_parts; combining the gathered parts by log-sum-exp must
give softmax attention over the whole context.  The per-part attention and
the combination are written here in numpy (the CUDA kernels need a GPU; the
GPU test checks tq_merge_lse itself), so this covers the collective: order,
shapes and the exchanged state."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

LOG2E = 1.4426950408889634


def part_state(q, k, v, scale):
    """Normalized output and (max, sum) in log2 units of one context part (fp64)."""
    s = (k @ q.T) * scale * LOG2E            # [T][H]
    m = s.max(0)
    w = np.exp2(s - m)
    return (w.T @ v) / w.sum(0)[:, None], np.stack([m, w.sum(0)], 1)


def combine(outs, lses):
    M = lses[:, :, 0].max(0)
    w = np.exp2(lses[:, :, 0] - M) * lses[:, :, 1]
    return (w[:, :, None] * outs).sum(0) / w.sum(0)[:, None]


def _worker(rank, world, port, shards, q, scale, result):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from compressed_domain_attention_tq_b200.context_parallel import gather_parts
        k, v = shards[rank]
        o, st = part_state(q, k, v, scale)
        outs, lses = gather_parts(torch.from_numpy(o[None].astype(np.float32)),
                                  torch.from_numpy(st[None].astype(np.float32)))
        result[rank] = (outs.numpy(), lses.numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.timeout(120)
def test_gather_and_combine_two_ranks():
    rng = np.random.default_rng(3)
    H, d, T = 4, 16, 300
    q = rng.standard_normal((H, d))
    k = rng.standard_normal((T, d)) * 2
    v = rng.standard_normal((T, d))
    scale = 1 / np.sqrt(d)
    cut = 113  # uneven shards
    shards = [(k[:cut], v[:cut]), (k[cut:], v[cut:])]
    with mp.Manager() as mgr:
        result = mgr.dict()
        mp.spawn(_worker, args=(2, _free_port(), shards, q, scale, result), nprocs=2, join=True)
        res = dict(result)
    full, _ = part_state(q, k, v, scale)
    for rank in (0, 1):
        outs, lses = res[rank]
        assert outs.shape == (2, 1, H, d) and lses.shape == (2, 1, H, 2)
        for r in (0, 1):  # rank order preserved, state exchanged exactly
            o_r, st_r = part_state(q, *shards[r], scale)
            np.testing.assert_allclose(outs[r, 0], o_r, rtol=1e-6, atol=1e-6)
            np.testing.assert_allclose(lses[r, 0], st_r, rtol=1e-6, atol=1e-6)
        got = combine(outs[:, 0].astype(np.float64), lses[:, 0].astype(np.float64))
        np.testing.assert_allclose(got, full, rtol=1e-5, atol=1e-6)


def test_shard_range_tiles_the_context():
    from compressed_domain_attention_tq_b200.context_parallel import shard_range
    for total in (1, 2, 7, 300, 131072, 1048576, 1048577):
        for world in (1, 2, 3, 4, 8):
            if total < world:
                with pytest.raises(ValueError):
                    shard_range(total, world, 0)
                continue
            spans = [shard_range(total, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(spans[r][1] == spans[r + 1][0] for r in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
            assert sizes == sorted(sizes, reverse=True)   # the longer shards come first


def _shard_worker(rank, world, port, T, result):
    """One rank of the bench's context-parallel split on CPU: its shard from
    make_kv_shard, numpy attention over it, the parts gathered."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from compressed_domain_attention_tq_b200 import workloads as wl
        from compressed_domain_attention_tq_b200.context_parallel import gather_parts, shard_range
        w = wl.shrink(wl.WORKLOADS["llama70b_gqa_128k"], T, num_kv_heads=1)
        t0, t1 = shard_range(T, world, rank)
        k, v = wl.make_kv_shard(w, 5, t0, t1)
        q = wl.make_query(w, 5)[0].double().numpy()          # [G][d] of kv head 0
        k = k[0, 0].double().numpy()
        v = v[0, 0].double().numpy()
        o, st = part_state(q, k, v, w.attn_scales[0])
        outs, lses = gather_parts(torch.from_numpy(o[None].astype(np.float32)),
                                  torch.from_numpy(st[None].astype(np.float32)))
        result[rank] = ((t0, t1), outs.numpy(), lses.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_bench_shard_split_and_gather_two_ranks():
    """The split bench.py --mode context-parallel uses, on two gloo ranks: the
    shards tile the context, and merging the gathered parts gives attention
    over the whole context (the concatenation of every rank's shard)."""
    from compressed_domain_attention_tq_b200 import workloads as wl
    from compressed_domain_attention_tq_b200.context_parallel import shard_range
    T, world = 301, 2
    with mp.Manager() as mgr:
        result = mgr.dict()
        mp.spawn(_shard_worker, args=(world, _free_port(), T, result), nprocs=world, join=True)
        res = dict(result)
    assert [res[r][0] for r in range(world)] == [shard_range(T, world, r) for r in range(world)]
    w = wl.shrink(wl.WORKLOADS["llama70b_gqa_128k"], T, num_kv_heads=1)
    ks, vs = zip(*(wl.make_kv_shard(w, 5, *shard_range(T, world, r)) for r in range(world)))
    k = torch.cat(ks, 2)[0, 0].double().numpy()
    v = torch.cat(vs, 2)[0, 0].double().numpy()
    q = wl.make_query(w, 5)[0].double().numpy()
    full, _ = part_state(q, k, v, w.attn_scales[0])
    for r in range(world):
        _, outs, lses = res[r]
        assert outs.shape == (world, 1) + full.shape and lses.shape == (world, 1, full.shape[0], 2)
        got = combine(outs[:, 0].astype(np.float64), lses[:, 0].astype(np.float64))
        np.testing.assert_allclose(got, full, rtol=1e-5, atol=1e-6)
