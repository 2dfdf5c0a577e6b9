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
