"""Context-parallel decode emulated on one GPU: each sequence's cache rows are
split into contiguous shards (separate caches, as the ranks would hold them),
each shard is decoded with tq_sdpa_int4_decode_lse, and tq_merge_lse combines
the parts.  The result must match the decode of the whole cache (same
arithmetic up to summation order) and pass the oracle gates."""
import math

import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_tq_b200 import _lib
from conftest import require_cuda
from helpers import THREADS, check_attention, oracle_cache, to_oracle, upload_cache

pytestmark = pytest.mark.gpu


def shard_cache(cache, starts, ends):
    """Rows [starts[b], ends[b]) of every kv head of sequence b, moved to rows 0.."""
    kp, ks, vp, vs = cache
    B, H = kp.shape[:2]
    cap = int(max(e - s for s, e in zip(starts, ends)))
    out = [np.zeros((B, H, cap) + a.shape[3:], a.dtype) for a in (kp, ks, vp, vs)]
    for b in range(B):
        n = ends[b] - starts[b]
        for src, dst in zip((kp, ks, vp, vs), out):
            dst[b, :, :n] = src[b, :, starts[b]:ends[b]]
    return out


@pytest.mark.parametrize("d,G", [(128, 8), (128, 2), (256, 2), (128, 16)])
def test_context_parallel_matches_whole_context(d, G):
    require_cuda()
    B, Hkv = 2, 2
    ctx = [2900, 1500]
    g = torch.Generator().manual_seed(d + G)
    T = max(ctx)
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16)
    signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)
    cache = oracle_cache(k, v, signs)
    scale = 1 / math.sqrt(d)
    dev = "cuda"
    qd, sg = q.to(dev), signs.to(dev)
    Hq = Hkv * G

    ws = torch.empty(_lib.decode_workspace_bytes(B, Hq, Hkv, d, T), dtype=torch.uint8, device=dev)
    full = torch.empty(B, Hq, d, device=dev)
    _lib.sdpa_int4_decode(qd, *upload_cache(cache), torch.tensor(ctx, dtype=torch.int32, device=dev),
                          T, sg, scale, full, ws)

    cuts = [(0, 700, 2100, 2900), (0, 1, 900, 1500)]  # per sequence; a one-token shard
    outs, lses = [], []
    for r in range(3):
        starts = [c[r] for c in cuts]
        ends = [c[r + 1] for c in cuts]
        n = [e - s for s, e in zip(starts, ends)]
        sc = upload_cache(shard_cache(cache, starts, ends))
        mx = max(n)
        ws_r = torch.empty(_lib.decode_workspace_bytes(B, Hq, Hkv, d, mx), dtype=torch.uint8, device=dev)
        o = torch.empty(B, Hq, d, device=dev)
        l = torch.empty(B, Hq, 2, device=dev)
        _lib.sdpa_int4_decode_lse(qd, *sc, torch.tensor(n, dtype=torch.int32, device=dev), mx, sg,
                                  scale, o, l, ws_r)
        outs.append(o)
        lses.append(l)
    merged = torch.empty(B, Hq, d, device=dev)
    _lib.merge_lse(torch.stack(outs).contiguous(), torch.stack(lses).contiguous(), merged)
    torch.cuda.synchronize()
    a, b = merged.cpu().numpy(), full.cpu().numpy()
    assert np.linalg.norm(a - b) <= 2e-6 * np.linalg.norm(b)
    want = oracle.sdpa_int4_decode(to_oracle(q), cache, ctx, signs.numpy(), scale, Hkv, threads=THREADS)
    check_attention(a, want, cache, ctx, G, f"context parallel d={d} G={G}")


def test_lse_of_one_part_reproduces_plain_decode():
    """The lse call's output equals the plain decode's, and merging a single
    part is the identity."""
    require_cuda()
    B, Hkv, G, d, T = 1, 2, 8, 128, 1000
    g = torch.Generator().manual_seed(7)
    k = torch.randn(B, Hkv, T, d, generator=g)
    v = torch.randn(B, Hkv, T, d, generator=g)
    q = torch.randn(B, Hkv * G, d, generator=g)
    cache = upload_cache(oracle_cache(k, v, None))
    dev = "cuda"
    ctx = torch.tensor([T], dtype=torch.int32, device=dev)
    ws = torch.empty(_lib.decode_workspace_bytes(B, Hkv * G, Hkv, d, T), dtype=torch.uint8, device=dev)
    o1 = torch.empty(B, Hkv * G, d, device=dev)
    o2 = torch.empty_like(o1)
    l = torch.empty(B, Hkv * G, 2, device=dev)
    _lib.sdpa_int4_decode(q.to(dev), *cache, ctx, T, None, 0.1, o1, ws)
    _lib.sdpa_int4_decode_lse(q.to(dev), *cache, ctx, T, None, 0.1, o2, l, ws)
    m = torch.empty_like(o1)
    _lib.merge_lse(o2[None].contiguous(), l[None].contiguous(), m)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert torch.allclose(m, o2, rtol=1e-6, atol=1e-7)
    assert bool((l[..., 1] >= 1.0).all())  # the sum includes the maximum's own weight 1


def _srft_and_cb_caches(B, Hkv, d, T, g):
    """Host inputs plus an SRFT and a 3-bit codebook cache of them (oracle-quantized)."""
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16)
    return k, v


@pytest.mark.parametrize("kind", ["srft", "cb3"])
def test_context_parallel_srft_and_codebook_caches(kind):
    """context_parallel's per-shard decode (decode_lse of each cache kind) merged with
    tq_merge_lse equals the whole-cache decode of the same kind."""
    require_cuda()
    from compressed_domain_attention_tq_b200 import CodebookKVCache, Int4KVCache
    B, Hkv, G, d = 1, 2, 4, (96 if kind == "srft" else 128)
    T = 2500
    g = torch.Generator().manual_seed(77 if kind == "srft" else 78)
    k, v = _srft_and_cb_caches(B, Hkv, d, T, g)
    q = torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16).cuda()
    signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)
    lam = torch.exp2(torch.empty(2, d).uniform_(-0.25, 0.25, generator=g))

    def make(cap):
        if kind == "srft":
            return Int4KVCache(B, Hkv, d, cap, signs=signs, rotation="srft", lambda_k=lam[0],
                               lambda_v=lam[1])
        return CodebookKVCache(B, Hkv, d, cap, 3, signs=signs)

    zero = torch.zeros(B, dtype=torch.int32, device="cuda")
    whole = make(T)
    whole.append(k.cuda(), v.cuda(), zero)
    full = whole.decode(q, torch.tensor([T], dtype=torch.int32, device="cuda"), T, 0.1)
    outs, lses = [], []
    for s0, s1 in ((0, 1000), (1000, 1001), (1001, T)):
        part = make(s1 - s0)
        part.append(k[:, :, s0:s1].contiguous().cuda(), v[:, :, s0:s1].contiguous().cuda(), zero)
        o = torch.empty(B, Hkv * G, d, device="cuda")
        l = torch.empty(B, Hkv * G, 2, device="cuda")
        part.decode_lse(q, torch.tensor([s1 - s0], dtype=torch.int32, device="cuda"), s1 - s0, 0.1, o, l)
        outs.append(o)
        lses.append(l)
    merged = torch.empty_like(full)
    _lib.merge_lse(torch.stack(outs).contiguous(), torch.stack(lses).contiguous(), merged)
    torch.cuda.synchronize()
    a, b = merged.cpu().numpy(), full.cpu().numpy()
    assert np.linalg.norm(a - b) <= 2e-6 * np.linalg.norm(b), np.linalg.norm(a - b) / np.linalg.norm(b)
