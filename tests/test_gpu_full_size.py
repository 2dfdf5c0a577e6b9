"""Parity at the full workload sizes, in the launch configuration bench.py times.

Each workload is generated on the GPU from its seed, quantized by the CUDA path
(one bulk tq_quantize_append call, then one single-token append as in a decode
step) and decoded over the whole context.  The oracle checks sampled outputs it
can compute one by one:
  - codes and scales of sampled token rows, from those rows' exact inputs;
  - the decode of sampled kv heads (all their query heads), over that head's
    GPU-written packed cache.
Gates as in the other GPU tests: rotation on -> at most 0.01% of codes differ,
each by 1, scales within 4 ulp (32 ulp with the SRFT rotation, whose fp32 FFT
error is relative to the whole row); attention rel-L2 <= 1e-4 and max-abs <=
1e-3 * max|v_hat| per (sequence, query head).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_tq_b200 import CodebookKVCache, Int4KVCache, UniformKVCache
from compressed_domain_attention_tq_b200 import workloads as wl
from conftest import require_cuda
from helpers import THREADS, check_attention, to_oracle

pytestmark = pytest.mark.gpu


def _run_workload(name, attn_scale=None, seed=0, sample_rows=64, sample_heads=2):
    require_cuda()
    dev = torch.device("cuda", 0)
    w = wl.WORKLOADS[name]
    B, Hq, Hkv, d = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim
    G = Hq // Hkv
    signs = wl.make_signs(d, seed) if w.rotation else None
    srft = w.rotation and w.rotation_kind == "srft"
    lk, lv = wl.make_lambdas(w, seed)
    ctx = wl.make_context_lengths(w, seed)
    cache = Int4KVCache(B, Hkv, d, w.capacity, dev, signs,
                        rotation="srft" if srft else "hadamard", lambda_k=lk, lambda_v=lv)
    k_all, v_all = wl.make_kv(w, seed, device=dev, tokens=w.capacity - 1)
    cache.append(k_all, v_all, torch.zeros(B, dtype=torch.int32, device=dev))
    k_new, v_new = wl.make_kv(w, seed, device=dev, tokens=1, token_offset=10_000_019)
    cache.append(k_new, v_new, ctx.to(dev))
    q = wl.make_query(w, seed, device=dev)
    scale = w.attn_scales[0] if attn_scale is None else attn_scale
    T = ctx + 1
    out = cache.decode(q, T.to(dev), int(T.max()), scale)
    torch.cuda.synchronize()
    gen = np.random.default_rng(seed + 7)
    sg = None if signs is None else signs.numpy()
    lk_h, lv_h = (None, None) if lk is None else (lk.numpy(), lv.numpy())
    scale_ulp = 32 if srft else (4 if sg is not None else 0)

    # ---- quantizer: sampled rows of the bulk call
    n_diff = n_tot = 0
    for _ in range(sample_rows):
        b, h = int(gen.integers(B)), int(gen.integers(Hkv))
        t = int(gen.integers(int(ctx[b])))
        xk = k_all[b:b + 1, h:h + 1, t:t + 1].contiguous().cpu()
        xv = v_all[b:b + 1, h:h + 1, t:t + 1].contiguous().cpu()
        ref = oracle.empty_cache(1, 1, 1, d)
        if srft:
            oracle.quantize_append_srft(to_oracle(xk), to_oracle(xv), np.zeros(1, np.int32), sg,
                                        lk_h, lv_h, ref)
        else:
            oracle.quantize_append(to_oracle(xk), to_oracle(xv), np.zeros(1, np.int32), sg, ref)
        for packed, scales, rp, rs in ((cache.k_packed, cache.k_scales, ref[0], ref[1]),
                                       (cache.v_packed, cache.v_scales, ref[2], ref[3])):
            got_codes = oracle.unpack(packed[b, h, t:t + 1].cpu().numpy(), d).astype(np.int64)
            want_codes = oracle.unpack(rp[0, 0], d).astype(np.int64)
            diff = np.abs(got_codes - want_codes)
            assert diff.max() <= (1 if sg is not None else 0), f"{name} b={b} h={h} t={t}"
            n_diff += int((diff > 0).sum())
            n_tot += diff.size
            got_s = scales[b, h, t].cpu().numpy().view(np.int32).astype(np.int64)
            want_s = rs[0, 0, 0].view(np.int32).astype(np.int64)
            assert np.abs(got_s - want_s).max() <= scale_ulp
    assert n_diff <= max(1e-4 * n_tot, 1), f"{name}: {n_diff}/{n_tot} codes differ"

    # ---- decode: sampled (sequence, kv head) pairs over the GPU-written cache
    got = out.cpu().numpy()
    q_host = to_oracle(q.cpu())
    for _ in range(sample_heads):
        b, h = int(gen.integers(B)), int(gen.integers(Hkv))
        Tb = int(T[b])
        sub = [np.ascontiguousarray(a[b:b + 1, h:h + 1, :Tb].cpu().numpy())
               for a in (cache.k_packed, cache.k_scales, cache.v_packed, cache.v_scales)]
        qs = np.ascontiguousarray(q_host[b:b + 1, h * G:(h + 1) * G])
        if srft:
            want = oracle.sdpa_int4_decode_srft(qs, sub, [Tb], sg, lk_h, lv_h, scale, 1,
                                                threads=THREADS)
        else:
            want = oracle.sdpa_int4_decode(qs, sub, [Tb], sg, scale, 1, threads=THREADS)
        check_attention(got[b:b + 1, h * G:(h + 1) * G], want, sub, [Tb], G,
                        f"{name} b={b} kv head {h}")
    return n_diff, n_tot


def test_full_size_tiny_mha_4k():
    _run_workload("tiny_mha_4k", sample_rows=128, sample_heads=4)


def test_full_size_llama70b_gqa_32k():
    _run_workload("llama70b_gqa_32k")


def test_full_size_llama70b_gqa_128k():
    _run_workload("llama70b_gqa_128k")


def test_full_size_ragged_b16():
    _run_workload("ragged_b16", sample_heads=3)


@pytest.mark.parametrize("scale", [1.0, 1 / 16.0])
def test_full_size_wide_d256(scale):
    _run_workload("wide_d256", attn_scale=scale)


def test_full_size_llama70b_gqa_128k_srft():
    _run_workload("llama70b_gqa_128k_srft")


def test_full_size_mha32_d96_32k():
    _run_workload("mha32_d96_32k", sample_heads=3)


def _run_workload_cb(name, seed=0, sample_rows=32, sample_heads=2):
    """Codebook and uniform low-bit workloads: bulk append by the CUDA path, one appended token,
    decode over the whole context; sampled rows' indices and scales and
    sampled kv heads' outputs against the oracle (same gates as the codebook
    tests: at most 0.01% of indices differ, each by one level, scales within 4
    ulp; attention rel-L2 <= 1e-4, max-abs <= 1e-3 max|v_hat|)."""
    from test_gpu_codebook import check_attention_cb
    require_cuda()
    dev = torch.device("cuda", 0)
    w = wl.WORKLOADS[name]
    B, Hq, Hkv, d, bits = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.cb_bits
    G = Hq // Hkv
    signs = wl.make_signs(d, seed) if w.rotation else None
    ctx = wl.make_context_lengths(w, seed)
    cache = (UniformKVCache(B, Hkv, d, w.capacity, bits, dev, signs) if w.cb_uniform
             else CodebookKVCache(B, Hkv, d, w.capacity, bits, dev, signs))
    k_all, v_all = wl.make_kv(w, seed, device=dev, tokens=w.capacity - 1)
    cache.append(k_all, v_all, torch.zeros(B, dtype=torch.int32, device=dev))
    k_new, v_new = wl.make_kv(w, seed, device=dev, tokens=1, token_offset=10_000_019)
    cache.append(k_new, v_new, ctx.to(dev))
    q = wl.make_query(w, seed, device=dev)
    scale = w.attn_scales[0]
    T = ctx + 1
    out = cache.decode(q, T.to(dev), int(T.max()), scale)
    torch.cuda.synchronize()
    gen = np.random.default_rng(seed + 7)
    sg = None if signs is None else signs.numpy()
    lv = cache.levels.cpu()

    n_diff = n_tot = 0
    for _ in range(sample_rows):
        b, h = int(gen.integers(B)), int(gen.integers(Hkv))
        t = int(gen.integers(int(ctx[b])))
        xk = k_all[b:b + 1, h:h + 1, t:t + 1].contiguous().cpu()
        xv = v_all[b:b + 1, h:h + 1, t:t + 1].contiguous().cpu()
        ref = oracle.empty_cb_cache(1, 1, 1, d, bits)
        if w.cb_uniform:
            oracle.quantize_append_uniform(to_oracle(xk), to_oracle(xv), np.zeros(1, np.int32), sg,
                                           bits, ref)
        else:
            oracle.quantize_append_cb(to_oracle(xk), to_oracle(xv), np.zeros(1, np.int32), sg, bits,
                                      lv.numpy(), ref)
        for packed, scales, rp, rs in ((cache.k_packed, cache.k_scales, ref[0], ref[1]),
                                       (cache.v_packed, cache.v_scales, ref[2], ref[3])):
            got_i = oracle.cb_unpack(packed[b, h, t:t + 1].cpu().numpy(), d, bits).astype(np.int64)
            want_i = oracle.cb_unpack(rp[0, 0], d, bits).astype(np.int64)
            diff = np.abs(got_i - want_i)
            assert diff.max() <= (1 if sg is not None else 0), f"{name} b={b} h={h} t={t}"
            n_diff += int((diff > 0).sum())
            n_tot += diff.size
            got_s = scales[b, h, t].cpu().numpy().view(np.int32).astype(np.int64)
            want_s = rs[0, 0, 0].view(np.int32).astype(np.int64)
            assert np.abs(got_s - want_s).max() <= (4 if sg is not None else 0)
    assert n_diff <= max(1e-4 * n_tot, 1), f"{name}: {n_diff}/{n_tot} indices differ"

    got = out.cpu().numpy()
    q_host = to_oracle(q.cpu())
    for _ in range(sample_heads):
        b, h = int(gen.integers(B)), int(gen.integers(Hkv))
        Tb = int(T[b])
        sub = [np.ascontiguousarray(a[b:b + 1, h:h + 1, :Tb].cpu().numpy())
               for a in (cache.k_packed, cache.k_scales, cache.v_packed, cache.v_scales)]
        qs = np.ascontiguousarray(q_host[b:b + 1, h * G:(h + 1) * G])
        want = oracle.sdpa_cb_decode(qs, sub, [Tb], sg, bits, lv.numpy(), scale, 1, threads=THREADS)
        check_attention_cb(got[b:b + 1, h * G:(h + 1) * G], want, sub, [Tb], G, bits, lv,
                           f"{name} b={b} kv head {h}")


@pytest.mark.parametrize("name", ["llama70b_gqa_128k_cb2", "llama70b_gqa_128k_cb3",
                                  "llama70b_gqa_128k_int2", "llama70b_gqa_128k_int3"])
def test_full_size_codebook_128k(name):
    _run_workload_cb(name)
