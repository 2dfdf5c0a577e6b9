"""tq_sdpa_int4_decode_append (one decode step in one call) against the two-call
step it replaces: tq_quantize_append of the new token at row T_b - 1, then
tq_sdpa_int4_decode.  The whole cache and the output must be bit-identical
(same quantizer arithmetic, same decode kernels and plan), and the two-call
step itself is checked against the oracle by the other GPU tests.  Covers the
tensor-core decodes (the kernel quantizes the new tokens itself), the CUDA-core
decode (small append launch first), clamped lengths and a one-token context."""
import math

import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_tq_b200 import _lib
from conftest import require_cuda
from helpers import THREADS, check_attention, oracle_cache, to_oracle, upload_cache

pytestmark = pytest.mark.gpu


def step_pair(B, Hkv, G, d, ctx, max_ctx, dtype=torch.bfloat16, seed=0, rot=True):
    cap = max_ctx + 3
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, Hkv, cap, d, generator=g).to(dtype)
    v = torch.randn(B, Hkv, cap, d, generator=g).to(dtype)
    q = torch.randn(B, Hkv * G, d, generator=g).to(dtype)
    k_new = torch.randn(B, Hkv, 1, d, generator=g).to(dtype)
    v_new = torch.randn(B, Hkv, 1, d, generator=g).to(dtype)
    signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8) if rot else None
    base = upload_cache(oracle_cache(k, v, signs))  # every row filled; row T_b - 1 gets replaced
    dev = "cuda"
    ctx_d = torch.tensor(ctx, dtype=torch.int32, device=dev)
    sg = None if signs is None else signs.to(dev)
    scale = 1 / math.sqrt(d)
    ws = torch.empty(_lib.decode_workspace_bytes(B, Hkv * G, Hkv, d, max_ctx), dtype=torch.uint8, device=dev)
    # two calls
    c2 = [t.clone() for t in base]
    pos = (torch.clamp(ctx_d, 1, max_ctx) - 1).to(torch.int32)
    _lib.quantize_append(k_new.to(dev), v_new.to(dev), pos, sg, *c2)
    out2 = torch.empty(B, Hkv * G, d, device=dev)
    _lib.sdpa_int4_decode(q.to(dev), *c2, ctx_d, max_ctx, sg, scale, out2, ws)
    torch.cuda.synchronize()
    flags2 = ws[: 4 * B].view(torch.int32).cpu().numpy().copy()
    # one call
    c1 = [t.clone() for t in base]
    out1 = torch.empty(B, Hkv * G, d, device=dev)
    _lib.sdpa_int4_decode_append(q.to(dev), k_new.to(dev), v_new.to(dev), *c1, ctx_d, max_ctx, sg,
                                 scale, out1, ws)
    torch.cuda.synchronize()
    flags1 = ws[: 4 * B].view(torch.int32).cpu().numpy().copy()
    for a, b in zip(c1, c2):
        assert torch.equal(a, b)
    assert not torch.equal(c1[0], base[0])  # the new rows were written
    np.testing.assert_array_equal(out1.cpu().numpy(), out2.cpu().numpy())
    np.testing.assert_array_equal(flags1, flags2)
    return c1, q, signs, out1, scale, flags1


@pytest.mark.parametrize("d,G", [(128, 8), (128, 5), (128, 2), (256, 2), (256, 4), (128, 16), (256, 8)])
def test_fused_step_matches_two_calls(d, G):
    require_cuda()
    step_pair(2, 2, G, d, [700, 1537], 1600, seed=d + G)


def test_fused_step_one_token_and_clamped():
    require_cuda()
    c, q, signs, out, scale, flags = step_pair(3, 2, 8, 128, [1, 40, 999], 64, seed=5)
    assert list(flags) == [0, 0, 1]


def test_fused_step_vs_oracle_fp32_inputs():
    """End to end against the oracle: fused step on fp32 inputs, rotation off
    (codes bit-exact), then the oracle decodes the written cache."""
    require_cuda()
    B, Hkv, G, d = 1, 2, 8, 128
    c, q, signs, out, scale, _ = step_pair(B, Hkv, G, d, [2049], 2100, dtype=torch.float32, seed=9,
                                           rot=False)
    cache = [t.cpu().numpy() for t in c]
    want = oracle.sdpa_int4_decode(to_oracle(q), cache, [2049], None, scale, Hkv, threads=THREADS)
    check_attention(out.cpu().numpy(), want, cache, [2049], G, "fused step")


def test_bound_decode_append_matches_plain_call_on_refilled_buffers():
    """Int4KVCache.bind_decode_append: the prepared step, called after the inputs are
    refilled in place, gives bit-identical caches and outputs to the plain call."""
    require_cuda()
    import torch
    from compressed_domain_attention_tq_b200 import Int4KVCache
    B, Hkv, G, d, T = 1, 2, 8, 128, 1200
    g = torch.Generator().manual_seed(91)
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).cuda()
    signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)
    caches = [Int4KVCache(B, Hkv, d, T + 4, signs=signs) for _ in range(2)]
    for c in caches:
        c.append(k, v, torch.zeros(B, dtype=torch.int32, device="cuda"))
    q = torch.empty(B, Hkv * G, d, dtype=torch.bfloat16, device="cuda")
    kn = torch.empty(B, Hkv, 1, d, dtype=torch.bfloat16, device="cuda")
    vn = torch.empty_like(kn)
    ctx = torch.empty(B, dtype=torch.int32, device="cuda")
    step, out_b = caches[0].bind_decode_append(q, kn, vn, ctx, T + 4, 0.09)
    for i in range(3):
        q.copy_(torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16))
        kn.copy_(torch.randn(B, Hkv, 1, d, generator=g).to(torch.bfloat16))
        vn.copy_(torch.randn(B, Hkv, 1, d, generator=g).to(torch.bfloat16))
        ctx.fill_(T + 1 + i)
        step()
        out_p = caches[1].decode_append(q, kn, vn, ctx, T + 4, 0.09)
        torch.cuda.synchronize()
        assert torch.equal(out_b, out_p)
    for a, b in zip((caches[0].k_packed, caches[0].k_scales, caches[0].v_packed, caches[0].v_scales),
                    (caches[1].k_packed, caches[1].k_scales, caches[1].v_packed, caches[1].v_scales)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("pinned", [True, False])
def test_host_buffer_step_matches_device_step(pinned):
    """tq_sdpa_int4_decode_append_host on host buffers writes the same cache rows
    and returns the same output (bit for bit) as the device-buffer step: pinned
    (mapped) buffers are read and written by the kernels directly, pageable ones
    are staged through the workspace by copies."""
    require_cuda()
    import torch
    from compressed_domain_attention_tq_b200 import Int4KVCache
    B, Hkv, G, d, T = 2, 2, 8, 128, 900
    g = torch.Generator().manual_seed(93)
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).cuda()
    signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)
    caches = [Int4KVCache(B, Hkv, d, T + 2, signs=signs) for _ in range(2)]
    for c in caches:
        c.append(k, v, torch.zeros(B, dtype=torch.int32, device="cuda"))
    q = torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, Hkv, 1, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, Hkv, 1, d, generator=g).to(torch.bfloat16)
    ctx = torch.tensor([T + 1, T - 40], dtype=torch.int32, device="cuda")
    if pinned:
        hq, hk, hv = q.pin_memory(), kn.pin_memory(), vn.pin_memory()
        hout = torch.empty(B, Hkv * G, d, dtype=torch.float32).pin_memory()
    else:
        hq, hk, hv = q.clone(), kn.clone(), vn.clone()
        hout = torch.empty(B, Hkv * G, d, dtype=torch.float32)
    step = caches[0].bind_decode_append_host(hq, hk, hv, ctx, T + 2, hout, 0.1)
    step()
    out_d = caches[1].decode_append(q.cuda(), kn.cuda(), vn.cuda(), ctx, T + 2, 0.1)
    torch.cuda.synchronize()
    assert torch.equal(hout, out_d.cpu())
    for a, b in zip((caches[0].k_packed, caches[0].k_scales, caches[0].v_packed, caches[0].v_scales),
                    (caches[1].k_packed, caches[1].k_scales, caches[1].v_packed, caches[1].v_scales)):
        assert torch.equal(a, b)


def test_graphed_host_buffer_step_matches_direct_calls():
    """bind_decode_append_host(graph=True): the step captured once into a CUDA
    graph and replayed gives, step after step with new host inputs, the same
    output and cache rows (bit for bit) as the direct host-buffer call."""
    require_cuda()
    from compressed_domain_attention_tq_b200 import Int4KVCache
    B, Hkv, G, d, T = 2, 2, 8, 128, 700
    g = torch.Generator().manual_seed(94)
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).cuda()
    signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)
    caches = [Int4KVCache(B, Hkv, d, T + 4, signs=signs) for _ in range(2)]
    for c in caches:
        c.append(k, v, torch.zeros(B, dtype=torch.int32, device="cuda"))
    ctx = torch.tensor([T + 1, T - 60], dtype=torch.int32, device="cuda")
    hosts = [(torch.zeros(B, Hkv * G, d, dtype=torch.bfloat16).pin_memory(),
              torch.zeros(B, Hkv, 1, d, dtype=torch.bfloat16).pin_memory(),
              torch.zeros(B, Hkv, 1, d, dtype=torch.bfloat16).pin_memory(),
              torch.zeros(B, Hkv * G, d, dtype=torch.float32).pin_memory()) for _ in range(2)]
    steps = [caches[0].bind_decode_append_host(*hosts[0][:3], ctx, T + 4, hosts[0][3], 0.1,
                                               graph=True),
             caches[1].bind_decode_append_host(*hosts[1][:3], ctx, T + 4, hosts[1][3], 0.1)]
    for i in range(3):
        q = torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16)
        kn = torch.randn(B, Hkv, 1, d, generator=g).to(torch.bfloat16)
        vn = torch.randn(B, Hkv, 1, d, generator=g).to(torch.bfloat16)
        for (hq, hk, hv, _), step in zip(hosts, steps):
            hq.copy_(q)
            hk.copy_(kn)
            hv.copy_(vn)
            step()
            torch.cuda.synchronize()
        assert torch.equal(hosts[0][3], hosts[1][3]), f"step {i}"
    for a, b in zip((caches[0].k_packed, caches[0].k_scales, caches[0].v_packed, caches[0].v_scales),
                    (caches[1].k_packed, caches[1].k_scales, caches[1].v_packed, caches[1].v_scales)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("case", ["unaligned", "fp32"])
def test_host_buffer_step_fallbacks_and_dtypes(case):
    """tq_sdpa_int4_decode_append_host with pinned buffers that are not 16-byte
    aligned (the staged copies are used instead of the gather kernel) and with
    fp32 inputs (the gather kernel moves 4-byte elements): bit-identical to the
    device-buffer step."""
    require_cuda()
    from compressed_domain_attention_tq_b200 import Int4KVCache
    B, Hkv, G, d, T = 1, 2, 8, 128, 600
    dt = torch.float32 if case == "fp32" else torch.bfloat16
    g = torch.Generator().manual_seed(95)
    k = torch.randn(B, Hkv, T, d, generator=g).to(dt).cuda()
    v = torch.randn(B, Hkv, T, d, generator=g).to(dt).cuda()
    signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)
    caches = [Int4KVCache(B, Hkv, d, T + 2, signs=signs) for _ in range(2)]
    for c in caches:
        c.append(k, v, torch.zeros(B, dtype=torch.int32, device="cuda"))
    q = torch.randn(B, Hkv * G, d, generator=g).to(dt)
    kn = torch.randn(B, Hkv, 1, d, generator=g).to(dt)
    vn = torch.randn(B, Hkv, 1, d, generator=g).to(dt)
    ctx = torch.tensor([T + 1], dtype=torch.int32, device="cuda")

    def pinned_like(t, shift):
        # a pinned buffer whose data starts `shift` elements into its allocation
        buf = torch.empty(t.numel() + shift, dtype=t.dtype).pin_memory()
        view = buf[shift:].view(t.shape)
        view.copy_(t)
        return view

    shift = 1 if case == "unaligned" else 0
    hq, hk, hv = pinned_like(q, shift), pinned_like(kn, shift), pinned_like(vn, shift)
    hout = pinned_like(torch.zeros(B, Hkv * G, d), shift)
    step = caches[0].bind_decode_append_host(hq, hk, hv, ctx, T + 2, hout, 0.1)
    step()
    out_d = caches[1].decode_append(q.cuda(), kn.cuda(), vn.cuda(), ctx, T + 2, 0.1)
    torch.cuda.synchronize()
    assert torch.equal(hout, out_d.cpu())
    for a, b in zip((caches[0].k_packed, caches[0].k_scales, caches[0].v_packed, caches[0].v_scales),
                    (caches[1].k_packed, caches[1].k_scales, caches[1].v_packed, caches[1].v_scales)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("kind,G,d", [("srft", 8, 128), ("cb2", 8, 128), ("cb3", 8, 128),
                                       ("srft", 4, 96), ("cb2", 2, 128)])
def test_host_buffer_step_srft_and_codebook(kind, G, d):
    """The host-buffer step of the SRFT and codebook caches (pinned buffers:
    gather kernel and direct output writes; then graph replay) equals their
    device-buffer step bit for bit, cache rows included, on the tensor-core
    decode and (d = 96, two heads per kv head) on the CUDA-core decode."""
    require_cuda()
    from compressed_domain_attention_tq_b200 import CodebookKVCache, Int4KVCache
    B, Hkv, T = 2, 2, 500
    g = torch.Generator().manual_seed(96)
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).cuda()
    signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)

    def make():
        if kind == "srft":
            lk = torch.rand(d, generator=g) * 0.5 + 0.75
            lv = torch.rand(d, generator=g) * 0.5 + 0.75
            return Int4KVCache(B, Hkv, d, T + 2, signs=signs, rotation="srft",
                               lambda_k=lk, lambda_v=lv)
        return CodebookKVCache(B, Hkv, d, T + 2, int(kind[2]), signs=signs)

    gstate = g.get_state()
    caches = []
    for _ in range(3):
        g.set_state(gstate)
        c = make()
        c.append(k, v, torch.zeros(B, dtype=torch.int32, device="cuda"))
        caches.append(c)
    q = torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, Hkv, 1, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, Hkv, 1, d, generator=g).to(torch.bfloat16)
    ctx = torch.tensor([T + 1, T - 30], dtype=torch.int32, device="cuda")
    outs = []
    for i, graph in enumerate((False, True)):
        hq, hk, hv = q.pin_memory(), kn.pin_memory(), vn.pin_memory()
        hout = torch.zeros(B, Hkv * G, d, dtype=torch.float32).pin_memory()
        step = caches[i].bind_decode_append_host(hq, hk, hv, ctx, T + 2, hout, 0.1, graph=graph)
        step()
        torch.cuda.synchronize()
        outs.append(hout.clone())
    out_d = caches[2].decode_append(q.cuda(), kn.cuda(), vn.cuda(), ctx, T + 2, 0.1)
    torch.cuda.synchronize()
    for o in outs:
        assert torch.equal(o, out_d.cpu())
    for c in caches[:2]:
        for a, b in zip((c.k_packed, c.k_scales, c.v_packed, c.v_scales),
                        (caches[2].k_packed, caches[2].k_scales, caches[2].v_packed,
                         caches[2].v_scales)):
            assert torch.equal(a, b)
