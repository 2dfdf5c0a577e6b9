"""GPU uniform low-bit variant (Open-TQ-Metal forum summary, future work:
int2; the int4 quantizer at 2 or 3 bits: s = fl32(amax / m), codes
clamp(rne(y / s), -m, m) stored as indices c + m in the codebook layout) vs
the oracle on the same inputs.

Bars as for the codebook variant: rotation off -> packed indices and scales
bit-identical; rotation on -> at most 0.01% of indices differ, each by one,
scales within 4 ulp; decode over the same packed cache (codebook decode with
the integer levels u - m) -> per head relative L2 <= 1e-4 and max abs <=
1e-3 * max|v_hat|.  At four bits the indices minus 7 must be the int4 codes
of tq_quantize_append bit for bit."""
import math

import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_tq_b200 import UniformKVCache, _lib
from conftest import require_cuda
from helpers import THREADS, to_oracle, upload_cache
from test_gpu_codebook import cb_decode, check_attention_cb, compare_cb
from test_gpu_decode import make_case, signs_for
from test_gpu_quantize import inputs, run_gpu

pytestmark = pytest.mark.gpu


def gpu_uniform_quantize(k, v, pos, signs, bits, cap):
    B, H, n, d = k.shape
    rb = d * bits // 8
    kp = torch.zeros(B, H, cap, rb, dtype=torch.uint8, device="cuda")
    vp = torch.zeros_like(kp)
    ks = torch.zeros(B, H, cap, d // 32, dtype=torch.float32, device="cuda")
    vs = torch.zeros_like(ks)
    _lib.quantize_append_uniform(k.cuda(), v.cuda(), torch.tensor(pos, dtype=torch.int32, device="cuda"),
                                 None if signs is None else signs.cuda(), bits, kp, ks, vp, vs)
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (kp, ks, vp, vs)]


def oracle_uniform_cache(k, v, signs, bits, cap=None, pos=None):
    B, H, n, d = k.shape
    cache = oracle.empty_cb_cache(B, H, n if cap is None else cap, d, bits)
    p = np.zeros(B, np.int32) if pos is None else np.asarray(pos, np.int32)
    oracle.quantize_append_uniform(to_oracle(k), to_oracle(v), p, None if signs is None else signs.numpy(),
                                   bits, cache, threads=THREADS)
    return cache


def test_uniform_levels_match_the_oracle():
    for bits in (2, 3, 4):
        np.testing.assert_array_equal(_lib.uniform_levels(bits).numpy(), oracle.uniform_levels(bits))


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rot", [False, True])
def test_uniform_quantize_matches_oracle(bits, d, dtype, rot):
    require_cuda()
    seed = bits * 100 + d + (1 if rot else 0) + 7
    B, H, n = 2, 3, 257
    k, v = inputs(B, H, n, d, dtype, seed)
    signs = signs_for(d, seed + 1) if rot else None
    got = gpu_uniform_quantize(k, v, [1, 4], signs, bits, n + 5)
    want = oracle_uniform_cache(k, v, signs, bits, n + 5, [1, 4])
    compare_cb(got, want, d, bits, rot, f"int{bits} d={d} {dtype} rot={rot}")


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("rot", [False, True])
def test_uniform_four_bits_gives_the_int4_codes(d, rot):
    """The uniform quantizer at four bits and the int4 quantizer (different
    kernels, different layouts) write the same codes and scales."""
    require_cuda()
    B, H, n = 1, 2, 300
    k, v = inputs(B, H, n, d, torch.float32, 40 + d)
    signs = signs_for(d, 41) if rot else None
    uni = gpu_uniform_quantize(k, v, [0], signs, 4, n)
    i4 = run_gpu(k, v, [0], signs, n)
    for (pu, su), (p4, s4) in (((uni[0], uni[1]), (i4[0], i4[1])), ((uni[2], uni[3]), (i4[2], i4[3]))):
        iu = oracle.cb_unpack(pu.reshape(-1, pu.shape[-1]), d, 4).astype(np.int64) - 7
        c4 = oracle.unpack(p4.reshape(-1, p4.shape[-1]), d).astype(np.int64)
        np.testing.assert_array_equal(iu, c4)
        np.testing.assert_array_equal(su.view(np.uint32), s4.view(np.uint32))


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("B,Hkv,G,d,ctx", [
    (1, 2, 8, 128, [1500]),      # tensor-core decode
    (2, 2, 6, 128, [3001, 517]),  # tensor-core decode, ragged, padding heads
    (2, 2, 1, 128, [777, 4100]),  # CUDA-core decode
    (1, 2, 4, 256, [1000]),
])
def test_uniform_decode_matches_oracle(bits, B, Hkv, G, d, ctx):
    require_cuda()
    seed = bits * 10 + G + d + 3
    T = max(ctx)
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, seed, heavy=True)
    signs = signs_for(d, seed + 1)
    lv = _lib.uniform_levels(bits)
    cache = oracle_uniform_cache(k, v, signs, bits)
    for scale in (1 / math.sqrt(d), 1.0):
        got = cb_decode(upload_cache(cache), q, ctx, T, signs, bits, lv, scale, Hkv)
        want = oracle.sdpa_cb_decode(to_oracle(q), cache, ctx, signs.numpy(), bits, lv.numpy(), scale,
                                     Hkv, threads=THREADS)
        check_attention_cb(got, want, cache, ctx, G, bits, lv,
                           f"int{bits} B={B} Hkv={Hkv} G={G} d={d} scale={scale:.3g}")


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("G", [6, 1])
def test_uniform_fused_step_equals_two_calls(bits, G):
    """UniformKVCache.decode_append (G = 6: the tensor-core decode quantizes the
    new token itself; G = 1: an append launch, then the CUDA-core decode) is
    bit-identical to append-then-decode, on a ragged batch with stale rows to
    overwrite, and the oracle agrees on the resulting cache."""
    require_cuda()
    B, Hkv, d, ctx = 2, 2, 128, [1800, 333]
    T = max(ctx)
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 600 + bits + G)
    signs = signs_for(d, 601 + bits)
    ct = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    kn = torch.stack([k[b, :, ctx[b] - 1] for b in range(B)])[:, :, None].contiguous().cuda()
    vn = torch.stack([v[b, :, ctx[b] - 1] for b in range(B)])[:, :, None].contiguous().cuda()
    outs, caches = [], []
    for fused in (True, False):
        c = UniformKVCache(B, Hkv, d, T, bits, signs=signs)
        c.append(k.cuda(), v.cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"))
        for b in range(B):
            c.k_packed[b, :, ctx[b] - 1:].fill_(0x5A)
            c.v_packed[b, :, ctx[b] - 1:].fill_(0xA5)
        if fused:
            out = c.decode_append(q.cuda(), kn, vn, ct, T)
        else:
            c.append(kn, vn, ct - 1)
            out = c.decode(q.cuda(), ct, T)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy())
        caches.append([t.cpu().numpy() for t in (c.k_packed, c.k_scales, c.v_packed, c.v_scales)])
    np.testing.assert_array_equal(outs[0], outs[1])
    for b in range(B):
        for a0, a1 in zip(caches[0], caches[1]):
            np.testing.assert_array_equal(a0[b, :, :ctx[b]], a1[b, :, :ctx[b]])
    # the appended rows are the uniform quantizer's (not the codebook rule's)
    for b in range(B):
        ref = oracle_uniform_cache(kn[b:b + 1].cpu(), vn[b:b + 1].cpu(), signs, bits)
        for a, r in ((caches[0][0], ref[0]), (caches[0][2], ref[2])):
            ia = oracle.cb_unpack(a[b, :, ctx[b] - 1], d, bits).astype(np.int64)
            ir = oracle.cb_unpack(r[0, :, 0], d, bits).astype(np.int64)
            assert np.abs(ia - ir).max() <= 1 and (ia != ir).mean() <= 0.01
    lv = c.levels.cpu()
    want = oracle.sdpa_cb_decode(to_oracle(q), caches[0], ctx, signs.numpy(), bits, lv.numpy(),
                                 1 / math.sqrt(d), Hkv, threads=THREADS)
    check_attention_cb(outs[0], want, caches[0], ctx, G, bits, lv, f"int{bits} G={G} fused step")


def test_uniform_host_step_matches_device_step():
    """The host-buffer step (pinned q, k_new, v_new and output) equals the device step."""
    require_cuda()
    B, Hkv, G, d, T, bits = 1, 2, 8, 128, 2000, 2
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 77)
    signs = signs_for(d, 78)
    ctx = torch.tensor([T], dtype=torch.int32, device="cuda")
    kn, vn = k[:, :, T - 1:].contiguous(), v[:, :, T - 1:].contiguous()
    outs = []
    for host in (False, True):
        c = UniformKVCache(B, Hkv, d, T, bits, signs=signs)
        c.append(k[:, :, :T - 1].cuda(), v[:, :, :T - 1].cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"))
        if host:
            h_q, h_k, h_v = (t.pin_memory() for t in (q, kn, vn))
            h_out = torch.empty(B, Hkv * G, d, dtype=torch.float32).pin_memory()
            step = c.bind_decode_append_host(h_q, h_k, h_v, ctx, T, h_out)
            step()
            torch.cuda.synchronize()
            outs.append(h_out.numpy().copy())
        else:
            out = c.decode_append(q.cuda(), kn.cuda(), vn.cuda(), ctx, T)
            torch.cuda.synchronize()
            outs.append(out.cpu().numpy())
    np.testing.assert_array_equal(outs[0], outs[1])
