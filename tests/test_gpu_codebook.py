"""GPU codebook variant (AdapTQ post: 2/3/4-bit Max-Lloyd indices, +-3 sigma
clipping, lookup-table scores) vs the oracle on the same inputs.

Bars: rotation off -> packed indices and scales bit-identical; rotation on ->
at most 0.01% of indices differ, each by one level, scales within 4 ulp;
decode over the same packed cache -> per head relative L2 <= 1e-4 and max
abs <= 1e-3 * max|v_hat|.  The codebook itself comes from libtq's generator
and is handed to both sides as an input."""
import math

import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_tq_b200 import CodebookKVCache, _lib
from conftest import require_cuda
from helpers import MAX_ABS_GATE, REL_L2_GATE, THREADS, to_oracle, upload_cache
from test_gpu_decode import make_case, signs_for
from test_gpu_quantize import inputs

pytestmark = pytest.mark.gpu


def levels_for(bits):
    return _lib.lloyd_max_gaussian(bits)


def gpu_cb_quantize(k, v, pos, signs, bits, levels, cap):
    B, H, n, d = k.shape
    rb = d * bits // 8
    kp = torch.zeros(B, H, cap, rb, dtype=torch.uint8, device="cuda")
    vp = torch.zeros_like(kp)
    ks = torch.zeros(B, H, cap, d // 32, dtype=torch.float32, device="cuda")
    vs = torch.zeros_like(ks)
    _lib.quantize_append_cb(k.cuda(), v.cuda(), torch.tensor(pos, dtype=torch.int32, device="cuda"),
                            None if signs is None else signs.cuda(), bits, levels.cuda(),
                            kp, ks, vp, vs)
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (kp, ks, vp, vs)]


def oracle_cb_cache(k, v, signs, bits, levels, cap=None, pos=None):
    B, H, n, d = k.shape
    cache = oracle.empty_cb_cache(B, H, n if cap is None else cap, d, bits)
    p = np.zeros(B, np.int32) if pos is None else np.asarray(pos, np.int32)
    oracle.quantize_append_cb(to_oracle(k), to_oracle(v), p, None if signs is None else signs.numpy(),
                              bits, levels.numpy(), cache, threads=THREADS)
    return cache


def compare_cb(got, want, d, bits, rot, label):
    n_diff = n_tot = 0
    for a, b in ((got[0], want[0]), (got[2], want[2])):
        ia = oracle.cb_unpack(a.reshape(-1, a.shape[-1]), d, bits).astype(np.int64)
        ib = oracle.cb_unpack(b.reshape(-1, b.shape[-1]), d, bits).astype(np.int64)
        diff = np.abs(ia - ib)
        if not rot:
            assert diff.max() == 0, label
        assert diff.max() <= 1, label
        n_diff += int((diff > 0).sum())
        n_tot += diff.size
    assert n_diff <= 1e-4 * n_tot, f"{label}: {n_diff}/{n_tot} indices differ"
    for a, b in ((got[1], want[1]), (got[3], want[3])):
        ulp = np.abs(a.view(np.int32).astype(np.int64) - b.view(np.int32).astype(np.int64))
        assert ulp.max() <= (4 if rot else 0), f"{label}: scale ulp {ulp.max()}"
    return n_diff, n_tot


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rot", [False, True])
def test_cb_quantize_matches_oracle(bits, d, dtype, rot):
    require_cuda()
    seed = bits * 100 + d + (1 if rot else 0)
    B, H, n = 2, 3, 257
    k, v = inputs(B, H, n, d, dtype, seed)
    signs = signs_for(d, seed + 1) if rot else None
    lv = levels_for(bits)
    got = gpu_cb_quantize(k, v, [1, 4], signs, bits, lv, n + 5)
    want = oracle_cb_cache(k, v, signs, bits, lv, n + 5, [1, 4])
    compare_cb(got, want, d, bits, rot, f"cb{bits} d={d} {dtype} rot={rot}")


def check_attention_cb(got, want, cache, ctx, G, bits, levels, label):
    _, _, vp, vs = cache
    d = want.shape[-1]
    c = levels.numpy().astype(np.float64)
    for b in range(want.shape[0]):
        for hk in range(want.shape[1] // G):
            T = int(ctx[b])
            idx = oracle.cb_unpack(vp[b, hk, :T], d, bits)
            vmax = float(np.max(np.abs(c[idx] * np.repeat(vs[b, hk, :T].astype(np.float64), 32, 1))))
            for h in range(hk * G, (hk + 1) * G):
                err = np.asarray(got[b, h], np.float64) - want[b, h]
                rel = np.linalg.norm(err) / max(np.linalg.norm(want[b, h]), 1e-300)
                ab = np.max(np.abs(err)) / max(vmax, 1e-300)
                assert rel <= REL_L2_GATE, f"{label} b={b} h={h}: rel-L2 {rel:.3e}"
                assert ab <= MAX_ABS_GATE, f"{label} b={b} h={h}: max-abs/max|v| {ab:.3e}"


def cb_decode(cache_dev, q, ctx, max_ctx, signs, bits, levels, scale, Hkv):
    B, Hq, d = q.shape
    ws = torch.empty(_lib.decode_cb_workspace_bytes(B, Hq, Hkv, d, max_ctx), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    kp, ks, vp, vs = cache_dev
    _lib.sdpa_cb_decode(q.cuda(), kp, ks, vp, vs, torch.tensor(ctx, dtype=torch.int32, device="cuda"),
                        max_ctx, None if signs is None else signs.cuda(), bits, levels.cuda(), scale,
                        out, ws)
    torch.cuda.synchronize()
    assert np.all(ws[: 4 * B].view(torch.int32).cpu().numpy() == 0)
    return out.cpu().numpy()


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("B,Hkv,G,d,ctx", [
    (1, 2, 8, 128, [1500]),
    (2, 2, 1, 128, [777, 4100]),
    (1, 1, 16, 128, [300]),
    (1, 2, 4, 256, [1000]),
    (1, 1, 3, 256, [1]),
])
def test_cb_decode_matches_oracle(bits, B, Hkv, G, d, ctx):
    require_cuda()
    seed = bits * 10 + G + d
    T = max(ctx)
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, seed, heavy=True)
    signs = signs_for(d, seed + 1)
    lv = levels_for(bits)
    cache = oracle_cb_cache(k, v, signs, bits, lv)
    scale = 1 / math.sqrt(d)
    got = cb_decode(upload_cache(cache), q, ctx, T, signs, bits, lv, scale, Hkv)
    want = oracle.sdpa_cb_decode(to_oracle(q), cache, ctx, signs.numpy(), bits, lv.numpy(), scale,
                                 Hkv, threads=THREADS)
    check_attention_cb(got, want, cache, ctx, G, bits, lv, f"cb{bits} B={B} Hkv={Hkv} G={G} d={d}")


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("G", [5, 6, 7, 8])
def test_cb_tensor_core_decode_ragged_batch(bits, G):
    """The tensor-core codebook decode (5..8 query heads per kv head, d = 128):
    two sequences of different lengths, each over several 256-token stages and
    split-K chunks, with ragged tails and (G < 8) padding heads."""
    require_cuda()
    B, Hkv, d, ctx = 2, 2, 128, [3001, 517]
    seed = 300 + 10 * bits + G
    T = max(ctx)
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, seed, heavy=True)
    signs = signs_for(d, seed + 1)
    lv = levels_for(bits)
    cache = oracle_cb_cache(k, v, signs, bits, lv)
    got = cb_decode(upload_cache(cache), q, ctx, T, signs, bits, lv, 1 / math.sqrt(d), Hkv)
    want = oracle.sdpa_cb_decode(to_oracle(q), cache, ctx, signs.numpy(), bits, lv.numpy(),
                                 1 / math.sqrt(d), Hkv, threads=THREADS)
    check_attention_cb(got, want, cache, ctx, G, bits, lv, f"cb{bits} G={G} ragged")


@pytest.mark.parametrize("bits,mul,off", [(2, 1e3, 0.3), (3, 1e-3, -0.2), (4, 37.0, 0.05)])
def test_cb_tensor_core_decode_custom_levels(bits, mul, off):
    """Levels other than the Gaussian codebook: asymmetric and far from 1 in
    magnitude (the tensor-core decode normalises them by a power of two before
    splitting them into f16 parts), at attn_scale 1.0 and 1/sqrt(d)."""
    require_cuda()
    B, Hkv, G, d, T = 1, 2, 8, 128, 1200
    seed = 400 + bits
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, seed)
    signs = signs_for(d, seed + 1)
    lv = ((levels_for(bits).double() + off) * mul).float()
    assert torch.all(lv[1:] > lv[:-1])
    cache = oracle_cb_cache(k, v, signs, bits, lv)
    for scale in (1 / math.sqrt(d), 1.0):
        got = cb_decode(upload_cache(cache), q, [T], T, signs, bits, lv, scale, Hkv)
        want = oracle.sdpa_cb_decode(to_oracle(q), cache, [T], signs.numpy(), bits, lv.numpy(),
                                     scale, Hkv, threads=THREADS)
        check_attention_cb(got, want, cache, [T], G, bits, lv,
                           f"cb{bits} levels x{mul}+{off} scale={scale:.3g}")


def test_cb_decode_rotation_off_fp32_query_attn_scale_one():
    require_cuda()
    B, Hkv, G, d, T, bits = 1, 2, 2, 128, 700, 3
    k, v, q = make_case(B, Hkv, G, d, T, torch.float32, 5)
    lv = levels_for(bits)
    cache = oracle_cb_cache(k, v, None, bits, lv)
    got = cb_decode(upload_cache(cache), q, [T], T, None, bits, lv, 1.0, Hkv)
    want = oracle.sdpa_cb_decode(to_oracle(q), cache, [T], None, bits, lv.numpy(), 1.0, Hkv,
                                 threads=THREADS)
    check_attention_cb(got, want, cache, [T], G, bits, lv, "cb3 rotation off")


def test_cb_engine_step_and_determinism():
    """CodebookKVCache: append + fused step equals append then decode, bit for
    bit, is deterministic, and agrees with the oracle on its own cache."""
    require_cuda()
    B, Hkv, G, d, T, bits = 1, 2, 8, 128, 2000, 2
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 7)
    signs = signs_for(d, 8)
    outs = []
    for fused in (True, False, True):
        c = CodebookKVCache(B, Hkv, d, T, bits, signs=signs)
        c.append(k[:, :, :T - 1].cuda(), v[:, :, :T - 1].cuda(),
                 torch.zeros(B, dtype=torch.int32, device="cuda"))
        ctx = torch.tensor([T], dtype=torch.int32, device="cuda")
        kn, vn = k[:, :, T - 1:].contiguous().cuda(), v[:, :, T - 1:].contiguous().cuda()
        if fused:
            out = c.decode_append(q.cuda(), kn, vn, ctx, T)
        else:
            c.append(kn, vn, ctx - 1)
            out = c.decode(q.cuda(), ctx, T)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy())
    np.testing.assert_array_equal(outs[0], outs[1])
    np.testing.assert_array_equal(outs[0], outs[2])
    cache = [t.cpu().numpy() for t in (c.k_packed, c.k_scales, c.v_packed, c.v_scales)]
    want = oracle.sdpa_cb_decode(to_oracle(q), cache, [T], signs.numpy(), bits, c.levels.cpu().numpy(),
                                 1 / math.sqrt(d), Hkv, threads=THREADS)
    check_attention_cb(outs[0], want, cache, [T], G, bits, c.levels.cpu(), "cb engine")


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_cb_fused_step_ragged_batch(bits):
    """decode_append on the tensor-core codebook path (the decode kernel
    quantizes each sequence's new token into row ctx - 1 itself): two
    sequences of different lengths, 6 query heads per kv head.  Bit-identical
    to append-then-decode, and the oracle agrees on the resulting cache."""
    require_cuda()
    B, Hkv, G, d, ctx = 2, 2, 6, 128, [1800, 333]
    T = max(ctx)
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 500 + bits)
    signs = signs_for(d, 501 + bits)
    ct = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    kn = torch.stack([k[b, :, ctx[b] - 1] for b in range(B)])[:, :, None].contiguous().cuda()
    vn = torch.stack([v[b, :, ctx[b] - 1] for b in range(B)])[:, :, None].contiguous().cuda()
    outs, caches = [], []
    for fused in (True, False):
        c = CodebookKVCache(B, Hkv, d, T, bits, signs=signs)
        c.append(k.cuda(), v.cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"))
        for b in range(B):  # rows ctx - 1 .. hold stale data the step must overwrite
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
    lv = c.levels.cpu()
    want = oracle.sdpa_cb_decode(to_oracle(q), caches[0], ctx, signs.numpy(), bits, lv.numpy(),
                                 1 / math.sqrt(d), Hkv, threads=THREADS)
    check_attention_cb(outs[0], want, caches[0], ctx, G, bits, lv, f"cb{bits} fused step")


def test_cb_tensor_core_decode_large_batch():
    """1030 ragged sequences (more than the decode's in-shared-memory item
    list holds): the tensor-core codebook decode walks every item of the plan."""
    require_cuda()
    B, Hkv, G, d, bits = 1030, 1, 8, 128, 3
    rng = np.random.default_rng(7)
    ctx = [int(x) for x in rng.integers(1, 400, size=B)]
    ctx[0] = 400
    T = max(ctx)
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 77)
    signs = signs_for(d, 78)
    lv = levels_for(bits)
    cache = oracle_cb_cache(k, v, signs, bits, lv)
    got = cb_decode(upload_cache(cache), q, ctx, T, signs, bits, lv, 1 / math.sqrt(d), Hkv)
    want = oracle.sdpa_cb_decode(to_oracle(q), cache, ctx, signs.numpy(), bits, lv.numpy(),
                                 1 / math.sqrt(d), Hkv, threads=THREADS)
    check_attention_cb(got, want, cache, ctx, G, bits, lv, "cb3 B=1030")
