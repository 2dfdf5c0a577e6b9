"""GPU SRFT variant (signs + orthonormal Hartley transform + per-coordinate
lambda; SRFT post, core method) vs the oracle on the same inputs.

Bars, as for the Hadamard rotation: quantize -> at most 0.01% of codes differ,
each by exactly 1; decode on the same packed cache -> per head relative L2 <=
1e-4 and max abs <= 1e-3 * max|v_hat|.  Scales (not required bit-exact with a
rotation) within 32 ulp: an fp32 FFT's rounding error is about
log2(d) * eps * |y|_2 per output element, i.e. relative to the whole row rather
than to each group's maximum; for Gaussian rows (|y|_2 / max_g ~ sqrt(d) / 3)
that is up to ~25 ulp of a group's scale at d = 96 .. 256.  The largest
difference measured on each case is printed."""
import math

import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_tq_b200 import _lib
from compressed_domain_attention_tq_b200.cache import Int4KVCache
from conftest import require_cuda
from helpers import THREADS, check_attention, to_oracle, upload_cache
from test_gpu_decode import make_case, signs_for
from test_gpu_quantize import compare, inputs

pytestmark = pytest.mark.gpu
SCALE_ULP = 32


def lam_for(d, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.exp2(torch.empty(d).uniform_(-1.0, 1.0, generator=g)).to(torch.float32)


def _np(t):
    return None if t is None else t.numpy()


def _dev(t):
    return None if t is None else t.to("cuda")


def gpu_quantize(k, v, pos, signs, lk, lv, cap):
    B, H, n, d = k.shape
    kp = torch.zeros(B, H, cap, d // 2, dtype=torch.uint8, device="cuda")
    vp = torch.zeros_like(kp)
    ks = torch.zeros(B, H, cap, d // 32, dtype=torch.float32, device="cuda")
    vs = torch.zeros_like(ks)
    _lib.quantize_append_srft(k.cuda(), v.cuda(), torch.tensor(pos, dtype=torch.int32, device="cuda"),
                              _dev(signs), _dev(lk), _dev(lv), kp, ks, vp, vs)
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (kp, ks, vp, vs)]


def oracle_srft_cache(k, v, signs, lk, lv, cap=None, pos=None):
    B, H, n, d = k.shape
    cache = oracle.empty_cache(B, H, n if cap is None else cap, d)
    p = np.zeros(B, np.int32) if pos is None else np.asarray(pos, np.int32)
    oracle.quantize_append_srft(to_oracle(k), to_oracle(v), p, _np(signs), _np(lk), _np(lv), cache,
                                threads=THREADS)
    return cache


@pytest.mark.parametrize("d", [32, 96, 128, 160, 192, 224, 256])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,n", [(1, 1, 1), (2, 3, 300), (1, 4, 700)])
def test_srft_quantize_matches_oracle(d, dtype, B, H, n):
    require_cuda()
    seed = 3 * d + n + B
    k, v = inputs(B, H, n, d, dtype, seed)
    signs, lk, lv = signs_for(d, seed + 1), lam_for(d, seed + 2), lam_for(d, seed + 3)
    cap = n + 5
    pos = [(2 * b + 1) % 5 for b in range(B)]
    got = gpu_quantize(k, v, pos, signs, lk, lv, cap)
    want = oracle_srft_cache(k, v, signs, lk, lv, cap, pos)
    ulp = max(int(np.abs(a.view(np.int32).astype(np.int64) - b.view(np.int32).astype(np.int64)).max())
              for a, b in ((got[1], want[1]), (got[3], want[3])))
    n_diff, n_tot = compare(got, want, d, True, f"srft d={d} {dtype} B={B} H={H} n={n}", SCALE_ULP)
    print(f"srft quantize d={d} {dtype} B={B} H={H} n={n}: codes differing {n_diff}/{n_tot}, "
          f"max scale ulp {ulp}")


def test_srft_quantize_without_signs_or_lambda():
    require_cuda()
    d, B, H, n = 96, 1, 2, 64
    k, v = inputs(B, H, n, d, torch.float32, 5)
    got = gpu_quantize(k, v, [0], None, None, None, n)
    want = oracle_srft_cache(k, v, None, None, None)
    compare(got, want, d, True, "srft without signs and lambda", SCALE_ULP)


def srft_decode(cache_dev, q, ctx, max_ctx, signs, lk, lv, scale, Hkv):
    B, Hq, d = q.shape
    ws = torch.empty(_lib.decode_srft_workspace_bytes(B, Hq, Hkv, d, max_ctx), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    kp, ks, vp, vs = cache_dev
    _lib.sdpa_int4_decode_srft(q.cuda(), kp, ks, vp, vs,
                               torch.tensor(ctx, dtype=torch.int32, device="cuda"), max_ctx,
                               _dev(signs), _dev(lk), _dev(lv), scale, out, ws)
    torch.cuda.synchronize()
    assert np.all(ws[: 4 * B].view(torch.int32).cpu().numpy() == 0)
    return out.cpu().numpy()


def srft_parity(B, Hkv, G, d, ctx, dtype=torch.bfloat16, scale=None, seed=0, lam=True, signs=True):
    T = max(ctx)
    k, v, q = make_case(B, Hkv, G, d, T, dtype, seed, heavy=True)
    sg = signs_for(d, seed + 1) if signs else None
    lk, lv = (lam_for(d, seed + 2), lam_for(d, seed + 3)) if lam else (None, None)
    cache = oracle_srft_cache(k, v, sg, lk, lv)
    scale = 1 / math.sqrt(d) if scale is None else scale
    got = srft_decode(upload_cache(cache), q, ctx, T, sg, lk, lv, scale, Hkv)
    want = oracle.sdpa_int4_decode_srft(to_oracle(q), cache, ctx, _np(sg), _np(lk), _np(lv), scale,
                                        Hkv, threads=THREADS)
    return check_attention(got, want, cache, ctx, G, f"srft B={B} Hkv={Hkv} G={G} d={d} ctx={ctx}")


@pytest.mark.parametrize("B,Hkv,G,d,ctx", [
    (1, 2, 1, 96, [1000]),            # MHA, CUDA-core decode
    (2, 2, 4, 96, [777, 1290]),       # ragged batch
    (1, 1, 3, 160, [257]),            # odd number of query heads (pairs)
    (1, 2, 8, 128, [1500]),           # tensor-core decode, heads on rows
    (1, 3, 3, 128, [700]),            # tensor-core decode, dims on rows, odd Hq
    (1, 1, 4, 256, [600]),            # tensor-core decode, d = 256
    (1, 2, 16, 192, [300]),           # CUDA-core decode, 16 heads per kv head
    (1, 1, 2, 32, [64]),              # smallest width
    (2, 1, 1, 224, [1, 5]),           # one-token and tiny contexts
    (1, 1, 2, 64, [4097]),            # several chunks and a ragged tail
])
def test_srft_decode_matches_oracle(B, Hkv, G, d, ctx):
    require_cuda()
    srft_parity(B, Hkv, G, d, ctx, seed=d + G)


def test_srft_decode_fp32_query_and_attn_scale_one():
    require_cuda()
    srft_parity(1, 2, 4, 96, [900], dtype=torch.float32, scale=1.0, seed=11)


def test_srft_decode_without_lambda_or_signs():
    require_cuda()
    srft_parity(1, 1, 2, 96, [500], lam=False, seed=12)
    srft_parity(1, 1, 2, 160, [500], signs=False, seed=13)


@pytest.mark.parametrize("d,G", [(96, 4), (128, 4), (128, 8), (256, 2)])
def test_srft_decode_append_equals_two_calls_and_oracle(d, G):
    """The fused step writes the same cache row and gives the same output as
    quantize-append then decode; both agree with the oracle.  d = 96 runs the
    CUDA-core decode, d = 128 and 256 the tensor-core decode, each after the
    preparation kernel (new token and query rotation in one launch)."""
    require_cuda()
    B, Hkv, T = 2, 2, 900
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 21)
    sg, lk, lv = signs_for(d, 22), lam_for(d, 23), lam_for(d, 24)
    ctx = [T, T - 100]
    cache0 = oracle_srft_cache(k, v, sg, lk, lv)
    newk, newv = k[:, :, :1].clone() * 3, v[:, :, :1].clone() * 3
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    outs, caches = [], []
    for fused in (True, False):
        kp, ks, vp, vs = upload_cache(cache0)
        out = torch.empty(B, Hkv * G, d, dtype=torch.float32, device="cuda")
        ws = torch.empty(_lib.decode_srft_workspace_bytes(B, Hkv * G, Hkv, d, T), dtype=torch.uint8,
                         device="cuda")
        if fused:
            _lib.sdpa_int4_decode_append_srft(q.cuda(), newk.cuda(), newv.cuda(), kp, ks, vp, vs, ctx_t,
                                              T, sg.cuda(), lk.cuda(), lv.cuda(), 0.1, out, ws)
        else:
            _lib.quantize_append_srft(newk.cuda(), newv.cuda(), ctx_t - 1, sg.cuda(), lk.cuda(),
                                      lv.cuda(), kp, ks, vp, vs)
            _lib.sdpa_int4_decode_srft(q.cuda(), kp, ks, vp, vs, ctx_t, T, sg.cuda(), lk.cuda(),
                                       lv.cuda(), 0.1, out, ws)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy())
        caches.append([t.cpu().numpy() for t in (kp, ks, vp, vs)])
    np.testing.assert_array_equal(outs[0], outs[1])
    for a, b in zip(*caches):
        np.testing.assert_array_equal(a, b)
    want = oracle.sdpa_int4_decode_srft(to_oracle(q), caches[0], ctx, sg.numpy(), lk.numpy(),
                                        lv.numpy(), 0.1, Hkv, threads=THREADS)
    check_attention(outs[0], want, caches[0], ctx, G, "srft fused step")


def test_srft_decode_is_deterministic():
    require_cuda()
    B, Hkv, G, d, T = 1, 2, 8, 128, 3000
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 31)
    sg, lk, lv = signs_for(d, 32), lam_for(d, 33), lam_for(d, 34)
    cache = upload_cache(oracle_srft_cache(k, v, sg, lk, lv))
    a = srft_decode(cache, q, [T], T, sg, lk, lv, 0.09, Hkv)
    b = srft_decode(cache, q, [T], T, sg, lk, lv, 0.09, Hkv)
    np.testing.assert_array_equal(a, b)


def test_srft_cache_engine_end_to_end():
    """Int4KVCache(rotation='srft'): GPU quantize + GPU decode against the
    oracle's quantize + decode on the same inputs (the caches may differ in a
    rare code by one; the attention gates hold)."""
    require_cuda()
    B, Hkv, G, d, T = 1, 2, 4, 160, 1200
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 41)
    sg, lk, lv = signs_for(d, 42), lam_for(d, 43), lam_for(d, 44)
    c = Int4KVCache(B, Hkv, d, T, signs=sg, rotation="srft", lambda_k=lk, lambda_v=lv)
    c.append(k.cuda(), v.cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"))
    out = c.decode(q.cuda(), torch.tensor([T], dtype=torch.int32, device="cuda"), T)
    torch.cuda.synchronize()
    cache = [t.cpu().numpy() for t in (c.k_packed, c.k_scales, c.v_packed, c.v_scales)]
    want = oracle.sdpa_int4_decode_srft(to_oracle(q), cache, [T], sg.numpy(), lk.numpy(), lv.numpy(),
                                        1 / math.sqrt(d), Hkv, threads=THREADS)
    check_attention(out.cpu().numpy(), want, cache, [T], G, "srft engine")
    ref = oracle_srft_cache(k, v, sg, lk, lv)
    compare(cache, ref, d, True, "srft engine cache", SCALE_ULP)


def test_srft_decode_large_ragged_batch():
    """1030 ragged sequences with the SRFT rotation on the tensor-core decode
    (query rotation kernel over every sequence, items past short sequences)."""
    require_cuda()
    B, Hkv, G, d = 1030, 1, 8, 128
    rng = np.random.default_rng(9)
    ctx = [int(x) for x in rng.integers(1, 300, size=B)]
    ctx[0] = 300
    T = max(ctx)
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 91)
    sg, lk, lv = signs_for(d, 92), lam_for(d, 93), lam_for(d, 94)
    cache = oracle_srft_cache(k, v, sg, lk, lv)
    got = srft_decode(upload_cache(cache), q, ctx, T, sg, lk, lv, 0.09, Hkv)
    want = oracle.sdpa_int4_decode_srft(to_oracle(q), cache, ctx, sg.numpy(), lk.numpy(),
                                        lv.numpy(), 0.09, Hkv, threads=THREADS)
    check_attention(got, want, cache, ctx, G, "srft B=1030")
