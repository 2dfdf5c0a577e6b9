"""GPU decode attention vs the oracle on the same (oracle-quantized) cache.

The oracle quantizes the seeded inputs; that cache is uploaded and both the
CUDA path and the oracle attend over it.  Gates: per (sequence, query head)
relative L2 <= 1e-4 and max abs <= 1e-3 * max|v_hat|.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_tq_b200 import _lib
from conftest import require_cuda
from helpers import THREADS, check_attention, oracle_cache, to_oracle, upload_cache

pytestmark = pytest.mark.gpu


def make_case(B, Hkv, G, d, T_cap, dtype, seed, heavy=False, outliers=False):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, Hkv, T_cap, d, generator=g)
    v = torch.randn(B, Hkv, T_cap, d, generator=g)
    if outliers:
        k[..., [3, 17, 64, 100 % d]] *= 10
    if heavy:
        m = torch.rand(B, 1, T_cap, 1, generator=g) < 0.02
        k = torch.where(m, k * 8, k)
        v = torch.where(m, v * 8, v)
    q = torch.randn(B, Hkv * G, d, generator=g)
    return k.to(dtype), v.to(dtype), q.to(dtype)


def run_decode(cache_dev, q, ctx, max_ctx, signs, scale, Hkv):
    B, Hq, d = q.shape
    dev = "cuda"
    ws = torch.empty(_lib.decode_workspace_bytes(B, Hq, Hkv, d, max_ctx), dtype=torch.uint8, device=dev)
    out = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
    kp, ks, vp, vs = cache_dev
    _lib.sdpa_int4_decode(q.to(dev), kp, ks, vp, vs, torch.tensor(ctx, dtype=torch.int32, device=dev),
                          max_ctx, None if signs is None else signs.to(dev), scale, out, ws)
    torch.cuda.synchronize()
    flags = ws[: 4 * B].view(torch.int32).cpu().numpy()
    return out.cpu().numpy(), flags


def signs_for(d, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)


def parity(B, Hkv, G, d, ctx, dtype=torch.bfloat16, rot=True, scale=None, seed=0, heavy=False,
           outliers=False, max_ctx=None):
    max_ctx = max(ctx) if max_ctx is None else max_ctx
    T_cap = max(max(ctx), max_ctx)
    k, v, q = make_case(B, Hkv, G, d, T_cap, dtype, seed, heavy, outliers)
    signs = signs_for(d, seed + 1) if rot else None
    cache = oracle_cache(k, v, signs)
    scale = 1 / math.sqrt(d) if scale is None else scale
    got, flags = run_decode(upload_cache(cache), q, ctx, max_ctx, signs, scale, Hkv)
    want = oracle.sdpa_int4_decode(to_oracle(q), cache, ctx, None if signs is None else signs.numpy(),
                                   scale, Hkv, threads=THREADS)
    assert np.all(flags == 0)
    return check_attention(got, want, cache, ctx, G, f"B={B} Hkv={Hkv} G={G} d={d} ctx={ctx}")


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("G", [1, 2, 8, 16])
@pytest.mark.parametrize("T", [1, 31, 64, 65, 1000])
def test_decode_small_shapes(d, G, T):
    require_cuda()
    parity(1, 2, G, d, [T], seed=d + G + T)


@pytest.mark.parametrize("d", [128, 256])
def test_decode_chunk_boundaries(d):
    require_cuda()
    B, Hkv, G = 1, 1, 8
    for T in (2500, 8000):
        chunk = _lib.decode_chunk_tokens(B, Hkv * G, Hkv, d, T)
        for t in sorted({chunk - 1, chunk, chunk + 1, 2 * chunk + 5, T}):
            if 1 <= t <= T:
                parity(B, Hkv, G, d, [t], seed=t, max_ctx=T)


@pytest.mark.parametrize("G", [3, 5, 6, 7])
@pytest.mark.parametrize("scale", [None, 1.0])
def test_decode_group_sizes_with_unused_head_columns(G, scale):
    """3..7 query heads per kv head: the tensor-core decode's MMA tiles are
    sized for 4 or 8 heads, so some head columns carry no query; contexts of
    several 384-token stages with ragged last stages."""
    require_cuda()
    parity(2, 2, G, 128, [1000, 2893], scale=scale, seed=60 + G)


@pytest.mark.parametrize("rot", [False, True])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_tiny_mha_full_size(rot, dtype):
    """Tiny MHA decode at its full size: B=1, 4 heads, d=128, 4096 tokens."""
    require_cuda()
    parity(1, 4, 1, 128, [4096], dtype=dtype, rot=rot, seed=11)


def test_decode_ragged_batch_heavy_rows():
    require_cuda()
    ctx = [1, 700, 2049, 3000, 64, 4096]
    parity(len(ctx), 2, 8, 128, ctx, seed=21, heavy=True)


def test_decode_outlier_channels():
    require_cuda()
    parity(1, 8, 8, 128, [3333], seed=31, outliers=True)


@pytest.mark.parametrize("scale", [1.0, 1 / 16.0])
def test_decode_wide_head_attn_scales(scale):
    """d=256, G=2, at attn_scale 1.0 (peaked softmax) and 1/sqrt(256)."""
    require_cuda()
    parity(2, 2, 2, 256, [3000, 1777], scale=scale, seed=41)


def test_decode_attn_scale_one_d128_peaked():
    require_cuda()
    parity(1, 2, 8, 128, [2000], scale=1.0, seed=51)


@pytest.mark.parametrize("B,G", [(1100, 8), (1030, 2)])
def test_decode_large_batch_without_item_list(B, G):
    """More sequences than the tensor-core decode's in-shared-memory item list
    holds (1024): the kernel walks every (sequence, kv head, chunk) of the plan,
    and the items past a short sequence's end do no work.  Ragged lengths from 1
    to 700 tokens against the oracle for every sequence."""
    require_cuda()
    rng = np.random.default_rng(B + G)
    ctx = [int(x) for x in rng.integers(1, 701, size=B)]
    ctx[0] = 700
    parity(B, 1, G, 128, ctx, seed=B + G)


def test_decode_flags_and_clamping():
    require_cuda()
    B, Hkv, G, d, T = 3, 1, 4, 128, 200
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 61)
    signs = signs_for(d, 62)
    cache = oracle_cache(k, v, signs)
    # max_ctx = 160: 0 is below 1 and 999 above 160, both flagged and clamped
    got, flags = run_decode(upload_cache(cache), q, [0, 150, 999], 160, signs, 0.1, Hkv)
    assert list(flags) == [1, 0, 1]
    want = oracle.sdpa_int4_decode(to_oracle(q), cache, [1, 150, 160], signs.numpy(), 0.1, Hkv)
    check_attention(got, want, cache, [1, 150, 160], G, "clamped")


def test_decode_is_deterministic():
    require_cuda()
    B, Hkv, G, d, T = 1, 2, 8, 128, 5000
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 71)
    signs = signs_for(d, 72)
    cache = upload_cache(oracle_cache(k, v, signs))
    a, _ = run_decode(cache, q, [T], T, signs, 0.08, Hkv)
    b, _ = run_decode(cache, q, [T], T, signs, 0.08, Hkv)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("d,G", [(128, 8), (128, 2), (256, 2)])
def test_decode_zero_v_prefix(d, G):
    """V exactly zero on the first tokens (zero V scales), then random: the
    V-scale exponent is first chosen after real tokens already count in the
    softmax sum, which must then be rescaled with the accumulators.  An
    all-zero V must give an exact zero output."""
    require_cuda()
    B, Hkv, T = 1, 2, 3000
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 81)
    signs = signs_for(d, 82)
    for zero_to in (700, T):
        vz = v.clone()
        vz[:, :, :zero_to] = 0
        cache = oracle_cache(k, vz, signs)
        got, flags = run_decode(upload_cache(cache), q, [T], T, signs, 1 / math.sqrt(d), Hkv)
        assert np.all(flags == 0)
        if zero_to == T:
            assert np.all(got == 0.0)
            continue
        want = oracle.sdpa_int4_decode(to_oracle(q), cache, [T], signs.numpy(), 1 / math.sqrt(d),
                                       Hkv, threads=THREADS)
        check_attention(got, want, cache, [T], G, f"zero V prefix d={d} G={G}")


def test_injected_launch_failure_enqueues_nothing():
    """Host-side fault injection: the call reports TQ_ERR_CUDA and leaves the output alone."""
    require_cuda()
    B, Hkv, G, d, T = 1, 2, 8, 128, 300
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 61)
    cache = upload_cache(oracle_cache(k, v, None))
    ws = torch.empty(_lib.decode_workspace_bytes(B, Hkv * G, Hkv, d, T), dtype=torch.uint8, device="cuda")
    out = torch.full((B, Hkv * G, d), 7.0, device="cuda")
    _lib.set_test_hooks(_lib.TEST_HOOK_FAIL_LAUNCH)
    try:
        with pytest.raises(_lib.TQError) as err:
            _lib.sdpa_int4_decode(q.cuda(), *cache, torch.tensor([T], dtype=torch.int32, device="cuda"), T,
                                  None, 0.1, out, ws)
    finally:
        _lib.set_test_hooks(0)
    assert err.value.status == _lib.TQ_ERR_CUDA
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


@pytest.mark.parametrize("hooks", [0, 4], ids=["mma_sync", "tcgen05"])
def test_starved_pipeline_gives_up_and_context_stays_usable(hooks):
    """The tensor-core decode's waits for its copies are bounded: with each CTA's
    first copy withheld (test hook), the waits run out after about two seconds, the
    kernel ends, the heads' outputs are NaN, and the next call on the same context
    is correct."""
    require_cuda()
    B, Hkv, G, d, T = 1, 2, 8, 128, 3000
    k, v, q = make_case(B, Hkv, G, d, T, torch.bfloat16, 62)
    cache = oracle_cache(k, v, None)
    dev = upload_cache(cache)
    _lib.set_test_hooks(hooks | _lib.TEST_HOOK_STARVE_PIPELINE)
    try:
        got, _ = run_decode(dev, q, [T], T, None, 0.1, Hkv)
    finally:
        _lib.set_test_hooks(hooks)
    assert np.all(np.isnan(got))
    try:
        got, flags = run_decode(dev, q, [T], T, None, 0.1, Hkv)
    finally:
        _lib.set_test_hooks(0)
    want = oracle.sdpa_int4_decode(to_oracle(q), cache, [T], None, 0.1, Hkv, threads=THREADS)
    check_attention(got, want, cache, [T], G, "after a starved call")
