"""The tensor-core bulk quantizer (quantize_tc.cu) against the oracle.

Bulk quantize-appends (more than 8192 vectors) of bf16 vectors at head_dim 128
and 256 with rotation run the rotation as a bf16 tcgen05 product on 128-vector
tiles (at 256: two 128-wide products P, Q and y = (P +- Q) / 16);
TQ_TEST_HOOK_BUTTERFLY_QUANTIZE selects the fp32 butterfly kernel instead.
Bars as in test_gpu_quantize: at most 0.01% of codes differ from the oracle's,
each by 1, scales within 4 ulp.  Cases: ragged last tiles, several sequences
with different start positions, rows past the capacity skipped, extreme
values (bf16 subnormals, values near the bf16 maximum, wide exponent spreads
inside one vector, zero vectors), agreement with the butterfly kernel, and the
bounded waits running out.
"""
import numpy as np
import pytest
import torch

from compressed_domain_attention_tq_b200 import _lib
from conftest import require_cuda
from helpers import oracle_cache
from test_gpu_quantize import compare, inputs

pytestmark = pytest.mark.gpu


def _quantize(k, v, pos, signs, cap, hooks=0):
    B, H, n, d = k.shape
    dev = "cuda"
    kp = torch.full((B, H, cap, d // 2), 0xAB, dtype=torch.uint8, device=dev)
    vp = kp.clone()
    ks = torch.full((B, H, cap, d // 32), -1.0, dtype=torch.float32, device=dev)
    vs = ks.clone()
    _lib.set_test_hooks(hooks)
    try:
        _lib.quantize_append(k.to(dev), v.to(dev), torch.tensor(pos, dtype=torch.int32, device=dev),
                             signs.to(dev), kp, ks, vp, vs)
        torch.cuda.synchronize()
    finally:
        _lib.set_test_hooks(0)
    return [t.cpu().numpy() for t in (kp, ks, vp, vs)]


def _signs(d, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("B,H,n,pos,extra", [
    (1, 8, 1100, [0], 3),          # 8800 vectors per tensor: 68.75 tiles
    (3, 2, 1501, [0, 7, 100], 0),  # rows of the last two sequences run past the capacity
    (2, 5, 1000, [3, 0], 9),
])
def test_tc_quantize_matches_oracle(d, B, H, n, pos, extra):
    require_cuda()
    k, v = inputs(B, H, n, d, torch.bfloat16, 31 * n + B + d)
    signs = _signs(d, n)
    cap = n + extra
    assert 2 * B * H * n > 8192   # the bulk path
    ref = oracle_cache(k, v, signs, capacity=cap + max(pos), pos=pos)
    got = _quantize(k, v, pos, signs, cap)
    ref = [r[:, :, :cap] for r in ref]
    # rows the call does not write keep their fill; the oracle's cache has zeros there
    for b, p in enumerate(pos):
        end = min(p + n, cap)
        for arr, fill in ((got[0], 0xAB), (got[2], 0xAB), (got[1], -1.0), (got[3], -1.0)):
            assert np.all(arr[b, :, :p] == fill) and np.all(arr[b, :, end:] == fill)
            arr[b, :, :p] = 0
            arr[b, :, end:] = 0
    compare(got, ref, d, True, f"B={B} H={H} n={n} pos={pos}")


@pytest.mark.parametrize("d", [128, 256])
def test_tc_quantize_agrees_with_butterfly_kernel(d):
    """Same inputs through both bulk kernels: the rotations differ only in the
    order of fp32 roundings, so codes match except at near-ties."""
    require_cuda()
    B, H, n = 2, 4, 1300
    k, v = inputs(B, H, n, d, torch.bfloat16, 77)
    signs = _signs(d, 78)
    tc = _quantize(k, v, [0, 5], signs, n + 5)
    bf = _quantize(k, v, [0, 5], signs, n + 5, _lib.TEST_HOOK_BUTTERFLY_QUANTIZE)
    n_diff, n_tot = compare(tc, bf, d, True, "tcgen05 vs butterfly")
    assert n_diff <= 1e-5 * n_tot


@pytest.mark.parametrize("d", [128, 256])
def test_tc_quantize_bit_identical_to_butterfly_kernel_on_exact_inputs(d):
    """Small-integer inputs times a power of two per vector: every partial sum
    of both rotations is exact, so both kernels round the same rotated values
    and must give identical bits (scale division by 7, reciprocal bracket,
    fallbacks and packing all included).  Zero vectors included.  (Against the
    oracle such inputs are a poor case: many y / s fall exactly on a
    half-integer in exact arithmetic, where fl(D c) and the oracle's correctly
    rounded rotation may round apart; oracle parity is the other tests'.)"""
    require_cuda()
    B, H, n = 1, 6, 1500
    g = torch.Generator().manual_seed(21)
    ints = torch.randint(-8, 9, (B, H, n, d), generator=g).float()
    ints[:, :, 5] = 0
    ints[:, :, 6] = 0
    ints[:, :, 6, 40] = 3
    e = torch.randint(-40, 41, (B, H, n, 1), generator=g).float()
    x = (ints * torch.exp2(e)).to(torch.bfloat16)
    assert torch.equal(x.float(), ints * torch.exp2(e))
    y = (-x.float() * 0.5).to(torch.bfloat16)
    signs = _signs(d, 22)
    tc = _quantize(x, y, [0], signs, n)
    bf = _quantize(x, y, [0], signs, n, _lib.TEST_HOOK_BUTTERFLY_QUANTIZE)
    for a, b in zip(tc, bf):
        np.testing.assert_array_equal(a.view(np.uint8), b.view(np.uint8))


@pytest.mark.parametrize("d", [128, 256])
def test_tc_quantize_extreme_values(d):
    """bf16 subnormals, values near the bf16 maximum over d (no fp32
    overflow in the rotation), one huge and many tiny values in one vector,
    single spikes and zero vectors, inside a bulk call."""
    require_cuda()
    n = 4500
    g = torch.Generator().manual_seed(11)
    x = torch.randn(1, 2, n, d, generator=g)
    sub = torch.finfo(torch.float32).tiny  # 2^-126
    special = [
        torch.full((d,), 3.0) * sub * 0.25,                        # all subnormal
        torch.where(torch.arange(d) % 2 == 0, 1.0, 0.5) * sub * 0.03,
        torch.cat([torch.ones(1), torch.full((d - 1,), sub * 0.5)]),  # one normal, rest subnormal
        torch.linspace(-1.0, 1.0, d) * 2.0 ** 119,                 # near the bf16 maximum / 2^8
        torch.cat([torch.full((1,), 1e30), torch.full((d - 1,), 1e-30)]),
        torch.cat([torch.full((3,), -2.0 ** 100), torch.randn(d - 3, generator=g)]),
        torch.eye(d)[17] * 5.0,
        torch.zeros(d),
        torch.full((d,), -1e-36),
    ]
    for i, row in enumerate(special):
        x[0, i % 2, 10 * i + 3] = row
        x[0, (i + 1) % 2, n - 1 - i] = row
    k = x.to(torch.bfloat16)
    v = (-x).to(torch.bfloat16)
    signs = _signs(d, 12)
    ref = oracle_cache(k, v, signs, capacity=n, pos=[0])
    got = _quantize(k, v, [0], signs, n)
    compare(got, ref, d, True, "extremes")


@pytest.mark.parametrize("d", [128, 256])
def test_tc_quantize_starved_pipeline_writes_nan_scales_then_recovers(d):
    """With every CTA's first copy withheld the kernel's bounded waits run out:
    every written row gets NaN scales.  The next call on the context is
    correct."""
    require_cuda()
    B, H, n = 1, 8, 1100
    k, v = inputs(B, H, n, d, torch.bfloat16, 5)
    signs = _signs(d, 6)
    bad = _quantize(k, v, [0], signs, n, _lib.TEST_HOOK_STARVE_PIPELINE)
    assert np.all(np.isnan(bad[1])) and np.all(np.isnan(bad[3]))
    good = _quantize(k, v, [0], signs, n)
    ref = oracle_cache(k, v, signs, capacity=n, pos=[0])
    compare(good, ref, d, True, "after the starved call")
