"""The tensor-core SRFT bulk quantizer (quantize_srft_tc.cu) against the oracle.

Bulk appends (more than 8192 vectors) of bf16 vectors at head_dim 32, 64, 96
and 128 form y = lambda (.) F (sigma (.) x) as a bf16 product with the
Hartley matrix split into three bf16 parts, accumulated in fp32 in tensor
memory.  TQ_TEST_HOOK_BUTTERFLY_QUANTIZE selects the CUDA-core SRFT kernels
instead.  Bars as in test_gpu_srft: at most 0.01% of codes differ from the
oracle's, each by 1, scales within 32 ulp.  Cases: every width (d = 32 and 96
take the 64-byte swizzled chunk), ragged last tiles, start positions, rows
past the capacity, lambda spread 2^U(-1, 1) and none, agreement with the
CUDA-core kernels, and the bounded waits running out."""
import numpy as np
import pytest
import torch

from compressed_domain_attention_tq_b200 import _lib
from conftest import require_cuda
from test_gpu_decode import signs_for
from test_gpu_quantize import compare, inputs
from test_gpu_srft import SCALE_ULP, _dev, lam_for, oracle_srft_cache

pytestmark = pytest.mark.gpu


def _quantize(k, v, pos, signs, lk, lv, cap, hooks=0):
    B, H, n, d = k.shape
    kp = torch.full((B, H, cap, d // 2), 0xAB, dtype=torch.uint8, device="cuda")
    vp = kp.clone()
    ks = torch.full((B, H, cap, d // 32), -1.0, dtype=torch.float32, device="cuda")
    vs = ks.clone()
    _lib.set_test_hooks(hooks)
    try:
        _lib.quantize_append_srft(k.cuda(), v.cuda(), torch.tensor(pos, dtype=torch.int32, device="cuda"),
                                  _dev(signs), _dev(lk), _dev(lv), kp, ks, vp, vs)
        torch.cuda.synchronize()
    finally:
        _lib.set_test_hooks(0)
    return [t.cpu().numpy() for t in (kp, ks, vp, vs)]


def _written_only(got, pos, n, cap):
    """Rows a call does not write keep their fill; zero them like the oracle's cache."""
    for b, p in enumerate(pos):
        end = min(p + n, cap)
        for arr, fill in ((got[0], 0xAB), (got[2], 0xAB), (got[1], -1.0), (got[3], -1.0)):
            assert np.all(arr[b, :, :p] == fill) and np.all(arr[b, :, end:] == fill)
            arr[b, :, :p] = 0
            arr[b, :, end:] = 0


@pytest.mark.parametrize("d", [32, 64, 96, 128])
@pytest.mark.parametrize("B,H,n,pos,extra,lam", [
    (1, 8, 1100, [0], 3, True),
    (3, 2, 1501, [0, 7, 100], 0, True),   # rows past the capacity
    (2, 5, 900, [3, 0], 9, False),        # lambda none (ones)
])
def test_srft_tc_quantize_matches_oracle(d, B, H, n, pos, extra, lam):
    require_cuda()
    seed = 5 * d + n + B
    k, v = inputs(B, H, n, d, torch.bfloat16, seed)
    signs = signs_for(d, seed + 1)
    lk, lv = (lam_for(d, seed + 2), lam_for(d, seed + 3)) if lam else (None, None)
    cap = n + extra
    assert 2 * B * H * n > 8192
    got = _quantize(k, v, pos, signs, lk, lv, cap)
    want = oracle_srft_cache(k, v, signs, lk, lv, cap + max(pos), pos)
    want = [w[:, :, :cap] for w in want]
    _written_only(got, pos, n, cap)
    n_diff, n_tot = compare(got, want, d, True, f"srft tc d={d} B={B} H={H} n={n}", SCALE_ULP)
    ulp = max(int(np.abs(a.view(np.int32).astype(np.int64) - b.view(np.int32).astype(np.int64)).max())
              for a, b in ((got[1], want[1]), (got[3], want[3])))
    print(f"srft tc d={d}: codes differing {n_diff}/{n_tot}, max scale ulp {ulp}")


@pytest.mark.parametrize("d", [96, 128])
def test_srft_tc_agrees_with_cuda_core_kernels(d):
    require_cuda()
    B, H, n = 1, 6, 1500
    k, v = inputs(B, H, n, d, torch.bfloat16, 90 + d)
    signs, lk, lv = signs_for(d, 91), lam_for(d, 92), lam_for(d, 93)
    tc = _quantize(k, v, [0], signs, lk, lv, n)
    cc = _quantize(k, v, [0], signs, lk, lv, n, _lib.TEST_HOOK_BUTTERFLY_QUANTIZE)
    n_diff, n_tot = compare(tc, cc, d, True, f"srft tensor core vs CUDA cores d={d}", SCALE_ULP)
    assert n_diff <= 1e-4 * n_tot


def test_srft_tc_starved_pipeline_writes_nan_scales_then_recovers():
    require_cuda()
    B, H, n, d = 1, 8, 1100, 96
    k, v = inputs(B, H, n, d, torch.bfloat16, 7)
    signs, lk, lv = signs_for(d, 8), lam_for(d, 9), lam_for(d, 10)
    bad = _quantize(k, v, [0], signs, lk, lv, n, _lib.TEST_HOOK_STARVE_PIPELINE)
    assert np.all(np.isnan(bad[1])) and np.all(np.isnan(bad[3]))
    good = _quantize(k, v, [0], signs, lk, lv, n)
    want = oracle_srft_cache(k, v, signs, lk, lv, n, [0])
    compare(good, want, d, True, "after the starved call", SCALE_ULP)
