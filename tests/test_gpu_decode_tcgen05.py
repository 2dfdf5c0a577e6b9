"""The tcgen05 / tensor-memory decode kernel (decode_tc.cu) against the oracle.

libtq's default int4 decode at head_dim 128 is the warp-level mma.sync
kernel; the tcgen05 kernel is the alternative selected with the test hook
TQ_TEST_HOOK_TCGEN05_DECODE.  The decode tests below are the same functions as
in the modules they come from (same cases, same gates: rel-L2 <= 1e-4 and
max-abs <= 1e-3 max|v_hat| per head against the oracle), collected again here
and run with that kernel selected.  They cover tiles with a ragged tail,
chunk boundaries, batches with and without the item list, the lazy softmax
reference moving (attn_scale 1.0, heavy rows, outliers, V exactly zero on a
prefix), the fused append, the SRFT cache's rotated queries and the softmax
state for context parallelism.  Two more tests compare the two kernels.
"""
import math

import numpy as np
import pytest
import torch

from compressed_domain_attention_tq_b200 import _lib
from conftest import require_cuda
from helpers import oracle_cache, upload_cache

from test_gpu_decode import (test_decode_attn_scale_one_d128_peaked, test_decode_chunk_boundaries,  # noqa: F401
                             test_decode_flags_and_clamping, test_decode_is_deterministic,
                             test_decode_large_batch_without_item_list, test_decode_outlier_channels,
                             test_decode_ragged_batch_heavy_rows, test_decode_small_shapes,
                             test_decode_tiny_mha_full_size, test_decode_zero_v_prefix)
from test_gpu_decode_append import (test_fused_step_matches_two_calls, test_fused_step_one_token_and_clamped,  # noqa: F401
                                    test_fused_step_vs_oracle_fp32_inputs)
from test_gpu_srft import (test_srft_decode_append_equals_two_calls_and_oracle,  # noqa: F401
                           test_srft_decode_matches_oracle)
from test_gpu_context_parallel import (test_context_parallel_matches_whole_context,  # noqa: F401
                                       test_lse_of_one_part_reproduces_plain_decode)
from test_gpu_full_size import test_full_size_llama70b_gqa_128k, test_full_size_ragged_b16  # noqa: F401

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def tcgen05_decode():
    """Select the tcgen05 kernel for every decode call of the test."""
    _lib.set_test_hooks(_lib.TEST_HOOK_TCGEN05_DECODE)
    yield
    _lib.set_test_hooks(0)


def _decode(cache_dev, q, ctx, T, signs, scale, Hkv):
    B, Hq, d = q.shape
    ws = torch.empty(_lib.decode_workspace_bytes(B, Hq, Hkv, d, T), dtype=torch.uint8, device="cuda")
    out = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    kp, ks, vp, vs = cache_dev
    _lib.sdpa_int4_decode(q.cuda(), kp, ks, vp, vs, torch.tensor(ctx, dtype=torch.int32, device="cuda"), T,
                          signs.cuda(), scale, out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("G,ctx,scale", [(8, [5000], None), (5, [2000, 7777], None), (8, [3000], 1.0),
                                         (1, [129], None)])
def test_tcgen05_matches_mma_sync_kernel(G, ctx, scale):
    """Both kernels on the same cache: same result to far inside the oracle gate
    (they differ only in the order of fp32 roundings)."""
    require_cuda()
    B, Hkv, d, T = len(ctx), 2, 128, max(ctx)
    g = torch.Generator().manual_seed(G * 100 + T)
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16)
    signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)
    dev = upload_cache(oracle_cache(k, v, signs))
    scale = 1 / math.sqrt(d) if scale is None else scale
    tc = _decode(dev, q, ctx, T, signs, scale, Hkv)
    _lib.set_test_hooks(0)
    ref = _decode(dev, q, ctx, T, signs, scale, Hkv)
    rel = np.linalg.norm(tc - ref) / np.linalg.norm(ref)
    assert rel < 2e-6, rel


def test_tcgen05_starved_pipeline_returns_nan_then_recovers():
    """The kernel's bounded waits run out when every CTA's first copy is
    withheld: NaN outputs, and the next call on the context is correct."""
    require_cuda()
    B, Hkv, G, d, T = 1, 2, 8, 128, 3000
    g = torch.Generator().manual_seed(5)
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16)
    signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)
    dev = upload_cache(oracle_cache(k, v, signs))
    _lib.set_test_hooks(_lib.TEST_HOOK_TCGEN05_DECODE | _lib.TEST_HOOK_STARVE_PIPELINE)
    bad = _decode(dev, q, [T], T, signs, 0.1, Hkv)
    _lib.set_test_hooks(_lib.TEST_HOOK_TCGEN05_DECODE)
    assert np.all(np.isnan(bad))
    good = _decode(dev, q, [T], T, signs, 0.1, Hkv)
    _lib.set_test_hooks(0)
    ref = _decode(dev, q, [T], T, signs, 0.1, Hkv)
    assert np.linalg.norm(good - ref) / np.linalg.norm(ref) < 2e-6
