"""The allocation-free decode entry point, tq_sdpa_int4_decode_static_scratch.

Some callers cannot allocate device memory: a plug-in inside a host framework
that owns all device memory, or a latency-critical caller that cannot accept
cudaMalloc's device-wide synchronization.  For them libtq keeps its decode
scratch in a built-in device array of TQ_STATIC_SCRATCH_BYTES.  These tests
check that this entry point gives the same attention as tq_sdpa_int4_decode
with a caller workspace, on two calls in a row (the array keeps the previous
call's contents), and that sizes beyond the array are rejected before any
launch.  This file is collected last on purpose: if it fails, a run that stops
at the first failure has already run every other test.
"""
import math

import numpy as np
import pytest
import torch

from compressed_domain_attention_tq_b200 import _lib
from conftest import require_cuda
from helpers import check_attention, oracle_cache, upload_cache


def test_static_scratch_rejects_sizes_beyond_the_array():
    """Host-only: the size check comes before any CUDA call."""
    B, Hq, Hkv, d, T = 256, 64, 8, 128, 131072
    need = _lib.decode_workspace_bytes(B, Hq, Hkv, d, T)
    assert need > _lib.STATIC_SCRATCH_BYTES
    P = lambda x: __import__("ctypes").c_void_p(x)
    rc = _lib.load().tq_sdpa_int4_decode_static_scratch(
        P(4096), _lib.TQ_BF16, B, Hq, Hkv, d, 32, P(4096), P(4096), P(4096), P(4096), T,
        P(4096), T, None, 1 / math.sqrt(d), P(4096), None)
    assert rc == _lib.TQ_ERR_SCRATCH_LIMIT
    assert "scratch" in _lib.status_string(rc)


@pytest.mark.gpu
@pytest.mark.parametrize("B,Hkv,G,d,ctx", [(2, 2, 8, 128, [3000, 1777]), (1, 2, 2, 256, [2500])])
def test_static_scratch_matches_caller_workspace_twice(B, Hkv, G, d, ctx):
    require_cuda()
    dev = "cuda"
    T = max(ctx)
    g = torch.Generator().manual_seed(B * 1000 + d)
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16)
    signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)
    cache = oracle_cache(k, v, signs)
    kp, ks, vp, vs = upload_cache(cache, dev)
    ctx_d = torch.tensor(ctx, dtype=torch.int32, device=dev)
    sg = signs.to(dev)
    scale = 1 / math.sqrt(d)
    assert _lib.decode_workspace_bytes(B, Hkv * G, Hkv, d, T) <= _lib.STATIC_SCRATCH_BYTES

    ws = torch.empty(_lib.decode_workspace_bytes(B, Hkv * G, Hkv, d, T), dtype=torch.uint8,
                     device=dev)
    outs = []
    for call in range(2):
        q = torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16).to(dev)
        want = torch.empty(B, Hkv * G, d, dtype=torch.float32, device=dev)
        got = torch.full((B, Hkv * G, d), float("nan"), dtype=torch.float32, device=dev)
        _lib.sdpa_int4_decode(q, kp, ks, vp, vs, ctx_d, T, sg, scale, want, ws)
        _lib.sdpa_int4_decode_static_scratch(q, kp, ks, vp, vs, ctx_d, T, sg, scale, got)
        torch.cuda.synchronize()
        got, want = got.cpu().numpy(), want.cpu().numpy()
        assert np.all(np.isfinite(got)), f"call {call}: non-finite output"
        check_attention(got, want.astype(np.float64), cache, ctx, G, f"static scratch call {call}")
        outs.append(got)
    assert not np.array_equal(outs[0], outs[1])   # the two calls used different queries
