"""The allocation-free decode entry point, tq_sdpa_int4_decode_static_scratch.

Some callers cannot allocate device memory: a plug-in inside a host framework
that owns all device memory, or a latency-critical caller that cannot accept
cudaMalloc's device-wide synchronization.  For them libtq keeps its decode
scratch in a built-in device array of TQ_STATIC_SCRATCH_BYTES.  These tests
check that this entry point gives exactly the output of tq_sdpa_int4_decode
with a caller workspace (same kernels, same plan), on two calls in a row (the
array keeps the previous call's contents), that a call allocates no device
memory, that it works in a second CUDA context on the same GPU (the array's
address is looked up per context), and that invalid arguments and sizes beyond
the array are rejected before any launch.  This file is collected last on
purpose: if it fails, a run that stops at the first failure has already run
every other test.
"""
import ctypes
import math
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

from compressed_domain_attention_tq_b200 import _lib
from conftest import require_cuda
from helpers import oracle_cache, upload_cache

P = ctypes.c_void_p


def _static_call(q, B, Hq, Hkv, d, T, q_ptr=P(4096), head_dim=None):
    return _lib.load().tq_sdpa_int4_decode_static_scratch(
        q_ptr, _lib.TQ_BF16, B, Hq, Hkv, d if head_dim is None else head_dim, 32, P(4096), P(4096),
        P(4096), P(4096), T, P(4096), T, None, 1 / math.sqrt(d), P(4096), None)


def test_static_scratch_rejects_sizes_beyond_the_array():
    """Host-only: sizes whose workspace exceeds the array are rejected before any
    CUDA call (the pointers are only checked for NULL and alignment)."""
    B, Hq, Hkv, d, T = 256, 64, 8, 128, 131072
    assert _lib.decode_workspace_bytes(B, Hq, Hkv, d, T) > _lib.STATIC_SCRATCH_BYTES
    rc = _static_call(None, B, Hq, Hkv, d, T)
    assert rc == _lib.TQ_ERR_SCRATCH_LIMIT
    assert "scratch" in _lib.status_string(rc)


def test_static_scratch_reports_invalid_arguments_first():
    """Host-only: an invalid call is reported as tq_sdpa_int4_decode reports it,
    whatever its sizes: a NULL query or a misaligned pointer is an invalid
    argument, head_dim 64 is unsupported."""
    B, Hq, Hkv, d, T = 256, 64, 8, 128, 131072
    assert _static_call(None, B, Hq, Hkv, d, T, q_ptr=None) == _lib.TQ_ERR_INVALID_ARG
    assert _static_call(None, B, Hq, Hkv, d, T, q_ptr=P(4100)) == _lib.TQ_ERR_INVALID_ARG
    assert _static_call(None, B, Hq, Hkv, d, T, head_dim=64) == _lib.TQ_ERR_UNSUPPORTED


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
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        _lib.sdpa_int4_decode_static_scratch(q, kp, ks, vp, vs, ctx_d, T, sg, scale, got)
        torch.cuda.synchronize()
        if call == 1:  # warmed up: the call takes no device memory
            assert torch.cuda.mem_get_info()[0] == free_before
        got, want = got.cpu().numpy(), want.cpu().numpy()
        assert np.all(np.isfinite(got)), f"call {call}: non-finite output"
        # the same kernels and plan as the caller-workspace call: the same bits
        np.testing.assert_array_equal(got, want, err_msg=f"static scratch call {call}")
        outs.append(got)
    assert not np.array_equal(outs[0], outs[1])   # the two calls used different queries


_SECOND_CONTEXT = textwrap.dedent(r'''
    import ctypes, math, sys
    import numpy as np
    lib = ctypes.CDLL(sys.argv[1])
    cu = ctypes.CDLL("libcuda.so.1")
    def ok(rc, what):
        if rc != 0:
            raise SystemExit(f"{what} failed: {rc}")
    P, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    lib.tq_sdpa_int4_decode_static_scratch.argtypes = [P, i32, i32, i32, i32, i32, i32, P, P, P, P, i64,
                                                       P, i32, P, f32, P, P]
    lib.tq_sdpa_int4_decode.argtypes = [P, i32, i32, i32, i32, i32, i32, P, P, P, P, i64, P, i32, P, f32,
                                        P, P, ctypes.c_size_t, P]
    lib.tq_decode_workspace_bytes.argtypes = [i32] * 5
    lib.tq_decode_workspace_bytes.restype = ctypes.c_size_t
    B, Hq, Hkv, d, T = 1, 16, 2, 128, 3000
    rng = np.random.default_rng(7)
    host = {
        "q": rng.standard_normal((B, Hq, d)).astype(np.float32),
        "kp": rng.integers(0, 256, (B, Hkv, T, d // 2), dtype=np.uint8),
        "vp": rng.integers(0, 256, (B, Hkv, T, d // 2), dtype=np.uint8),
        "ks": rng.uniform(0.05, 0.5, (B, Hkv, T, d // 32)).astype(np.float32),
        "vs": rng.uniform(0.05, 0.5, (B, Hkv, T, d // 32)).astype(np.float32),
        "ctx": np.array([T], dtype=np.int32),
    }
    ok(cu.cuInit(0), "cuInit")
    dev = ctypes.c_int()
    ok(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")
    ws_bytes = lib.tq_decode_workspace_bytes(B, Hq, Hkv, d, T)

    def run_in_current_context():
        ptr = {}
        for name, a in host.items():
            p = ctypes.c_uint64()
            ok(cu.cuMemAlloc_v2(ctypes.byref(p), ctypes.c_size_t(a.nbytes)), "cuMemAlloc")
            ok(cu.cuMemcpyHtoD_v2(p, a.ctypes.data_as(P), ctypes.c_size_t(a.nbytes)), "cuMemcpyHtoD")
            ptr[name] = P(p.value)
        outs = []
        for kind in ("static", "workspace"):
            o = ctypes.c_uint64()
            ok(cu.cuMemAlloc_v2(ctypes.byref(o), ctypes.c_size_t(B * Hq * d * 4)), "cuMemAlloc")
            if kind == "static":
                rc = lib.tq_sdpa_int4_decode_static_scratch(ptr["q"], 0, B, Hq, Hkv, d, 32, ptr["kp"],
                                                            ptr["ks"], ptr["vp"], ptr["vs"], T, ptr["ctx"],
                                                            T, None, 1 / math.sqrt(d), P(o.value), None)
            else:
                w = ctypes.c_uint64()
                ok(cu.cuMemAlloc_v2(ctypes.byref(w), ctypes.c_size_t(ws_bytes)), "cuMemAlloc")
                rc = lib.tq_sdpa_int4_decode(ptr["q"], 0, B, Hq, Hkv, d, 32, ptr["kp"], ptr["ks"], ptr["vp"],
                                             ptr["vs"], T, ptr["ctx"], T, None, 1 / math.sqrt(d), P(o.value),
                                             P(w.value), ws_bytes, None)
            ok(rc, kind + " decode")
            ok(cu.cuCtxSynchronize(), "cuCtxSynchronize")
            out = np.empty((B, Hq, d), dtype=np.float32)
            ok(cu.cuMemcpyDtoH_v2(out.ctypes.data_as(P), P(o.value), ctypes.c_size_t(out.nbytes)), "DtoH")
            outs.append(out)
        return outs

    # a context of the caller's own on the GPU, then the device's primary context
    ctx = P()
    ok(cu.cuCtxCreate_v2(ctypes.byref(ctx), 0, dev), "cuCtxCreate")
    a_static, a_ws = run_in_current_context()
    prim = P()
    ok(cu.cuDevicePrimaryCtxRetain(ctypes.byref(prim), dev), "cuDevicePrimaryCtxRetain")
    ok(cu.cuCtxSetCurrent(prim), "cuCtxSetCurrent")
    b_static, b_ws = run_in_current_context()
    assert np.all(np.isfinite(a_static))
    assert np.array_equal(a_static, a_ws) and np.array_equal(b_static, b_ws), "static != workspace"
    assert np.array_equal(a_static, b_static), "contexts differ"
    print("ok")
''')


@pytest.mark.gpu
def test_static_scratch_in_a_second_cuda_context():
    """The array's device address belongs to the context the call runs in: in a
    context the caller created with the driver API and then in the device's
    primary context, the call gives exactly the caller-workspace result (run in
    a child process that uses no torch)."""
    require_cuda()
    r = subprocess.run([sys.executable, "-c", _SECOND_CONTEXT, _lib.LIB_PATH], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
