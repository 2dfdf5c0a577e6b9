"""C-ABI boundary checks that need no GPU: the library loads, exports every
symbol include/tq.h declares, and rejects invalid calls on the host before
any launch (these calls never reach the CUDA runtime)."""
import ctypes
import os
import re

import pytest

from compressed_domain_attention_tq_b200 import _lib
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "tq.h")


def declared_symbols():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(tq_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from compressed_domain_attention_tq_b200 import build
    build.build()
    return _lib.load()


def test_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert set(_lib.SYMBOLS) <= set(syms) or set(syms) <= set(_lib.SYMBOLS) or syms
    assert len(syms) >= 5
    for s in syms:
        assert hasattr(lib, s), f"libtq.so does not export {s}"


def test_only_declared_symbols_are_exported(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted({ln.split()[-1] for ln in out.splitlines() if " T " in ln and ln.split()[-1].startswith("tq_")})
    assert exported == declared_symbols()


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4):
        assert _lib.status_string(code)
    assert "unknown" in _lib.status_string(7)


@pytest.mark.parametrize("B,Hq,Hkv,d,T", [(1, 4, 4, 128, 4096), (1, 64, 8, 128, 32769),
                                          (1, 64, 8, 128, 131073), (16, 64, 8, 128, 65536),
                                          (4, 32, 16, 256, 65536), (3, 8, 1, 256, 1)])
def test_decode_plan_properties(lib, B, Hq, Hkv, d, T):
    chunk = _lib.decode_chunk_tokens(B, Hq, Hkv, d, T)
    ws = _lib.decode_workspace_bytes(B, Hq, Hkv, d, T)
    # whole pipeline stages of the decode that serves the shape: 384 tokens at d = 128 with
    # 5..8 query heads per kv head, 256 at d = 128 with 1..4, 128 otherwise
    G = Hq // Hkv
    stage = 384 if (d == 128 and 5 <= G <= 8) else 256 if (d == 128 and G <= 4) else 128
    assert chunk % stage == 0 and chunk >= 128
    n_chunks = -(-T // chunk)
    # (sequence, kv head, chunk) items fill their waves over the 148 SMs well
    if T >= 128 * 148:
        items = B * Hkv * n_chunks
        assert items / (-(-items // 148) * 148) >= 0.85
    assert (n_chunks - 1) * chunk < T <= n_chunks * chunk
    header = -(-4 * B // 256) * 256
    assert ws == header + 4 * B * Hq * n_chunks * (d + 4)
    assert _lib.decode_workspace_bytes(B, Hq, Hkv, d, T) == ws          # deterministic


@pytest.mark.parametrize("args", [(0, 8, 8, 128, 10), (1, 6, 4, 128, 10), (1, 8, 8, 96, 10),
                                  (1, 8, 8, 128, 0)])
def test_decode_plan_rejects_invalid_sizes(lib, args):
    assert _lib.decode_workspace_bytes(*args) == 0
    assert _lib.decode_chunk_tokens(*args) == 0


class FakeBuffers:
    """Aligned host memory standing in for device pointers; the calls below
    fail validation before anything dereferences them."""

    def __init__(self):
        self.buf = ctypes.create_string_buffer(1 << 16)
        base = ctypes.addressof(self.buf)
        self.base = (base + 255) // 256 * 256

    def p(self, off=0):
        return ctypes.c_void_p(self.base + off)


def quantize(lib, fb, **kw):
    a = dict(k=fb.p(0), v=fb.p(256), dtype=1, B=1, H=8, n=1, d=128, group=32, pos=fb.p(512),
             signs=None, kp=fb.p(1024), ks=fb.p(2048), vp=fb.p(3072), vs=fb.p(4096), cap=16,
             stream=None)
    a.update(kw)
    return lib.tq_quantize_append(a["k"], a["v"], a["dtype"], a["B"], a["H"], a["n"], a["d"],
                                  a["group"], a["pos"], a["signs"], a["kp"], a["ks"], a["vp"],
                                  a["vs"], a["cap"], a["stream"])


def decode(lib, fb, **kw):
    a = dict(q=fb.p(0), dtype=1, B=1, Hq=8, Hkv=2, d=128, group=32, kp=fb.p(1024), ks=fb.p(2048),
             vp=fb.p(3072), vs=fb.p(4096), cap=64, ctx=fb.p(512), max_ctx=64, signs=None,
             scale=0.125, out=fb.p(8192), ws=fb.p(16384), ws_bytes=1 << 15, stream=None)
    a.update(kw)
    return lib.tq_sdpa_int4_decode(a["q"], a["dtype"], a["B"], a["Hq"], a["Hkv"], a["d"],
                                   a["group"], a["kp"], a["ks"], a["vp"], a["vs"], a["cap"],
                                   a["ctx"], a["max_ctx"], a["signs"], a["scale"], a["out"],
                                   a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), _lib.TQ_ERR_INVALID_ARG), (dict(pos=None), _lib.TQ_ERR_INVALID_ARG),
    (dict(vs=None), _lib.TQ_ERR_INVALID_ARG), (dict(dtype=7), _lib.TQ_ERR_INVALID_ARG),
    (dict(B=0), _lib.TQ_ERR_INVALID_ARG), (dict(n=0), _lib.TQ_ERR_INVALID_ARG),
    (dict(cap=0), _lib.TQ_ERR_INVALID_ARG), (dict(n=20, cap=16), _lib.TQ_ERR_INVALID_ARG),
    (dict(d=64), _lib.TQ_ERR_UNSUPPORTED), (dict(d=96), _lib.TQ_ERR_UNSUPPORTED),
    (dict(group=64), _lib.TQ_ERR_UNSUPPORTED), ("misaligned_k", _lib.TQ_ERR_INVALID_ARG),
    ("misaligned_scales", _lib.TQ_ERR_INVALID_ARG)])
def test_quantize_rejects_on_host(lib, kw, code):
    fb = FakeBuffers()
    if kw == "misaligned_k":
        kw = dict(k=fb.p(2))
    elif kw == "misaligned_scales":
        kw = dict(ks=fb.p(2052))
    assert quantize(lib, fb, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), _lib.TQ_ERR_INVALID_ARG), (dict(ctx=None), _lib.TQ_ERR_INVALID_ARG),
    (dict(out=None), _lib.TQ_ERR_INVALID_ARG), (dict(dtype=2), _lib.TQ_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), _lib.TQ_ERR_INVALID_ARG), (dict(Hq=1, Hkv=2), _lib.TQ_ERR_INVALID_ARG),
    (dict(max_ctx=0), _lib.TQ_ERR_INVALID_ARG), (dict(max_ctx=65), _lib.TQ_ERR_INVALID_ARG),
    (dict(scale=0.0), _lib.TQ_ERR_INVALID_ARG), (dict(scale=-1.0), _lib.TQ_ERR_INVALID_ARG),
    (dict(scale=float("inf")), _lib.TQ_ERR_INVALID_ARG), (dict(scale=float("nan")), _lib.TQ_ERR_INVALID_ARG),
    (dict(d=64), _lib.TQ_ERR_UNSUPPORTED), (dict(group=16), _lib.TQ_ERR_UNSUPPORTED),
    (dict(Hq=34, Hkv=2), _lib.TQ_ERR_UNSUPPORTED), (dict(ws=None), _lib.TQ_ERR_WORKSPACE),
    (dict(ws_bytes=100), _lib.TQ_ERR_WORKSPACE), ("misaligned_q", _lib.TQ_ERR_INVALID_ARG),
    ("misaligned_ws", _lib.TQ_ERR_INVALID_ARG)])
def test_decode_rejects_on_host(lib, kw, code):
    fb = FakeBuffers()
    if kw == "misaligned_q":
        kw = dict(q=fb.p(4))
    elif kw == "misaligned_ws":
        kw = dict(ws=fb.p(16392))
    assert decode(lib, fb, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(packed=None), _lib.TQ_ERR_INVALID_ARG), (dict(scales=None), _lib.TQ_ERR_INVALID_ARG),
    (dict(out=None), _lib.TQ_ERR_INVALID_ARG), (dict(dtype=3), _lib.TQ_ERR_INVALID_ARG),
    (dict(n_seq=0), _lib.TQ_ERR_INVALID_ARG), (dict(rows=0), _lib.TQ_ERR_INVALID_ARG),
    (dict(rows=65, stride=64), _lib.TQ_ERR_INVALID_ARG), (dict(d=80), _lib.TQ_ERR_UNSUPPORTED),
    (dict(d=288), _lib.TQ_ERR_UNSUPPORTED), (dict(group=16), _lib.TQ_ERR_UNSUPPORTED),
    (dict(out=8), _lib.TQ_ERR_INVALID_ARG)])
def test_dequantize_rejects_on_host(lib, kw, code):
    fb = FakeBuffers()
    a = dict(packed=fb.p(1024), scales=fb.p(2048), n_seq=2, rows=64, stride=64, d=128, group=32,
             out=fb.p(4096), dtype=1, stream=None)
    if kw.get("out") == 8:
        kw = dict(out=fb.p(4104))
    a.update(kw)
    assert lib.tq_dequantize(a["packed"], a["scales"], a["n_seq"], a["rows"], a["stride"], a["d"],
                             a["group"], a["out"], a["dtype"], a["stream"]) == code


@pytest.mark.parametrize("kw,code", [
    (dict(k_new=None), _lib.TQ_ERR_INVALID_ARG), (dict(v_new=None), _lib.TQ_ERR_INVALID_ARG),
    (dict(kv_dtype=5), _lib.TQ_ERR_INVALID_ARG), (dict(k_new=20), _lib.TQ_ERR_INVALID_ARG),
    (dict(q=None), _lib.TQ_ERR_INVALID_ARG), (dict(d=64), _lib.TQ_ERR_UNSUPPORTED),
    (dict(max_ctx=65), _lib.TQ_ERR_INVALID_ARG), (dict(ws_bytes=100), _lib.TQ_ERR_WORKSPACE)])
def test_decode_append_rejects_on_host(lib, kw, code):
    fb = FakeBuffers()
    a = dict(q=fb.p(0), dtype=1, k_new=fb.p(32768), v_new=fb.p(36864), kv_dtype=1, B=1, Hq=8, Hkv=2,
             d=128, group=32, kp=fb.p(1024), ks=fb.p(2048), vp=fb.p(3072), vs=fb.p(4096), cap=64,
             ctx=fb.p(512), max_ctx=64, signs=None, scale=0.125, out=fb.p(8192), ws=fb.p(16384),
             ws_bytes=1 << 15, stream=None)
    if kw.get("k_new") == 20:
        kw = dict(k_new=fb.p(32788))
    a.update(kw)
    assert lib.tq_sdpa_int4_decode_append(
        a["q"], a["dtype"], a["k_new"], a["v_new"], a["kv_dtype"], a["B"], a["Hq"], a["Hkv"], a["d"],
        a["group"], a["kp"], a["ks"], a["vp"], a["vs"], a["cap"], a["ctx"], a["max_ctx"], a["signs"],
        a["scale"], a["out"], a["ws"], a["ws_bytes"], a["stream"]) == code


def test_lse_calls_reject_on_host(lib):
    fb = FakeBuffers()
    # merge: NULL, sizes, head_dim, misaligned
    assert lib.tq_merge_lse(None, fb.p(0), 2, 1, 8, 128, fb.p(4096), None) == _lib.TQ_ERR_INVALID_ARG
    assert lib.tq_merge_lse(fb.p(0), fb.p(2048), 0, 1, 8, 128, fb.p(4096), None) == _lib.TQ_ERR_INVALID_ARG
    assert lib.tq_merge_lse(fb.p(0), fb.p(2048), 2, 1, 8, 80, fb.p(4096), None) == _lib.TQ_ERR_UNSUPPORTED
    assert lib.tq_merge_lse(fb.p(0), fb.p(2052), 2, 1, 8, 128, fb.p(4096), None) == _lib.TQ_ERR_INVALID_ARG
    # decode_lse: NULL lse, misaligned lse
    for lse in (None, fb.p(20484)):
        assert lib.tq_sdpa_int4_decode_lse(fb.p(0), 1, 1, 8, 2, 128, 32, fb.p(1024), fb.p(2048),
                                           fb.p(3072), fb.p(4096), 64, fb.p(512), 64, None, 0.125,
                                           fb.p(8192), lse, fb.p(16384), 1 << 15, None) == _lib.TQ_ERR_INVALID_ARG


def test_workspace_size_is_exact_threshold(lib):
    fb = FakeBuffers()
    need = _lib.decode_workspace_bytes(1, 8, 2, 128, 64)
    assert decode(lib, fb, ws_bytes=need - 1) == _lib.TQ_ERR_WORKSPACE


def test_product_path_has_no_oracle_import():
    """The product package never imports the oracle (test infrastructure)."""
    pkg = os.path.join(ROOT, "compressed_domain_attention_tq_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".h", ".cuh", ".cpp")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "oracle.c" not in txt and "liboracle" not in txt, f


def test_codebook_generator_matches_oracle(lib):
    """libtq's Gaussian Max-Lloyd codebook (host code) equals the oracle's in fp32."""
    import numpy as np

    import oracle
    for bits in (2, 3, 4):
        np.testing.assert_array_equal(_lib.lloyd_max_gaussian(bits).numpy(),
                                      oracle.lloyd_max_gaussian(bits).astype(np.float32))


def test_codebook_calls_reject_on_host(lib):
    fb = FakeBuffers()
    args = lambda **kw: dict(dict(k=fb.p(0), v=fb.p(4096), dtype=1, B=1, H=2, n=3, d=128, group=32,
                                  bits=2, levels=fb.p(8192), pos=fb.p(512), signs=None,
                                  kp=fb.p(1024), ks=fb.p(2048), vp=fb.p(3072), vs=fb.p(16384),
                                  cap=16, stream=None), **kw)
    def q(**kw):
        a = args(**kw)
        return lib.tq_quantize_append_cb(a["k"], a["v"], a["dtype"], a["B"], a["H"], a["n"], a["d"],
                                         a["group"], a["bits"], a["levels"], a["pos"], a["signs"],
                                         a["kp"], a["ks"], a["vp"], a["vs"], a["cap"], a["stream"])
    assert q(bits=1) == _lib.TQ_ERR_UNSUPPORTED and q(bits=5) == _lib.TQ_ERR_UNSUPPORTED
    assert q(levels=None) == _lib.TQ_ERR_INVALID_ARG and q(levels=fb.p(8194)) == _lib.TQ_ERR_INVALID_ARG
    assert q(d=96) == _lib.TQ_ERR_UNSUPPORTED and q(k=None) == _lib.TQ_ERR_INVALID_ARG
    assert lib.tq_lloyd_max_gaussian(5, None) == _lib.TQ_ERR_UNSUPPORTED
    assert lib.tq_lloyd_max_gaussian(2, None) == _lib.TQ_ERR_INVALID_ARG
    assert _lib.decode_cb_workspace_bytes(1, 8, 2, 96, 64) == 0
    assert _lib.decode_cb_workspace_bytes(1, 8, 2, 128, 64) > 0
    def dec(bits=2, levels=fb.p(8192), ws_bytes=1 << 15):
        return lib.tq_sdpa_cb_decode(fb.p(0), 1, 1, 8, 2, 128, 32, bits, levels, fb.p(1024),
                                     fb.p(2048), fb.p(3072), fb.p(4096), 64, fb.p(512), 64, None,
                                     0.125, fb.p(8192), fb.p(16384), ws_bytes, None)
    assert dec(bits=7) == _lib.TQ_ERR_UNSUPPORTED
    assert dec(levels=None) == _lib.TQ_ERR_INVALID_ARG
    assert dec(ws_bytes=100) == _lib.TQ_ERR_WORKSPACE


def test_host_step_rejects_on_host(lib):
    fb = FakeBuffers()
    need = lib.tq_decode_append_host_workspace_bytes(1, 8, 2, 128, 64, 1, 1)
    assert need > _lib.decode_workspace_bytes(1, 8, 2, 128, 64)
    assert lib.tq_decode_append_host_workspace_bytes(1, 8, 2, 96, 64, 1, 1) == 0
    def call(q=fb.p(0), out=fb.p(4096), ws_bytes=1 << 16, d=128, qd=1):
        return lib.tq_sdpa_int4_decode_append_host(
            q, qd, fb.p(8192), fb.p(12288), 1, 1, 8, 2, d, 32, fb.p(1024), fb.p(2048), fb.p(3072),
            fb.p(4096), 64, fb.p(512), 64, None, 0.125, out, fb.p(16384), ws_bytes, None)
    assert call(q=None) == _lib.TQ_ERR_INVALID_ARG
    assert call(out=None) == _lib.TQ_ERR_INVALID_ARG
    assert call(d=96) == _lib.TQ_ERR_UNSUPPORTED
    assert call(qd=7) == _lib.TQ_ERR_INVALID_ARG
    assert call(ws_bytes=need - 1) == _lib.TQ_ERR_WORKSPACE


def test_variant_host_steps_reject_on_host(lib):
    """The SRFT and codebook host-buffer steps validate like the int4 one
    before anything is enqueued."""
    fb = FakeBuffers()
    need_s = lib.tq_decode_append_host_srft_workspace_bytes(1, 8, 2, 96, 64, 1, 1)
    need_c = lib.tq_decode_append_host_cb_workspace_bytes(1, 8, 2, 128, 64, 1, 1)
    assert need_s > 0 and need_c > 0
    assert lib.tq_decode_append_host_srft_workspace_bytes(1, 8, 2, 80, 64, 1, 1) == 0
    assert lib.tq_decode_append_host_cb_workspace_bytes(1, 8, 2, 96, 64, 1, 1) == 0

    def srft(q=fb.p(0), out=fb.p(4096), ws_bytes=1 << 16, d=96):
        return lib.tq_sdpa_int4_decode_append_srft_host(
            q, 1, fb.p(8192), fb.p(12288), 1, 1, 8, 2, d, 32, fb.p(1024), fb.p(2048), fb.p(3072),
            fb.p(4096), 64, fb.p(512), 64, None, None, None, 0.125, out, fb.p(16384), ws_bytes,
            None)

    assert srft(q=None) == _lib.TQ_ERR_INVALID_ARG
    assert srft(out=None) == _lib.TQ_ERR_INVALID_ARG
    assert srft(d=80) == _lib.TQ_ERR_UNSUPPORTED
    assert srft(ws_bytes=need_s - 1) == _lib.TQ_ERR_WORKSPACE

    def cb(bits=2, levels=fb.p(256), ws_bytes=1 << 16, d=128, q=fb.p(0)):
        return lib.tq_sdpa_cb_decode_append_host(
            q, 1, fb.p(8192), fb.p(12288), 1, 1, 8, 2, d, 32, bits, levels, fb.p(1024), fb.p(2048),
            fb.p(3072), fb.p(4096), 64, fb.p(512), 64, None, 0.125, fb.p(4096), fb.p(16384),
            ws_bytes, None)

    assert cb(bits=5) == _lib.TQ_ERR_UNSUPPORTED
    assert cb(d=96) == _lib.TQ_ERR_UNSUPPORTED
    assert cb(q=None) == _lib.TQ_ERR_INVALID_ARG
    assert cb(ws_bytes=need_c - 1) == _lib.TQ_ERR_WORKSPACE
    assert cb(levels=None) == _lib.TQ_ERR_INVALID_ARG
