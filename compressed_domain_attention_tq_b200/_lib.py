"""ctypes binding of libtq (include/tq.h).  Argument marshalling only: every
step of quantization and attention runs in the CUDA kernels of libtq.so.

There is no fallback: if libtq.so is missing or no CUDA device is present the
calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtq.so")

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_WORKSPACE, TQ_ERR_CUDA = 0, -1, -2, -3, -4
TQ_ERR_SCRATCH_LIMIT = -5
STATIC_SCRATCH_BYTES = 8 << 20   # TQ_STATIC_SCRATCH_BYTES in include/tq.h
TQ_F32, TQ_BF16 = 0, 1

SYMBOLS = ("tq_quantize_append", "tq_decode_workspace_bytes", "tq_decode_chunk_tokens",
           "tq_sdpa_int4_decode", "tq_sdpa_int4_decode_append", "tq_sdpa_int4_decode_lse",
           "tq_merge_lse", "tq_sdpa_int4_decode_static_scratch", "tq_dequantize",
           "tq_decode_srft_workspace_bytes", "tq_quantize_append_srft", "tq_sdpa_int4_decode_srft",
           "tq_sdpa_int4_decode_append_srft", "tq_lloyd_max_gaussian", "tq_decode_cb_workspace_bytes",
           "tq_quantize_append_cb", "tq_sdpa_cb_decode", "tq_sdpa_cb_decode_append",
           "tq_sdpa_int4_decode_srft_lse", "tq_sdpa_cb_decode_lse",
           "tq_decode_append_host_workspace_bytes", "tq_sdpa_int4_decode_append_host",
           "tq_decode_append_host_srft_workspace_bytes", "tq_sdpa_int4_decode_append_srft_host",
           "tq_decode_append_host_cb_workspace_bytes", "tq_sdpa_cb_decode_append_host",
           "tq_uniform_levels", "tq_quantize_append_uniform", "tq_sdpa_uniform_decode_append",
           "tq_sdpa_uniform_decode_append_host", "tq_status_string")

_lib = None


class TQError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def load() -> ctypes.CDLL:
    """Load libtq.so (built in-tree by compressed_domain_attention_tq_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: run `python -m compressed_domain_attention_tq_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    lib.tq_quantize_append.argtypes = [P, P, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, i64, P]
    lib.tq_quantize_append.restype = i32
    lib.tq_decode_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    lib.tq_decode_workspace_bytes.restype = sz
    lib.tq_decode_chunk_tokens.argtypes = [i32, i32, i32, i32, i32]
    lib.tq_decode_chunk_tokens.restype = i32
    lib.tq_sdpa_int4_decode.argtypes = [P, i32, i32, i32, i32, i32, i32, P, P, P, P, i64, P, i32,
                                        P, f32, P, P, sz, P]
    lib.tq_sdpa_int4_decode.restype = i32
    lib.tq_sdpa_int4_decode_append.argtypes = [P, i32, P, P, i32, i32, i32, i32, i32, i32, P, P, P, P,
                                               i64, P, i32, P, f32, P, P, sz, P]
    lib.tq_sdpa_int4_decode_append.restype = i32
    lib.tq_sdpa_int4_decode_lse.argtypes = [P, i32, i32, i32, i32, i32, i32, P, P, P, P, i64, P, i32,
                                            P, f32, P, P, P, sz, P]
    lib.tq_sdpa_int4_decode_lse.restype = i32
    lib.tq_merge_lse.argtypes = [P, P, i32, i32, i32, i32, P, P]
    lib.tq_merge_lse.restype = i32
    lib.tq_sdpa_int4_decode_static_scratch.argtypes = [P, i32, i32, i32, i32, i32, i32, P, P, P, P,
                                                       i64, P, i32, P, f32, P, P]
    lib.tq_sdpa_int4_decode_static_scratch.restype = i32
    lib.tq_dequantize.argtypes = [P, P, i32, i32, i64, i32, i32, P, i32, P]
    lib.tq_dequantize.restype = i32
    lib.tq_decode_srft_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    lib.tq_decode_srft_workspace_bytes.restype = sz
    lib.tq_quantize_append_srft.argtypes = [P, P, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P,
                                            P, i64, P]
    lib.tq_quantize_append_srft.restype = i32
    lib.tq_sdpa_int4_decode_srft.argtypes = [P, i32, i32, i32, i32, i32, i32, P, P, P, P, i64, P, i32,
                                             P, P, P, f32, P, P, sz, P]
    lib.tq_sdpa_int4_decode_srft.restype = i32
    lib.tq_sdpa_int4_decode_append_srft.argtypes = [P, i32, P, P, i32, i32, i32, i32, i32, i32, P, P,
                                                    P, P, i64, P, i32, P, P, P, f32, P, P, sz, P]
    lib.tq_sdpa_int4_decode_append_srft.restype = i32
    lib.tq_lloyd_max_gaussian.argtypes = [i32, P]
    lib.tq_lloyd_max_gaussian.restype = i32
    lib.tq_decode_cb_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    lib.tq_decode_cb_workspace_bytes.restype = sz
    lib.tq_quantize_append_cb.argtypes = [P, P, i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P,
                                          P, i64, P]
    lib.tq_quantize_append_cb.restype = i32
    lib.tq_sdpa_cb_decode.argtypes = [P, i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, i64, P,
                                      i32, P, f32, P, P, sz, P]
    lib.tq_sdpa_cb_decode.restype = i32
    lib.tq_sdpa_cb_decode_append.argtypes = [P, i32, P, P, i32, i32, i32, i32, i32, i32, i32, P, P,
                                             P, P, P, i64, P, i32, P, f32, P, P, sz, P]
    lib.tq_sdpa_cb_decode_append.restype = i32
    lib.tq_sdpa_int4_decode_srft_lse.argtypes = [P, i32, i32, i32, i32, i32, i32, P, P, P, P, i64,
                                                 P, i32, P, P, P, f32, P, P, P, sz, P]
    lib.tq_sdpa_int4_decode_srft_lse.restype = i32
    lib.tq_sdpa_cb_decode_lse.argtypes = [P, i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, i64, P,
                                          i32, P, f32, P, P, P, sz, P]
    lib.tq_sdpa_cb_decode_lse.restype = i32
    lib.tq_decode_append_host_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32]
    lib.tq_decode_append_host_workspace_bytes.restype = sz
    lib.tq_sdpa_int4_decode_append_host.argtypes = [P, i32, P, P, i32, i32, i32, i32, i32, i32, P,
                                                    P, P, P, i64, P, i32, P, f32, P, P, sz, P]
    lib.tq_sdpa_int4_decode_append_host.restype = i32
    for name in ("tq_decode_append_host_srft_workspace_bytes", "tq_decode_append_host_cb_workspace_bytes"):
        getattr(lib, name).argtypes = [i32, i32, i32, i32, i32, i32, i32]
        getattr(lib, name).restype = sz
    lib.tq_sdpa_int4_decode_append_srft_host.argtypes = [P, i32, P, P, i32, i32, i32, i32, i32, i32,
                                                         P, P, P, P, i64, P, i32, P, P, P, f32, P, P,
                                                         sz, P]
    lib.tq_sdpa_int4_decode_append_srft_host.restype = i32
    lib.tq_sdpa_cb_decode_append_host.argtypes = [P, i32, P, P, i32, i32, i32, i32, i32, i32, i32, P,
                                                  P, P, P, P, i64, P, i32, P, f32, P, P, sz, P]
    lib.tq_sdpa_cb_decode_append_host.restype = i32
    lib.tq_uniform_levels.argtypes = [i32, P]
    lib.tq_uniform_levels.restype = i32
    lib.tq_quantize_append_uniform.argtypes = [P, P, i32, i32, i32, i32, i32, i32, i32, P, P, P, P,
                                               P, P, i64, P]
    lib.tq_quantize_append_uniform.restype = i32
    lib.tq_sdpa_uniform_decode_append.argtypes = lib.tq_sdpa_cb_decode_append.argtypes
    lib.tq_sdpa_uniform_decode_append.restype = i32
    lib.tq_sdpa_uniform_decode_append_host.argtypes = lib.tq_sdpa_cb_decode_append_host.argtypes
    lib.tq_sdpa_uniform_decode_append_host.restype = i32
    lib.tq_status_string.argtypes = [i32]
    lib.tq_status_string.restype = ctypes.c_char_p
    lib.tq_set_test_hooks.argtypes = [ctypes.c_uint32]
    lib.tq_set_test_hooks.restype = None
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().tq_status_string(status).decode()


# tq_set_test_hooks bits (include/tq.h); testing and kernel comparisons only
TEST_HOOK_FAIL_LAUNCH = 1
TEST_HOOK_STARVE_PIPELINE = 2
TEST_HOOK_TCGEN05_DECODE = 4
TEST_HOOK_BUTTERFLY_QUANTIZE = 8


def set_test_hooks(hooks: int) -> None:
    """Process-wide test switches of libtq (0 = normal operation)."""
    load().tq_set_test_hooks(int(hooks))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TQ_F32
    if t.dtype == torch.bfloat16:
        return TQ_BF16
    raise TypeError(f"expected float32 or bfloat16, got {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("all tensors must be contiguous CUDA tensors")


def quantize_append(k, v, pos, signs, k_packed, k_scales, v_packed, v_scales, stream=None):
    """Quantize k, v [B][Hkv][n_new][d] into cache rows pos[b] .. pos[b]+n_new-1."""
    _need_cuda(k, v, pos, signs, k_packed, k_scales, v_packed, v_scales)
    B, H, n, d = k.shape
    rc = load().tq_quantize_append(_ptr(k), _ptr(v), _dtype_code(k), B, H, n, d, 32, _ptr(pos),
                                   _ptr(signs), _ptr(k_packed), _ptr(k_scales), _ptr(v_packed),
                                   _ptr(v_scales), k_packed.shape[2], _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_quantize_append")


def decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_ctx) -> int:
    return int(load().tq_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_ctx))


def decode_chunk_tokens(batch, num_q_heads, num_kv_heads, head_dim, max_ctx) -> int:
    return int(load().tq_decode_chunk_tokens(batch, num_q_heads, num_kv_heads, head_dim, max_ctx))


def sdpa_int4_decode(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, max_ctx, signs,
                     attn_scale, out, workspace, stream=None):
    """out[B][Hq][d] (fp32) = attention of q over the packed cache (see include/tq.h)."""
    _need_cuda(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, out, workspace)
    B, Hq, d = q.shape
    Hkv = k_packed.shape[1]
    rc = load().tq_sdpa_int4_decode(_ptr(q), _dtype_code(q), B, Hq, Hkv, d, 32, _ptr(k_packed),
                                    _ptr(k_scales), _ptr(v_packed), _ptr(v_scales),
                                    k_packed.shape[2], _ptr(ctx_lens), int(max_ctx), _ptr(signs),
                                    float(attn_scale), _ptr(out), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_sdpa_int4_decode")


def sdpa_int4_decode_lse(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, max_ctx, signs,
                         attn_scale, out, lse, workspace, stream=None):
    """sdpa_int4_decode that also writes lse[B][Hq][2] = (max in log2 units, sum) per head."""
    _need_cuda(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, out, lse, workspace)
    B, Hq, d = q.shape
    Hkv = k_packed.shape[1]
    rc = load().tq_sdpa_int4_decode_lse(_ptr(q), _dtype_code(q), B, Hq, Hkv, d, 32, _ptr(k_packed),
                                        _ptr(k_scales), _ptr(v_packed), _ptr(v_scales),
                                        k_packed.shape[2], _ptr(ctx_lens), int(max_ctx), _ptr(signs),
                                        float(attn_scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_sdpa_int4_decode_lse")


def merge_lse(outs, lses, out, stream=None):
    """out[B][Hq][d] from outs[R][B][Hq][d] and lses[R][B][Hq][2] over R disjoint context parts."""
    _need_cuda(outs, lses, out)
    R, B, Hq, d = outs.shape
    rc = load().tq_merge_lse(_ptr(outs), _ptr(lses), R, B, Hq, d, _ptr(out), _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_merge_lse")


def _decode_append_args(q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens, max_ctx,
                        signs, attn_scale, out, workspace, stream):
    _need_cuda(q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, out, workspace)
    if k_new.dtype != v_new.dtype:
        raise TypeError("k_new and v_new must share dtype")
    B, Hq, d = q.shape
    Hkv = k_packed.shape[1]
    i32, f32, sz = ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    return (_ptr(q), i32(_dtype_code(q)), _ptr(k_new), _ptr(v_new), i32(_dtype_code(k_new)), i32(B),
            i32(Hq), i32(Hkv), i32(d), i32(32), _ptr(k_packed), _ptr(k_scales), _ptr(v_packed),
            _ptr(v_scales), ctypes.c_int64(k_packed.shape[2]), _ptr(ctx_lens), i32(int(max_ctx)),
            _ptr(signs), f32(float(attn_scale)), _ptr(out), _ptr(workspace),
            sz(workspace.numel() * workspace.element_size()), _stream(stream))


def sdpa_int4_decode_append(q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens,
                            max_ctx, signs, attn_scale, out, workspace, stream=None):
    """One decode step: quantize k_new, v_new [B][Hkv][1][d] into row ctx_lens[b]-1
    of the cache, then out[B][Hq][d] = attention of q over rows 0..ctx_lens[b]-1."""
    rc = load().tq_sdpa_int4_decode_append(*_decode_append_args(
        q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens, max_ctx, signs,
        attn_scale, out, workspace, stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_sdpa_int4_decode_append")


class BoundCall:
    """A libtq call whose arguments were checked and marshalled once: each call
    enqueues the same work again on the same buffers and stream (a decode loop
    that refills its input buffers and reuses its output).  Saves the per-call
    Python work of building the C arguments."""

    def __init__(self, fn, args, where, keep):
        self._fn, self._args, self._where = fn, args, where
        self._keep = keep  # the tensors behind the pointers stay alive with the call

    def __call__(self):
        rc = self._fn(*self._args)
        if rc != TQ_OK:
            raise TQError(rc, self._where)


class GraphedCall:
    """A prepared call captured once into a CUDA graph: each call replays the
    graph on the current stream, so the work the library call enqueues is
    launched at once instead of call by call from the host.  make_call(stream)
    builds the call on a stream; it runs once uncaptured first (the library's
    one-time per-kernel set-up), then is captured.  Host buffers must be
    pinned; a replay uses what the buffers hold when it runs."""

    def __init__(self, make_call):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            first = make_call(side)
            first()
        torch.cuda.current_stream().wait_stream(side)
        self._graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self._graph):
            captured = make_call(torch.cuda.current_stream())
            captured()
        self._keep = (first, captured)

    def __call__(self):
        self._graph.replay()


def bind_sdpa_int4_decode_append(q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens,
                                 max_ctx, signs, attn_scale, out, workspace, stream=None) -> BoundCall:
    """sdpa_int4_decode_append prepared for repeated calls on the same buffers."""
    args = _decode_append_args(q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens,
                               max_ctx, signs, attn_scale, out, workspace, stream)
    keep = (q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, out, workspace)
    return BoundCall(load().tq_sdpa_int4_decode_append, args, "tq_sdpa_int4_decode_append", keep)


def sdpa_int4_decode_static_scratch(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, max_ctx,
                                    signs, attn_scale, out, stream=None):
    """sdpa_int4_decode using libtq's built-in device scratch instead of a
    caller workspace (for callers that cannot allocate; see include/tq.h)."""
    _need_cuda(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, out)
    B, Hq, d = q.shape
    Hkv = k_packed.shape[1]
    rc = load().tq_sdpa_int4_decode_static_scratch(
        _ptr(q), _dtype_code(q), B, Hq, Hkv, d, 32, _ptr(k_packed), _ptr(k_scales),
        _ptr(v_packed), _ptr(v_scales), k_packed.shape[2], _ptr(ctx_lens), int(max_ctx),
        _ptr(signs), float(attn_scale), _ptr(out), _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_sdpa_int4_decode_static_scratch")


def dequantize(packed, scales, rows, out, stream=None):
    """out[B][Hkv][rows][d] (fp32 or bf16) = scale * code of rows 0 .. rows-1 of
    each sequence of a packed cache [B][Hkv][capacity][d/2] (rotated basis)."""
    _need_cuda(packed, scales, out)
    B, H, cap, half = packed.shape
    rc = load().tq_dequantize(_ptr(packed), _ptr(scales), B * H, int(rows), cap, 2 * half, 32,
                              _ptr(out), _dtype_code(out), _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_dequantize")


# ------------------------------------------------------------------ SRFT variant
# The rotation of "SRFT + int4 KV-cache on Apple Silicon" (core method): the
# orthonormal discrete Hartley transform with random signs, then per-coordinate
# scales lambda_k / lambda_v (float32 [d] CUDA tensors, or None for ones).

def decode_srft_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_ctx) -> int:
    return int(load().tq_decode_srft_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim,
                                                     max_ctx))


def quantize_append_srft(k, v, pos, signs, lambda_k, lambda_v, k_packed, k_scales, v_packed,
                         v_scales, stream=None):
    """Quantize k, v [B][Hkv][n_new][d] with the SRFT rotation into rows pos[b] .. pos[b]+n_new-1."""
    _need_cuda(k, v, pos, signs, lambda_k, lambda_v, k_packed, k_scales, v_packed, v_scales)
    B, H, n, d = k.shape
    rc = load().tq_quantize_append_srft(_ptr(k), _ptr(v), _dtype_code(k), B, H, n, d, 32, _ptr(pos),
                                        _ptr(signs), _ptr(lambda_k), _ptr(lambda_v),
                                        _ptr(k_packed), _ptr(k_scales), _ptr(v_packed),
                                        _ptr(v_scales), k_packed.shape[2], _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_quantize_append_srft")


def sdpa_int4_decode_srft(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, max_ctx, signs,
                          lambda_k, lambda_v, attn_scale, out, workspace, stream=None):
    """out[B][Hq][d] (fp32, unrotated) = attention of q over an SRFT cache."""
    _need_cuda(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, lambda_k, lambda_v, out,
               workspace)
    B, Hq, d = q.shape
    Hkv = k_packed.shape[1]
    rc = load().tq_sdpa_int4_decode_srft(
        _ptr(q), _dtype_code(q), B, Hq, Hkv, d, 32, _ptr(k_packed), _ptr(k_scales), _ptr(v_packed),
        _ptr(v_scales), k_packed.shape[2], _ptr(ctx_lens), int(max_ctx), _ptr(signs),
        _ptr(lambda_k), _ptr(lambda_v), float(attn_scale), _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_sdpa_int4_decode_srft")


def sdpa_int4_decode_append_srft(q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens,
                                 max_ctx, signs, lambda_k, lambda_v, attn_scale, out, workspace,
                                 stream=None):
    """One decode step over an SRFT cache (append of k_new, v_new at row ctx_lens[b]-1, then attend)."""
    _need_cuda(q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, lambda_k,
               lambda_v, out, workspace)
    if k_new.dtype != v_new.dtype:
        raise TypeError("k_new and v_new must share dtype")
    B, Hq, d = q.shape
    Hkv = k_packed.shape[1]
    rc = load().tq_sdpa_int4_decode_append_srft(
        _ptr(q), _dtype_code(q), _ptr(k_new), _ptr(v_new), _dtype_code(k_new), B, Hq, Hkv, d, 32,
        _ptr(k_packed), _ptr(k_scales), _ptr(v_packed), _ptr(v_scales), k_packed.shape[2],
        _ptr(ctx_lens), int(max_ctx), _ptr(signs), _ptr(lambda_k), _ptr(lambda_v),
        float(attn_scale), _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_sdpa_int4_decode_append_srft")


# ------------------------------------------------------------ codebook variant
# AdapTQ's Max-Lloyd codebook indices at 2, 3 or 4 bits (see include/tq.h).

def lloyd_max_gaussian(bits: int) -> torch.Tensor:
    """The Gaussian Max-Lloyd codebook (float32 CPU tensor of 2**bits levels), from libtq."""
    out = torch.empty(1 << bits, dtype=torch.float32)
    rc = load().tq_lloyd_max_gaussian(bits, ctypes.c_void_p(out.data_ptr()))
    if rc != TQ_OK:
        raise TQError(rc, "tq_lloyd_max_gaussian")
    return out


def uniform_levels(bits: int) -> torch.Tensor:
    """The levels of a uniform low-bit cache, u - (2^(bits-1) - 1) (float32 CPU tensor), from libtq."""
    out = torch.empty(1 << bits, dtype=torch.float32)
    rc = load().tq_uniform_levels(bits, ctypes.c_void_p(out.data_ptr()))
    if rc != TQ_OK:
        raise TQError(rc, "tq_uniform_levels")
    return out


def quantize_append_uniform(k, v, pos, signs, bits, k_packed, k_scales, v_packed, v_scales,
                            stream=None):
    """Quantize k, v [B][Hkv][n_new][d] into uniform low-bit cache rows pos[b] .. pos[b]+n_new-1."""
    _need_cuda(k, v, pos, signs, k_packed, k_scales, v_packed, v_scales)
    B, H, n, d = k.shape
    rc = load().tq_quantize_append_uniform(_ptr(k), _ptr(v), _dtype_code(k), B, H, n, d, 32, int(bits),
                                           _ptr(pos), _ptr(signs), _ptr(k_packed), _ptr(k_scales),
                                           _ptr(v_packed), _ptr(v_scales), k_packed.shape[2],
                                           _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_quantize_append_uniform")


def sdpa_uniform_decode_append(q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens,
                               max_ctx, signs, bits, levels, attn_scale, out, workspace, stream=None):
    """One decode step over a uniform low-bit cache (levels = uniform_levels(bits) on the device)."""
    _need_cuda(q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, levels,
               out, workspace)
    if k_new.dtype != v_new.dtype:
        raise TypeError("k_new and v_new must share dtype")
    B, Hq, d = q.shape
    Hkv = k_packed.shape[1]
    rc = load().tq_sdpa_uniform_decode_append(
        _ptr(q), _dtype_code(q), _ptr(k_new), _ptr(v_new), _dtype_code(k_new), B, Hq, Hkv, d, 32,
        int(bits), _ptr(levels), _ptr(k_packed), _ptr(k_scales), _ptr(v_packed), _ptr(v_scales),
        k_packed.shape[2], _ptr(ctx_lens), int(max_ctx), _ptr(signs), float(attn_scale), _ptr(out),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_sdpa_uniform_decode_append")


def decode_cb_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_ctx) -> int:
    return int(load().tq_decode_cb_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_ctx))


def quantize_append_cb(k, v, pos, signs, bits, levels, k_packed, k_scales, v_packed, v_scales,
                       stream=None):
    """Quantize k, v [B][Hkv][n_new][d] into codebook-cache rows pos[b] .. pos[b]+n_new-1."""
    _need_cuda(k, v, pos, signs, levels, k_packed, k_scales, v_packed, v_scales)
    B, H, n, d = k.shape
    rc = load().tq_quantize_append_cb(_ptr(k), _ptr(v), _dtype_code(k), B, H, n, d, 32, int(bits),
                                      _ptr(levels), _ptr(pos), _ptr(signs), _ptr(k_packed),
                                      _ptr(k_scales), _ptr(v_packed), _ptr(v_scales),
                                      k_packed.shape[2], _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_quantize_append_cb")


def sdpa_cb_decode(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, max_ctx, signs, bits,
                   levels, attn_scale, out, workspace, stream=None):
    """out[B][Hq][d] (fp32) = attention of q over a codebook cache."""
    _need_cuda(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, levels, out, workspace)
    B, Hq, d = q.shape
    Hkv = k_packed.shape[1]
    rc = load().tq_sdpa_cb_decode(
        _ptr(q), _dtype_code(q), B, Hq, Hkv, d, 32, int(bits), _ptr(levels), _ptr(k_packed),
        _ptr(k_scales), _ptr(v_packed), _ptr(v_scales), k_packed.shape[2], _ptr(ctx_lens),
        int(max_ctx), _ptr(signs), float(attn_scale), _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_sdpa_cb_decode")


def sdpa_cb_decode_append(q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens,
                          max_ctx, signs, bits, levels, attn_scale, out, workspace, stream=None):
    """One decode step over a codebook cache (append at row ctx_lens[b]-1, then attend)."""
    _need_cuda(q, k_new, v_new, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, levels,
               out, workspace)
    if k_new.dtype != v_new.dtype:
        raise TypeError("k_new and v_new must share dtype")
    B, Hq, d = q.shape
    Hkv = k_packed.shape[1]
    rc = load().tq_sdpa_cb_decode_append(
        _ptr(q), _dtype_code(q), _ptr(k_new), _ptr(v_new), _dtype_code(k_new), B, Hq, Hkv, d, 32,
        int(bits), _ptr(levels), _ptr(k_packed), _ptr(k_scales), _ptr(v_packed), _ptr(v_scales),
        k_packed.shape[2], _ptr(ctx_lens), int(max_ctx), _ptr(signs), float(attn_scale), _ptr(out),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_sdpa_cb_decode_append")


def sdpa_int4_decode_srft_lse(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, max_ctx, signs,
                              lambda_k, lambda_v, attn_scale, out, lse, workspace, stream=None):
    """sdpa_int4_decode_srft that also writes lse[B][Hq][2] per head."""
    _need_cuda(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, lambda_k, lambda_v, out,
               lse, workspace)
    B, Hq, d = q.shape
    Hkv = k_packed.shape[1]
    rc = load().tq_sdpa_int4_decode_srft_lse(
        _ptr(q), _dtype_code(q), B, Hq, Hkv, d, 32, _ptr(k_packed), _ptr(k_scales), _ptr(v_packed),
        _ptr(v_scales), k_packed.shape[2], _ptr(ctx_lens), int(max_ctx), _ptr(signs),
        _ptr(lambda_k), _ptr(lambda_v), float(attn_scale), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_sdpa_int4_decode_srft_lse")


def sdpa_cb_decode_lse(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, max_ctx, signs, bits,
                       levels, attn_scale, out, lse, workspace, stream=None):
    """sdpa_cb_decode that also writes lse[B][Hq][2] per head."""
    _need_cuda(q, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, levels, out, lse, workspace)
    B, Hq, d = q.shape
    Hkv = k_packed.shape[1]
    rc = load().tq_sdpa_cb_decode_lse(
        _ptr(q), _dtype_code(q), B, Hq, Hkv, d, 32, int(bits), _ptr(levels), _ptr(k_packed),
        _ptr(k_scales), _ptr(v_packed), _ptr(v_scales), k_packed.shape[2], _ptr(ctx_lens),
        int(max_ctx), _ptr(signs), float(attn_scale), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != TQ_OK:
        raise TQError(rc, "tq_sdpa_cb_decode_lse")


# -------------------------------------------------- host-buffer decode step

def decode_append_host_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_ctx,
                                       q_dtype=torch.bfloat16, kv_dtype=torch.bfloat16,
                                       kind="int4") -> int:
    """Workspace bytes of a host-buffer step; kind: "int4", "srft" or "cb"."""
    code = {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16}
    fn = {"int4": "tq_decode_append_host_workspace_bytes",
          "srft": "tq_decode_append_host_srft_workspace_bytes",
          "cb": "tq_decode_append_host_cb_workspace_bytes"}[kind]
    return int(getattr(load(), fn)(batch, num_q_heads, num_kv_heads, head_dim, max_ctx,
                                   code[q_dtype], code[kv_dtype]))


def _host(*ts):
    for t in ts:
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("the step's inputs and output must be contiguous host tensors")


def bind_sdpa_int4_decode_append_host(q_host, k_new_host, v_new_host, k_packed, k_scales, v_packed,
                                      v_scales, ctx_lens, max_ctx, signs, attn_scale, out_host,
                                      workspace, stream=None) -> BoundCall:
    """A prepared decode step whose q, k_new, v_new and output live in (pinned) host
    memory: each call enqueues their copies, the step and the copy back on the stream."""
    _host(q_host, k_new_host, v_new_host, out_host)
    _need_cuda(k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, workspace)
    if k_new_host.dtype != v_new_host.dtype:
        raise TypeError("k_new and v_new must share dtype")
    B, Hq, d = q_host.shape
    Hkv = k_packed.shape[1]
    i32, f32, sz = ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    args = (_ptr(q_host), i32(_dtype_code(q_host)), _ptr(k_new_host), _ptr(v_new_host),
            i32(_dtype_code(k_new_host)), i32(B), i32(Hq), i32(Hkv), i32(d), i32(32), _ptr(k_packed),
            _ptr(k_scales), _ptr(v_packed), _ptr(v_scales), ctypes.c_int64(k_packed.shape[2]),
            _ptr(ctx_lens), i32(int(max_ctx)), _ptr(signs), f32(float(attn_scale)), _ptr(out_host),
            _ptr(workspace), sz(workspace.numel() * workspace.element_size()), _stream(stream))
    keep = (q_host, k_new_host, v_new_host, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs,
            out_host, workspace)
    return BoundCall(load().tq_sdpa_int4_decode_append_host, args,
                     "tq_sdpa_int4_decode_append_host", keep)


def bind_sdpa_int4_decode_append_srft_host(q_host, k_new_host, v_new_host, k_packed, k_scales,
                                           v_packed, v_scales, ctx_lens, max_ctx, signs, lambda_k,
                                           lambda_v, attn_scale, out_host, workspace,
                                           stream=None) -> BoundCall:
    """bind_sdpa_int4_decode_append_host for an SRFT-rotated cache."""
    _host(q_host, k_new_host, v_new_host, out_host)
    _need_cuda(k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, lambda_k, lambda_v,
               workspace)
    if k_new_host.dtype != v_new_host.dtype:
        raise TypeError("k_new and v_new must share dtype")
    B, Hq, d = q_host.shape
    Hkv = k_packed.shape[1]
    i32, f32, sz = ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    args = (_ptr(q_host), i32(_dtype_code(q_host)), _ptr(k_new_host), _ptr(v_new_host),
            i32(_dtype_code(k_new_host)), i32(B), i32(Hq), i32(Hkv), i32(d), i32(32), _ptr(k_packed),
            _ptr(k_scales), _ptr(v_packed), _ptr(v_scales), ctypes.c_int64(k_packed.shape[2]),
            _ptr(ctx_lens), i32(int(max_ctx)), _ptr(signs), _ptr(lambda_k), _ptr(lambda_v),
            f32(float(attn_scale)), _ptr(out_host), _ptr(workspace),
            sz(workspace.numel() * workspace.element_size()), _stream(stream))
    keep = (q_host, k_new_host, v_new_host, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs,
            lambda_k, lambda_v, out_host, workspace)
    return BoundCall(load().tq_sdpa_int4_decode_append_srft_host, args,
                     "tq_sdpa_int4_decode_append_srft_host", keep)


def bind_sdpa_cb_decode_append_host(q_host, k_new_host, v_new_host, k_packed, k_scales, v_packed,
                                    v_scales, ctx_lens, max_ctx, signs, bits, levels, attn_scale,
                                    out_host, workspace, stream=None, uniform=False) -> BoundCall:
    """bind_sdpa_int4_decode_append_host for a codebook cache (uniform: a uniform
    low-bit cache, tq_sdpa_uniform_decode_append_host)."""
    _host(q_host, k_new_host, v_new_host, out_host)
    _need_cuda(k_packed, k_scales, v_packed, v_scales, ctx_lens, signs, levels, workspace)
    if k_new_host.dtype != v_new_host.dtype:
        raise TypeError("k_new and v_new must share dtype")
    B, Hq, d = q_host.shape
    Hkv = k_packed.shape[1]
    i32, f32, sz = ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    args = (_ptr(q_host), i32(_dtype_code(q_host)), _ptr(k_new_host), _ptr(v_new_host),
            i32(_dtype_code(k_new_host)), i32(B), i32(Hq), i32(Hkv), i32(d), i32(32), i32(int(bits)),
            _ptr(levels), _ptr(k_packed), _ptr(k_scales), _ptr(v_packed), _ptr(v_scales),
            ctypes.c_int64(k_packed.shape[2]), _ptr(ctx_lens), i32(int(max_ctx)), _ptr(signs),
            f32(float(attn_scale)), _ptr(out_host), _ptr(workspace),
            sz(workspace.numel() * workspace.element_size()), _stream(stream))
    keep = (q_host, k_new_host, v_new_host, k_packed, k_scales, v_packed, v_scales, ctx_lens, signs,
            levels, out_host, workspace)
    name = "tq_sdpa_uniform_decode_append_host" if uniform else "tq_sdpa_cb_decode_append_host"
    return BoundCall(getattr(load(), name), args, name, keep)
