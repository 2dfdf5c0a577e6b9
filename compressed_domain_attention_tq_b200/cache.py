"""Int4KVCache: the packed int4 KV cache of one attention layer on one GPU.

The call shape follows the AdapTQ engine (AdapTQ post, section "native Python
API": an engine of fixed dim, heads and capacity with append(k, v) and
compute(q)).  Torch only provides the device buffers and the stream; both
operations run in libtq's kernels.

rotation="hadamard" (default): signs + Walsh-Hadamard rotation (or none when
signs is None), head_dim 128 or 256.  rotation="srft": the SRFT post's variant
(core method): signs + orthonormal discrete Hartley transform, then the
per-coordinate scales lambda_k / lambda_v (float32 [d], None = ones); head_dim
any multiple of 32 up to 256.
"""
from __future__ import annotations

import math

import torch

from . import _lib


class Int4KVCache:
    def __init__(self, batch: int, num_kv_heads: int, head_dim: int, capacity: int,
                 device="cuda", signs: torch.Tensor | None = None, rotation: str = "hadamard",
                 lambda_k: torch.Tensor | None = None, lambda_v: torch.Tensor | None = None):
        if head_dim % 32:
            raise ValueError("head_dim must be a multiple of 32")
        if rotation not in ("hadamard", "srft"):
            raise ValueError("rotation must be 'hadamard' or 'srft'")
        if rotation == "hadamard" and (lambda_k is not None or lambda_v is not None):
            raise ValueError("lambda_k / lambda_v belong to the srft rotation")
        self.srft = rotation == "srft"
        self.batch, self.num_kv_heads, self.head_dim, self.capacity = batch, num_kv_heads, head_dim, capacity
        dev = torch.device(device)
        shape = (batch, num_kv_heads, capacity)
        self.k_packed = torch.zeros(*shape, head_dim // 2, dtype=torch.uint8, device=dev)
        self.v_packed = torch.zeros(*shape, head_dim // 2, dtype=torch.uint8, device=dev)
        self.k_scales = torch.zeros(*shape, head_dim // 32, dtype=torch.float32, device=dev)
        self.v_scales = torch.zeros(*shape, head_dim // 32, dtype=torch.float32, device=dev)
        self.signs = None if signs is None else signs.to(device=dev, dtype=torch.int8).contiguous()
        self.lambda_k = None if lambda_k is None else lambda_k.to(device=dev, dtype=torch.float32).contiguous()
        self.lambda_v = None if lambda_v is None else lambda_v.to(device=dev, dtype=torch.float32).contiguous()
        self._ws = None

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.k_packed, self.v_packed, self.k_scales, self.v_scales))

    def append(self, k: torch.Tensor, v: torch.Tensor, pos: torch.Tensor, stream=None) -> None:
        """Quantize k, v [B][Hkv][n][d] into rows pos[b] .. pos[b]+n-1."""
        if self.srft:
            _lib.quantize_append_srft(k, v, pos, self.signs, self.lambda_k, self.lambda_v,
                                      self.k_packed, self.k_scales, self.v_packed, self.v_scales,
                                      stream)
            return
        _lib.quantize_append(k, v, pos, self.signs, self.k_packed, self.k_scales, self.v_packed,
                             self.v_scales, stream)

    def workspace(self, num_q_heads: int, max_ctx: int) -> torch.Tensor:
        sizer = _lib.decode_srft_workspace_bytes if self.srft else _lib.decode_workspace_bytes
        need = sizer(self.batch, num_q_heads, self.num_kv_heads, self.head_dim, max_ctx)
        if need == 0:
            raise ValueError("invalid decode sizes")
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.k_packed.device)
        return self._ws

    def decode(self, q: torch.Tensor, ctx_lens: torch.Tensor, max_ctx: int,
               attn_scale: float | None = None, out: torch.Tensor | None = None, stream=None):
        """Attention of q [B][Hq][d] over rows 0..ctx_lens[b]-1; returns fp32 [B][Hq][d]."""
        if attn_scale is None:
            attn_scale = 1.0 / math.sqrt(self.head_dim)
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        ws = self.workspace(q.shape[1], max_ctx)
        if self.srft:
            _lib.sdpa_int4_decode_srft(q, self.k_packed, self.k_scales, self.v_packed, self.v_scales,
                                       ctx_lens, max_ctx, self.signs, self.lambda_k, self.lambda_v,
                                       attn_scale, out, ws, stream)
            return out
        _lib.sdpa_int4_decode(q, self.k_packed, self.k_scales, self.v_packed, self.v_scales,
                              ctx_lens, max_ctx, self.signs, attn_scale, out, ws, stream)
        return out

    def decode_lse(self, q: torch.Tensor, ctx_lens: torch.Tensor, max_ctx: int, attn_scale: float,
                   out: torch.Tensor, lse: torch.Tensor, stream=None):
        """decode that also writes each head's softmax state lse[B][Hq][2] (for merging
        outputs over disjoint parts of a context)."""
        ws = self.workspace(q.shape[1], max_ctx)
        if self.srft:
            _lib.sdpa_int4_decode_srft_lse(q, self.k_packed, self.k_scales, self.v_packed,
                                           self.v_scales, ctx_lens, max_ctx, self.signs,
                                           self.lambda_k, self.lambda_v, attn_scale, out, lse, ws,
                                           stream)
        else:
            _lib.sdpa_int4_decode_lse(q, self.k_packed, self.k_scales, self.v_packed, self.v_scales,
                                      ctx_lens, max_ctx, self.signs, attn_scale, out, lse, ws, stream)
        return out

    def decode_append(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                      ctx_lens: torch.Tensor, max_ctx: int, attn_scale: float | None = None,
                      out: torch.Tensor | None = None, stream=None):
        """One decode step: append k_new, v_new [B][Hkv][1][d] at row ctx_lens[b]-1, then
        attend q [B][Hq][d] over rows 0..ctx_lens[b]-1 (lengths include the new token)."""
        if attn_scale is None:
            attn_scale = 1.0 / math.sqrt(self.head_dim)
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        ws = self.workspace(q.shape[1], max_ctx)
        if self.srft:
            _lib.sdpa_int4_decode_append_srft(q, k_new, v_new, self.k_packed, self.k_scales,
                                              self.v_packed, self.v_scales, ctx_lens, max_ctx,
                                              self.signs, self.lambda_k, self.lambda_v, attn_scale,
                                              out, ws, stream)
            return out
        _lib.sdpa_int4_decode_append(q, k_new, v_new, self.k_packed, self.k_scales, self.v_packed,
                                     self.v_scales, ctx_lens, max_ctx, self.signs, attn_scale, out,
                                     ws, stream)
        return out

    def bind_decode_append(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                           ctx_lens: torch.Tensor, max_ctx: int, attn_scale: float | None = None,
                           out: torch.Tensor | None = None, stream=None):
        """decode_append prepared once for a serving loop that refills q, k_new, v_new and
        ctx_lens in place: returns (step, out), where step() enqueues one decode step on
        these buffers (the Hadamard-rotated cache; one C call per step)."""
        if self.srft:
            raise NotImplementedError("bind_decode_append runs on Hadamard-rotated caches")
        if attn_scale is None:
            attn_scale = 1.0 / math.sqrt(self.head_dim)
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        ws = self.workspace(q.shape[1], max_ctx)
        step = _lib.bind_sdpa_int4_decode_append(q, k_new, v_new, self.k_packed, self.k_scales,
                                                 self.v_packed, self.v_scales, ctx_lens, max_ctx,
                                                 self.signs, attn_scale, out, ws, stream)
        return step, out

    def bind_decode_append_host(self, q_host: torch.Tensor, k_new_host: torch.Tensor,
                                v_new_host: torch.Tensor, ctx_lens: torch.Tensor, max_ctx: int,
                                out_host: torch.Tensor, attn_scale: float | None = None,
                                stream=None, graph: bool = False):
        """A prepared decode step on HOST buffers (q, k_new, v_new, out; pin them): each
        call of the returned step runs tq_sdpa_int4_decode_append_host (or its SRFT form;
        on pinned, mapped buffers a gather kernel reads the inputs and the merge writes the
        output directly).  graph=True captures that call once into a CUDA graph (after
        running it once) and each call of the step replays the graph on the current stream."""
        if attn_scale is None:
            attn_scale = 1.0 / math.sqrt(self.head_dim)
        need = _lib.decode_append_host_workspace_bytes(self.batch, q_host.shape[1], self.num_kv_heads,
                                                       self.head_dim, max_ctx, q_host.dtype,
                                                       k_new_host.dtype,
                                                       "srft" if self.srft else "int4")
        if need == 0:
            raise ValueError("invalid decode sizes")
        ws = torch.empty(need, dtype=torch.uint8, device=self.k_packed.device)

        def make(s):
            if self.srft:
                return _lib.bind_sdpa_int4_decode_append_srft_host(
                    q_host, k_new_host, v_new_host, self.k_packed, self.k_scales, self.v_packed,
                    self.v_scales, ctx_lens, max_ctx, self.signs, self.lambda_k, self.lambda_v,
                    attn_scale, out_host, ws, s)
            return _lib.bind_sdpa_int4_decode_append_host(q_host, k_new_host, v_new_host,
                                                          self.k_packed, self.k_scales,
                                                          self.v_packed, self.v_scales, ctx_lens,
                                                          max_ctx, self.signs, attn_scale, out_host,
                                                          ws, s)
        return _lib.GraphedCall(make) if graph else make(stream)

    def dequantize(self, rows: int, dtype=torch.bfloat16, stream=None):
        """Dequantized K and V of rows 0 .. rows-1 of every sequence, [B][Hkv][rows][d]
        in the rotated basis (scale * code; not used by decode)."""
        k = torch.empty(self.batch, self.num_kv_heads, rows, self.head_dim, dtype=dtype,
                        device=self.k_packed.device)
        v = torch.empty_like(k)
        _lib.dequantize(self.k_packed, self.k_scales, rows, k, stream)
        _lib.dequantize(self.v_packed, self.v_scales, rows, v, stream)
        return k, v


class CodebookKVCache:
    """The codebook variant of the cache (AdapTQ post: 2-, 3- or 4-bit indices
    into a Max-Lloyd codebook; int2 is the 2-bit case): the same calls as
    Int4KVCache.  levels: float32 [2**bits] increasing (default: the Gaussian
    Max-Lloyd codebook from libtq); signs: the Hadamard rotation, or None."""

    def __init__(self, batch: int, num_kv_heads: int, head_dim: int, capacity: int, bits: int = 2,
                 device="cuda", signs: torch.Tensor | None = None,
                 levels: torch.Tensor | None = None):
        if head_dim not in (128, 256):
            raise ValueError("head_dim must be 128 or 256")
        if bits not in (2, 3, 4):
            raise ValueError("bits must be 2, 3 or 4")
        self.batch, self.num_kv_heads, self.head_dim, self.capacity = batch, num_kv_heads, head_dim, capacity
        self.bits = bits
        dev = torch.device(device)
        rb = head_dim * bits // 8
        shape = (batch, num_kv_heads, capacity)
        self.k_packed = torch.zeros(*shape, rb, dtype=torch.uint8, device=dev)
        self.v_packed = torch.zeros(*shape, rb, dtype=torch.uint8, device=dev)
        self.k_scales = torch.zeros(*shape, head_dim // 32, dtype=torch.float32, device=dev)
        self.v_scales = torch.zeros(*shape, head_dim // 32, dtype=torch.float32, device=dev)
        self.signs = None if signs is None else signs.to(device=dev, dtype=torch.int8).contiguous()
        if levels is None:
            levels = _lib.lloyd_max_gaussian(bits)
        self.levels = levels.to(device=dev, dtype=torch.float32).contiguous()
        self._ws = None

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.k_packed, self.v_packed, self.k_scales, self.v_scales))

    def append(self, k: torch.Tensor, v: torch.Tensor, pos: torch.Tensor, stream=None) -> None:
        _lib.quantize_append_cb(k, v, pos, self.signs, self.bits, self.levels, self.k_packed,
                                self.k_scales, self.v_packed, self.v_scales, stream)

    def workspace(self, num_q_heads: int, max_ctx: int) -> torch.Tensor:
        need = _lib.decode_cb_workspace_bytes(self.batch, num_q_heads, self.num_kv_heads,
                                              self.head_dim, max_ctx)
        if need == 0:
            raise ValueError("invalid decode sizes")
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.k_packed.device)
        return self._ws

    def decode(self, q: torch.Tensor, ctx_lens: torch.Tensor, max_ctx: int,
               attn_scale: float | None = None, out: torch.Tensor | None = None, stream=None):
        if attn_scale is None:
            attn_scale = 1.0 / math.sqrt(self.head_dim)
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        ws = self.workspace(q.shape[1], max_ctx)
        _lib.sdpa_cb_decode(q, self.k_packed, self.k_scales, self.v_packed, self.v_scales, ctx_lens,
                            max_ctx, self.signs, self.bits, self.levels, attn_scale, out, ws, stream)
        return out

    def decode_append(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                      ctx_lens: torch.Tensor, max_ctx: int, attn_scale: float | None = None,
                      out: torch.Tensor | None = None, stream=None):
        if attn_scale is None:
            attn_scale = 1.0 / math.sqrt(self.head_dim)
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        ws = self.workspace(q.shape[1], max_ctx)
        _lib.sdpa_cb_decode_append(q, k_new, v_new, self.k_packed, self.k_scales, self.v_packed,
                                   self.v_scales, ctx_lens, max_ctx, self.signs, self.bits,
                                   self.levels, attn_scale, out, ws, stream)
        return out

    def bind_decode_append_host(self, q_host: torch.Tensor, k_new_host: torch.Tensor,
                                v_new_host: torch.Tensor, ctx_lens: torch.Tensor, max_ctx: int,
                                out_host: torch.Tensor, attn_scale: float | None = None,
                                stream=None, graph: bool = False):
        """Int4KVCache.bind_decode_append_host for the codebook cache
        (tq_sdpa_cb_decode_append_host)."""
        if attn_scale is None:
            attn_scale = 1.0 / math.sqrt(self.head_dim)
        need = _lib.decode_append_host_workspace_bytes(self.batch, q_host.shape[1], self.num_kv_heads,
                                                       self.head_dim, max_ctx, q_host.dtype,
                                                       k_new_host.dtype, "cb")
        if need == 0:
            raise ValueError("invalid decode sizes")
        ws = torch.empty(need, dtype=torch.uint8, device=self.k_packed.device)

        def make(s):
            return _lib.bind_sdpa_cb_decode_append_host(q_host, k_new_host, v_new_host,
                                                        self.k_packed, self.k_scales, self.v_packed,
                                                        self.v_scales, ctx_lens, max_ctx, self.signs,
                                                        self.bits, self.levels, attn_scale,
                                                        out_host, ws, s)
        return _lib.GraphedCall(make) if graph else make(stream)

    def decode_lse(self, q: torch.Tensor, ctx_lens: torch.Tensor, max_ctx: int, attn_scale: float,
                   out: torch.Tensor, lse: torch.Tensor, stream=None):
        """decode that also writes each head's softmax state lse[B][Hq][2]."""
        ws = self.workspace(q.shape[1], max_ctx)
        _lib.sdpa_cb_decode_lse(q, self.k_packed, self.k_scales, self.v_packed, self.v_scales,
                                ctx_lens, max_ctx, self.signs, self.bits, self.levels, attn_scale,
                                out, lse, ws, stream)
        return out


class UniformKVCache(CodebookKVCache):
    """The uniform low-bit variant (Open-TQ-Metal forum summary, future work:
    int2; the int4 quantizer at bits = 2 or 3): per group of 32 rotated
    coordinates s = fl32(amax / m), m = 2^(bits-1) - 1, codes
    clamp(rne(y / s), -m, m) stored as indices c + m in the codebook layout.
    Decoded as a codebook cache whose levels are the integers u - m (the
    levels attribute); the same calls as Int4KVCache."""

    def __init__(self, batch: int, num_kv_heads: int, head_dim: int, capacity: int, bits: int = 2,
                 device="cuda", signs: torch.Tensor | None = None):
        super().__init__(batch, num_kv_heads, head_dim, capacity, bits, device, signs,
                         levels=_lib.uniform_levels(bits))

    def append(self, k: torch.Tensor, v: torch.Tensor, pos: torch.Tensor, stream=None) -> None:
        _lib.quantize_append_uniform(k, v, pos, self.signs, self.bits, self.k_packed, self.k_scales,
                                     self.v_packed, self.v_scales, stream)

    def decode_append(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                      ctx_lens: torch.Tensor, max_ctx: int, attn_scale: float | None = None,
                      out: torch.Tensor | None = None, stream=None):
        if attn_scale is None:
            attn_scale = 1.0 / math.sqrt(self.head_dim)
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        ws = self.workspace(q.shape[1], max_ctx)
        _lib.sdpa_uniform_decode_append(q, k_new, v_new, self.k_packed, self.k_scales, self.v_packed,
                                        self.v_scales, ctx_lens, max_ctx, self.signs, self.bits,
                                        self.levels, attn_scale, out, ws, stream)
        return out

    def bind_decode_append_host(self, q_host: torch.Tensor, k_new_host: torch.Tensor,
                                v_new_host: torch.Tensor, ctx_lens: torch.Tensor, max_ctx: int,
                                out_host: torch.Tensor, attn_scale: float | None = None,
                                stream=None, graph: bool = False):
        """Int4KVCache.bind_decode_append_host for the uniform cache
        (tq_sdpa_uniform_decode_append_host)."""
        if attn_scale is None:
            attn_scale = 1.0 / math.sqrt(self.head_dim)
        need = _lib.decode_append_host_workspace_bytes(self.batch, q_host.shape[1], self.num_kv_heads,
                                                       self.head_dim, max_ctx, q_host.dtype,
                                                       k_new_host.dtype, "cb")
        if need == 0:
            raise ValueError("invalid decode sizes")
        ws = torch.empty(need, dtype=torch.uint8, device=self.k_packed.device)

        def make(s):
            return _lib.bind_sdpa_cb_decode_append_host(q_host, k_new_host, v_new_host,
                                                        self.k_packed, self.k_scales, self.v_packed,
                                                        self.v_scales, ctx_lens, max_ctx, self.signs,
                                                        self.bits, self.levels, attn_scale,
                                                        out_host, ws, s, uniform=True)
        return _lib.GraphedCall(make) if graph else make(stream)
