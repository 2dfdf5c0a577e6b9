"""Seeded synthetic workloads for int4 KV-cache decode.

This module only draws random inputs; it holds none of the method's
arithmetic (no rotation, quantization or attention).  Both the CUDA path and
the CPU oracle are fed from it.

The shapes stand in for the model runs on the pages (Open-TQ-Metal abstract:
Llama 3.1 70B at 128K context and Gemma 4 with attn_scale = 1.0; AdapTQ post,
performance section: 4 heads x d=128 x 4096 cached tokens; SRFT post: head
widths that are not powers of two).  No model weights or datasets are used:
K, V and Q are i.i.d. normal draws with the structure each workload names
(fixed outlier K channels, heavy-tailed token rows, ragged context lengths).
The SRFT variant's per-coordinate scales lambda come from calibration on the
pages; here they are drawn from the seed (2^U(-s, s) per coordinate, s = 1/4:
close to one, as a variance-equalizing calibration over these i.i.d. inputs
would give; the parity tests use a wider spread).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    context: int                  # cached tokens before the per-step append
    capacity: int                 # cache rows per (sequence, kv head)
    in_dtype: torch.dtype         # dtype of K, V, Q inputs
    rotation: bool
    attn_scales: tuple
    outlier_channels: int = 0     # K channels per kv head multiplied by outlier_scale
    outlier_scale: float = 1.0
    heavy_row_frac: float = 0.0   # fraction of token rows (K and V) multiplied by heavy_scale
    heavy_scale: float = 1.0
    ragged: tuple | None = None   # (lo, hi): per-sequence context ~ U{lo..hi}
    append_per_step: int = 1      # tokens quantize-appended per decode step
    rotation_kind: str = "hadamard"   # "hadamard" or "srft" (when rotation is on)
    cb_bits: int = 0                  # codebook variant: bits per index (2, 3, 4); 0 = int4
    cb_uniform: bool = False          # with cb_bits: the uniform low-bit variant (abs-max, index c + m)
    lambda_spread: float = 0.25       # srft: lambda = 2^U(-spread, spread) per coordinate
    notes: str = field(default="", compare=False)

    @property
    def group(self) -> int:
        return 32


WORKLOADS = {
    "tiny_mha_4k": Workload(
        "tiny_mha_4k", batch=1, num_q_heads=4, num_kv_heads=4, head_dim=128, context=4096,
        capacity=4097, in_dtype=torch.float32, rotation=False,
        attn_scales=(1 / math.sqrt(128),),
        notes="MHA, fp32 N(0,1); run with rotation off and on"),
    "llama70b_gqa_32k": Workload(
        "llama70b_gqa_32k", batch=1, num_q_heads=64, num_kv_heads=8, head_dim=128,
        context=32768, capacity=32769, in_dtype=torch.bfloat16, rotation=True,
        attn_scales=(1 / math.sqrt(128),), outlier_channels=4, outlier_scale=10.0,
        notes="64/8 GQA, bf16, 4 fixed K channels per head x10"),
    "llama70b_gqa_128k": Workload(
        "llama70b_gqa_128k", batch=1, num_q_heads=64, num_kv_heads=8, head_dim=128,
        context=131072, capacity=131073, in_dtype=torch.bfloat16, rotation=True,
        attn_scales=(1 / math.sqrt(128),), outlier_channels=4, outlier_scale=10.0,
        notes="64/8 GQA at 128K, bf16, outlier K channels; plus bulk prefill quantize"),
    "ragged_b16": Workload(
        "ragged_b16", batch=16, num_q_heads=64, num_kv_heads=8, head_dim=128, context=65536,
        capacity=65537, in_dtype=torch.bfloat16, rotation=True,
        attn_scales=(1 / math.sqrt(128),), heavy_row_frac=0.02, heavy_scale=8.0,
        ragged=(8192, 65536),
        notes="batch 16, per-sequence length U{8192..65536}, 2% token rows x8"),
    "wide_d256": Workload(
        "wide_d256", batch=4, num_q_heads=32, num_kv_heads=16, head_dim=256, context=65536,
        capacity=65537, in_dtype=torch.bfloat16, rotation=True,
        attn_scales=(1.0, 1 / 16.0),
        notes="32/16 GQA, d=256; attn_scale 1.0 and 1/sqrt(256)"),
    "llama70b_gqa_1m": Workload(
        "llama70b_gqa_1m", batch=1, num_q_heads=64, num_kv_heads=8, head_dim=128,
        context=1048576, capacity=1048577, in_dtype=torch.bfloat16, rotation=True,
        attn_scales=(1 / math.sqrt(128),), outlier_channels=4, outlier_scale=10.0,
        notes="the 64/8 GQA layer at 1M tokens: the context-parallel decode's long case"),
    "llama70b_gqa_128k_srft": Workload(
        "llama70b_gqa_128k_srft", batch=1, num_q_heads=64, num_kv_heads=8, head_dim=128,
        context=131072, capacity=131073, in_dtype=torch.bfloat16, rotation=True,
        attn_scales=(1 / math.sqrt(128),), outlier_channels=4, outlier_scale=10.0,
        rotation_kind="srft",
        notes="the 128K GQA layer with the SRFT rotation and per-coordinate lambdas"),
    "llama70b_gqa_128k_cb2": Workload(
        "llama70b_gqa_128k_cb2", batch=1, num_q_heads=64, num_kv_heads=8, head_dim=128,
        context=131072, capacity=131073, in_dtype=torch.bfloat16, rotation=True,
        attn_scales=(1 / math.sqrt(128),), outlier_channels=4, outlier_scale=10.0, cb_bits=2,
        notes="the 128K GQA layer with 2-bit Max-Lloyd codebook indices (AdapTQ; int2)"),
    "llama70b_gqa_128k_cb3": Workload(
        "llama70b_gqa_128k_cb3", batch=1, num_q_heads=64, num_kv_heads=8, head_dim=128,
        context=131072, capacity=131073, in_dtype=torch.bfloat16, rotation=True,
        attn_scales=(1 / math.sqrt(128),), outlier_channels=4, outlier_scale=10.0, cb_bits=3,
        notes="the 128K GQA layer with 3-bit Max-Lloyd codebook indices (AdapTQ)"),
    "llama70b_gqa_128k_int2": Workload(
        "llama70b_gqa_128k_int2", batch=1, num_q_heads=64, num_kv_heads=8, head_dim=128,
        context=131072, capacity=131073, in_dtype=torch.bfloat16, rotation=True,
        attn_scales=(1 / math.sqrt(128),), outlier_channels=4, outlier_scale=10.0, cb_bits=2,
        cb_uniform=True,
        notes="the 128K GQA layer with uniform int2 codes (abs-max, codes -1..1; Open-TQ-Metal int2)"),
    "llama70b_gqa_128k_int3": Workload(
        "llama70b_gqa_128k_int3", batch=1, num_q_heads=64, num_kv_heads=8, head_dim=128,
        context=131072, capacity=131073, in_dtype=torch.bfloat16, rotation=True,
        attn_scales=(1 / math.sqrt(128),), outlier_channels=4, outlier_scale=10.0, cb_bits=3,
        cb_uniform=True,
        notes="the 128K GQA layer with uniform int3 codes (abs-max, codes -3..3)"),
    "mha32_d96_32k": Workload(
        "mha32_d96_32k", batch=1, num_q_heads=32, num_kv_heads=32, head_dim=96, context=32768,
        capacity=32769, in_dtype=torch.bfloat16, rotation=True,
        attn_scales=(1 / math.sqrt(96),), outlier_channels=4, outlier_scale=10.0,
        rotation_kind="srft",
        notes="32-head MHA at head_dim 96 (not a power of two), SRFT rotation, 32K context"),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_signs(head_dim: int, seed: int) -> torch.Tensor:
    """Random +-1 int8 signs for the rotation (CPU tensor, from the seed)."""
    g = _gen(1_000_003 + seed, "cpu")
    return (torch.randint(0, 2, (head_dim,), generator=g, dtype=torch.int8) * 2 - 1).to(torch.int8)


def make_lambdas(w: Workload, seed: int):
    """SRFT workloads: (lambda_k, lambda_v), float32 [d] CPU tensors of
    2^U(-spread, spread); (None, None) otherwise."""
    if not (w.rotation and w.rotation_kind == "srft"):
        return None, None
    g = _gen(4_000_003 + seed, "cpu")
    e = torch.empty(2, w.head_dim).uniform_(-w.lambda_spread, w.lambda_spread, generator=g)
    lam = torch.exp2(e).to(torch.float32)
    return lam[0].contiguous(), lam[1].contiguous()


def make_context_lengths(w: Workload, seed: int) -> torch.Tensor:
    """Per-sequence cached context (int32, CPU)."""
    if w.ragged is None:
        return torch.full((w.batch,), w.context, dtype=torch.int32)
    lo, hi = w.ragged
    g = _gen(2_000_003 + seed, "cpu")
    return torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int32)


def make_outlier_channels(w: Workload, seed: int) -> torch.Tensor:
    """[Hkv][outlier_channels] fixed channel indices per kv head (CPU int64)."""
    g = _gen(3_000_003 + seed, "cpu")
    if w.outlier_channels == 0:
        return torch.zeros((w.num_kv_heads, 0), dtype=torch.int64)
    return torch.stack([torch.randperm(w.head_dim, generator=g)[:w.outlier_channels]
                        for _ in range(w.num_kv_heads)])


def make_kv(w: Workload, seed: int, device="cpu", tokens: int | None = None,
            token_offset: int = 0) -> tuple[torch.Tensor, torch.Tensor]:
    """K, V of shape [B][Hkv][tokens][d] in w.in_dtype.

    Rows are drawn N(0,1); the workload's structure (outlier K channels, heavy
    token rows) is applied as plain input scaling.  `token_offset` shifts the
    seed stream so a per-step append token differs from the cached ones.
    """
    n = w.capacity if tokens is None else tokens
    g = _gen(seed * 7919 + token_offset + 17, device)
    shape = (w.batch, w.num_kv_heads, n, w.head_dim)
    k = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if w.outlier_channels:
        ch = make_outlier_channels(w, seed).to(device)
        for h in range(w.num_kv_heads):
            k[:, h, :, ch[h]] *= w.outlier_scale
    if w.heavy_row_frac > 0:
        m = torch.rand((w.batch, 1, n, 1), generator=g, device=device) < w.heavy_row_frac
        k = torch.where(m, k * w.heavy_scale, k)
        v = torch.where(m, v * w.heavy_scale, v)
    return k.to(w.in_dtype), v.to(w.in_dtype)


def make_kv_shard(w: Workload, seed: int, start: int, stop: int, device="cpu"):
    """K, V of context tokens [start, stop) of every sequence, as held by one
    rank of a context-parallel decode ([B][Hkv][stop - start][d]).  The whole
    context is defined as the concatenation of its shards, each drawn from
    its own start offset, so a rank draws only its own tokens."""
    return make_kv(w, seed, device=device, tokens=stop - start, token_offset=20_000_033 + start)


def make_query(w: Workload, seed: int, device="cpu", step: int = 0) -> torch.Tensor:
    """Q of shape [B][Hq][d] (one decode token) in w.in_dtype."""
    g = _gen(seed * 104729 + 31 + step, device)
    q = torch.randn((w.batch, w.num_q_heads, w.head_dim), generator=g, device=device,
                    dtype=torch.float32)
    return q.to(w.in_dtype)


def shrink(w: Workload, context: int, batch: int | None = None,
           num_kv_heads: int | None = None) -> Workload:
    """Same structure at a smaller size (parity tests the oracle finishes in seconds)."""
    nk = w.num_kv_heads if num_kv_heads is None else num_kv_heads
    G = w.num_q_heads // w.num_kv_heads
    rag = None
    if w.ragged is not None:
        rag = (max(1, context // 8), context)
    return Workload(w.name + f"_small{context}", batch=w.batch if batch is None else batch,
                    num_q_heads=G * nk, num_kv_heads=nk, head_dim=w.head_dim, context=context,
                    capacity=context + w.append_per_step, in_dtype=w.in_dtype,
                    rotation=w.rotation, attn_scales=w.attn_scales,
                    outlier_channels=w.outlier_channels, outlier_scale=w.outlier_scale,
                    heavy_row_frac=w.heavy_row_frac, heavy_scale=w.heavy_scale, ragged=rag,
                    append_per_step=w.append_per_step, rotation_kind=w.rotation_kind,
                    lambda_spread=w.lambda_spread, cb_bits=w.cb_bits, cb_uniform=w.cb_uniform)
