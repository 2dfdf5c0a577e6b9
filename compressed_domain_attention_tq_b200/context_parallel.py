"""Context-parallel decode: each rank of a process group holds a contiguous
token shard of every sequence's packed cache (an Int4KVCache of its own), and
one decode step attends over the union of the shards.

Each rank attends its shard with tq_sdpa_int4_decode_lse, which also returns
every head's softmax state (max and sum); the ranks all-gather those outputs
and states (Hq x (d + 2) floats per sequence: tens of KB, a single collective),
and every rank combines them with tq_merge_lse.  The exchange is the split-K
log-sum-exp merge taken across GPUs; the packed cache itself never moves.  The
new token of a step is appended by the rank that owns the newest tokens, as an
ordinary Int4KVCache.append on that rank.

torch.distributed provides only the collective (NCCL between GPUs); the local
decode and the merge run in libtq's kernels.
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist

from . import _lib


def shard_range(total: int, world: int, rank: int) -> tuple[int, int]:
    """Tokens [start, stop) of a `total`-token context held by `rank` of `world`:
    contiguous shards in rank order, the first total % world ranks one token
    longer.  Every rank holds at least one token (total >= world)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    if total < world:
        raise ValueError(f"{total} tokens cannot give each of {world} ranks a shard")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def gather_parts(out: torch.Tensor, lse: torch.Tensor, group=None):
    """All-gather every rank's out [B][Hq][d] and lse [B][Hq][2] (float32):
    returns (outs [R][B][Hq][d], lses [R][B][Hq][2]) in rank order.  With one
    rank (or no initialized process group) the parts are views of out and lse."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world == 1:
        return out.unsqueeze(0), lse.unsqueeze(0)
    n_out = out.numel()
    packed = torch.cat([out.reshape(-1), lse.reshape(-1)])
    g = torch.empty(world, packed.numel(), dtype=packed.dtype, device=packed.device)
    dist.all_gather(list(g.unbind(0)), packed, group=group)  # rows of g, in rank order
    outs = g[:, :n_out].reshape(world, *out.shape).contiguous()
    lses = g[:, n_out:].reshape(world, *lse.shape).contiguous()
    return outs, lses


def decode(cache, q: torch.Tensor, ctx_lens: torch.Tensor, max_ctx: int,
           attn_scale: float | None = None, out: torch.Tensor | None = None, group=None,
           stream=None) -> torch.Tensor:
    """Attention of q [B][Hq][d] over the union of every rank's shard.

    cache      this rank's Int4KVCache or CodebookKVCache (its shard, rows 0 .. ctx_lens[b]-1);
               every rotation and code format the caches support.
    ctx_lens   this rank's shard lengths (device int32 [B], each >= 1).
    max_ctx    host bound on this rank's ctx_lens.
    Every rank calls this with the same q, attn_scale and group; every rank
    returns the full output (fp32 [B][Hq][d], unrotated basis)."""
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(cache.head_dim)
    B, Hq, d = q.shape
    local = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    lse = torch.empty(B, Hq, 2, dtype=torch.float32, device=q.device)
    cache.decode_lse(q, ctx_lens, max_ctx, attn_scale, local, lse, stream)
    outs, lses = gather_parts(local, lse, group)
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    _lib.merge_lse(outs, lses, out, stream)
    return out
