"""Test helpers: tensor <-> oracle conversion and the parity gates.

Gates (decode attention vs the oracle on the same packed cache): per
(sequence, query head) relative L2 error <= 1e-4, and max abs error <=
1e-3 * max|v_hat| over that sequence's attended value rows of the kv head.
"""
import os

import numpy as np
import torch

import oracle

REL_L2_GATE = 1e-4
MAX_ABS_GATE = 1e-3
THREADS = os.cpu_count() or 1


def to_oracle(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def oracle_cache(k, v, signs, capacity=None, pos=None):
    """Quantize host tensors k, v [B][H][T][d] with the oracle into a new cache."""
    B, H, T, d = k.shape
    cap = T if capacity is None else capacity
    cache = oracle.empty_cache(B, H, cap, d)
    p = np.zeros(B, np.int32) if pos is None else np.asarray(pos, np.int32)
    oracle.quantize_append(to_oracle(k), to_oracle(v), p, None if signs is None else signs.numpy(),
                           cache, threads=THREADS)
    return cache


def upload_cache(cache, device="cuda"):
    return [torch.from_numpy(np.ascontiguousarray(a)).to(device) for a in cache]


def vhat_absmax(cache, b, h, T):
    _, _, vp, vs = cache
    d = vp.shape[-1] * 2
    codes = oracle.unpack(vp[b, h, :T], d).astype(np.float64)
    return float(np.max(np.abs(codes * np.repeat(vs[b, h, :T].astype(np.float64), 32, axis=1))))


def check_attention(got, want, cache, ctx, G, label=""):
    """Apply both gates per (b, q head); returns (worst rel-L2, worst abs ratio)."""
    got = np.asarray(got, np.float64)
    B, Hq, d = want.shape
    worst_rel, worst_abs = 0.0, 0.0
    for b in range(B):
        for hk in range(Hq // G):
            vmax = vhat_absmax(cache, b, hk, int(ctx[b]))
            for h in range(hk * G, (hk + 1) * G):
                err = got[b, h] - want[b, h]
                rel = np.linalg.norm(err) / max(np.linalg.norm(want[b, h]), 1e-300)
                ab = np.max(np.abs(err)) / max(vmax, 1e-300)
                worst_rel, worst_abs = max(worst_rel, rel), max(worst_abs, ab)
                assert rel <= REL_L2_GATE, f"{label} b={b} h={h}: rel-L2 {rel:.3e}"
                assert ab <= MAX_ABS_GATE, f"{label} b={b} h={h}: max-abs/max|v| {ab:.3e}"
    return worst_rel, worst_abs
