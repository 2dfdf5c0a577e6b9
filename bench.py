#!/usr/bin/env python
"""Benchmark: one decode step of the int4 KV-cache path on B200.

A step = quantize-append of one new token (K and V of every kv head) into the
packed int4 cache + sdpa_int4 decode of one query token over the whole
context, on the 64/8-head, d=128, 128K-context Llama-3.1-70B-shaped layer
(synthetic seeded inputs, bf16), made with one tq_sdpa_int4_decode_append call
(the two-call step, append then decode, is timed beside it).  Prints one JSON
line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...   (weak scaling, N replicas)

Timing: one CUDA graph of exactly K steps replayed between CUDA events on the
launching stream (a second graph of K decodes splits the step into quantize-append
and decode).  The steps rotate over copies of the packed cache, as many as it
takes for their bytes to exceed twice the L2, so no step reads bytes its
predecessor left in the L2.  Barrier + synchronize around the timed region, max
over ranks.  The per-step distribution (median, P95) comes from graphs of 10
steps replayed at least 20 times between events.  e2e: the same step through the
public API with host buffers, timed per step.  A "configs" block repeats the
step measurement for the other synthetic configurations (1-GPU runs).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sdpa_int4 decode µs/step + effective KV GB/s (% of 8 TB/s) at 128K ctx"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
    ap.add_argument("--workload", default="llama70b_gqa_128k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the other configurations' block")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--context", type=int, default=0,
                    help="the workload at this many cached tokens per sequence (same batch and "
                         "heads): small cases for profiling captures; 0 = the workload's own")
    ap.add_argument("--mode", choices=["replicas", "context-parallel"], default="replicas",
                    help="replicas: each rank decodes its own copy of the workload (no collective); "
                         "context-parallel: one context split into contiguous token shards over the "
                         "ranks, per step a shard decode, an NCCL all-gather of the (o, max, sum) "
                         "parts and tq_merge_lse")
    ap.add_argument("--decode-kernel", choices=["mma_sync", "tcgen05"], default="mma_sync",
                    help="int4 decode kernel at head_dim 128 (mma_sync: the default; tcgen05: "
                         "the tensor-memory kernel, for comparison)")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def replica(cache):
    """A second cache object holding copies of `cache`'s packed tensors (same
    contents at other addresses), with its own workspace."""
    import copy
    c = copy.copy(cache)
    for name in ("k_packed", "v_packed", "k_scales", "v_scales"):
        setattr(c, name, getattr(cache, name).clone())
    c._ws = None
    return c


def rotation_count(step_bytes, l2_bytes, cap_bytes=4 << 30, cache_bytes=None):
    """Cache copies the timed steps rotate over: enough that the bytes read by
    consecutive steps exceed twice the L2 (at least 2), within cap_bytes."""
    n = max(2, -(-2 * l2_bytes // max(step_bytes, 1)))
    if cache_bytes:
        n = max(2, min(n, cap_bytes // cache_bytes))
    return int(n)


def window_times(torch, stream, fn, n_rot, windows, per_window):
    """Per-step times (s) of `windows` replays of a graph of `per_window` calls
    fn(i) (i rotating over n_rot caches), each replay between CUDA events."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(per_window):
            fn(i % n_rot)
    g.replay()
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(windows + 1)]
    evs[0].record(stream)
    for r in range(windows):
        g.replay()
        evs[r + 1].record(stream)
    torch.cuda.synchronize()
    t = [evs[r].elapsed_time(evs[r + 1]) / 1e3 / per_window for r in range(windows)]
    del g
    return t


def percentile(xs, p):
    xs = sorted(xs)
    return xs[min(len(xs) - 1, max(0, int(math.ceil(p / 100.0 * len(xs))) - 1))]


def kv_bytes(w, ctx_tokens):
    """Packed codes + fp32 scales of K and V read by one decode (all sequences)."""
    code_bytes = w.head_dim * w.cb_bits // 8 if w.cb_bits else w.head_dim // 2
    per_vec = code_bytes + 4 * (w.head_dim // 32)
    return 2 * per_vec * w.num_kv_heads * int(sum(ctx_tokens))


# Sources that determine each profiled kernel's code and launch shape; a
# committed DRAM-traffic figure counts only while their hash is unchanged.
KERNEL_SOURCES = {
    "decode": ["decode_mma.cu", "quantize_vector.cuh", "cb_vector.cuh", "tq_internal.h", "tq_api.cu"],
    "quantize_bulk": ["quantize_tc.cu", "tc_ptx.cuh", "quantize.cu", "tq_internal.h", "tq_api.cu"],
}


def kernel_source_hash(kernel_key):
    """Hash of the code in a kernel's sources: comments and layout do not count."""
    import re
    h = hashlib.sha256()
    cs = os.path.join(ROOT, "compressed_domain_attention_tq_b200", "csrc")
    for f in sorted(KERNEL_SOURCES[kernel_key]):
        with open(os.path.join(cs, f), encoding="utf-8") as fh:
            code = fh.read()
        code = re.sub(r"/\*.*?\*/", " ", code, flags=re.S)
        code = re.sub(r"//[^\n]*", " ", code)
        code = " ".join(code.split())
        h.update(f.encode() + code.encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources and this workload (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if (not e or e.get("source_hash") != kernel_source_hash(kernel_key)
            or e.get("workload_name") != workload):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.proc = None
        self.path = f"/tmp/tq_clocks_{os.getpid()}.csv"
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for ln in f:
                parts = [x.strip() for x in ln.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.remove(self.path)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def dist_setup(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def prefill_timing(torch, cache, k_all, v_all, pos0, stream, flush, w, srft=False):
    """The bulk prefill of k_all, v_all [B][Hkv][n][d] into rows 0 .. n-1 of
    `cache` (one quantize-append call): the minimum of 3 calls timed with CUDA
    events, each after an L2 flush (a write of `flush`), and its HBM roofline
    fraction over the bytes the call must move (bf16 inputs read once, codes
    and fp32 scales written once)."""
    times = []
    for i in range(4):
        flush.fill_(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cache.append(k_all, v_all, pos0)
        e1.record(stream)
        torch.cuda.synchronize()
        if i:
            times.append(e0.elapsed_time(e1) / 1e3)
    t = min(times)
    B, _, n, d = k_all.shape
    nvec = 2 * B * k_all.shape[1] * n
    code_bytes = d * w.cb_bits // 8 if w.cb_bits else d // 2
    moved = k_all.numel() * k_all.element_size() * 2 + nvec * (code_bytes + 4 * (d // 32))
    hbm_peak, peak_kind = measured_peaks()
    tc_rotation = (w.rotation and not w.cb_bits and k_all.dtype == torch.bfloat16 and nvec > 8192
                   and ((not srft and d in (128, 256)) or (srft and d <= 128)))
    return {"tokens": int(n), "us": round(t * 1e6, 2),
            "tokens_per_s": round(B * n / t, 1),
            "GB_per_s": round(moved / t / 1e9, 1), "ns_per_vec": round(t / nvec * 1e9, 4),
            "bytes_moved": int(moved),
            "roofline_frac": round(moved / t / 1e9 / hbm_peak, 3), "peak_kind": peak_kind,
            "kernel": (("quantize_srft_tc_kernel (Hartley transform as a tcgen05 product, "
                        "three bf16 parts)" if srft else
                        "quantize_tc256_kernel (H_2 x H_128: two tcgen05 bf16 products)" if d == 256 else
                        "quantize_tc_kernel (rotation as a tcgen05 bf16 product)") if tc_rotation
                       else "CUDA-core quantize kernel"),
            "timing": "min of 3 calls, each after a 256 MiB L2 flush"}


def run_tq(args):
    import torch
    import torch.distributed as dist

    import compressed_domain_attention_tq_b200 as tq
    from compressed_domain_attention_tq_b200 import workloads as wl

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    from compressed_domain_attention_tq_b200 import _lib
    _lib.set_test_hooks(_lib.TEST_HOOK_TCGEN05_DECODE if args.decode_kernel == "tcgen05" else 0)
    w = wl.WORKLOADS[args.workload]
    if args.context:
        w = wl.shrink(w, context=args.context)
    seed = args.seed + 1000 * rank
    B, Hq, Hkv, d, T = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.context
    stream = torch.cuda.current_stream()

    signs = wl.make_signs(d, seed) if w.rotation else None
    srft = w.rotation and w.rotation_kind == "srft"
    lk, lv = wl.make_lambdas(w, seed)
    ctx = wl.make_context_lengths(w, seed)                    # cached tokens per sequence
    if w.cb_bits and w.cb_uniform:
        cache = tq.UniformKVCache(B, Hkv, d, w.capacity, w.cb_bits, dev, signs)
    elif w.cb_bits:
        cache = tq.CodebookKVCache(B, Hkv, d, w.capacity, w.cb_bits, dev, signs)
    else:
        cache = tq.Int4KVCache(B, Hkv, d, w.capacity, dev, signs,
                               rotation="srft" if srft else "hadamard", lambda_k=lk, lambda_v=lv)
    k_all, v_all = wl.make_kv(w, seed, device=dev, tokens=w.capacity - 1)
    pos0 = torch.zeros(B, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    # bulk prefill: all cached tokens quantized in one call
    prefill = None
    if not args.no_prefill:
        prefill = prefill_timing(torch, cache, k_all, v_all, pos0, stream, flush, w, srft)
    else:
        cache.append(k_all, v_all, pos0)
    # host copy of sequence 0's first kv heads for the fidelity report
    n_fid = min(2, Hkv)
    ctx0 = int(ctx[0])
    fid_k = k_all[0, :n_fid, :ctx0].float().cpu() if rank == 0 else None
    fid_v = v_all[0, :n_fid, :ctx0].float().cpu() if rank == 0 else None
    del k_all, v_all

    # per-step inputs: one new token appended after the cached context
    k_new, v_new = wl.make_kv(w, seed, device=dev, tokens=1, token_offset=10_000_019)
    q = wl.make_query(w, seed, device=dev)
    pos = ctx.to(dev)
    ctx_dev = (ctx + 1).to(dev)
    max_ctx = int((ctx + 1).max())
    out = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
    scale = w.attn_scales[0]
    ws = cache.workspace(Hq, max_ctx)

    # The timed steps rotate over copies of the packed cache (same contents, other
    # addresses), enough that consecutive steps' bytes exceed twice the L2: no step
    # re-reads bytes its predecessor left in the L2.
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    kvb_step = kv_bytes(w, (ctx + 1).tolist())
    n_rot = rotation_count(kvb_step, l2_bytes, cache_bytes=cache.nbytes())
    caches = [cache] + [replica(cache) for _ in range(n_rot - 1)]
    del flush

    def step(i):  # one decode step in one call: append the new token, then attend
        caches[i].decode_append(q, k_new, v_new, ctx_dev, max_ctx, scale, out)

    def dec(i):
        caches[i].decode(q, ctx_dev, max_ctx, scale, out)

    def two(i):  # the same step as two calls (append, then decode)
        caches[i].append(k_new, v_new, pos)
        caches[i].decode(q, ctx_dev, max_ctx, scale, out)

    for i in range(max(args.warmup, n_rot)):
        step(i % n_rot)
    torch.cuda.synchronize()
    # Device timing: one CUDA graph holds exactly K steps (quantize-append + decode),
    # replayed once between CUDA events, so per-launch host and graph-launch latency
    # is amortised; a second graph of K decodes splits the step.
    g_step, g_dec, g_two = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    for g, fn in ((g_step, step), (g_dec, dec), (g_two, two)):
        with torch.cuda.graph(g):
            for i in range(args.steps):
                fn(i % n_rot)
    for i in range(max(1, args.warmup // args.steps + 1)):
        g_step.replay()
        g_dec.replay()
        g_two.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid)) if rank == 0 else None
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    ev[0].record(stream)
    g_step.replay()
    ev[1].record(stream)
    g_dec.replay()
    ev[2].record(stream)
    g_two.replay()
    ev[3].record(stream)
    torch.cuda.synchronize()
    # the per-step distribution: graphs of 10 steps, replayed >= 20 times
    win = window_times(torch, stream, step, n_rot, max(20, args.steps // 10), 10)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    step_s = ev[0].elapsed_time(ev[1]) / 1e3 / args.steps
    dec_s = ev[1].elapsed_time(ev[2]) / 1e3 / args.steps
    two_s = ev[2].elapsed_time(ev[3]) / 1e3 / args.steps
    q_s = max(step_s - dec_s, 0.0)
    p50_s, p95_s = percentile(win, 50), percentile(win, 95)
    if world > 1:
        tt = torch.tensor([step_s, dec_s, q_s, two_s, p50_s, p95_s], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        step_s, dec_s, q_s, two_s, p50_s, p95_s = tt.tolist()
    del g_step, g_dec, g_two

    # end to end through the C ABI with HOST buffers: the step's q, k_new, v_new and
    # output are pinned host tensors; tq_sdpa_int4_decode_append_host enqueues their
    # copies and the step in one call (a prepared call, Int4KVCache.bind_decode_append_host).
    # Caches without that call: one pinned copy up, the public step call, one copy back.
    h_q, h_k, h_v = (t.cpu().pin_memory() for t in (q, k_new, v_new))
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (h_q, h_k, h_v))
    host_steps = [c.bind_decode_append_host(h_q, h_k, h_v, ctx_dev, max_ctx, h_out, scale, graph=True)
                  for c in caches]

    e2e_t = []
    for i in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        host_steps[i % n_rot]()
        b.record(stream)
        b.synchronize()
        if i >= args.warmup:
            e2e_t.append(a.elapsed_time(b) / 1e3)
    e2e_s = sum(e2e_t) / len(e2e_t)
    if world > 1:
        tt = torch.tensor([e2e_s], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_s = tt.item()

    # comparisons on the same GPU (rank 0): bf16 dequantize-then-attend, and
    # fidelity of this path's output to unquantized fp64 attention
    baseline = fid = None
    if rank == 0:
        import numpy as np
        cache.decode(q, ctx_dev, max_ctx, scale, out)
        Qm, Om = basis_maps(d, signs, lk, lv, srft, dev)
        khat = None
        if not w.cb_bits:  # tq_dequantize reads the int4 layout
            bl = dequant_attend_baseline(cache, q, ctx_dev, max_ctx, scale, Qm, Om,
                                         min(args.steps, 50), 3, stream)
            o_ours, o_bl = out.double().flatten(1), bl.pop("out").double().flatten(1)
            bl["cosine_vs_int4_path_min"] = round(float(torch.nn.functional.cosine_similarity(
                o_ours, o_bl, dim=1).min()), 5)
            bl["int4_decode_speedup"] = round(bl["dequantize_then_attend_us"] / (dec_s * 1e6), 2)
            baseline = bl
            khat, _ = cache.dequantize(ctx0 + 1, torch.float32)
            khat = khat[0, :n_fid].cpu().numpy()
        G = Hq // Hkv
        fid_k = np.concatenate([fid_k.numpy(), k_new[0, :n_fid].float().cpu().numpy()], 1)
        fid_v = np.concatenate([fid_v.numpy(), v_new[0, :n_fid].float().cpu().numpy()], 1)
        fid = fidelity(fid_k, fid_v, q[0, :n_fid * G].float().cpu().numpy(),
                       out[0, :n_fid * G].cpu().numpy(), khat, Qm.cpu().numpy(), scale, G)
        fid["sample"] = f"sequence 0, kv heads 0..{n_fid - 1} ({n_fid * G} query heads), {ctx0 + 1} tokens"
        del khat

    kvb = kv_bytes(w, (ctx + 1).tolist())
    mma = not w.cb_bits and ((d == 128 and Hq // Hkv <= 8) or (d == 256 and Hq // Hkv <= 4))
    mma_cb = bool(w.cb_bits) and d == 128 and 5 <= Hq // Hkv <= 8
    cb_name = (f"uniform int{w.cb_bits} codes" if w.cb_uniform else f"{w.cb_bits}-bit Max-Lloyd codebook")
    cb_call = "tq_sdpa_uniform_decode_append" if w.cb_uniform else "tq_sdpa_cb_decode_append"
    if mma_cb:
        launches_per_step = 2
        step_desc = (f"{cb_call} ({cb_name}): the tensor-core "
                     "decode kernel quantizes the new token of each kv head into the cache, then "
                     "attends (split-K kernel + merge, 2 launches)")
    elif w.cb_bits:
        launches_per_step = 3
        step_desc = (f"{cb_call} ({cb_name}): quantize-append "
                     "of the new token, split-K decode, merge (3 launches)")
    elif srft:
        launches_per_step = 3
        step_desc = ("tq_sdpa_int4_decode_append_srft: one launch quantizes the new token (SRFT) and "
                     "rotates the queries, then split-K decode and merge with the inverse transform "
                     "(3 launches)")
    elif mma:
        launches_per_step = 2
        step_desc = ("tq_sdpa_int4_decode_append: the decode kernel quantizes the new token of each "
                     "kv head into the cache, then attends (split-K kernel + merge, 2 launches)")
    else:
        launches_per_step = 3
        step_desc = ("tq_sdpa_int4_decode_append: quantize-append of the new token, split-K "
                     "decode, merge (3 launches)")
    qo_bytes = q.numel() * q.element_size() + out.numel() * out.element_size()
    algo = kvb + qo_bytes
    peak, peak_kind = measured_peaks()
    dec_gbs = algo / dec_s / 1e9
    value = world * kvb / step_s / 1e9
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 5),
        "us_per_step": round(step_s * 1e6, 2), "decode_us": round(dec_s * 1e6, 2),
        "p50_us": round(p50_s * 1e6, 2), "p95_us": round(p95_s * 1e6, 2),
        "distribution": f"{len(win)} replays of a 10-step graph (per-step mean of each replay)",
        "append_in_step_us": round(q_s * 1e6, 2),
        "two_call_step_us": round(two_s * 1e6, 2),
        "pct_of_8TBps": round(100 * kvb / step_s / 1e9 / NOMINAL_HBM_GBS, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": (f"{cb_name} (codebook layout), fp32 accumulation" if w.cb_bits
                  else "int4 codes, fp32 accumulation"), "data": "synthetic (seeded N(0,1), bf16)",
        "config": {"workload": w.name, "batch": B, "q_heads": Hq, "kv_heads": Hkv, "head_dim": d,
                   "context": max_ctx, "decode_kernel": args.decode_kernel,
                   "rotation": (w.rotation_kind if w.rotation else False),
                   "codes": cb_name if w.cb_bits else "int4",
                   "attn_scale": scale,
                   "kv_bytes_per_step": kvb,
                   "l2": (f"rotated over {n_rot} caches: consecutive steps read {n_rot * kvb} B "
                          f"of packed cache, more than twice the {l2_bytes} B L2"),
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm",
                     "kernel": (f"{cb_name} decode on the codebook path (split-K + merge)" if w.cb_bits
                                else "sdpa_int4 decode (split-K + merge)"),
                     "achieved": round(dec_gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(dec_gbs / peak, 4), "peak_kind": peak_kind,
                     "algorithmic_bytes": algo, "traffic": ncu_traffic("decode", w.name)},
        "e2e": {"value": round(world * kvb / e2e_s / 1e9, 1), "unit": "GB/s",
                "us_per_step": round(e2e_s * 1e6, 2),
                "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(h_out.numel() * h_out.element_size())},
        "gpu_launches": launches_per_step * args.steps,
        "step": step_desc,
        "timing": "device: one CUDA graph of K steps replayed between CUDA events on the "
                  "launching stream (decode split from a K-decode graph; the two-call step "
                  "from a third graph); e2e: per step, the host-buffer decode step "
                  "(tq_sdpa_int4_decode_append_host, or its SRFT / codebook form) on pinned "
                  "host buffers (a gather kernel reads q, k_new, v_new over the bus, the merge "
                  "writes the output into host memory), replayed from a CUDA graph "
                  "(cache.bind_decode_append_host(graph=True)), between CUDA events",
        "clocks": clocks,
        "bulk_prefill": prefill,
        "bf16_dequantize_then_attend": baseline,
        "fidelity_vs_unquantized_fp64": fid,
    }
    if rank == 0 and world == 1 and not args.no_configs:
        res["configs"] = measure_configs(args, dev, stream, seed, peak)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, seed)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# The other synthetic configurations, each measured like the main workload's
# step (rotation over cache copies, graph timing, windows for median / P95,
# e2e through the host-buffer call): (workload, rotation on?, attn_scale index).
CONFIGS = (("tiny_mha_4k", False, 0), ("tiny_mha_4k", True, 0), ("llama70b_gqa_32k", True, 0),
           ("ragged_b16", True, 0), ("wide_d256", True, 0), ("wide_d256", True, 1))


def measure_config(name, rot, scale_idx, args, dev, stream, seed, peak, want_fidelity=False):
    """One configuration on this GPU: the bulk prefill of its cached context
    (one quantize-append call), the decode step as the fused append + decode
    (tq_sdpa_int4_decode_append), the decode alone, their median and P95 over
    graph replays, the host-buffer e2e step, and the decode's roofline fraction."""
    import dataclasses

    import torch

    import compressed_domain_attention_tq_b200 as tq
    from compressed_domain_attention_tq_b200 import workloads as wl
    w = dataclasses.replace(wl.WORKLOADS[name], rotation=rot)
    B, Hq, Hkv, d = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim
    scale = w.attn_scales[scale_idx]
    signs = wl.make_signs(d, seed) if rot else None
    ctx = wl.make_context_lengths(w, seed)
    cache = tq.Int4KVCache(B, Hkv, d, w.capacity, dev, signs)
    k_all, v_all = wl.make_kv(w, seed, device=dev, tokens=w.capacity - 1)
    pos0 = torch.zeros(B, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    prefill = prefill_timing(torch, cache, k_all, v_all, pos0, stream, flush, w)
    del flush
    fid_in = None
    k_new, v_new = wl.make_kv(w, seed, device=dev, tokens=1, token_offset=10_000_019)
    if want_fidelity:  # sequence 0's first two kv heads, unquantized, with the appended token
        c0 = int(ctx[0])
        fid_in = (torch.cat([k_all[0, :2, :c0], k_new[0, :2]], 1).float().cpu().numpy(),
                  torch.cat([v_all[0, :2, :c0], v_new[0, :2]], 1).float().cpu().numpy())
    del k_all, v_all
    q = wl.make_query(w, seed, device=dev)
    ctx_dev = (ctx + 1).to(dev)
    max_ctx = int((ctx + 1).max())
    out = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    kvb = kv_bytes(w, (ctx + 1).tolist())
    n_rot = rotation_count(kvb, l2_bytes, cache_bytes=cache.nbytes())
    caches = [cache] + [replica(cache) for _ in range(n_rot - 1)]

    def step(i):
        caches[i].decode_append(q, k_new, v_new, ctx_dev, max_ctx, scale, out)

    def dec(i):
        caches[i].decode(q, ctx_dev, max_ctx, scale, out)

    steps = max(n_rot, 40 // n_rot * n_rot)
    for i in range(max(args.warmup, n_rot)):
        step(i % n_rot)
    torch.cuda.synchronize()
    res = {}
    for key, fn in (("step", step), ("decode", dec)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(steps):
                fn(i % n_rot)
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        res[key] = e0.elapsed_time(e1) / 1e3 / steps
        del g
    win = window_times(torch, stream, step, n_rot, 20, 10)
    # e2e: the host-buffer step (pinned q, k_new, v_new in, output out), per step
    h_q, h_k, h_v = (t.cpu().pin_memory() for t in (q, k_new, v_new))
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hs = [c.bind_decode_append_host(h_q, h_k, h_v, ctx_dev, max_ctx, h_out, scale, graph=True)
          for c in caches]
    e2e = []
    for i in range(args.warmup + 20):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        hs[i % n_rot]()
        b.record(stream)
        b.synchronize()
        if i >= args.warmup:
            e2e.append(a.elapsed_time(b) / 1e3)
    algo = kvb + q.numel() * q.element_size() + out.numel() * out.element_size()
    entry = {
        "workload": w.name, "rotation": "hadamard" if rot else False, "attn_scale": scale,
        "batch": B, "q_heads": Hq, "kv_heads": Hkv, "head_dim": d, "context_max": max_ctx,
        "kv_bytes_per_step": kvb,
        "us_per_step": round(res["step"] * 1e6, 2), "decode_us": round(res["decode"] * 1e6, 2),
        "p50_us": round(percentile(win, 50) * 1e6, 2), "p95_us": round(percentile(win, 95) * 1e6, 2),
        "kv_GB_per_s": round(kvb / res["step"] / 1e9, 1),
        "roofline_frac": round(algo / res["decode"] / 1e9 / peak, 4),
        "e2e_us": round(sum(e2e) / len(e2e) * 1e6, 2),
        "l2": f"rotated over {n_rot} caches",
        "prefill": {k_: prefill[k_] for k_ in ("tokens", "us", "GB_per_s", "roofline_frac", "kernel")},
    }
    if want_fidelity:
        caches[0].decode(q, ctx_dev, max_ctx, scale, out)
        G = Hq // Hkv
        entry["_fidelity_out"] = out[0, :2 * G].cpu().numpy()
        entry["_fidelity_in"] = (fid_in, q[0, :2 * G].float().cpu().numpy(), signs, G)
    del caches, hs
    torch.cuda.synchronize()
    return entry


def measure_configs(args, dev, stream, seed, peak):
    """The CONFIGS block, and the wide-head configuration's fidelity at
    attn_scale 1.0 against 1/16 (directional error 1 - cosine to unquantized
    attention, and their ratio)."""
    import torch
    entries, fid = [], {}
    for name, rot, si in CONFIGS:
        e = measure_config(name, rot, si, args, dev, stream, seed, peak, want_fidelity=name == "wide_d256")
        if "_fidelity_out" in e:
            (k_h, v_h), q_h, signs, G = e.pop("_fidelity_in")
            o = e.pop("_fidelity_out")
            Qm, _ = basis_maps(e["head_dim"], signs, None, None, False, torch.device("cpu"))
            f = fidelity(k_h, v_h, q_h, o, None, Qm.numpy(), e["attn_scale"], G)
            fid[e["attn_scale"]] = f
            e["fidelity_vs_unquantized_fp64"] = f
        entries.append(e)
        torch.cuda.empty_cache()
    block = {"entries": entries}
    if len(fid) == 2:
        lo, hi = min(fid), max(fid)
        err = {s_: 1.0 - fid[s_]["cosine_mean"] for s_ in fid}
        block["wide_d256_attn_scale_directional_error"] = {
            "one_minus_cosine_mean_at_1.0": round(err[hi], 7),
            "one_minus_cosine_mean_at_1/16": round(err[lo], 7),
            "ratio": round(err[hi] / err[lo], 2) if err[lo] > 0 else None,
            "sample": "sequence 0, kv heads 0..1, unquantized fp64 softmax attention vs the int4 path"}
    return block


def rotation_matrix(d, signs, device):
    """R = H_d diag(signs) / sqrt(d) (Sylvester H_d) as fp64 on `device`; identity without signs."""
    import torch
    if signs is None:
        return torch.eye(d, dtype=torch.float64, device=device)
    H = torch.ones(1, 1, dtype=torch.float64)
    while H.shape[0] < d:
        H = torch.cat([torch.cat([H, H], 1), torch.cat([H, -H], 1)], 0)
    return (H * signs.double().cpu()[None, :] / math.sqrt(d)).to(device)


def basis_maps(d, signs, lk, lv, srft, device):
    """(Qm, Om), fp64 on `device`: q_r = Qm q takes a query into the cache's basis and
    o = Om o_r takes an output back.  Hadamard: R and R^T.  SRFT: diag(1/lambda_k) F
    diag(signs) and diag(signs) F diag(1/lambda_v), F the orthonormal Hartley matrix
    (Re - Im of the unitary DFT matrix)."""
    import torch
    if not srft:
        R = rotation_matrix(d, signs, device)
        return R, R.T.contiguous()
    X = torch.fft.fft(torch.eye(d, dtype=torch.float64), dim=0)
    F = (X.real - X.imag) / math.sqrt(d)
    one = torch.ones(d, dtype=torch.float64)
    s = one if signs is None else signs.double().cpu()
    ik = one if lk is None else 1.0 / lk.double().cpu()
    iv = one if lv is None else 1.0 / lv.double().cpu()
    return ((ik[:, None] * F * s[None, :]).to(device), (s[:, None] * F * iv[None, :]).to(device))


def dequant_attend_baseline(cache, q, ctx_dev, max_ctx, scale, Qm, Om, steps, warmup, stream):
    """In-house bf16 dequantize-then-attend on the same GPU: every step
    materializes bf16 K and V from the packed cache (tq_dequantize, one pass)
    and runs torch's bf16 scaled_dot_product_attention over them (query rotated
    into the cache basis by Qm, output back by Om).  Also times the attention
    alone on the materialized bf16 cache (what a bf16 KV cache would cost)."""
    import torch
    import torch.nn.functional as F

    from compressed_domain_attention_tq_b200 import _lib
    B, Hq, d = q.shape
    Hkv = cache.k_packed.shape[1]
    dev = q.device
    Qf, Of = Qm.float(), Om.float()
    Kb = torch.empty(B, Hkv, max_ctx, d, dtype=torch.bfloat16, device=dev)
    Vb = torch.empty_like(Kb)
    lens = ctx_dev.long()
    mask = None
    if int(lens.min()) < max_ctx:  # ragged batch: mask each sequence's tail
        mask = (torch.arange(max_ctx, device=dev)[None, :] < lens[:, None])[:, None, None, :]
    out = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)

    def attend():
        qr = (q.float() @ Qf.T).to(torch.bfloat16)[:, :, None, :]
        o = F.scaled_dot_product_attention(qr, Kb, Vb, attn_mask=mask, scale=scale, enable_gqa=True)
        out.copy_(o[:, :, 0].float() @ Of.T)

    def full():
        _lib.dequantize(cache.k_packed, cache.k_scales, max_ctx, Kb)
        _lib.dequantize(cache.v_packed, cache.v_scales, max_ctx, Vb)
        attend()

    for _ in range(warmup):
        full()
    torch.cuda.synchronize()
    res = {}
    for name, fn in (("dequantize_then_attend", full), ("attend_only_bf16_cache", attend)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(steps):
                fn()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        res[name + "_us"] = round(a.elapsed_time(b) * 1e3 / steps, 2)
        del g
    res["bf16_cache_bytes"] = 2 * Kb.numel() * Kb.element_size()
    res["out"] = out
    return res


def fidelity(k_h, v_h, q_h, out_h, khat_h, Qm, scale, G):
    """Fidelity of the int4 path to unquantized fp64 attention (report only).

    k_h, v_h [n][T][d] unquantized (unrotated) inputs of n kv heads; q_h [n*G][d];
    out_h [n*G][d] the CUDA path's output; khat_h [n][T][d] dequantized keys
    (cache basis); Qm the query's map into that basis.  Cosine similarity of each query head's output with exact
    softmax attention, and agreement of argmax_t q.k between the unquantized
    and the dequantized keys."""
    import numpy as np
    cos, agree = [], []
    for h in range(k_h.shape[0]):
        K, V = k_h[h].astype(np.float64), v_h[h].astype(np.float64)
        Q = q_h[h * G:(h + 1) * G].astype(np.float64)
        S = K @ Q.T * scale
        P = np.exp(S - S.max(0, keepdims=True))
        O = (P.T @ V) / P.sum(0)[:, None]
        Og = out_h[h * G:(h + 1) * G].astype(np.float64)
        cos += list((O * Og).sum(1) / (np.linalg.norm(O, axis=1) * np.linalg.norm(Og, axis=1)))
        if khat_h is not None:
            Sq = khat_h[h].astype(np.float64) @ (Q @ Qm.T).T
            agree += list(S.argmax(0) == Sq.argmax(0))
    return {"cosine_min": round(float(min(cos)), 7), "cosine_mean": round(float(np.mean(cos)), 7),
            "top1_qk_argmax_agreement": round(float(np.mean(agree)), 4) if agree else None,
            "query_heads": len(cos)}


def oracle_sample(w, seed, kv_head=0):
    """Inputs of one kv head (its G query heads) at the full context, from the
    seeded CPU generator, quantized by the oracle."""
    import numpy as np
    import torch

    import oracle
    from compressed_domain_attention_tq_b200 import workloads as wl

    k, v = wl.make_kv(w, seed, device="cpu", tokens=w.capacity)
    k = k[:1, kv_head:kv_head + 1].contiguous()
    v = v[:1, kv_head:kv_head + 1].contiguous()
    G = w.num_q_heads // w.num_kv_heads
    q = wl.make_query(w, seed)[:1, kv_head * G:(kv_head + 1) * G].contiguous()

    def bits(t):
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()

    signs = wl.make_signs(w.head_dim, seed).numpy() if w.rotation else None
    lk, lv = wl.make_lambdas(w, seed)
    lam = None if lk is None else (lk.numpy(), lv.numpy())
    if w.cb_bits:
        cache = oracle.empty_cb_cache(1, 1, w.capacity, w.head_dim, w.cb_bits)
    else:
        cache = oracle.empty_cache(1, 1, w.capacity, w.head_dim)
    thr = oracle.max_threads()
    levels = None
    if w.cb_bits:
        levels = (oracle.uniform_levels(w.cb_bits) if w.cb_uniform
                  else oracle.lloyd_max_gaussian(w.cb_bits).astype(np.float32))
    s = dict(k_new=bits(k[:, :, -1:]), v_new=bits(v[:, :, -1:]), q=bits(q), signs=signs, lam=lam,
             cache=cache, threads=thr, G=G, T=w.capacity - 1, cb_bits=w.cb_bits, levels=levels,
             cb_uniform=w.cb_uniform)
    t0 = time.perf_counter()
    oracle_append(s, bits(k[:, :, :-1]), bits(v[:, :, :-1]), 0)
    s["prefill_s"] = time.perf_counter() - t0
    return s


def oracle_append(s, k, v, pos):
    import oracle
    if s["cb_bits"] and s["cb_uniform"]:
        oracle.quantize_append_uniform(k, v, [pos], s["signs"], s["cb_bits"], s["cache"],
                                       threads=s["threads"])
    elif s["cb_bits"]:
        oracle.quantize_append_cb(k, v, [pos], s["signs"], s["cb_bits"], s["levels"], s["cache"],
                                  threads=s["threads"])
    elif s["lam"] is None:
        oracle.quantize_append(k, v, [pos], s["signs"], s["cache"], threads=s["threads"])
    else:
        oracle.quantize_append_srft(k, v, [pos], s["signs"], s["lam"][0], s["lam"][1], s["cache"],
                                    threads=s["threads"])


def oracle_step(s, w):
    import oracle
    oracle_append(s, s["k_new"], s["v_new"], s["T"])
    if s["cb_bits"]:
        return oracle.sdpa_cb_decode(s["q"], s["cache"], [s["T"] + 1], s["signs"], s["cb_bits"],
                                     s["levels"], w.attn_scales[0], 1, threads=s["threads"])
    if s["lam"] is None:
        return oracle.sdpa_int4_decode(s["q"], s["cache"], [s["T"] + 1], s["signs"],
                                       w.attn_scales[0], 1, threads=s["threads"])
    return oracle.sdpa_int4_decode_srft(s["q"], s["cache"], [s["T"] + 1], s["signs"], s["lam"][0],
                                        s["lam"][1], w.attn_scales[0], 1, threads=s["threads"])


def cpu_baseline(w, seed):
    s = oracle_sample(w, seed)
    ts = []
    for _ in range(3):
        t0 = time.perf_counter()
        oracle_step(s, w)
        ts.append(time.perf_counter() - t0)
    t = min(ts)
    kvb = kv_bytes(w, [s["T"] + 1]) // w.num_kv_heads
    cores = s["threads"]
    s["threads"] = 1  # the same step on one core, once
    t0 = time.perf_counter()
    oracle_step(s, w)
    t1 = time.perf_counter() - t0
    return {"value": round(kvb / t / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "us_per_step_sample": round(t * 1e6, 1),
            "single_thread": {"value": round(kvb / t1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                              "us_per_step_sample": round(t1 * 1e6, 1)},
            "sample": (f"kv head 0 of {w.num_kv_heads} ({s['G']} query heads) at {s['T'] + 1}-token "
                       f"context: quantize-append 1 token + decode, best of 3; oracle prefill of the "
                       f"sample took {s['prefill_s']:.1f} s")}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from compressed_domain_attention_tq_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    s = oracle_sample(w, args.seed)
    for _ in range(args.warmup):
        oracle_step(s, w)
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(s, w)
        ts.append(time.perf_counter() - t0)
    t = sum(ts) / len(ts)
    kvb = kv_bytes(w, [s["T"] + 1]) // w.num_kv_heads
    val = kvb / t / 1e9
    sample = (f"kv head 0 of {w.num_kv_heads} ({s['G']} query heads) at {s['T'] + 1}-token context; "
              f"each step = oracle quantize-append of 1 token + fp64 decode")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1), bf16)",
        "config": {"workload": w.name, "batch": 1, "q_heads": s["G"], "kv_heads": 1,
                   "head_dim": w.head_dim, "context": s["T"] + 1},
        "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": s["threads"], "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def cp_measure(name, args, world, rank, dev, stream, l2_bytes):
    """Context-parallel decode of one workload: this rank's shard timings (s),
    max over ranks, and the byte counts."""
    import torch
    import torch.distributed as dist

    import compressed_domain_attention_tq_b200 as tq
    from compressed_domain_attention_tq_b200 import _lib
    from compressed_domain_attention_tq_b200 import context_parallel as cp
    from compressed_domain_attention_tq_b200 import workloads as wl
    w = wl.WORKLOADS[name]
    if w.ragged is not None or w.cb_bits or (w.rotation and w.rotation_kind == "srft"):
        raise ValueError(f"context-parallel bench: {name} is not an equal-length int4 workload")
    B, Hq, Hkv, d, T = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.context
    seed = args.seed  # one global context: every rank draws from the same seed
    t0, t1 = cp.shard_range(T, world, rank)
    n = t1 - t0
    signs = wl.make_signs(d, seed) if w.rotation else None
    cache = tq.Int4KVCache(B, Hkv, d, n, dev, signs)
    chunk = 1 << 18  # draw and quantize the shard in pieces (bounded bf16 staging)
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        k, v = wl.make_kv_shard(w, seed, t0 + c0, t0 + c1, device=dev)
        cache.append(k, v, torch.full((B,), c0, dtype=torch.int32, device=dev))
        del k, v
    q = wl.make_query(w, seed, device=dev)
    scale = w.attn_scales[0]
    ctx_dev = torch.full((B,), n, dtype=torch.int32, device=dev)
    shard_bytes = kv_bytes(w, [n] * B)
    total_bytes = kv_bytes(w, [T] * B)
    n_rot = rotation_count(shard_bytes, l2_bytes, cache_bytes=cache.nbytes())
    caches = [cache] + [replica(cache) for _ in range(n_rot - 1)]
    local = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
    lse = torch.empty(B, Hq, 2, dtype=torch.float32, device=dev)
    out = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
    K = args.steps

    def shard(i):
        caches[i % n_rot].decode_lse(q, ctx_dev, n, scale, local, lse)

    parts = cp.gather_parts(local, lse)

    def merge():
        _lib.merge_lse(parts[0], parts[1], out)

    def step(i):
        nonlocal parts
        shard(i)
        parts = cp.gather_parts(local, lse)
        merge()

    for i in range(max(args.warmup, n_rot)):
        step(i)
    torch.cuda.synchronize()

    def graph_time(fn):  # K calls in one CUDA graph, replayed between events
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(K):
                fn(i)
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) / 1e3 / K

    def eager_time(fn):  # K calls enqueued back to back, between events
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(K):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3 / K

    # end to end: q from pinned host memory, the step, the output back to pinned host memory
    h_q = q.cpu().pin_memory()
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def host_step(i):
        q.copy_(h_q, non_blocking=True)
        step(i)
        h_out.copy_(out, non_blocking=True)

    shard_s = graph_time(shard)
    merge_s = graph_time(lambda i: merge())
    gather_s = eager_time(lambda i: cp.gather_parts(local, lse))
    step_s = eager_time(step)
    e2e_s = eager_time(host_step)
    t = torch.tensor([shard_s, gather_s, merge_s, step_s, e2e_s], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    shard_s, gather_s, merge_s, step_s, e2e_s = t.tolist()
    # the merged output against this rank's own whole-context decode is not
    # available (no rank holds the whole context); report the output's norm
    # agreement across ranks instead: every rank must hold the same result
    chk = out.double().norm().reshape(1)
    if world > 1:
        lo, hi = chk.clone(), chk.clone()
        dist.all_reduce(lo, op=dist.ReduceOp.MIN)
        dist.all_reduce(hi, op=dist.ReduceOp.MAX)
        same = bool(lo.item() == hi.item())
    else:
        same = True
    del caches, cache
    torch.cuda.empty_cache()
    return {"workload": name, "context": T, "shard_tokens": [cp.shard_range(T, world, r)[1] -
                                                               cp.shard_range(T, world, r)[0]
                                                               for r in range(world)],
            "shard_bytes_max": kv_bytes(w, [cp.shard_range(T, world, 0)[1]] * B),
            "kv_bytes": total_bytes, "step_s": step_s, "shard_s": shard_s, "gather_s": gather_s,
            "merge_s": merge_s, "n_rot": n_rot, "outputs_equal_across_ranks": same,
            "gather_bytes_per_rank": int((local.numel() + lse.numel()) * 4), "e2e_s": e2e_s,
            "h2d_bytes": int(h_q.numel() * h_q.element_size()),
            "d2h_bytes": int(h_out.numel() * h_out.element_size())}


def run_context_parallel(args):
    """bench.py --mode context-parallel: one context split over the ranks."""
    import torch
    import torch.distributed as dist
    from compressed_domain_attention_tq_b200 import _lib
    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    _lib.set_test_hooks(_lib.TEST_HOOK_TCGEN05_DECODE if args.decode_kernel == "tcgen05" else 0)
    stream = torch.cuda.current_stream()
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    peak, peak_kind = measured_peaks()
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid)) if rank == 0 else None
    main_r = cp_measure(args.workload, args, world, rank, dev, stream, l2_bytes)
    long_r = cp_measure("llama70b_gqa_1m", args, world, rank, dev, stream, l2_bytes)
    clocks = sampler.stop() if sampler else None

    def entry(r):
        return {"workload": r["workload"], "context": r["context"], "shard_tokens": r["shard_tokens"],
                "us_per_step": round(r["step_s"] * 1e6, 2),
                "kv_GB_per_s": round(r["kv_bytes"] / r["step_s"] / 1e9, 1),
                "shard_decode_us": round(r["shard_s"] * 1e6, 2),
                "gather_us": round(r["gather_s"] * 1e6, 2),
                "merge_lse_us": round(r["merge_s"] * 1e6, 2),
                "shard_roofline_frac": round(r["shard_bytes_max"] / r["shard_s"] / 1e9 / peak, 4),
                "outputs_equal_across_ranks": r["outputs_equal_across_ranks"],
                "l2": f"shard decodes rotated over {r['n_rot']} cache copies"}

    m = main_r
    res = {
        "metric": METRIC, "value": round(m["kv_bytes"] / m["step_s"] / 1e9, 1), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(m["step_s"] * 1e3, 5), "us_per_step": round(m["step_s"] * 1e6, 2),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "int4 codes, fp32 accumulation", "data": "synthetic (seeded N(0,1), bf16)",
        "config": {"workload": m["workload"], "mode": "context-parallel", "context": m["context"],
                   "parallelism": f"context shards x{world}",
                   "partitioning": ("contiguous token shards of the one sequence, rank r holding "
                                    "tokens [r T / N, (r + 1) T / N); per step every rank decodes its "
                                    "shard (tq_sdpa_int4_decode_lse), the ranks all-gather the "
                                    "(o, max, sum) parts over NCCL, every rank merges them "
                                    "(tq_merge_lse)"),
                   "gather_bytes_per_rank": m["gather_bytes_per_rank"], "decode_kernel": args.decode_kernel},
        "context_parallel": entry(m),
        "long_context": entry(long_r),
        "roofline": {"bound": "hbm", "kernel": "sdpa_int4 decode of one shard (split-K + merge)",
                     "achieved": round(m["shard_bytes_max"] / m["shard_s"] / 1e9, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(m["shard_bytes_max"] / m["shard_s"] / 1e9 / peak, 4),
                     "peak_kind": peak_kind, "traffic": None},
        "e2e": {"value": round(m["kv_bytes"] / m["e2e_s"] / 1e9, 1), "unit": "GB/s",
                "us_per_step": round(m["e2e_s"] * 1e6, 2), "h2d_bytes_per_step": m["h2d_bytes"],
                "d2h_bytes_per_step": m["d2h_bytes"]},
        "gpu_launches": 3 * args.steps,
        "step": ("per rank: tq_sdpa_int4_decode_lse on its shard (split-K kernel + merge, 2 launches), "
                 "NCCL all_gather of the (o, max, sum) parts, tq_merge_lse (1 launch)"),
        "timing": ("shard decode and tq_merge_lse: K calls in one CUDA graph each, between CUDA "
                   "events; gather and the whole step: K eager calls back to back between events "
                   "(includes host enqueue time where it exceeds the device time); e2e: the eager "
                   "step with q copied in from pinned host memory and the output copied back; "
                   "every figure the max over ranks"),
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.mode == "context-parallel":
        run_context_parallel(args)
    else:
        run_tq(args)


if __name__ == "__main__":
    main()
