#!/usr/bin/env python
"""Benchmark of the structured-mask attention hot path on B200.

Step = one pass of the DFlash hot path over one batch of the long-context
workload (B=1, H=32, KVH=8, d=128, bf16, 32768 context keys, 2048 draft blocks
of 16, is_causal=True, full-attention layer): the analytic block map
(dfa_block_map) followed by the tensor-core forward (dfa_attn_fwd) on it.
Metric: kept-tile TFLOP/s = 4 * 128 * 128 * d * H * (FULL + PARTIAL 128x128
tiles) / time.  Inputs are resident in HBM and larger than L2 (268 MB of Q,
268 MB of K/V), so no flush is needed between steps.

``--impl reference`` times the float64 CPU oracle (dense mask + dense
softmax attention) on a bounded sample of the same workload on the host
cores.  Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as wl  # noqa: E402

METRIC = "masked-attn fwd TFLOP/s (kept tiles) & % bf16 peak; top-k mask GB/s, 1 B200"
WORKLOAD = wl.DFLASH_LONG_FULL
TILE = 128
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tile_flops(d: int, heads: int, kept_tiles: int) -> float:
    return 4.0 * TILE * TILE * d * heads * kept_tiles


def config_dict(w, extra=None):
    c = {"workload": f"{w.name}: B={w.batch}, H={w.heads}, KVH={w.kv_heads}, d={w.head_dim}, "
                     f"{w.dtype}, ctx_len={w.ctx_len}, {w.n_blocks} blocks of {w.block_size}, "
                     f"is_causal={w.is_causal}, layer={'sliding W=%d' % w.sliding_window if w.layer_type else 'full'}",
         "global_batch": w.batch, "seq_len": w.n_k, "l2": "inputs larger than L2 (no flush)"}
    if extra:
        c.update(extra)
    return c


# ---------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"sma_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------- helpers


def max_over_ranks(ms: float, world: int, device) -> float:
    """The job's time: the slowest rank's, returned on every rank (one
    all-reduce; a single process returns its own)."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank: float, ms_per_step: float) -> float:
    """Units per second of the whole job: every rank processes its own
    units_per_rank each step (replicas, weak scaling) in ms_per_step."""
    return world * units_per_rank / (ms_per_step * 1e-3)


def timed(fn, stream, reps, warmup):
    """Average ms of fn() over reps, CUDA events on `stream`."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(reps):
        fn()
    e.record(stream)
    torch.cuda.synchronize()
    return s.elapsed_time(e) / reps


# Committed ncu summaries of the headline kernel's DRAM traffic carry two
# machine-readable lines: the bytes (read + write) of one launch and a
# SHA-256 of the kernel's sources when the counters were taken.  The figure is
# reported only while the sources still hash the same; once the kernel
# changes it is stale and roofline.traffic is null.
KERNEL_SOURCES = ("structured_mask_attention_analytic_b200/csrc/attn_tc.cu",
                  "structured_mask_attention_analytic_b200/csrc/device_common.cuh")


def kernel_source_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(workload_name: str):
    """(bytes per launch, summary path) from the committed ncu traffic summary
    of the workload's attention launch, if it was captured on the current
    kernel sources, else (None, reason)."""
    path = os.path.join(ROOT, "profiles", f"attn_tc_{workload_name}_traffic.md")
    if not os.path.exists(path):
        return None, "no ncu traffic summary for this workload"
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.startswith("- "):
                key, val = line[2:].split(":", 1)
                vals[key.strip()] = val.strip().strip("`")
    if "traffic_bytes_per_launch" not in vals or "kernel_source_sha256" not in vals:
        return None, "summary lacks traffic_bytes_per_launch / kernel_source_sha256"
    if vals["kernel_source_sha256"] != kernel_source_sha256():
        return None, "stale: kernel sources changed since the capture"
    return float(vals["traffic_bytes_per_launch"]), os.path.relpath(path, ROOT)


def timed_graph(fn, reps, warmup):
    """Average ms of one replay of a CUDA graph holding one fn() call (the
    same launches without the Python / ctypes issue time between them)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    side = torch.cuda.current_stream()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(side)
    for _ in range(reps):
        g.replay()
    e.record(side)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / reps
    del g
    return ms


def dflash_case(w, dev, seed=None):
    q, k, v, anchors = wl.dflash_inputs(w, seed)
    return tuple(t.to(dev) for t in (q, k, v, anchors))


# ---------------------------------------------------------------- our arm


def run_ours(args, rank, world, dev):
    import structured_mask_attention_analytic_b200 as sma

    peaks, peak_src = load_peaks()
    w = workload_by_name(args.workload)
    q, k, v, anchors = dflash_case(w, dev, seed=w.seed + rank)
    stream = torch.cuda.current_stream(dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.batch, w.heads, w.n_q), dtype=torch.float32, device=dev)
    nq_t, nk_t = sma.dfa_block_map_dims(w.batch, w.n_blocks, w.block_size, w.ctx_len, w.is_causal,
                                        w.layer_type, w.sliding_window)
    bm = [torch.empty((w.batch, nq_t), dtype=torch.int32, device=dev),
          torch.empty((w.batch, nq_t, nk_t), dtype=torch.int32, device=dev),
          torch.empty((w.batch, nq_t), dtype=torch.int32, device=dev),
          torch.empty((w.batch, nq_t, nk_t), dtype=torch.int32, device=dev)]

    def block_map():
        r = sma.dfa_block_map(anchors, w.ctx_len, w.block_size, w.is_causal, w.layer_type,
                              w.sliding_window)
        for dst, src in zip(bm, r):
            dst.copy_(src)  # noqa -- keeps the map in fixed buffers (not timed)

    # map once to count kept tiles
    block_map()
    torch.cuda.synchronize()
    kept = int((bm[0] + bm[2]).sum().item())
    flops = tile_flops(w.head_dim, w.heads, kept)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    from structured_mask_attention_analytic_b200 import _native as nat
    import ctypes
    lib = nat.load()
    desc = nat.DfaMaskDesc(w.batch, w.n_blocks, w.block_size, w.ctx_len, w.is_causal, w.layer_type,
                           w.sliding_window)
    maps = nat.DfaBlockMapPtrs(bm[0].data_ptr(), bm[1].data_ptr(), bm[2].data_ptr(), bm[3].data_ptr())
    st = ctypes.c_void_p(stream.cuda_stream)
    qs, ks, vs, os_ = (nat.i64_array(t.stride()[:3]) for t in (q, k, v, out))

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        nat.check(lib.dfa_block_map(ctypes.byref(desc), ctypes.c_void_p(anchors.data_ptr()),
                                    ctypes.c_void_p(bm[0].data_ptr()), ctypes.c_void_p(bm[1].data_ptr()),
                                    ctypes.c_void_p(bm[2].data_ptr()), ctypes.c_void_p(bm[3].data_ptr()), st))
        if evs:
            evs[1].record(stream)
        nat.check(lib.dfa_attn_fwd(ctypes.byref(desc), ctypes.c_void_p(anchors.data_ptr()), nat.SMA_BF16,
                                   w.heads, w.kv_heads, w.head_dim, ctypes.c_float(0.0),
                                   ctypes.c_void_p(q.data_ptr()), qs, ctypes.c_void_p(k.data_ptr()), ks,
                                   ctypes.c_void_p(v.data_ptr()), vs, ctypes.c_void_p(out.data_ptr()), os_,
                                   ctypes.c_void_p(lse.data_ptr()), ctypes.byref(maps), None, 0, st))
        if evs:
            evs[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(ev[i])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert sma.device_status(dev) == 0
    total_ms = t0.elapsed_time(t1)
    attn_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(args.steps)]
    map_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(world, flops, ms_per_step) / 1e12
    attn_avg = sum(attn_ms) / len(attn_ms)
    achieved = flops / (attn_avg * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    if args.traffic_bytes is not None:
        traffic, traffic_src = args.traffic_bytes, "--traffic-bytes"
    else:
        traffic, traffic_src = measured_traffic(w.name)

    # end to end: host buffers in pinned memory, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        qh, kh, vh, ah = (t.cpu().pin_memory() for t in (q, k, v, anchors))
        oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        lh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        qd, kd, vd, ad = (torch.empty_like(t) for t in (q, k, v, anchors))
        ws = torch.empty(sma.dfa_attn_fwd_workspace_size(w.batch, w.n_blocks, w.block_size, w.ctx_len,
                                                         w.heads, w.kv_heads, w.head_dim, w.is_causal,
                                                         w.layer_type, w.sliding_window),
                         dtype=torch.uint8, device=dev)

        def e2e_step():
            for d_, h_ in ((qd, qh), (kd, kh), (vd, vh), (ad, ah)):
                d_.copy_(h_, non_blocking=True)
            _, lse_step = sma.dfa_attn_fwd(qd, kd, vd, ad, w.ctx_len, w.block_size, w.is_causal,
                                           w.layer_type, w.sliding_window, out=out, workspace=ws)
            oh.copy_(out, non_blocking=True)
            lh.copy_(lse_step, non_blocking=True)

        e_ms = timed(e2e_step, stream, args.e2e_steps, 2)
        h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh, ah))
        d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()
        e_ms = max_over_ranks(e_ms, world, dev)
        e2e = {"value": job_throughput(world, flops, e_ms) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}
        del qh, kh, vh, oh

    details = {}
    if not args.no_details and rank == 0:
        details = run_details(sma, dev, stream, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_tiles)

    res = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16, sorted random anchors)",
        "config": config_dict(w, {"parallelism": f"replicas x{world} (one long-context batch per GPU)",
                                  "kept_tiles": kept, "flops_per_step": flops}),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "traffic": traffic, "traffic_source": traffic_src,
                     "kernel": "attn_tc_kernel<128, DFlash, bf16>",
                     "peak_source": f"{peak_src} bf16 dense burst",
                     "frac_of_spec_2250": achieved / 2250.0,
                     # context: the measured sustained figure (a GEMM loop held
                     # under the power cap), for runs whose clocks show the cap
                     "frac_of_sustained": achieved / float(peaks["bf16_tflops_sustained"]),
                     "attn_ms": attn_avg, "block_map_ms": sum(map_ms) / len(map_ms)},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 2 * args.steps, "clocks": clk,
        "details": details,
    }
    return res


DETAILS = ("dflash", "dflash_bwd", "spec_generate", "varlen", "broadcast_prefill", "broadcast_decode", "topk", "topk_wide")


def run_details(sma, dev, stream, peaks, only=None):
    """Other workloads, each timed alone (events on the launch stream).
    ``only`` restricts the run to one group of DETAILS."""
    out = {}
    pk_t, pk_b = float(peaks["bf16_tflops"]), float(peaks["hbm_gbs"])

    def want(name):
        return only is None or only == name

    # DFlash: sliding layer of the long-context workload, both training layers
    for w in ((wl.DFLASH_LONG_SLIDING, wl.DFLASH_TRAIN_FULL, wl.DFLASH_TRAIN_SLIDING) if want("dflash") else ()):
        q, k, v, anchors = dflash_case(w, dev)
        bmap = sma.dfa_block_map(anchors, w.ctx_len, w.block_size, w.is_causal, w.layer_type, w.sliding_window)
        kept = int((bmap[0] + bmap[2]).sum().item())
        o = torch.empty_like(q)
        ms = timed(lambda: sma.dfa_attn_fwd(q, k, v, anchors, w.ctx_len, w.block_size, w.is_causal, w.layer_type,
                                            w.sliding_window, out=o, block_map=bmap), stream, 10, 3)
        tf = tile_flops(w.head_dim, w.heads, kept) / (ms * 1e-3) / 1e12
        out[w.name] = {"ms": ms, "TFLOP/s": tf, "frac_bf16_peak": tf / pk_t, "kept_tiles": kept}
        del q, k, v, o

    # backward of the DFlash layers: 5 products per kept tile (2.5x the forward's work)
    for w in ((wl.DFLASH_TRAIN_FULL, wl.DFLASH_TRAIN_SLIDING, wl.DFLASH_LONG_FULL) if want("dflash_bwd") else ()):
        q, k, v, anchors = dflash_case(w, dev)
        args = (anchors, w.ctx_len, w.block_size, w.is_causal, w.layer_type, w.sliding_window)
        bmap = sma.dfa_block_map(*args)
        kept = int((bmap[0] + bmap[2]).sum().item())
        o, lse = sma.dfa_attn_fwd(q, k, v, *args)
        do = torch.randn_like(q)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(sma.dfa_attn_bwd_workspace_size(q.shape[0], anchors.shape[1], w.block_size, w.ctx_len,
                                                         w.heads, w.kv_heads, w.head_dim, w.is_causal, w.layer_type,
                                                         w.sliding_window), dtype=torch.uint8, device=dev)
        ms = timed(lambda: sma.dfa_attn_bwd(q, k, v, o, lse, do, *args, dq=dq, dk=dk, dv=dv, workspace=ws),
                   stream, 5, 2)
        tf = 2.5 * tile_flops(w.head_dim, w.heads, kept) / (ms * 1e-3) / 1e12
        out[w.name + "_bwd"] = {"ms": ms, "TFLOP/s": tf, "frac_bf16_peak": tf / pk_t, "kept_tiles": kept,
                                "status": sma.device_status()}
        del q, k, v, o, lse, do, dq, dk, dv, ws
        torch.cuda.empty_cache()

    if want("spec_generate"):
        # DFlash inference: one block of 16 draft queries after a 32k context (HBM-bound: K/V read once)
        wd = wl.DFLASH_LONG_FULL
        bs, lc = wd.block_size, wd.ctx_len
        g = torch.Generator(device=dev).manual_seed(7)
        q = torch.randn((1, bs, wd.heads, wd.head_dim), device=dev, generator=g).to(torch.bfloat16)
        k = torch.randn((1, lc + bs, wd.kv_heads, wd.head_dim), device=dev, generator=g).to(torch.bfloat16)
        v = torch.randn_like(k)
        cl = torch.tensor([lc], dtype=torch.int32, device=dev)
        o = torch.empty_like(q)
        call = lambda: sma.dflash_spec_generate_fwd(q, k, v, cl, lc, True, out=o)
        ms_eager = timed(call, stream, 20, 3)
        ms = timed_graph(call, 20, 3)  # block map, attention, combine: one graph replay
        nbytes = 2 * k.numel() * 2 + 2 * q.numel() * 2
        out["spec_generate_32k"] = {"ms": ms, "GB/s": nbytes / (ms * 1e-3) / 1e9,
                                    "frac_hbm_peak": nbytes / (ms * 1e-3) / 1e9 / pk_b, "bytes": nbytes,
                                    "timing": "CUDA graph replay of the call's 3 launches",
                                    "ms_python_calls": ms_eager}
        del q, k, v, o

    if want("varlen"):
        # packed causal training batch: 12 sequences of random lengths up to 8192 (seed 5), H 32 / KVH 8, d 128
        rng = np.random.default_rng(5)
        lens = rng.integers(256, 8193, size=12).tolist()
        cu = torch.tensor(np.cumsum([0] + lens), dtype=torch.int32, device=dev)
        total = int(sum(lens))
        g = torch.Generator(device=dev).manual_seed(5)
        q = torch.randn((total, 32, 128), device=dev, generator=g).to(torch.bfloat16)
        k = torch.randn((total, 8, 128), device=dev, generator=g).to(torch.bfloat16)
        v = torch.randn_like(k)
        o = torch.empty_like(q)
        ms = timed(lambda: sma.varlen_attn_fwd(q, k, v, cu, cu, max(lens), max(lens), True, out=o), stream, 10, 3)
        kept = sum(sum(1 for a in range(-(-L // TILE)) for c in range(-(-L // TILE)) if c <= a) for L in lens)
        tf = tile_flops(128, 32, kept) / (ms * 1e-3) / 1e12
        out["varlen_causal_12seq"] = {"ms": ms, "TFLOP/s": tf, "frac_bf16_peak": tf / pk_t, "tokens": total,
                                      "kept_tiles_per_head": kept}
        # backward of the same batch: 5 products per kept tile (2.5x the forward's work)
        o, lse = sma.varlen_attn_fwd(q, k, v, cu, cu, max(lens), max(lens), True, out=o)
        do = torch.randn(q.shape, device=dev, generator=g).to(torch.bfloat16)
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
        ms_b = timed(lambda: sma.varlen_attn_bwd(q, k, v, o, lse, do, cu, cu, max(lens), max(lens), True,
                                                 dq=grads[0], dk=grads[1], dv=grads[2]), stream, 5, 2)
        tf_b = 2.5 * tile_flops(128, 32, kept) / (ms_b * 1e-3) / 1e12
        out["varlen_causal_12seq_bwd"] = {"ms": ms_b, "TFLOP/s": tf_b, "frac_bf16_peak": tf_b / pk_t,
                                          "status": sma.device_status()}
        del q, k, v, o, do, grads

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    if want("broadcast_prefill"):
        _detail_prefill(sma, dev, stream, out, pk_t)
    if want("broadcast_decode"):
        _detail_decode(sma, dev, stream, out, pk_b, flush)
    if want("topk"):
        _detail_topk(sma, dev, stream, out, pk_t, pk_b, flush)
    if want("topk_wide"):
        _detail_topk_wide(sma, dev, stream, out, pk_b)
    del flush
    torch.cuda.empty_cache()
    return out


def _detail_prefill(sma, dev, stream, out, pk_t):
    w = wl.BROADCAST_PREFILL
    q, k, v, mask, bias = (None if t is None else t.to(dev) for t in wl.masked_inputs(w))
    codes = sma.mask_tile_summary(mask, w.n_k)
    kept_per_bh = int((codes != 0).sum().item())
    o = torch.empty_like(q)
    ws = torch.empty(sma.masked_attn_fwd_workspace_size(w.batch, w.heads, w.kv_heads, w.n_q, w.n_k, w.head_dim,
                                                        tuple(mask.shape)), dtype=torch.uint8, device=dev)
    ms = timed(lambda: sma.masked_attn_fwd(q, k, v, mask, bias, w.is_causal, out=o, workspace=ws), stream, 10, 3)
    tf = tile_flops(w.head_dim, w.heads * w.batch, kept_per_bh) / (ms * 1e-3) / 1e12
    ms_sum = timed(lambda: sma.mask_tile_summary(mask, w.n_k), stream, 10, 3)
    mbytes = mask.numel()
    out[w.name] = {"ms": ms, "TFLOP/s": tf, "frac_bf16_peak": tf / pk_t, "kept_tiles_per_bh": kept_per_bh,
                   "mask_summary_ms": ms_sum, "mask_summary_GB/s": mbytes / (ms_sum * 1e-3) / 1e9}
    del q, k, v, mask, bias, o


def _detail_decode(sma, dev, stream, out, pk_b, flush):
    # decode (swapped grouped-head path): HBM-bound
    w = wl.BROADCAST_DECODE
    q, k, v, mask, bias = (None if t is None else t.to(dev) for t in wl.masked_inputs(w))
    o = torch.empty_like(q)
    ws = torch.empty(sma.masked_attn_fwd_workspace_size(w.batch, w.heads, w.kv_heads, 1, w.n_k, w.head_dim),
                     dtype=torch.uint8, device=dev)

    def dec():
        sma.masked_attn_fwd(q, k, v, None, bias, False, out=o, workspace=ws)

    # K/V (537 MB) exceed L2; time with a flush between calls anyway (flush excluded)
    times = []
    for _ in range(13):
        flush.fill_(1)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        dec()
        e.record(stream)
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e))
    ms = statistics.median(times[3:])
    nbytes = 2 * k.numel() * 2 + bias.numel() * 2 + q.numel() * 2 * 2
    gbs = nbytes / (ms * 1e-3) / 1e9
    out[w.name] = {"ms": ms, "GB/s": gbs, "frac_hbm_peak": gbs / pk_b, "bytes": nbytes}
    del q, k, v, bias, o


def _detail_topk(sma, dev, stream, out, pk_t, pk_b, flush):
    # top-k mask, then attention under it
    w = wl.TOPK
    bias, pre = (t.to(dev) for t in wl.topk_inputs(w))
    keep = torch.empty(bias.shape, dtype=torch.bool, device=dev)
    times = []
    for _ in range(13):
        flush.fill_(1)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        sma.dynamic_topk_mask(bias, w.n_k, w.window, pre, out=keep)
        e.record(stream)
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e))
    ms = statistics.median(times[3:])
    nbytes = bias.numel() * 2 + pre.numel() + keep.numel()
    out[w.name + "_mask"] = {"ms": ms, "GB/s": nbytes / (ms * 1e-3) / 1e9, "bytes": nbytes,
                             "frac_hbm_peak": nbytes / (ms * 1e-3) / 1e9 / pk_b,
                             "note": "0.8 MB of traffic: launch-latency bound"}
    q, k, v = (t.to(dev) for t in wl.topk_attention_inputs(w))
    o = torch.empty_like(q)
    ms = timed(lambda: sma.masked_attn_fwd(q, k, v, keep, None, True, out=o), stream, 10, 3)
    off = w.n_k - w.n_q
    qt_n, kt_n = -(-w.n_q // TILE), -(-w.n_k // TILE)
    kept = sum(1 for a in range(qt_n) for c in range(kt_n) if c * TILE <= min((a + 1) * TILE, w.n_q) - 1 + off)
    tf = tile_flops(w.head_dim, w.heads * w.batch, kept) / (ms * 1e-3) / 1e12
    out[w.name + "_attention"] = {"ms": ms, "TFLOP/s": tf, "frac_bf16_peak": tf / pk_t, "kept_tiles_per_bh": kept}
    # index-gather path over the same mask: compacted key tiles per (b, kv head, q tile)
    ws = torch.empty(sma.sparse_attn_fwd_workspace_size(q.dtype, w.batch, w.heads, w.kv_heads, w.n_q, w.n_k,
                                                        w.head_dim, tuple(keep.shape), max_keys=w.window),
                     dtype=torch.uint8, device=dev)
    ms_g = timed(lambda: sma.sparse_attn_fwd(q, k, v, keep, None, True, max_keys=w.window, out=o, workspace=ws),
                 stream, 10, 3)
    km = keep[:, :, 0, :w.n_k].cpu()
    ctiles = 0
    for row in km.reshape(-1, w.n_k):
        idx = torch.nonzero(row).flatten()
        for a in range(qt_n):
            lim = int(torch.searchsorted(idx, min((a + 1) * TILE, w.n_q) - 1 + off, right=True))
            ctiles += -(-lim // TILE)
    group = w.heads // w.kv_heads
    tf_c = tile_flops(w.head_dim, group, ctiles) / (ms_g * 1e-3) / 1e12
    out[w.name + "_attention_gather"] = {
        "ms": ms_g, "speedup_vs_dense_walk": ms / ms_g,
        "TFLOP/s_compacted_tiles": tf_c, "frac_bf16_peak": tf_c / pk_t,
        "TFLOP/s_dense_tile_equivalent": tile_flops(w.head_dim, w.heads * w.batch, kept) / (ms_g * 1e-3) / 1e12,
        "compacted_tiles": ctiles}
    del q, k, v, o, bias, pre, keep, ws


def _detail_topk_wide(sma, dev, stream, out, pk_b):
    w = wl.TOPK_WIDE
    bias, pre = (t.to(dev) for t in wl.topk_inputs(w))
    keep = torch.empty(bias.shape, dtype=torch.bool, device=dev)
    ms = timed(lambda: sma.dynamic_topk_mask(bias, w.n_k, w.window, pre, out=keep), stream, 5, 2)
    nbytes = bias.numel() * 2 + pre.numel() + keep.numel()
    out[w.name + "_mask"] = {"ms": ms, "GB/s": nbytes / (ms * 1e-3) / 1e9, "frac_hbm_peak": nbytes / (ms * 1e-3) / 1e9 / pk_b,
                             "bytes": nbytes}
    del bias, pre, keep


# ---------------------------------------------------------------- oracle arm


class OracleSampler:
    """The float64 CPU oracle (dense mask + dense softmax attention) on chosen
    query tiles of a DFlash workload, all heads; inputs drawn once."""

    def __init__(self, w):
        from oracle import attention as at
        from oracle import dflash_mask as dm
        from oracle import tiles as tl

        self.at, self.dm, self.tl, self.w = at, dm, tl, w
        q, k, v, anchors = wl.dflash_inputs(w)
        self.q = q
        self.k, self.v = k.double().numpy(), v.double().numpy()
        self.a = anchors.numpy()
        self.causal = dm.resolve_in_block_causal(w.is_causal, w.layer_type)
        self.win = dm.resolve_window(w.layer_type, w.sliding_window) if w.layer_type == dm.LAYER_SLIDING else None
        self.threads = at.host_threads()
        self.qt_n = -(-w.n_q // TILE)

    def spread(self, n):
        return sorted(set(int(round(x)) for x in np.linspace(0, self.qt_n - 1, n)))

    def run(self, tiles):
        """Seconds spent in the oracle and kept-tile FLOPs of the sample."""
        w, dm, tl = self.w, self.dm, self.tl
        rows = [(t * TILE, min((t + 1) * TILE, w.n_q)) for t in tiles]
        kept = 0
        for (r0, r1) in rows:
            keep = dm.dflash_keep_rows(self.a[:1], w.ctx_len, w.block_size, self.causal, self.win, r0, r1)[0]
            kept += int((tl.tile_codes(keep, w.n_k) != tl.EMPTY).sum())
        qs = np.concatenate([self.q[:, r0:r1].double().numpy() for r0, r1 in rows], axis=1)
        starts = np.concatenate([np.full(r1 - r0, r0 - i * TILE) for i, (r0, r1) in enumerate(rows)])

        def keep_rows(b, q0, q1):
            off = int(starts[q0])
            return dm.dflash_keep_rows(self.a[b:b + 1], w.ctx_len, w.block_size, self.causal, self.win,
                                       q0 + off, q1 + off)

        try:
            from threadpoolctl import threadpool_limits
            ctx = threadpool_limits(1)
        except Exception:  # pragma: no cover
            import contextlib
            ctx = contextlib.nullcontext()
        with ctx:
            t0 = time.perf_counter()
            self.at.attention(qs, self.k, self.v, keep_rows=keep_rows, workers=self.threads, row_chunk=TILE)
            sec = time.perf_counter() - t0
        return sec, tile_flops(w.head_dim, w.heads, kept)


def cpu_baseline(w, n_tiles):
    s = OracleSampler(w)
    tiles = s.spread(n_tiles)
    sec, flops = s.run(tiles)
    return {"value": flops / sec / 1e12, "unit": "TFLOP/s", "cores": s.threads, "kind": "oracle",
            "sample": f"{len(tiles)} of {s.qt_n} query tiles spread over the sequence (all {w.heads} heads; "
                      f"float64 dense mask + softmax over all {w.n_k} keys); kept-tile FLOPs of the sample "
                      f"/ {sec:.1f} s"}


def run_reference(args, rank, world):
    """The oracle as the reference arm: every step (warm-up included) is one
    query tile of the workload, cycling over tiles spread along the sequence."""
    if rank != 0:
        return None
    w = workload_by_name(args.workload)
    s = OracleSampler(w)
    order = s.spread(16)
    for i in range(args.warmup):
        s.run([order[i % len(order)]])
    secs, flops = [], []
    for i in range(args.steps):
        sec, f = s.run([order[i % len(order)]])
        secs.append(sec)
        flops.append(f)
    v = sum(flops) / sum(secs) / 1e12
    sample = (f"one of {s.qt_n} query tiles per step (all {w.heads} heads), cycling over 16 tiles spread "
              f"along the sequence; float64 oracle on {s.threads} host threads")
    return {"metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * sum(secs) / len(secs), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(w, {"parallelism": "host cores"}), "impl": "reference",
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": s.threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


DFLASH_WORKLOADS = {x.name: x for x in (wl.DFLASH_LONG_FULL, wl.DFLASH_LONG_SLIDING, wl.DFLASH_TRAIN_FULL,
                                         wl.DFLASH_TRAIN_SLIDING)}


def workload_by_name(name):
    return DFLASH_WORKLOADS[name]


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(DFLASH_WORKLOADS), default=WORKLOAD.name,
                    help="DFlash workload of the step (default: the long-context full layer)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-tiles", type=int, default=8, help="query tiles in the oracle sample")
    ap.add_argument("--no-details", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=DETAILS, default=None,
                    help="time only this group of secondary workloads and print their JSON (profiling aid)")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="DRAM bytes per attention launch from an ncu capture (reported as roofline.traffic)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.only is not None:
        import structured_mask_attention_analytic_b200 as sma
        peaks, _ = load_peaks()
        print(json.dumps({"only": args.only,
                          "details": run_details(sma, dev, torch.cuda.current_stream(dev), peaks, args.only)}))
        return 0
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        res = run_ours(args, rank, world, dev)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
