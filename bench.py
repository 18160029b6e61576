#!/usr/bin/env python
"""Benchmark of the bifocal attention hot path on B200.

One step = one bifocal prefill of a Qwen3-8B-shaped layer at L = 131072 (32
query / 8 KV heads, head_dim 128, w_pretrained 32768 -> G = 4, w0 = 4096) plus
one bifocal decode token against a 131072-token base-RoPE cache (Qwen3-4B
shape: 32 / 8 heads, head_dim 128).  Inputs are seeded synthetic bf16 data
(rope_context_extension_sm_b200.inputs), resident in HBM before timing; both
the prefill inputs (1.5 GB) and the cache (512 MiB) are larger than L2.  The
prefill is the whole jl_bifocal_prefill call with a preallocated key workspace:
the keys' rotation, then the attention kernel.

Prints ONE JSON line (rank 0).  ``value`` is useful prefill TFLOP/s (each causal
(q, k) pair counted once at 4 * head_dim flops per query head), aggregated over
ranks; decode latency, the plain comparators, the roofline of the dominant
kernel, the end-to-end number through host buffers and the CPU oracle baseline
ride along in the same line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With --gpus N > 1 (under torchrun) every rank runs an independent replica of the
step; there is no collective on the data path (the method does not need one).
``--impl reference`` times the CPU oracle (the only reference implementation
this method has) on a bounded sample of the same workload.
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
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rope_context_extension_sm_b200 import inputs as I  # noqa: E402

PREFILL = I.QWEN3_8B_128K
DECODE = I.DECODE_QWEN3_4B
DECODE_L = 131072
METRIC = "bifocal prefill useful TFLOP/s at 128K (frac of BF16 peak); decode us/token"
UNIT = "TFLOP/s"
WORKLOAD = "qwen3_8b_prefill_L131072_G4_w0_4096 + qwen3_4b_decode_L131072"


def _config():
    return {
        "workload": WORKLOAD,
        "seq_len": PREFILL.seqlens[0],
        "n_q_heads": PREFILL.n_q_heads,
        "n_kv_heads": PREFILL.n_kv_heads,
        "head_dim": PREFILL.head_dim,
        "w0": PREFILL.w0,
        "w_pretrained": PREFILL.w_pretrained,
        "G": I.QWEN3_8B_128K.seqlens[0] // PREFILL.w_pretrained,
        "decode_cache_len": DECODE_L,
        "decode_heads": [DECODE.n_q_heads, DECODE.n_kv_heads],
        "l2": "inputs larger than L2 (prefill 1.5 GB, decode cache 512 MiB); no flush needed",
        "parallelism": "replicas",
    }


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["bf16_tflops"], p["bf16_tflops_sustained"], p["hbm_gbs"], "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, 1400.0, 6650.0, "fallback"


def _source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


PREFILL_SRC = ["rope_context_extension_sm_b200/csrc/jl_prefill.cuh", "rope_context_extension_sm_b200/csrc/jl_device.cuh"]


def _profiled(kernel, files, key):
    """A figure from the committed ncu summary (profiles/traffic.txt), if it was taken on this
    source: DRAM bytes per launch, or the tensor pipe's active fraction."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.txt")) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_hash") != _source_hash(files):
        return None
    return rec.get(key)


def _traffic(kernel, files):
    return _profiled(kernel, files, "dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def _dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def _barrier(world):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def _max_over_ranks(x, world, device="cuda"):
    """Max of a per-rank device time over all ranks (the slowest rank sets the step time)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world, units_per_rank, steps, max_total_ms):
    """Whole-job throughput of N independent replicas: all ranks' units over the slowest rank's time."""
    return world * units_per_rank * steps / (max_total_ms * 1e-3)


def _measure_other_configs(jl, dev, sustained, hbm, _time, _time_graph):
    """The other workloads the metric is reported on, each on its own synthetic inputs.

    - Qwen3-1.7B layer at L = 65536 (G = 2) for every w0 of the window sweep.
    - The packed batch of 8 log-uniform sequences (4K-128K).
    - A batched decode: 8 entries, cache lengths 8K-128K (each its own G), one token each.
    """
    res = {}
    cfg = I.QWEN3_1P7B
    q, k, v, cu = [t.to(dev) for t in I.prefill_inputs(cfg)]
    L = cfg.seqlens[0]
    cos, sin = jl.jl_rope_tables(L, cfg.head_dim, cfg.rope_base, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((cfg.n_q_heads, L), dtype=torch.float32, device=dev)
    kws = torch.empty(jl.jl_bifocal_prefill_workspace_size(L, cfg.n_kv_heads, cfg.head_dim), dtype=torch.uint8,
                      device=dev)
    flops = cfg.useful_flops()
    sweep = {}
    for _ in range(10):  # ~0.2 s of the same work first, so every point runs at the steady-state clock
        jl.jl_bifocal_prefill(q, k, v, cu, L, cfg.w0, cfg.w_pretrained, cos, sin, out=out, lse=lse, workspace=kws)
    for w0 in I.W0_SWEEP:
        fn = lambda w0=w0: jl.jl_bifocal_prefill(q, k, v, cu, L, w0, cfg.w_pretrained, cos, sin, out=out, lse=lse,
                                                 workspace=kws)
        fn()
        ms = _time(fn, 5)
        sweep[str(w0)] = {"ms": round(ms, 3), "useful_tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                          "frac_of_bf16_peak_measured_sustained": round(flops / (ms * 1e-3) / 1e12 / sustained, 4)}
    pl = lambda: jl.jl_plain_prefill(q, k, v, cu, L, cos, sin, out=out, lse=lse, workspace=kws)
    pl()
    ms = _time(pl, 5)
    res["qwen3_1p7b_L65536_G2"] = {"w0_sweep": sweep, "plain_ms": round(ms, 3),
                                   "plain_useful_tflops": round(flops / (ms * 1e-3) / 1e12, 2)}
    del q, k, v, out, lse, cos, sin, kws

    cfg = I.VARLEN
    q, k, v, cu = [t.to(dev) for t in I.prefill_inputs(cfg)]
    mx = cfg.max_seqlen
    cos, sin = jl.jl_rope_tables(mx, cfg.head_dim, cfg.rope_base, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((cfg.n_q_heads, q.shape[0]), dtype=torch.float32, device=dev)
    kws = torch.empty(jl.jl_bifocal_prefill_workspace_size(q.shape[0], cfg.n_kv_heads, cfg.head_dim),
                      dtype=torch.uint8, device=dev)
    flops = cfg.useful_flops()
    fn = lambda: jl.jl_bifocal_prefill(q, k, v, cu, mx, cfg.w0, cfg.w_pretrained, cos, sin, out=out, lse=lse,
                                       workspace=kws)
    fn()
    ms = _time(fn, 3)
    res["varlen_8seq"] = {"seqlens": list(cfg.seqlens), "ms": round(ms, 3),
                          "useful_tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                          "frac_of_bf16_peak_measured_sustained": round(flops / (ms * 1e-3) / 1e12 / sustained, 4)}
    del q, k, v, out, lse

    dc = DECODE
    lens = [8192, 16384, 32768, 49152, 65536, 98304, 114688, 131072]
    B, stride = len(lens), max(lens)
    gen = torch.Generator(device=dev).manual_seed(11)  # timing-only inputs, drawn on the device
    kc = torch.randn((B, stride, dc.n_kv_heads, dc.head_dim), generator=gen, device=dev).to(torch.bfloat16)
    vc = torch.randn((B, stride, dc.n_kv_heads, dc.head_dim), generator=gen, device=dev).to(torch.bfloat16)
    qd = torch.randn((B, dc.n_q_heads, dc.head_dim), generator=gen, device=dev).to(torch.bfloat16)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    dcos, dsin = jl.jl_rope_tables(stride, dc.head_dim, dc.rope_base, device=dev)
    ws = torch.empty(jl.jl_bifocal_decode_workspace_size(B, dc.n_q_heads, dc.head_dim, stride), dtype=torch.uint8,
                     device=dev)
    dout = torch.empty_like(qd)
    dlse = torch.empty((B, dc.n_q_heads), dtype=torch.float32, device=dev)
    fn = lambda: jl.jl_bifocal_decode(qd, kc, vc, sl, stride, dc.w0, dc.w_pretrained, dcos, dsin, out=dout, lse=dlse,
                                      workspace=ws)
    us = _time_graph([fn], 100) * 1e3
    kv_bytes = sum(2 * Lb * dc.n_kv_heads * dc.head_dim * 2 for Lb in lens)
    res["batched_decode_8"] = {"cache_lens": lens, "us_per_step": round(us, 2),
                               "hbm_gbs": round(kv_bytes / (us * 1e-6) / 1e9, 1),
                               "frac_of_hbm_measured": round(kv_bytes / (us * 1e-6) / 1e9 / hbm, 4)}
    return res


def _measure_next_rows(jl, dev, stream, q, k, v, cu, cos, sin, out, lse, fused_ms, dk, dv, dq, dsl, dout, dlse,
                       dws, dec_ms, hbm, sustained, _time, _time_graph):
    """Device time of the rows built beyond the hot path, on the bench's own shapes.

    - Literal three-pass prefill: the Qwen3-8B layer at L = 131072.
    - KV-cache fill: the same layer's K/V into a base-RoPE cache.
    - Prefill writing that cache itself (jl_bifocal_prefill_and_cache).
    - Decode append: one token.
    - Chunked prefill: the last 8192 queries of the 131072-token sequence against the cache
      of the first 122880 tokens plus the chunk.
    - Paged decode: the 131072-token Qwen3-4B cache in 128-token pages in permuted order.
    - Interpolation prefill: the remote pairs at scaled frequencies, lambda = 1/G.
    """
    L = PREFILL.seqlens[0]
    d, hq, hkv = PREFILL.head_dim, PREFILL.n_q_heads, PREFILL.n_kv_heads
    useful = PREFILL.useful_flops()
    rows = {}

    # literal inclusion-exclusion: three passes through the same kernel + the LSE merge
    ws3 = torch.empty(3 * L * hq * d * 4 + 3 * L * hq * 4, dtype=torch.uint8, device=dev)
    three = lambda: jl.jl_bifocal_prefill_three_pass(q, k, v, cu, L, PREFILL.w0, PREFILL.w_pretrained, cos, sin,
                                                      out=out, lse=lse, workspace=ws3)
    three()
    ms = _time(three, 2)
    rows["three_pass_prefill"] = {"ms": round(ms, 3), "useful_tflops": round(useful / (ms * 1e-3) / 1e12, 2),
                                  "frac_of_bf16_peak_measured_sustained": round(useful / (ms * 1e-3) / 1e12 / sustained, 4),
                                  "time_vs_fused": round(ms / fused_ms, 4)}
    del ws3

    # KV-cache fill: raw K, V -> R(j) k and v, one cache entry of L positions
    kc = torch.empty((1, L, hkv, d), dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    fill = lambda: jl.jl_kv_cache_fill(k, v, cu, cos, sin, kc, vc)
    fill()
    ms = _time(fill, 10)
    fill_bytes = 4 * L * hkv * d * 2 + L * (d // 2) * 4 * 2  # K, V read + written, one table row pair per token
    rows["kv_cache_fill"] = {"ms": round(ms, 4), "algorithmic_bytes": fill_bytes,
                             "gbs": round(fill_bytes / (ms * 1e-3) / 1e9, 1),
                             "frac_of_hbm_measured": round(fill_bytes / (ms * 1e-3) / 1e9 / hbm, 4)}

    # the same cache written by jl_bifocal_prefill_and_cache alongside the attention (key workspace)
    pac = lambda: jl.jl_bifocal_prefill_and_cache(q, k, v, cu, L, PREFILL.w0, PREFILL.w_pretrained, cos, sin, kc, vc,
                                                  out=out, lse=lse)
    pac()
    ms = _time(pac, 2)
    rows["prefill_and_cache"] = {"ms": round(ms, 3), "useful_tflops": round(useful / (ms * 1e-3) / 1e12, 2),
                                 "time_vs_prefill": round(ms / fused_ms, 4)}

    # decode append: rotate one token's query, write its key and value (launch-bound)
    sl1 = torch.tensor([L], dtype=torch.int32, device=dev)
    q1 = q[:1].clone()
    k1, v1 = k[:1].clone(), v[:1].clone()
    q1_out = torch.empty_like(q1)
    app = lambda: jl.jl_decode_append(q1, k1, v1, sl1, cos, sin, kc, vc, q_out=q1_out)
    rows["decode_append"] = {"us": round(_time_graph([app], 200) * 1e3, 3)}

    # chunked prefill: the last chunk of queries against the (filled) cache
    chunk = 8192
    past = L - chunk
    qc = q[past:].contiguous()
    cu_c = torch.tensor([0, chunk], dtype=torch.int32, device=dev)
    past_t = torch.tensor([past], dtype=torch.int32, device=dev)
    outc = torch.empty_like(qc)
    lsec = torch.empty((hq, chunk), dtype=torch.float32, device=dev)
    chk = lambda: jl.jl_bifocal_prefill_chunk(qc, cu_c, past_t, chunk, L, kc, vc, PREFILL.w0, PREFILL.w_pretrained,
                                              cos, sin, out=outc, lse=lsec)
    chk()
    ms = _time(chk, 5)
    chunk_flops = 4.0 * d * hq * sum(range(past + 1, L + 1))
    rows["chunked_prefill"] = {"chunk": chunk, "past": past, "ms": round(ms, 3),
                               "useful_tflops": round(chunk_flops / (ms * 1e-3) / 1e12, 2),
                               "frac_of_bf16_peak_measured_sustained":
                                   round(chunk_flops / (ms * 1e-3) / 1e12 / sustained, 4)}
    del kc, vc, qc, outc

    # paged decode: the decode cache as 128-token pages in a permuted pool
    page = 128
    n_pages = DECODE_L // page
    perm = torch.randperm(n_pages, generator=torch.Generator().manual_seed(7)).to(dev)
    kp = torch.empty((n_pages, page, DECODE.n_kv_heads, DECODE.head_dim), dtype=torch.bfloat16, device=dev)
    vp = torch.empty_like(kp)
    kp[perm] = dk.view(n_pages, page, DECODE.n_kv_heads, DECODE.head_dim)
    vp[perm] = dv.view(n_pages, page, DECODE.n_kv_heads, DECODE.head_dim)
    table = perm.to(torch.int32).view(1, n_pages).contiguous()
    pgd = lambda: jl.jl_bifocal_decode_paged(dq, kp, vp, table, dsl, DECODE_L, DECODE.w0, DECODE.w_pretrained, cos,
                                             sin, out=dout, lse=dlse, workspace=dws)
    us = _time_graph([pgd], 200) * 1e3
    kv_bytes = 2 * DECODE_L * DECODE.n_kv_heads * DECODE.head_dim * 2
    rows["paged_decode"] = {"page_size": page, "us_per_token": round(us, 2),
                            "frac_of_hbm_measured": round(kv_bytes / (us * 1e-6) / 1e9 / hbm, 4),
                            "time_vs_contiguous": round(us / (dec_ms * 1e3), 4)}
    del kp, vp

    # frequency-interpolation variant of the remote window (position interpolation, lambda = 1/G)
    G = jl.jl_group_size(L, PREFILL.w_pretrained)
    cr, sr = jl.jl_rope_tables_scaled(L, d, PREFILL.rope_base, [1.0 / G] * (d // 2), device=dev)
    itp = lambda: jl.jl_interp_prefill(q, k, v, cu, L, PREFILL.w0, cos, sin, cr, sr, out=out, lse=lse)
    itp()
    ms = _time(itp, 2)
    rows["interp_prefill"] = {"lambda": "1/G", "ms": round(ms, 3),
                              "useful_tflops": round(useful / (ms * 1e-3) / 1e12, 2),
                              "frac_of_bf16_peak_measured_sustained": round(useful / (ms * 1e-3) / 1e12 / sustained, 4),
                              "time_vs_bifocal": round(ms / fused_ms, 4)}
    del cr, sr
    return rows


def _measure_walk(jl, dev, stream, dk, dv, cos, sin):
    """The generation walk of the decode workload: 256 tokens at query positions 98176 .. 98431,
    crossing L = 98304 -> 98305 where G goes from 3 to 4.  Each step appends the token (its query
    rotated to R(i) q, its key rotated into the base-RoPE cache, its value stored) and decodes it
    against the cache with the correction rotation on the fly.  Every step is timed on the device
    with its own pair of CUDA events; the same walk through the plain decode is the comparator.
    The tokens' q/k/v are seeded random bf16; the cache rows before the walk are the bench's."""
    first, steps = DECODE.walk_first_pos, DECODE.walk_steps
    max_len = first + steps
    hq, hkv, d = DECODE.n_q_heads, DECODE.n_kv_heads, DECODE.head_dim
    gen = torch.Generator(device=dev).manual_seed(5)
    wq = torch.randn((steps, 1, hq, d), generator=gen, device=dev).to(torch.bfloat16)
    wk = torch.randn((steps, 1, hkv, d), generator=gen, device=dev).to(torch.bfloat16)
    wv = torch.randn((steps, 1, hkv, d), generator=gen, device=dev).to(torch.bfloat16)
    sls = torch.arange(first + 1, first + steps + 1, dtype=torch.int32, device=dev).view(steps, 1)
    qt = torch.empty((1, hq, d), dtype=torch.bfloat16, device=dev)
    out = torch.empty_like(qt)
    lse = torch.empty((1, hq), dtype=torch.float32, device=dev)
    ws = torch.empty(jl.jl_bifocal_decode_workspace_size(1, hq, d, max_len), dtype=torch.uint8, device=dev)

    def step(t, plain):
        jl.jl_decode_append(wq[t], wk[t], wv[t], sls[t], cos, sin, dk, dv, q_out=qt)
        if plain:
            jl.jl_plain_decode(qt, dk, dv, sls[t], max_len, cos, sin, out=out, lse=lse, workspace=ws)
        else:
            jl.jl_bifocal_decode(qt, dk, dv, sls[t], max_len, DECODE.w0, DECODE.w_pretrained, cos, sin, out=out,
                                 lse=lse, workspace=ws)

    def walk(plain):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        ev[0].record(stream)
        for t in range(steps):
            step(t, plain)
            ev[t + 1].record(stream)
        torch.cuda.synchronize()
        return [ev[t].elapsed_time(ev[t + 1]) * 1e3 for t in range(steps)]

    walk(False)  # warm: every launch shape of the walk once
    walk(True)
    bif, pln = walk(False), walk(True)
    jl.jl_sync_status()
    Ls = [first + t + 1 for t in range(steps)]
    before = [t for t in range(steps) if jl.jl_group_size(Ls[t], DECODE.w_pretrained) == 3]
    after = [t for t in range(steps) if jl.jl_group_size(Ls[t], DECODE.w_pretrained) == 4]

    def stats(xs):
        return {"min": round(min(xs), 2), "median": round(statistics.median(xs), 2), "max": round(max(xs), 2)}

    def side(ts):
        b, p = [bif[t] for t in ts], [pln[t] for t in ts]
        return {"steps": len(ts), "L": [Ls[ts[0]], Ls[ts[-1]]], "us_per_token": stats(b), "plain_us_per_token": stats(p),
                "overhead_vs_plain": round(statistics.median(b) / statistics.median(p) - 1.0, 4)}

    boundary = Ls.index(first + 128)  # the last step at G = 3 (L = 98304) and the first at G = 4
    return {
        "tokens": steps, "query_positions": [first, first + steps - 1], "G": [3, 4],
        "step": "jl_decode_append + jl_bifocal_decode (plain: jl_decode_append + jl_plain_decode)",
        "us_per_token": stats(bif), "plain_us_per_token": stats(pln),
        "overhead_vs_plain": round(statistics.median(bif) / statistics.median(pln) - 1.0, 4),
        "G3_side": side(before), "G4_side": side(after),
        "around_boundary_us": {str(Ls[t]): round(bif[t], 2) for t in range(boundary - 2, boundary + 3)},
        "plain_around_boundary_us": {str(Ls[t]): round(pln[t], 2) for t in range(boundary - 2, boundary + 3)},
    }


# --------------------------------------------------------------- our arm ----

def _build_decode_cache(L):
    """A resident cache of L positions: random bf16 rows stand for base-rotated keys."""
    k_raw, v = I.decode_raw_inputs(DECODE, L)
    return k_raw, v


def run_ours(args, world, rank, local):
    from rope_context_extension_sm_b200 import build
    if rank == 0:
        build.build()
    if world > 1:
        torch.distributed.barrier()
    from rope_context_extension_sm_b200 import jetlong as jl

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    L = PREFILL.seqlens[0]
    # ---- inputs (host, seeded), then resident in HBM ----
    q_h, k_h, v_h, cu_h = I.prefill_inputs(PREFILL)
    q_h, k_h, v_h = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    q, k, v, cu = q_h.to(dev), k_h.to(dev), v_h.to(dev), cu_h.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((PREFILL.n_q_heads, L), dtype=torch.float32, device=dev)
    cos, sin = jl.jl_rope_tables(L, PREFILL.head_dim, PREFILL.rope_base, device=dev)
    dk_h, dv_h = _build_decode_cache(DECODE_L)
    dk, dv = dk_h.to(dev), dv_h.to(dev)
    dq_h = I.decode_queries(DECODE, 1)[0].contiguous().pin_memory()
    dq = dq_h.to(dev)
    dsl = torch.tensor([DECODE_L], dtype=torch.int32, device=dev)
    dout = torch.empty_like(dq)
    dlse = torch.empty((1, DECODE.n_q_heads), dtype=torch.float32, device=dev)
    dws = torch.empty(jl.jl_bifocal_decode_workspace_size(1, DECODE.n_q_heads, DECODE.head_dim, DECODE_L),
                      dtype=torch.uint8, device=dev)
    # the prefill's rotated keys (base and remote rows), written by its first kernel each call
    kws = torch.empty(jl.jl_bifocal_prefill_workspace_size(L, PREFILL.n_kv_heads, PREFILL.head_dim),
                      dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def prefill():
        jl.jl_bifocal_prefill(q, k, v, cu, L, PREFILL.w0, PREFILL.w_pretrained, cos, sin, out=out, lse=lse,
                              workspace=kws)

    def decode():
        jl.jl_bifocal_decode(dq, dk, dv, dsl, DECODE_L, DECODE.w0, DECODE.w_pretrained, cos, sin, out=dout,
                             lse=dlse, workspace=dws)

    for _ in range(args.warmup):
        prefill()
        decode()
    jl.jl_sync_status()

    sampler = ClockSampler(local)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    _barrier(world)
    sampler.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(K):
        ev[s][0].record(stream)
        prefill()
        ev[s][1].record(stream)
        decode()
        ev[s][2].record(stream)
    t_end.record(stream)
    _barrier(world)
    clocks = sampler.stop()
    jl.jl_sync_status()
    total_ms = _max_over_ranks(t_start.elapsed_time(t_end), world)
    pre_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(K)]
    dec_ms = [ev[s][1].elapsed_time(ev[s][2]) for s in range(K)]
    pre_avg = _max_over_ranks(sum(pre_ms) / K, world)
    dec_avg = _max_over_ranks(sum(dec_ms) / K, world)

    flops = PREFILL.useful_flops()
    value = replica_throughput(world, flops, K, total_ms) / 1e12  # whole job, prefill flops over the step time
    prefill_tflops = flops / (pre_avg * 1e-3) / 1e12
    burst, sustained, hbm, peak_kind = _peaks()
    kv_bytes = 2 * DECODE_L * DECODE.n_kv_heads * DECODE.head_dim * 2
    dec_gbs = kv_bytes / (dec_avg * 1e-3) / 1e9

    # ---- plain comparators, same run ----
    def plain_prefill():
        jl.jl_plain_prefill(q, k, v, cu, L, cos, sin, out=out, lse=lse, workspace=kws)

    def plain_decode():
        jl.jl_plain_decode(dq, dk, dv, dsl, DECODE_L, cos, sin, out=dout, lse=dlse, workspace=dws)

    def _time(fn, n):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    def _time_graph(fns, reps):
        """Device time per call of the calls in fns, captured once into a CUDA graph and replayed
        reps times back to back (no host launch gaps between decode tokens)."""
        for f in fns:  # once-per-process setup (kernel attributes) happens outside the capture
            f()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for f in fns:
                f()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / (reps * len(fns))

    plain_pre_ms = _time(plain_prefill, max(1, min(K, 3)))
    plain_dec_ms = _max_over_ranks(_time_graph([plain_decode], 200), world)
    bif_dec_ms_loop = _max_over_ranks(_time_graph([decode], 200), world)

    # ---- decode at the other cache lengths (rotating caches so each launch streams from HBM) ----
    sweep = {}
    for Ld in DECODE.cache_lens:
        if Ld == DECODE_L:
            sweep[str(Ld)] = {"us": bif_dec_ms_loop * 1e3, "plain_us": plain_dec_ms * 1e3}
            continue
        bytes_one = 2 * Ld * DECODE.n_kv_heads * DECODE.head_dim * 2
        n_rot = max(1, int(math.ceil(2 * 126e6 / bytes_one)))
        caches = [(dk[:, :Ld].contiguous(), dv[:, :Ld].contiguous()) for _ in range(n_rot)]
        sl = torch.tensor([Ld], dtype=torch.int32, device=dev)
        ws = torch.empty(jl.jl_bifocal_decode_workspace_size(1, DECODE.n_q_heads, DECODE.head_dim, Ld),
                         dtype=torch.uint8, device=dev)

        def dstep(kk, vv, plain=False):
            if plain:
                jl.jl_plain_decode(dq, kk, vv, sl, Ld, cos, sin, out=dout, lse=dlse, workspace=ws)
            else:
                jl.jl_bifocal_decode(dq, kk, vv, sl, Ld, DECODE.w0, DECODE.w_pretrained, cos, sin, out=dout,
                                     lse=dlse, workspace=ws)

        reps = max(1, 200 // n_rot)
        bif = [lambda kk=kk, vv=vv: dstep(kk, vv) for kk, vv in caches]
        pln = [lambda kk=kk, vv=vv: dstep(kk, vv, True) for kk, vv in caches]
        sweep[str(Ld)] = {"us": _time_graph(bif, reps) * 1e3, "plain_us": _time_graph(pln, reps) * 1e3,
                          "rotating_caches": n_rot}
        del caches
    for Ld, rec in sweep.items():
        rec["overhead_vs_plain"] = rec["us"] / rec["plain_us"] - 1.0
        rec["hbm_gbs"] = 2 * int(Ld) * DECODE.n_kv_heads * DECODE.head_dim * 2 / (rec["us"] * 1e-6) / 1e9
    jl.jl_sync_status()

    # ---- the 256-token generation walk across the G = 3 -> 4 boundary ----
    decode_walk = _measure_walk(jl, dev, stream, dk, dv, cos, sin)

    # ---- rows beyond the hot path, each measured on its own workload ----
    next_rows = _measure_next_rows(jl, dev, stream, q, k, v, cu, cos, sin, out, lse, pre_avg, dk, dv, dq, dsl,
                                   dout, dlse, dws, bif_dec_ms_loop, hbm, sustained, _time, _time_graph)
    jl.jl_sync_status()
    other_configs = _measure_other_configs(jl, dev, sustained, hbm, _time, _time_graph)
    jl.jl_sync_status()

    # ---- end to end through host buffers (H2D inputs, D2H outputs inside the timed region) ----
    # Every step copies its inputs in from pinned host memory and its results out. The copies
    # run on their own streams against double-buffered device tensors, so step s+1's inputs
    # arrive and step s-1's results leave while step s computes; the timed region runs from
    # the first input copy to the last result copy.
    e2e_steps = max(2, K)
    devbuf = [dict(q=q, k=k, v=v, dq=dq, out=out, lse=lse, dout=dout),
              dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v), dq=torch.empty_like(dq),
                   out=torch.empty_like(out), lse=torch.empty_like(lse), dout=torch.empty_like(dout))]
    hostout = [dict(out=torch.empty_like(q_h).pin_memory(),
                    lse=torch.empty((PREFILL.n_q_heads, L), dtype=torch.float32).pin_memory(),
                    dout=torch.empty_like(dq_h).pin_memory()) for _ in range(2)]
    h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_out = [torch.cuda.Event() for _ in range(e2e_steps)]

    def copy_in(s_):
        d = devbuf[s_ % 2]
        with torch.cuda.stream(h2d_stream):
            if s_ >= 2:
                h2d_stream.wait_event(ev_done[s_ - 2])  # step s-2 has finished reading this buffer
            for name, src in (("q", q_h), ("k", k_h), ("v", v_h), ("dq", dq_h)):
                d[name].copy_(src, non_blocking=True)
            ev_in[s_].record(h2d_stream)

    _barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    h2d_stream.wait_event(a)
    copy_in(0)
    for s_ in range(e2e_steps):
        d = devbuf[s_ % 2]
        stream.wait_event(ev_in[s_])
        if s_ >= 2:
            stream.wait_event(ev_out[s_ - 2])  # step s-2's results have left this buffer
        jl.jl_bifocal_prefill(d["q"], d["k"], d["v"], cu, L, PREFILL.w0, PREFILL.w_pretrained, cos, sin,
                              out=d["out"], lse=d["lse"], workspace=kws)
        jl.jl_bifocal_decode(d["dq"], dk, dv, dsl, DECODE_L, DECODE.w0, DECODE.w_pretrained, cos, sin,
                             out=d["dout"], lse=dlse, workspace=dws)
        ev_done[s_].record(stream)
        if s_ + 1 < e2e_steps:
            copy_in(s_ + 1)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(ev_done[s_])
            ho = hostout[s_ % 2]
            for name in ("out", "lse", "dout"):
                ho[name].copy_(d[name], non_blocking=True)
            ev_out[s_].record(d2h_stream)
    stream.wait_event(ev_out[e2e_steps - 1])
    b.record(stream)
    _barrier(world)
    out_h, lse_h, dout_h = hostout[0]["out"], hostout[0]["lse"], hostout[0]["dout"]
    e2e_ms = _max_over_ranks(a.elapsed_time(b) / e2e_steps, world)
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h, dq_h))
    d2h = sum(t.numel() * t.element_size() for t in (out_h, lse_h, dout_h))

    res = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, outlier-scaled key channels)",
        "config": _config(),
        "prefill": {
            "ms": round(pre_avg, 4),
            "useful_tflops": round(prefill_tflops, 2),
            "frac_of_bf16_peak_measured_sustained": round(prefill_tflops / sustained, 4),
            "frac_of_bf16_peak_measured_burst": round(prefill_tflops / burst, 4),
            "frac_of_bf16_nominal_2250": round(prefill_tflops / 2250.0, 4),
            "plain_ms": round(plain_pre_ms, 4),
            "plain_useful_tflops": round(flops / (plain_pre_ms * 1e-3) / 1e12, 2),
            "bifocal_over_plain_time": round(pre_avg / plain_pre_ms, 4),
            # clock-normalised: useful flops per SM cycle at the median SM clock of the timed region,
            # against the tensor pipe's 8192 dense bf16 flops per SM cycle
            "sm_mhz_median": clocks["sm_mhz"] if clocks else None,
            "useful_flop_per_sm_cycle": (round(flops / (pre_avg * 1e-3 * clocks["sm_mhz"] * 1e6 * 148), 1)
                                         if clocks else None),
            "tensor_frac_at_measured_clock": (round(flops / (pre_avg * 1e-3 * clocks["sm_mhz"] * 1e6 * 148) / 8192, 4)
                                              if clocks else None),
        },
        "decode": {
            # back-to-back tokens: one decode call captured in a CUDA graph, replayed 200 times
            "us_per_token": round(bif_dec_ms_loop * 1e3, 2),
            "cache_len": DECODE_L,
            "hbm_gbs": round(kv_bytes / (bif_dec_ms_loop * 1e-3) / 1e9, 1),
            "frac_of_hbm_measured": round(kv_bytes / (bif_dec_ms_loop * 1e-3) / 1e9 / hbm, 4),
            "frac_of_hbm_nominal_8000": round(kv_bytes / (bif_dec_ms_loop * 1e-3) / 1e9 / 8000.0, 4),
            # the one token of each timed step, right after that step's 147 ms prefill
            "us_in_step": round(dec_avg * 1e3, 2),
            "hbm_gbs_in_step": round(dec_gbs, 1),
            "plain_us_per_token": round(plain_dec_ms * 1e3, 2),
            "overhead_vs_plain": round(bif_dec_ms_loop / plain_dec_ms - 1.0, 4),
            "sweep": {k_: {kk: (round(vv, 3) if isinstance(vv, float) else vv) for kk, vv in r.items()}
                      for k_, r in sweep.items()},
            "walk": decode_walk,
        },
        "next_rows": next_rows,
        "other_configs": other_configs,
        "roofline": {
            "kernel": "jl_prefill_kernel<128,2>",
            "bound": "tensor",
            "achieved": round(prefill_tflops, 2),
            "peak": sustained,
            "peak_kind": f"{peak_kind} bf16 sustained (kernel timed inside a long loop)",
            "unit": "TFLOP/s",
            "frac": round(prefill_tflops / sustained, 4),
            "traffic": _traffic("prefill", PREFILL_SRC),
            "tensor_pipe_active": _profiled("prefill", PREFILL_SRC, "tensor_pipe_active_pct"),
            # the timed call is the whole jl_bifocal_prefill: the keys' rotation kernel, then this kernel
            "duration_includes": "jl_key_rotate_kernel",
            "algorithmic_bytes_per_launch": int(sum(t.numel() * t.element_size() for t in (q, k, v, out, lse))),
        },
        "e2e": {
            "value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 3),
            "unit": UNIT,
            "ms_per_step": round(e2e_ms, 3),
            "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h),
        },
        # per step: the key rotation and the prefill kernel, the decode split kernel and its merge
        "gpu_launches": 4 * K,
        "clocks": clocks,
    }
    if rank == 0 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
    return res


# ----------------------------------------------------- CPU oracle (baseline) ----

def _host_cores():
    """Cores this process may run on (affinity-aware nproc)."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def _cpu_prefill_rows(O, seconds, inputs=None):
    """The fp64 oracle on rows drawn uniformly from the second half of the 128K sequence, all
    query heads of KV head 0, for about `seconds` of oracle time."""
    if inputs is None:
        q_h, k_h, v_h, _ = I.prefill_inputs(PREFILL)
    else:
        q_h, k_h, v_h = inputs
    L = PREFILL.seqlens[0]
    qb, kb, vb = I.bf16_bits(q_h), I.bf16_bits(k_h), I.bf16_bits(v_h)
    group = PREFILL.n_q_heads // PREFILL.n_kv_heads
    rng = np.random.default_rng(7)
    n = 8
    done_rows, done_flops, spent = 0, 0.0, 0.0
    while spent < seconds:
        pos = rng.integers(L // 2, L, n)
        head = rng.integers(0, group, n)  # KV head 0's query heads
        t0 = time.perf_counter()
        O.bifocal_rows(qb, kb, vb, L, pos, head, w0=PREFILL.w0, w_pretrained=PREFILL.w_pretrained,
                       rope_base=PREFILL.rope_base)
        spent += time.perf_counter() - t0
        done_rows += n
        done_flops += float(np.sum(4.0 * PREFILL.head_dim * (pos + 1)))
        n = min(n * 2, 256)
    return done_rows, done_flops, spent


def _cpu_decode(O):
    """The oracle's decode step (fp64) on the decode workload: one step at each cache length, and
    the four steps of the 256-token walk on either side of the G = 3 -> 4 boundary (L = 98303 ..
    98306).  The whole walk is extrapolated from those four and labelled an estimate."""
    cfg = DECODE
    first, steps = cfg.walk_first_pos, cfg.walk_steps
    max_len = max(max(cfg.cache_lens), first + steps)
    k_raw, v = I.decode_raw_inputs(cfg, max_len)  # random rows stand for base-rotated keys
    kb, vb = I.bf16_bits(k_raw[0]), I.bf16_bits(v[0])
    qb = I.bf16_bits(I.decode_queries(cfg, 1)[0, 0])

    def one(L):
        t0 = time.perf_counter()
        O.decode_step(qb, kb[:L], vb[:L], L, w0=cfg.w0, w_pretrained=cfg.w_pretrained, rope_base=cfg.rope_base)
        return time.perf_counter() - t0

    per_len = {str(L): round(one(L) * 1e6, 1) for L in cfg.cache_lens}
    walk_L = [first + 127, first + 128, first + 129, first + 130]
    walk_s = [one(L) for L in walk_L]
    return {
        "unit": "us/token",
        "us_per_token_at_cache_len": per_len,
        "walk_sample": {"L": walk_L, "G": [O.group_size(L, cfg.w_pretrained) for L in walk_L],
                        "us_per_token": [round(t * 1e6, 1) for t in walk_s]},
        "walk_256_tokens_estimate_s": round(statistics.mean(walk_s) * steps, 2),
    }


def _cpu_tiny(O):
    """Config 1 (L = 256, one head, head_dim 64, G = 4, w0 = 32) in full: every row."""
    cfg = I.TINY
    q, k, v, _ = I.prefill_inputs(cfg)
    L = cfg.seqlens[0]
    qb, kb, vb = I.bf16_bits(q), I.bf16_bits(k), I.bf16_bits(v)
    pos, head = np.arange(L), np.zeros(L, dtype=np.int64)
    reps, t0 = 0, time.perf_counter()
    while reps < 3 or time.perf_counter() - t0 < 0.5:
        O.bifocal_rows(qb, kb, vb, L, pos, head, w0=cfg.w0, w_pretrained=cfg.w_pretrained, rope_base=cfg.rope_base)
        reps += 1
    dt = (time.perf_counter() - t0) / reps
    return {"ms_per_layer": round(dt * 1e3, 3), "useful_tflops": cfg.useful_flops() / dt / 1e12,
            "sample": f"the whole tiny layer ({L} rows), mean of {reps} runs"}


def cpu_baseline(seconds=15.0, inputs=None, with_decode=True):
    """The fp64 oracle as it stands, timed on the host cores: a bounded sample of the 128K prefill
    (the headline metric's unit), plus the decode step and the tiny layer."""
    from oracle import oracle as O
    done_rows, done_flops, spent = _cpu_prefill_rows(O, seconds, inputs)
    res = {
        "value": done_flops / spent / 1e12,
        "unit": UNIT,
        "cores": _host_cores(),
        "omp_threads": O.num_threads(),
        "kind": "oracle",
        "sample": f"{done_rows} query rows of the L=131072 prefill (positions in [65536, 131072), KV head 0), "
                  f"{spent:.1f} s; useful flops of those rows / time",
        "full_layer_estimate_s": PREFILL.useful_flops() / (done_flops / spent),
    }
    if with_decode:
        res["decode"] = _cpu_decode(O)
        res["tiny"] = _cpu_tiny(O)
    return res


def run_reference(args, world, rank):
    if rank != 0:
        return None
    q_h, k_h, v_h, _ = I.prefill_inputs(PREFILL)
    inputs = (q_h, k_h, v_h)
    for _ in range(args.warmup):
        cpu_baseline(seconds=0.5, inputs=inputs, with_decode=False)
    per_step = max(2.0, min(20.0, 150.0 / max(1, args.steps)))
    vals, step_s = [], []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        vals.append(cpu_baseline(seconds=per_step, inputs=inputs, with_decode=False))
        step_s.append(time.perf_counter() - t0)
    v = statistics.mean(r["value"] for r in vals)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": v,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": statistics.mean(step_s) * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16, outlier-scaled key channels)",
        "config": _config(),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": vals[0]["cores"], "omp_threads": vals[0]["omp_threads"],
                         "kind": "oracle", "sample": vals[0]["sample"] + f"; each step a sample of {per_step:.0f} s"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res))
        return
    world, rank, local = _dist_setup(args.gpus)
    try:
        res = run_ours(args, world, rank, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
