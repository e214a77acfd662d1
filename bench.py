#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

Headline: causal GQA prefill, batch 2, 32 query / 8 KV heads, head dim 128, 8192 tokens,
bf16 in / fp32 accumulate, in TFLOP/s (algorithmic FLOPs: the causal half only), printed last.
Before it, one compact JSON line per secondary workload: the split-KV decodes (ragged bf16
64K-128K cache; FP8 E4M3, INT8 and INT4 caches of 32768 tokens; paged and multi-token variants)
in KV GB/s, the packed varlen prefill, and the streamed causal prefill over 2^20 host-resident
tokens, each against the measured roofline and the oracle timed on the host cores; the headline
line repeats them as a summary.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-stream]

Under torchrun (N > 1) every rank runs the same workload on its own GPU (independent
replicas: weak scaling, no collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from exact_long_context_tmem_b200 import inputs as I  # noqa: E402

METRIC = "prefill attn TFLOP/s & decode KV GB/s at 1 B200, as fraction of roofline"
HEADLINE = "prefill_b2_h32g8_d128_s8192"
DECODE_WORKLOADS = (("decode_bf16", "decode_b4_h32g8_d128_ragged64k_128k"),
                    ("decode_fp8", "decode_fp8_b16_h32g8_d128_t32768"),
                    ("decode_int8", "decode_int8_b16_h32g8_d128_t32768"),
                    ("decode_int4", "decode_int4_b16_h32g8_d128_t32768"))
STREAM = "stream_b1_h32g8_d128_s1m_chunk64k"
L2_BYTES = 126 * 10**6

# DRAM bytes (read + write) per launch from one ncu capture of each kernel on its bench workload.
# A value is reported only while the kernel's sources still hash to the ones the counters were
# taken from; otherwise the traffic is unknown (null).
NCU_TRAFFIC = {
    "prefill": {"sources": ('ptx.cuh', 'status.cuh', 'prefill.cuh'), "sha1": "1f04feae59dccef5",
        "bytes": 319281920 + 103592448},
    "decode_b4_h32g8_d128_ragged64k_128k": {"sources": ('ptx.cuh', 'status.cuh', 'decode.cuh'), "sha1": "6b6cf2c3fc7aa803",
        "bytes": 1549382144 + 4482816},
    "decode_fp8_b16_h32g8_d128_t32768": {"sources": ('ptx.cuh', 'status.cuh', 'decode.cuh', 'decode_fp8.cuh'), "sha1": "b3ac03fa062a074c",
        "bytes": 1147788288 + 4960000},
    "decode_int8_b16_h32g8_d128_t32768": {"sources": ('ptx.cuh', 'status.cuh', 'decode.cuh', 'decode_int.cuh'), "sha1": "ea38a1d9e25a36f6",
        "bytes": 1147653376 + 5013760},
    "decode_int4_b16_h32g8_d128_t32768": {"sources": ('ptx.cuh', 'status.cuh', 'decode.cuh', 'decode_int.cuh'), "sha1": "ea38a1d9e25a36f6",
        "bytes": 601052928 + 4892416},
}


def ncu_traffic(key):
    import hashlib
    e = NCU_TRAFFIC.get(key)
    if not e:
        return None
    m = hashlib.sha1()
    for f in e["sources"]:
        with open(os.path.join(ROOT, "exact_long_context_tmem_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    return e["bytes"] if m.hexdigest()[:16] == e["sha1"] else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ distributed plumbing

def dist_init(n_gpus, backend=None):
    """One process per GPU under torchrun: NCCL with the device bound, or gloo (CPU plumbing
    tests).  Returns (world, rank, local rank)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = backend or "nccl"
        timeout = datetime.timedelta(seconds=300)
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timeout)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The largest of every rank's x (a device time): one all-reduce, on the GPU under NCCL."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.lines = []
        self.dev = device_index

    def start(self):
        try:
            ident = None
            try:
                ident = str(torch.cuda.get_device_properties(self.dev).uuid)
                if not ident.startswith("GPU-"):
                    ident = "GPU-" + ident
            except Exception:  # noqa: BLE001
                ident = str(self.dev)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", ident], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:  # noqa: BLE001
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:  # noqa: BLE001
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ workloads

def prefill_flops(w):
    # causal: row i sees i+1 keys; QK^T and PV are 2*D FLOPs per (row, key) each
    pairs = w.S * (w.S + 1) // 2 if w.causal else w.S * w.T
    return 4.0 * w.D * w.B * w.Hq * pairs


def decode_bytes(w, lens):
    tok = int(lens.sum())
    row = w.D // 2 if w.kv_bits == 4 else (w.D if (w.kv_fp8 or w.kv_bits == 8) else 2 * w.D)  # bytes per K or V row
    per_tok = w.Hkv * row * 2
    if w.kv_fp8 or w.kv_bits:
        per_tok += w.Hkv * 4 * 2  # k and v scales
    qo = w.B * w.Hq * w.D * 2 * 2 + w.B * w.Hq * 4
    return tok * per_tok + qo


def bench_prefill(w, steps, warmup, world, dev, pk):
    from exact_long_context_tmem_b200 import attn as A

    q, k, v = I.prefill_inputs(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o = torch.empty((w.B, w.S, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.S, w.Hq), dtype=torch.float32, device=dev)
    for _ in range(warmup):
        A.attn_prefill(qd, kd, vd, causal=True, o=o, lse=lse)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # Clocks: the timed region is shorter than nvidia-smi's 200 ms period, so the same launches
    # keep the GPU loaded for ~0.4 s right before it and the samples cover both.
    sampler = ClockSampler(dev.index or 0)
    sampler.start()
    soak = max(1, int(0.4e15 / prefill_flops(w)))  # ~0.4 s at ~1 PFLOP/s
    for _ in range(min(soak, 2000)):
        A.attn_prefill(qd, kd, vd, causal=True, o=o, lse=lse)
    barrier(world)
    torch.cuda.synchronize()
    t0.record()
    for i in range(steps):
        ev[i][0].record()
        A.attn_prefill(qd, kd, vd, causal=True, o=o, lse=lse)
        ev[i][1].record()
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    total_ms = max_over_ranks(t0.elapsed_time(t1), world)
    launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    flops = prefill_flops(w)

    # End to end through the public call with host buffers: every step uploads its Q/K/V from
    # pinned host memory, runs attn_prefill and downloads O and LSE.  Steps are double-buffered on
    # three streams (upload, compute, download), so step i+1's upload overlaps step i's compute
    # and step i-1's download; the region is timed with events from the first upload to the last
    # download.
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    bufs = []
    for _ in range(2):
        bufs.append({"q": torch.empty_like(qd), "k": torch.empty_like(kd), "v": torch.empty_like(vd),
                     "o": torch.empty_like(o), "lse": torch.empty_like(lse),
                     "oh": torch.empty(o.shape, dtype=o.dtype, pin_memory=True),
                     "lh": torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True),
                     "in_ready": torch.cuda.Event(), "comp_done": torch.cuda.Event(), "out_done": torch.cuda.Event()})
    up, comp, down = torch.cuda.Stream(), torch.cuda.current_stream(), torch.cuda.Stream()

    def e2e_steps(count, t_start=None, t_end=None):
        for i in range(count):
            bb = bufs[i & 1]
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(bb["comp_done"])
                if i == 0 and t_start is not None:
                    t_start.record(up)
                bb["q"].copy_(qh, non_blocking=True)
                bb["k"].copy_(kh, non_blocking=True)
                bb["v"].copy_(vh, non_blocking=True)
                bb["in_ready"].record(up)
            comp.wait_event(bb["in_ready"])
            if i >= 2:
                comp.wait_event(bb["out_done"])
            A.attn_prefill(bb["q"], bb["k"], bb["v"], causal=True, o=bb["o"], lse=bb["lse"], stream=comp)
            bb["comp_done"].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(bb["comp_done"])
                bb["oh"].copy_(bb["o"], non_blocking=True)
                bb["lh"].copy_(bb["lse"], non_blocking=True)
                bb["out_done"].record(down)
                if i == count - 1 and t_end is not None:
                    t_end.record(down)

    e2e_steps(max(2, warmup))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_n = max(4, steps // 2)
    barrier(world)
    torch.cuda.synchronize()
    e2e_steps(e2e_n, e0, e1)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_n
    h2d = (q.numel() + k.numel() + v.numel()) * 2
    d2h = o.numel() * 2 + lse.numel() * 4
    achieved = flops / (launch_ms * 1e-3) / 1e12
    return {
        "total_ms": total_ms, "ms_per_step": total_ms / steps, "launch_ms": launch_ms, "flops": flops,
        "tflops": flops * world / (total_ms / steps * 1e-3) / 1e12,
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_tflops"], 4),
                     "traffic": ncu_traffic("prefill"),
                     "peak_kind": f"bf16 dense, burst, {pk['source']}",
                     "frac_of_sustained": (round(achieved / pk["bf16_tflops_sustained"], 4)
                                           if pk.get("bf16_tflops_sustained") else None)},
        "e2e": {"value": round(flops * world / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clocks, "launches": steps,
    }


PAGE_SIZE = 512


def bench_decode(name, steps, warmup, world, dev, pk, paged=False, n_q=1):
    """Split-KV decode of a decode workload; paged=True lays the same cache out as a pool of
    PAGE_SIZE-token pages in seeded random order with a page table (attn_decode_paged); n_q > 1
    decodes the last n_q cache tokens of every sequence in one pass (attn_decode_multi)."""
    from exact_long_context_tmem_b200 import attn as A

    w = I.WORKLOADS[name]
    d = I.decode_inputs(w)
    d_contig = d
    lens = d["kv_lens"]
    Tmax = d["Tmax"]
    if paged:
        d = I.paged_inputs(d, PAGE_SIZE, seed=w.seed + 7)
        Tmax = d["page_table"].shape[1] * PAGE_SIZE
        table = d["page_table"].to(dev)
    qd, ld = d["q"].to(dev), lens.to(dev)
    if w.kv_fp8 or w.kv_bits:
        kd, vd = d["k_codes"].to(dev), d["v_codes"].to(dev)
        ks, vs = d["k_scale"].to(dev), d["v_scale"].to(dev)
    else:
        kd, vd = d["k"].to(dev), d["v"].to(dev)
        ks = vs = None
    if n_q > 1:
        qd = I.randn_bf16((w.B, n_q, w.Hq, w.D), I.generator(w.seed + 11)).to(dev)
    o = torch.empty((w.B, n_q, w.Hq, w.D) if n_q > 1 else (w.B, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, n_q, w.Hq) if n_q > 1 else (w.B, w.Hq), dtype=torch.float32, device=dev)
    nbytes = A.attn_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, Tmax) * n_q
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    splits = A.attn_decode_num_splits(w.B, w.Hq, w.Hkv, w.D, Tmax)

    def step():
        if n_q > 1:
            A.attn_decode_multi(qd, kd, vd, ld, k_scale=ks, v_scale=vs, o=o, lse=lse, ws=ws)
        elif paged:
            A.attn_decode_paged(qd, kd, vd, table, ld, k_scale=ks, v_scale=vs, o=o, lse=lse, ws=ws)
        else:
            A.attn_decode_splitkv(qd, kd, vd, ld, k_scale=ks, v_scale=vs, o=o, lse=lse, ws=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    call_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev), world)
    nb = decode_bytes(w, lens)
    gbs = nb / (call_ms * 1e-3) / 1e9
    suffix = (f"_paged{PAGE_SIZE}" if paged else "") + (f"_multi{n_q}" if n_q > 1 else "")
    return {"workload": name + suffix, "value": round(gbs * world, 1), "unit": "GB/s",
            "ms_per_step": round(call_ms, 4),
            "splits": splits, "kv_tokens": int(lens.sum()), "bytes_per_step": nb,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / pk["hbm_gbs"], 4),
                         "traffic": None if (paged or n_q > 1) else ncu_traffic(name),
                         "timed": "split kernel + merge kernel (one API call)"},
            "launches": steps * (2 if splits > 1 else 1),
            "cpu_baseline": decode_oracle_sample(w, d_contig, n_q) if world == 1 else None}


VARLEN = "prefill_varlen_b16_h32g8_d128_ragged512_2048"


def bench_prefill_varlen(steps, warmup, world, dev, pk):
    """Packed variable-length causal prefill (attn_prefill_varlen), inputs resident on the device."""
    from exact_long_context_tmem_b200 import attn as A

    w = I.WORKLOADS[VARLEN]
    d = I.varlen_inputs(w)
    qd, kd, vd, cu = d["q"].to(dev), d["k"].to(dev), d["v"].to(dev), d["cu"].to(dev)
    max_s = int(d["lens"].max())
    o = torch.empty_like(qd)
    lse = torch.empty((qd.shape[0], w.Hq), dtype=torch.float32, device=dev)

    def step():
        A.attn_prefill_varlen(qd, kd, vd, cu, cu, max_s, causal=True, o=o, lse=lse)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev), world)
    flops = sum(4.0 * w.D * w.Hq * int(n) * (int(n) + 1) / 2 for n in d["lens"])
    tf = flops / (ms * 1e-3) / 1e12
    return {"workload": VARLEN, "value": round(tf * world, 1), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
            "tokens": int(d["lens"].sum()), "flops_per_step": flops,
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(tf / pk["bf16_tflops"], 4), "traffic": None}, "launches": steps,
            "cpu_baseline": varlen_oracle_sample(w, d) if world == 1 else None}


def varlen_oracle_sample(w, d):
    """Time the float64 oracle on the first packed sequence of the varlen workload (all heads);
    returns a cpu_baseline dict in TFLOP/s (causal pairs only, as the GPU line counts them)."""
    from oracle import attention as O

    n = int(d["lens"][0])
    cu = torch.tensor([0, n], dtype=torch.int32)
    t = time.perf_counter()
    O.prefill_varlen(d["q"][:n], d["k"][:n], d["v"][:n], cu, cu, scale=w.scale, causal=True)
    dt = time.perf_counter() - t
    flops = 4.0 * w.D * w.Hq * n * (n + 1) / 2
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": host_threads(), "kind": "oracle",
            "sample": f"sequence 0 of {w.B} ({n} tokens, {w.Hq} heads, {dt:.2f} s)"}


STREAM_SMALL = "stream_b1_h32g8_d128_s128k_chunk16k"


def bench_stream(dev, pk, name=STREAM):
    """The streamed causal prefill over 2^20 host-resident tokens (attn_chunked_stream: pinned host
    Q/K/V/O/LSE, 64K-token key chunks, 16e9-byte device budget), run once.  Reports TFLOP/s over the
    device span from the first upload to the end of the last copy back, the prefill tasks' own rate
    against the tensor roofline, copy-engine GB/s of each direction (bytes / summed copy time), and
    the overlap fraction (compute time / device span: 1 = every copy hidden)."""
    from exact_long_context_tmem_b200 import attn as A

    w = I.WORKLOADS[name]
    g = I.generator(w.seed)
    shape_q = (w.B, w.S, w.Hq, w.D)
    shape_kv = (w.B, w.S, w.Hkv, w.D)
    t_gen = time.perf_counter()
    q = I.randn_bf16(shape_q, g, out=torch.empty(shape_q, dtype=torch.bfloat16, pin_memory=True))
    k = I.randn_bf16(shape_kv, g, out=torch.empty(shape_kv, dtype=torch.bfloat16, pin_memory=True))
    v = I.randn_bf16(shape_kv, g, out=torch.empty(shape_kv, dtype=torch.bfloat16, pin_memory=True))
    o = torch.empty(shape_q, dtype=torch.bfloat16, pin_memory=True)
    lse = torch.empty((w.B, w.S, w.Hq), dtype=torch.float32, pin_memory=True)
    t_gen = time.perf_counter() - t_gen
    torch.cuda.nvtx.range_push("attn_chunked_stream")  # the range a profiler can measure as a whole
    _, _, st = A.attn_chunked_stream(q, k, v, causal=True, chunk_tokens=w.chunk_tokens, budget_bytes=w.budget_bytes,
                                     o_h=o, lse_h=lse)
    torch.cuda.nvtx.range_pop()
    flops = prefill_flops(w)
    tf = flops / (st.ms_device * 1e-3) / 1e12
    busy_tf = flops / (st.ms_compute_busy * 1e-3) / 1e12
    line = {"workload": name, "value": round(tf, 1), "unit": "TFLOP/s", "ms_per_step": round(st.ms_device, 1),
            "flops_per_step": flops, "q_block": st.plan.q_block, "kv_chunk": st.plan.kv_chunk,
            "tasks": st.plan.n_tasks, "device_bytes": st.plan.device_bytes, "device_budget": w.budget_bytes,
            "roofline": {"bound": "tensor", "achieved": round(busy_tf, 1), "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(busy_tf / pk["bf16_tflops"], 4), "traffic": None,
                         "timed": "prefill tasks + block finishes, summed CUDA-event time on the compute stream"},
            "copies": {"h2d_GBps": round(st.h2d_bytes / (st.ms_h2d * 1e-3) / 1e9, 2),
                       "d2h_GBps": round(st.d2h_bytes / (st.ms_d2h * 1e-3) / 1e9, 2),
                       "h2d_bytes": st.h2d_bytes, "d2h_bytes": st.d2h_bytes,
                       "ms_h2d": round(st.ms_h2d, 1), "ms_d2h": round(st.ms_d2h, 1),
                       "timed": "summed CUDA-event time of each copy batch on its stream"},
            "overlap": round(st.ms_compute_busy / st.ms_device, 4),
            "ms_compute_busy": round(st.ms_compute_busy, 1), "ms_call_wall": round(st.ms_total, 1),
            "e2e": {"value": round(tf, 1), "unit": "TFLOP/s", "h2d_bytes_per_step": st.h2d_bytes,
                    "d2h_bytes_per_step": st.d2h_bytes},
            "launches": 2 * st.plan.n_tasks, "input_gen_s": round(t_gen, 1),
            "cpu_baseline": stream_oracle_sample(w, q, k, v)}
    return line


def stream_oracle_sample(w, q, k, v, n_rows=4):
    """Time the float64 oracle on a bounded sample of the streamed workload: n_rows query rows
    from the end of the sequence (each sees about 2^20 keys) for the 4 query heads of KV head 0
    (the widening of that head's K and V to float64 inside the timed region).  TFLOP/s counts the
    causal pairs as the GPU line does."""
    from oracle import attention as O

    G = w.Hq // w.Hkv
    step = max(1, w.chunk_tokens or w.S // (n_rows + 1))
    rows = [r for r in (w.S - 1 - i * step for i in range(n_rows)) if r >= 0]
    t = time.perf_counter()
    O.attention(q[:, :, :G], k[:, :, :1], v[:, :, :1], scale=w.scale, causal=True, rows=rows)
    dt = time.perf_counter() - t
    flops = sum(4.0 * w.D * (r + 1) for r in rows) * G
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": host_threads(), "kind": "oracle",
            "sample": f"{n_rows} query rows near the end x {G} heads of KV head 0 ({dt:.1f} s)"}


# ------------------------------------------------------------------ oracle (CPU baseline)

def host_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:  # noqa: BLE001
        pass
    return len(os.sched_getaffinity(0))


def oracle_sample(w, n_rows, seed=4242):
    """Time the float64 oracle on n_rows sampled query rows (all batches and heads) of the
    prefill workload; returns (TFLOP/s of the sample, seconds, rows)."""
    from oracle import attention as O

    q, k, v = I.prefill_inputs(w)
    rows = I.sample_rows(w.S, n_rows, seed=seed)
    t = time.perf_counter()
    O.attention(q, k, v, scale=w.scale, causal=True, rows=rows)
    dt = time.perf_counter() - t
    flops = sum(4.0 * w.D * (r + 1) for r in rows) * w.B * w.Hq
    return flops / dt / 1e12, dt, rows


def oracle_rates(w, n_rows, seconds, tflops):
    """The oracle's sampled rate as query rows per second (each row over every batch and head),
    and the time the whole prefill workload would take at the sample's FLOP rate (an
    extrapolation, labelled as such: the oracle never runs the full configuration)."""
    return {"rows_per_s": round(n_rows / seconds, 3),
            "extrapolated_full_config_s": round(prefill_flops(w) / (tflops * 1e12), 1)}


def decode_oracle_sample(w, d, n_q=1):
    """Time the float64 oracle on a bounded sample of a decode workload: sequence 0 of the cache
    (every head; codes decoded to values first, as the oracle's input), single-token or n_q-token
    decode.  Returns a cpu_baseline dict in the bench's unit (cache GB/s of the sample)."""
    from oracle import attention as O

    lens = d["kv_lens"][:1]
    L = int(lens[0])
    if w.kv_bits or w.kv_fp8:
        if w.kv_bits:
            from oracle import intq
            dec = lambda c: intq.int_values(c[:1, :L], w.kv_bits)  # noqa: E731
        else:
            from oracle import fp8
            dec = lambda c: fp8.e4m3_decode(c[:1, :L])  # noqa: E731
        t = time.perf_counter()
        k, v = dec(d["k_codes"]), dec(d["v_codes"])
        ks, vs = d["k_scale"][:1, :L], d["v_scale"][:1, :L]
    else:
        t = time.perf_counter()
        k, v, ks, vs = d["k"][:1, :L], d["v"][:1, :L], None, None
    if n_q > 1:
        q = I.randn_bf16((1, n_q, w.Hq, w.D), I.generator(w.seed + 11))
        O.decode_multi(q, k, v, lens, scale=w.scale, k_scale=ks, v_scale=vs)
    else:
        O.decode(d["q"][:1], k, v, lens, scale=w.scale, k_scale=ks, v_scale=vs)
    dt = time.perf_counter() - t
    nb = L * (decode_bytes(w, torch.tensor([1])) - decode_bytes(w, torch.tensor([0])))
    return {"value": round(nb / dt / 1e9, 3), "unit": "GB/s", "cores": host_threads(), "kind": "oracle",
            "sample": f"sequence 0 of {w.B} ({L} tokens, {w.Hq} heads{f', {n_q} query tokens' if n_q > 1 else ''}), "
                      f"contiguous cache, codes decoded inside the timed region ({dt:.2f} s)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-stream", action="store_true", help="leave out the 1M-token streamed prefill")
    ap.add_argument("--cpu-rows", type=int, default=128)
    ap.add_argument("--workloads",
                    default="prefill,prefill_varlen,decode_bf16,decode_fp8,decode_bf16_paged,decode_fp8_paged,"
                            "decode_bf16_multi,decode_fp8_multi,decode_int8,decode_int4,stream",
                    help="comma list of prefill, prefill_varlen, stream, stream_small, "
                         "decode_{bf16,fp8,int8,int4}[_paged|_multi] (profiling runs select one)")
    args = ap.parse_args()
    w = I.WORKLOADS[HEADLINE]
    config = {"workload": HEADLINE, "batch": w.B, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.D,
              "seq_len": w.S, "causal": True, "io": "bf16 Q/K/V/O, fp32 LSE",
              "l2": "per step 192 MiB of inputs + 130 MiB of outputs > 126 MB L2; no flush",
              "parallelism": f"replicas x{args.gpus}"}
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        cores = host_threads()
        vals = []
        n_rows = max(4, args.cpu_rows // 8)
        for i in range(args.warmup + args.steps):
            tf, dt, rows = oracle_sample(w, n_rows, seed=9000 + i)
            if i >= args.warmup:
                vals.append((tf, dt))
        value = statistics.mean(v for v, _ in vals)
        line = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(1e3 * statistics.mean(d for _, d in vals), 1),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic N(0,1), seeded", "config": config, "impl": "reference",
                "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                 "sample": f"{n_rows} sampled query rows x {w.B} batch x {w.Hq} heads per step",
                                 **oracle_rates(w, n_rows, statistics.mean(d for _, d in vals), value)},
                "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    world, rank, local = dist_init(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from exact_long_context_tmem_b200 import attn as A
    A.lib()
    pk = peaks()
    sel = set(args.workloads.split(","))

    def emit(line):
        """A secondary workload: its own compact JSON line, printed before the headline line."""
        if rank == 0:
            print(json.dumps({"metric": METRIC, "kind": "secondary", "n_gpus": world, **line}), flush=True)

    pre = bench_prefill(w, args.steps, args.warmup, world, dev, pk) if "prefill" in sel else None
    summary = {}

    def note(line):
        summary[line["workload"]] = [line["value"], line["unit"], line["roofline"]["frac"]]
        emit(line)

    if not args.no_decode:
        for key, name in DECODE_WORKLOADS:
            if key in sel:
                note(bench_decode(name, args.steps, args.warmup, world, dev, pk))
            if key + "_paged" in sel:
                note(bench_decode(name, args.steps, args.warmup, world, dev, pk, paged=True))
            if key + "_multi" in sel:
                note(bench_decode(name, args.steps, args.warmup, world, dev, pk, n_q=4))
    if "prefill_varlen" in sel:
        note(bench_prefill_varlen(args.steps, args.warmup, world, dev, pk))
    st, site = A.attn_device_status(reset=True)
    if st != 0:
        raise SystemExit(f"device status {st} at wait site {site}")
    # The streamed 2^20-token prefill holds ~20 GiB of pinned host memory and takes ~10 s: one run,
    # on a single process (with several replicas it is left out).
    if "stream" in sel and not args.no_stream:
        if world == 1:
            note(bench_stream(dev, pk))
        elif rank == 0:
            summary[STREAM] = "left out with more than one process (host memory)"
    if "stream_small" in sel and world == 1:  # a 2^17-token streamed case, for profiling the host link
        note(bench_stream(dev, pk, STREAM_SMALL))
    cpu = None
    if pre is None:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "partial": True, "summary": summary}), flush=True)
        return
    if rank == 0 and world == 1:
        tf, dt, rows = oracle_sample(w, args.cpu_rows)
        cpu = {"value": round(tf, 6), "unit": "TFLOP/s", "cores": host_threads(), "kind": "oracle",
               "sample": f"{len(rows)} sampled query rows x {w.B} batch x {w.Hq} heads ({dt:.1f} s)",
               **oracle_rates(w, len(rows), dt, tf)}
    if rank == 0:
        line = {"metric": METRIC, "value": round(pre["tflops"], 2), "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(pre["ms_per_step"], 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic N(0,1), seeded", "config": config, "roofline": pre["roofline"],
                "cpu_baseline": cpu, "e2e": pre["e2e"], "clocks": pre["clocks"], "gpu_launches": pre["launches"],
                "summary": summary}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
