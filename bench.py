#!/usr/bin/env python3
"""Benchmark of the exact-attention hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic inputs:
  * prefill forward on the 8192-token workload (B=1, H=32, N=8192, d=128,
    causal), O and LSE  -> attn fwd TFLOP/s (the line's ``value``);
  * split-KV decode on the 32K-cache workload (B=16, H=32, Nkv=32768, d=128,
    64 chunks), partials + merge -> decode KV GB/s (``decode``).
Inputs are seeded i.i.d. N(0,1) bf16 (seeded_inputs.py), resident in HBM
before timing; they exceed the 126 MB L2 (192 MB prefill + 8.6 GB decode), so
no extra flush is needed between steps. Workloads whose device-resident bytes
fit in L2 (gpt2_1k and its variants, tiny) are timed cold: a buffer of twice
the L2 size is written before every timed step, outside the kernels' CUDA
events, and the line adds ``hot``, the same kernels back to back.

``--workload prefill_8k_bwd`` (or another ``*_bwd``) times the backward pass
(dQ, dK, dV) of that prefill workload instead, one attn_bwd call per step
(attn_bwd_deterministic with ``--deterministic``).

``--workload prefill_8k_fp8`` times the forward pass on e4m3 inputs
(attn_fwd_fp8) of that workload.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workloads instead (the reference arm); it never touches the GPU path.

Multi-GPU (torchrun): every rank runs the same step on its own batch (seed +
rank); the path has no data exchange, so scaling is weak and timings are the
max over ranks.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from seeded_inputs import WORKLOADS, make_qkv, make_workload  # noqa: E402

METRIC = "attn fwd TFLOP/s & % BF16 tensor peak; decode KV GB/s & % HBM peak"
PREFILL = WORKLOADS["prefill_8k"]
DECODE = WORKLOADS["decode_32k"]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p["bf16_tflops_sustained"]), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# --------------------------------------------------------------- work model --
def prefill_pairs(w):
    if w.causal:   # bottom-right aligned visible pairs
        tot = 0
        off = w.Nkv - w.Nq
        # rows i see min(Nkv, max(0, i + off + 1)) keys
        for i in range(w.Nq):
            tot += min(w.Nkv, max(0, i + off + 1))
        return tot
    return w.Nq * w.Nkv


def prefill_flops(w):
    return 4.0 * w.d * w.B * w.H * prefill_pairs(w)


def prefill_bytes(w):
    return w.B * w.H * (2 * w.Nq * w.d * 2 + 2 * w.Nkv * w.d * 2 + 4 * w.Nq)


def decode_kv_bytes(w):
    return 2.0 * w.B * w.H * w.Nkv * w.d * 2


def decode_partial_bytes(w):
    """Compulsory traffic of the partial kernel: q, K, V read; partials written."""
    return decode_kv_bytes(w) + w.B * w.H * (w.d * 2 + w.num_splits * (w.d + 1) * 4)


def bwd_flops(w):
    """Five products per visible pair (S, dP, dV, dK, dQ), 2 d FLOP each."""
    return 10.0 * w.d * w.B * w.H * prefill_pairs(w)


def bwd_bytes(w):
    """Compulsory traffic: Q, K, V, O, dO, LSE read; dQ, dK, dV written."""
    return w.B * w.H * (3 * w.Nq * w.d * 2 + 2 * w.Nkv * w.d * 2 + 4 * w.Nq
                        + w.Nq * w.d * 2 + 2 * w.Nkv * w.d * 2)


def merge_bytes(w):
    return w.B * w.H * (w.num_splits * (w.d + 1) * 4 + w.d * 2 + 4)


# ---------------------------------------------------------------- helpers --
def dist_env():
    """(world size, rank, local rank) as torch.distributed.run sets them.

    Parsed here rather than through the library's package, so that the
    reference arm (the CPU oracle) never loads the CUDA library."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    if ws < 1 or not 0 <= rank < ws:
        raise ValueError(f"bad rank {rank} for world size {ws}")
    return ws, rank, local


def rank_slice(w, rank):
    """This rank's slice of a workload that grows with the number of GPUs: the
    same shapes, drawn from the rank's own seed (its own batch entries for a
    prefill, its own shard of the keys for a decode)."""
    import dataclasses

    from exact_io_aware_70_b200.sharding import shard_seed
    return dataclasses.replace(w, seed=shard_seed(w.seed, rank))


def l2_flush_plan(resident_bytes, l2_bytes, reduced_batch):
    """(flush?, note) for a timed loop. Inputs that fit in L2 would be served from
    it when run back to back, so such workloads are timed cold: a buffer of twice
    the L2 size is written before every timed step, outside the kernels' events."""
    if reduced_batch:
        return False, "reduced batch for profiling"
    if resident_bytes < l2_bytes:
        return True, (f"inputs fit in L2 ({resident_bytes / 1e6:.1f} MB < {l2_bytes / 1e6:.0f} "
                      f"MB): a {2 * l2_bytes / 1e6:.0f} MB buffer is written before every timed "
                      "step to flush L2; kernel times exclude that write, ms_per_step includes "
                      "it; 'hot' gives the same kernels back to back")
    return False, (f"inputs larger than L2 ({resident_bytes / 1e6:.0f} MB > "
                   f"{l2_bytes / 1e6:.0f} MB); no flush")


class L2Flusher:
    """Callable that flushes L2 before a timed step when l2_flush_plan says so."""

    def __init__(self, tensors, dev, reduced_batch):
        import torch
        props = torch.cuda.get_device_properties(dev)
        l2 = int(getattr(props, "L2_cache_size", 0)) or (126 << 20)
        resident = sum(t.numel() * t.element_size() for t in tensors)
        self.active, self.note = l2_flush_plan(resident, l2, reduced_batch)
        self.buf = (torch.empty(2 * l2, dtype=torch.uint8, device=dev) if self.active else None)
        self.n = 0

    def __call__(self):
        if self.active:
            self.n += 1
            self.buf.fill_(self.n & 0xFF)


def timed_calls(step, K, flush, stream, ws, local):
    """Time K calls of step(): CUDA events on `stream` around each call, barrier
    and synchronize on both sides, L2 flushed before each call (outside its
    events) when `flush` is active. Returns (total ms, mean ms per call, the clock
    sampler, mean ms per call back to back without the flush or None)."""
    import torch
    import torch.distributed as dist

    def pairs():
        return [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(K)]
    ev = pairs()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for a, b in ev:
            flush()
            a.record(stream)
            step()
            b.record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
    total_ms = t0.elapsed_time(t1)
    call_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    hot_ms = None
    if flush.active:
        hev = pairs()
        for a, b in hev:
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
        hot_ms = statistics.mean(a.elapsed_time(b) for a, b in hev)
    return total_ms, call_ms, clk, hot_ms


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self, max_mhz_default=1965.0):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
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
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": max_mhz_default, "reasons": ["unsampled"],
                    "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else max_mhz_default,
                "reasons": sorted(reasons), "samples": len(sm)}


# The device code each kernel's DRAM traffic depends on (its own header and the
# PTX helpers it includes). A recorded figure is used only while these files
# hash to the value stored beside it.
KERNEL_SOURCES = {
    # attn_api.cu: the host sets the unit deal and head groups, which move the traffic
    "attn_fwd_sm100": ("fwd_sm100.cuh", "ptx_sm100.cuh", "tmem_wide.cuh", "attn_api.cu"),
    "attn_decode_partials": ("decode_sm100.cuh", "ptx_sm100.cuh"),
    "attn_lse_merge": ("decode_sm100.cuh", "ptx_sm100.cuh"),
    "attn_bwd_sm100": ("bwd_sm100.cuh", "ptx_sm100.cuh", "tmem_wide.cuh"),
    "attn_fwd_sm100_e4m3": ("fwd_sm100.cuh", "ptx_sm100.cuh", "tmem_wide.cuh", "attn_api.cu"),
}


def kernel_source_hash(kernel):
    """Hash of the kernel's device sources with // comments and blank lines
    dropped, so that editing a comment does not retire a recorded figure."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_70_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            for line in fh:
                code = re.sub(r"//.*", "", line).rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def recorded_traffic():
    """Per-launch DRAM traffic from the committed ncu summary, for each kernel
    whose sources still hash to the value recorded with its figure, keyed by
    (kernel name, workload)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    try:
        with open(path) as fh:
            text = fh.read()
    except OSError:
        return {}
    import re
    out = {}
    for name, _wl, nbytes, shash in re.findall(
            r"^\|\s*(attn_\w+)\s*\|\s*([\w ]+?)\s*\|\s*(\d+)\s*\|\s*([0-9a-f]{16})\s*\|",
            text, re.M):
        if name in KERNEL_SOURCES and shash == kernel_source_hash(name):
            out[(name, _wl)] = int(nbytes)
    return out


# ------------------------------------------------------------ CPU oracle --
def oracle_prefill_sample(budget_s, max_rows=None, max_heads=4, w=None):
    """Time the oracle on evenly spaced query rows of a prefill workload's heads
    (prefill_8k unless `w` names another).

    The row count grows until one head's sample takes a quarter of the budget
    (or covers every row); whole heads are then repeated while the budget lasts.
    """
    import numpy as np

    import oracle
    from seeded_inputs import bf16_bits, make_qkv
    w = PREFILL if w is None else w
    orc = oracle.get()
    q, k, v = make_qkv(1, max_heads, w.Nq, w.Nkv, w.d, w.seed)   # CPU generator
    hb = [(bf16_bits(q[0, h]), bf16_bits(k[0, h]), bf16_bits(v[0, h])) for h in range(max_heads)]
    nrows = 64
    while True:
        rows = np.linspace(0, w.Nq - 1, nrows).astype(np.int64)
        t0 = time.perf_counter()
        orc.attn_rows_bf16(*hb[0], rows, w.causal, w.scale)
        dt = time.perf_counter() - t0
        if dt > budget_s / 4 or nrows >= w.Nq or (max_rows and nrows >= max_rows):
            break
        nrows = min(w.Nq, nrows * 4)
    heads = 1
    while heads < max_heads and dt * (heads + 1) / heads < budget_s:
        t0 = time.perf_counter()
        orc.attn_rows_bf16(*hb[heads], rows, w.causal, w.scale)
        dt += time.perf_counter() - t0
        heads += 1
    flops = heads * sum(4.0 * w.d * (min(w.Nkv, max(0, int(r) + 1 + (w.Nkv - w.Nq)))
                                     if w.causal else w.Nkv) for r in rows)
    return {"flops": flops, "seconds": dt, "rows": int(nrows), "heads": heads,
            "cores": orc.num_threads()}


def oracle_decode_sample(budget_s):
    import oracle
    from seeded_inputs import bf16_bits, make_qkv
    w = DECODE
    orc = oracle.get()
    q, k, v = make_qkv(1, 2, 1, w.Nkv, w.d, w.seed)
    heads = 0
    t0 = time.perf_counter()
    while True:
        for h in range(2):
            orc.attn_rows_bf16(bf16_bits(q[0, h]), bf16_bits(k[0, h]), bf16_bits(v[0, h]), [0],
                               False, w.scale)
            heads += 1
        dt = time.perf_counter() - t0
        if dt > budget_s or heads >= 64:
            break
    return {"bytes": heads * 2.0 * w.Nkv * w.d * 2, "seconds": dt, "heads": heads,
            "cores": orc.num_threads()}


def cpu_baseline(budget_s=8.0):
    pf = oracle_prefill_sample(budget_s)
    dc = oracle_decode_sample(budget_s / 4)
    return {
        "value": pf["flops"] / pf["seconds"] / 1e12, "unit": "TFLOP/s", "cores": pf["cores"],
        "kind": "oracle",
        "sample": (f"fp64 oracle, {pf['rows']} evenly spaced query rows of each of "
                   f"{pf['heads']} heads of prefill_8k ({pf['flops'] / 1e9:.1f} GFLOP in {pf['seconds']:.2f} s); "
                   f"decode: {dc['heads']} (b,h) rows of decode_32k "
                   f"({dc['bytes'] / 1e9:.2f} GB of K/V in {dc['seconds']:.2f} s)"),
        "decode": {"value": dc["bytes"] / dc["seconds"] / 1e9, "unit": "GB/s"},
        "decode_sample": (f"fp64 oracle, {dc['heads']} (b,h) rows of decode_32k "
                          f"({dc['bytes'] / 1e9:.2f} GB of K/V in {dc['seconds']:.2f} s)"),
    }


def naive_comparison(dev, flash_ms_8k):
    """The naive three-step attention the pages contrast with (S = scale QK^T and
    P = softmax(S) written to HBM in bf16, then O = PV), run with torch on the
    same GPU: its time on prefill_8k against this library's, its accuracy on
    sampled rows against the oracle, and the device memory each needs at 2K,
    4K and 8K tokens (the pages' "10x less memory at 2K, 20x at 4K" claim).
    A comparison only: nothing of it is on the library's path."""
    import numpy as np
    import torch

    import exact_io_aware_70_b200 as ea
    w = PREFILL

    def naive(q, k, v):
        s_ = torch.matmul(q, k.transpose(-1, -2)) * w.scale       # S materialised (bf16)
        n = q.shape[2]
        s_.masked_fill_(torch.ones(n, n, dtype=torch.bool, device=dev).triu(1), float("-inf"))
        p_ = torch.softmax(s_, dim=-1)                              # P materialised (bf16)
        del s_
        return torch.matmul(p_, v)

    out = {"what": "torch bf16 matmul -> masked softmax -> matmul, S and P materialised"}
    q, k, v = make_workload(w, device="cuda")
    for _ in range(2):
        naive(q, k, v)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    reps = 5
    for _ in range(reps):
        o_n = naive(q, k, v)
    e1.record()
    torch.cuda.synchronize()
    naive_ms = e0.elapsed_time(e1) / reps
    out.update(workload="prefill_8k", naive_ms=naive_ms, flash_ms=flash_ms_8k,
               speedup=naive_ms / flash_ms_8k,
               score_matrix_bytes_per_head=w.Nq * w.Nkv * 2,
               score_matrix_bytes_total=w.B * w.H * w.Nq * w.Nkv * 2)
    # accuracy of the naive bf16 path on sampled rows of head 0 (oracle = fp64 definition)
    try:
        import oracle
        from seeded_inputs import bf16_bits
        rows = np.linspace(0, w.Nq - 1, 64).astype(np.int64)
        ro, _ = oracle.get().attn_rows_bf16(bf16_bits(q[0, 0].cpu()), bf16_bits(k[0, 0].cpu()),
                                            bf16_bits(v[0, 0].cpu()), rows, w.causal, w.scale)
        out["naive_max_abs_err_O_sampled"] = float(np.abs(o_n[0, 0, rows].float().cpu().numpy()
                                                          - ro).max())
    except Exception as exc:   # the comparison is informational
        out["naive_accuracy"] = f"not measured: {exc}"
    del q, k, v, o_n
    # peak device memory above the inputs, naive vs this library
    mem = {}
    for n in (2048, 4096, 8192):
        qn, kn, vn = make_qkv(1, w.H, n, n, w.d, 7, device="cuda")
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats()
        base = torch.cuda.memory_allocated()
        o_ = naive(qn, kn, vn)
        torch.cuda.synchronize()
        naive_extra = torch.cuda.max_memory_allocated() - base
        del o_
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats()
        base = torch.cuda.memory_allocated()
        of = torch.empty_like(qn)
        lf = torch.empty((1, w.H, n), dtype=torch.float32, device=dev)
        ea.attn_fwd(qn, kn, vn, of, lf, True, w.scale)
        torch.cuda.synchronize()
        flash_extra = torch.cuda.max_memory_allocated() - base
        mem[str(n)] = {"naive_bytes": int(naive_extra), "flash_bytes": int(flash_extra),
                       "ratio": naive_extra / flash_extra}
        del qn, kn, vn, of, lf
    out["memory_above_inputs_H32_d128"] = mem
    return out


def run_reference(args):
    """Reference arm: the oracle, as it stands, on bounded samples of the workload."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    sizes = []
    for _ in range(max(0, args.warmup)):
        oracle_prefill_sample(1.0, max_rows=256, max_heads=1)
    times = []
    flops = 0.0
    for _ in range(args.steps):
        r = oracle_prefill_sample(1.0, max_rows=256, max_heads=1)
        times.append(r["seconds"])
        flops = r["flops"]
        sizes.append(r["rows"])
    dc = oracle_decode_sample(1.0)
    value = flops / statistics.mean(times) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "prefill_8k (sampled rows) + decode_32k (sampled heads)",
                   "B": PREFILL.B, "H": PREFILL.H, "N": PREFILL.Nq, "d": PREFILL.d,
                   "causal": PREFILL.causal, "parallelism": "cpu"},
        "decode": {"value": dc["bytes"] / dc["seconds"] / 1e9, "unit": "GB/s"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": r["cores"],
                         "kind": "oracle",
                         "sample": f"{sizes[-1]} evenly spaced rows of one prefill_8k head per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def oracle_bwd_sample(w, budget_s):
    """Time the oracle's backward pass on leading square blocks of one head.

    For a causal square head, the first n query rows see only the first n keys,
    so the n x n leading block is itself a complete causal problem; n doubles
    until one call takes a quarter of the budget."""
    import oracle
    from seeded_inputs import make_dout
    orc = oracle.get()
    q, k, v = make_qkv(1, 1, w.Nq, w.Nkv, w.d, w.seed)
    do = make_dout(1, 1, w.Nq, w.d, w.seed)
    f64 = lambda t, n: t[0, 0, :n].double().numpy()
    n, dt, flops = 256, 0.0, 0.0
    while True:
        t0 = time.perf_counter()
        orc.attn_bwd_head_f64(f64(q, n), f64(k, n), f64(v, n), f64(do, n), w.causal, w.scale)
        dt = time.perf_counter() - t0
        flops = 10.0 * w.d * (n * (n + 1) // 2 if w.causal else n * n)
        if dt > budget_s / 4 or 2 * n > min(w.Nq, w.Nkv):
            break
        n *= 2
    return {"flops": flops, "seconds": dt, "n": n, "cores": orc.num_threads()}


def oracle_fp8_sample(w, budget_s):
    """Time the oracle's 8-bit entry on leading square blocks of one head (a
    causal head's first n rows see only its first n keys); n doubles until one
    call takes a quarter of the budget."""
    import oracle
    from seeded_inputs import fp8_codes, make_qkv_fp8
    orc = oracle.get()
    q8, k8, v8, qd, kd, vd = make_qkv_fp8(1, 1, w.Nq, w.Nkv, w.d, w.seed)
    n = 256
    while True:
        c = lambda t: fp8_codes(t[:, :, :n])
        t0 = time.perf_counter()
        orc.attn_fwd_fp8(c(q8), c(k8), c(v8), qd.numpy(), kd.numpy(), vd.numpy(), w.causal,
                         w.scale)
        dt = time.perf_counter() - t0
        flops = 4.0 * w.d * (n * (n + 1) // 2 if w.causal else n * n)
        if dt > budget_s / 4 or 2 * n > min(w.Nq, w.Nkv):
            break
        n *= 2
    return {"flops": flops, "seconds": dt, "n": n, "cores": orc.num_threads()}


def run_fp8(args):
    """Forward pass on e4m3 inputs (attn_fwd_fp8) of a prefill workload: codes and
    per-head descale factors drawn from the workload's seed; one call per step."""
    import torch
    import torch.distributed as dist

    import exact_io_aware_70_b200 as ea
    from exact_io_aware_70_b200.sharding import max_over_ranks
    from seeded_inputs import make_qkv_fp8

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    L = ea.lib
    w = _maybe_batch(WORKLOADS[args.workload[:-len("_fp8")]], args.batch)
    wr = rank_slice(w, rank)
    ins = make_qkv_fp8(w.B, w.H, w.Nq, w.Nkv, w.d, wr.seed, device="cuda")
    o = torch.empty((w.B, w.H, w.Nq, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    args_c = tuple(t.data_ptr() for t in ins) + (o.data_ptr(), lse.data_ptr(), w.B, w.H, w.Nq,
                                                 w.Nkv, w.d, int(w.causal), w.scale, sp)

    def step():
        rc = L.attn_fwd_fp8(*args_c)
        if rc != 0:
            raise RuntimeError(f"attn_fwd_fp8: {ea.attn_strerror(rc)}")

    flush = L2Flusher(list(ins) + [o, lse], dev, bool(args.batch))
    for _ in range(args.warmup):
        step()
    if ea.attn_status() != 0:
        raise RuntimeError("device status reported an error during warm-up")
    K = args.steps
    total_ms, call_ms, clk, hot_ms = timed_calls(step, K, flush, stream, ws, local)
    if ea.attn_status() != 0:
        raise RuntimeError("device status reported an error in the timed region")

    e2e = None
    if not args.no_e2e:
        hin = [t.cpu().pin_memory() for t in ins]
        hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (o, lse)]
        h2d = sum(t.numel() * t.element_size() for t in hin)
        d2h = sum(t.numel() * t.element_size() for t in hout)
        sets = [list(ins) + [o, lse], [torch.empty_like(t) for t in list(ins) + [o, lse]]]

        def run(b):
            q8, k8, v8, qd, kd, vd, O, Ls = sets[b]
            ea.attn_fwd_fp8(q8, k8, v8, qd, kd, vd, O, Ls, w.causal, w.scale)

        h2d_l = [(h, (sets[0][i], sets[1][i])) for i, h in enumerate(hin)]
        d2h_l = [((sets[0][6 + i], sets[1][6 + i]), h) for i, h in enumerate(hout)]
        pipelined_e2e(h2d_l, run, d2h_l, 2, stream)   # warm-up
        E = max(4, min(K, 6))
        ems = pipelined_e2e(h2d_l, run, d2h_l, E, stream)
        del sets
        if ea.attn_status() != 0:
            raise RuntimeError("device status reported an error in the e2e region")
        e2e = {"value": None, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems, "steps": E,
               "path": "pinned host -> copy (own stream) -> attn_fwd_fp8 -> copy back (own "
                       "stream), every step; two device buffer sets, so one step's copies "
                       "overlap the neighbouring steps' kernels; CUDA events"}
    vals = max_over_ranks([total_ms, call_ms] + ([e2e["ms_per_step"]] if e2e else []) +
                          ([hot_ms] if hot_ms is not None else []), device=dev)
    total_ms, call_ms = vals[0], vals[1]
    if hot_ms is not None:
        hot_ms = vals[-1]
    if e2e:
        e2e["ms_per_step"] = vals[2]
        e2e["value"] = ws * prefill_flops(w) / (vals[2] * 1e-3) / 1e12
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]
    a = prefill_flops(w) / (call_ms * 1e-3) / 1e12
    roof = {"kernel": "attn_fwd_sm100 (e4m3)", "bound": "tensor", "achieved": a,
            "peak": fp8_peak, "unit": "TFLOP/s", "frac": a / fp8_peak,
            "peak_note": "measured bf16 peak x 2 (nominal e4m3 / bf16 dense ratio)",
            "frac_of_bf16_peak": a / pk["bf16_tflops"],
            "traffic": recorded_traffic().get(("attn_fwd_sm100_e4m3", args.workload)),
            "algorithmic_bytes": prefill_bytes(w) // 2 + w.B * w.H * w.Nq * w.d,
            "algorithmic_flops": prefill_flops(w), "ms": call_ms}
    line = {
        "metric": "attn fwd (e4m3 inputs) TFLOP/s & % FP8 tensor peak",
        "value": ws * a, "unit": "TFLOP/s", "n_gpus": ws, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": args.workload, "B": w.B, "H": w.H, "N": w.Nq, "d": w.d,
                   "causal": w.causal, "flop_per_step": prefill_flops(w), "l2": flush.note,
                   "parallelism": (f"batch partitioned: one {w.B}-entry slice per GPU x{ws}"
                                   if ws > 1 else "1 GPU")},
        "roofline": roof,
        "peaks": dict(pk, note="of measured" if pk["source"] == "measured" else "of fallback"),
        "clocks": clk.summary(max_mhz_default=1965.0),
        "gpu_launches": K, "e2e": e2e,
    }
    if hot_ms is not None:
        line["hot"] = {"value": ws * prefill_flops(w) / (hot_ms * 1e-3) / 1e12,
                       "unit": "TFLOP/s", "ms": hot_ms, "note": "back to back, L2 not flushed"}
    if ws == 1 and not args.no_cpu_baseline:
        cb = oracle_fp8_sample(w, args.cpu_budget)
        line["cpu_baseline"] = {
            "value": cb["flops"] / cb["seconds"] / 1e12, "unit": "TFLOP/s", "cores": cb["cores"],
            "kind": "oracle",
            "sample": f"fp64 oracle on the decoded e4m3 inputs of the leading {cb['n']}x{cb['n']} "
                      f"block of one head ({cb['flops'] / 1e9:.1f} GFLOP in {cb['seconds']:.2f} s)"}
    print(json.dumps(line), flush=True)
    return 0


def run_bwd(args):
    """Backward pass (dQ, dK, dV) of a prefill workload: O and LSE come from one
    untimed forward call; each step is one attn_bwd call (three kernels)."""
    import torch
    import torch.distributed as dist

    import exact_io_aware_70_b200 as ea
    from exact_io_aware_70_b200.sharding import max_over_ranks
    from seeded_inputs import make_dout

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    L = ea.lib
    w = _maybe_batch(WORKLOADS[args.workload[:-len("_bwd")]], args.batch)
    wr = rank_slice(w, rank)
    q, k, v = make_workload(wr, device="cuda")
    do = make_dout(w.B, w.H, w.Nq, w.d, wr.seed, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    ea.attn_fwd(q, k, v, o, lse, w.causal, w.scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    work = torch.empty(ea.attn_bwd_workspace_bytes(w.B, w.H, w.Nq, w.d), dtype=torch.uint8,
                       device=dev)
    args_c = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
              lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), w.B, w.H, w.Nq, w.Nkv,
              w.d, int(w.causal), w.scale, work.data_ptr(), work.numel(), sp)

    det = bool(args.deterministic)
    entry = L.attn_bwd_deterministic if det else L.attn_bwd
    name = "attn_bwd_deterministic" if det else "attn_bwd"

    def step():
        rc = entry(*args_c)
        if rc != 0:
            raise RuntimeError(f"{name}: {ea.attn_strerror(rc)}")

    flush = L2Flusher([q, k, v, o, do, lse, dq, dk, dv, work], dev, bool(args.batch))
    for _ in range(args.warmup):
        step()
    if ea.attn_status() != 0:
        raise RuntimeError("device status reported an error during warm-up")
    K = args.steps
    total_ms, call_ms, clk, hot_ms = timed_calls(step, K, flush, stream, ws, local)
    if ea.attn_status() != 0:
        raise RuntimeError("device status reported an error in the timed region")

    e2e = None
    if not args.no_e2e:
        hin = [t.cpu().pin_memory() for t in (q, k, v, o, do, lse)]
        hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (dq, dk, dv)]
        h2d = sum(t.numel() * t.element_size() for t in hin)
        d2h = sum(t.numel() * t.element_size() for t in hout)

        tset = [q, k, v, o, do, lse, dq, dk, dv]
        sets = [tset, [torch.empty_like(t) for t in tset]]

        def run(b):
            Q, Kt, V, O, DO, Ls, DQ, DK, DV = sets[b]
            ea.attn_bwd(Q, Kt, V, O, DO, Ls, DQ, DK, DV, w.causal, w.scale, work,
                        deterministic=det)

        h2d_l = [(h, (sets[0][i], sets[1][i])) for i, h in enumerate(hin)]
        d2h_l = [((sets[0][6 + i], sets[1][6 + i]), h) for i, h in enumerate(hout)]
        pipelined_e2e(h2d_l, run, d2h_l, 2, stream)   # warm-up
        E = max(4, min(K, 6))
        ems = pipelined_e2e(h2d_l, run, d2h_l, E, stream)
        del sets
        if ea.attn_status() != 0:
            raise RuntimeError("device status reported an error in the e2e region")
        e2e = {"value": None, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems, "steps": E,
               "path": f"pinned host -> copy (own stream) -> {name} -> copy back (own stream), "
                       "every step; two device buffer sets, so one step's copies overlap the "
                       "neighbouring steps' kernels; CUDA events"}
    vals = max_over_ranks([total_ms, call_ms] + ([e2e["ms_per_step"]] if e2e else []) +
                          ([hot_ms] if hot_ms is not None else []), device=dev)
    total_ms, call_ms = vals[0], vals[1]
    if hot_ms is not None:
        hot_ms = vals[-1]
    if e2e:
        e2e["ms_per_step"] = vals[2]
        e2e["value"] = ws * bwd_flops(w) / (vals[2] * 1e-3) / 1e12
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    pk = peaks()
    a = bwd_flops(w) / (call_ms * 1e-3) / 1e12
    roof = {"kernel": (f"{name} ({'kv bound + ' if det else ''}preprocess + attn_bwd_sm100 + "
                       "postprocess, timed as one call)"),
            "bound": "tensor", "achieved": a, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
            "frac": a / pk["bf16_tflops"], "frac_of_sustained": a / pk["bf16_tflops_sustained"],
            "traffic": recorded_traffic().get(
                ("attn_bwd_sm100", args.workload + ("_deterministic" if det else ""))),
            "algorithmic_bytes": bwd_bytes(w), "algorithmic_flops": bwd_flops(w), "ms": call_ms}
    line = {
        "metric": "attn bwd TFLOP/s & % BF16 tensor peak",
        "value": ws * a, "unit": "TFLOP/s", "n_gpus": ws, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "B": w.B, "H": w.H, "N": w.Nq, "d": w.d,
                   "causal": w.causal, "flop_per_step": bwd_flops(w), "l2": flush.note,
                   "entry": name,
                   "parallelism": (f"batch partitioned: one {w.B}-entry slice per GPU x{ws}"
                                   if ws > 1 else "1 GPU")},
        "roofline": roof,
        "peaks": dict(pk, note="of measured" if pk["source"] == "measured" else "of fallback"),
        "clocks": clk.summary(max_mhz_default=1965.0),
        "gpu_launches": (4 if det else 3) * K, "e2e": e2e,
    }
    if hot_ms is not None:
        line["hot"] = {"value": ws * bwd_flops(w) / (hot_ms * 1e-3) / 1e12,
                       "unit": "TFLOP/s", "ms": hot_ms, "note": "back to back, L2 not flushed"}
    if ws == 1 and not args.no_cpu_baseline:
        cb = oracle_bwd_sample(w, args.cpu_budget)
        line["cpu_baseline"] = {
            "value": cb["flops"] / cb["seconds"] / 1e12, "unit": "TFLOP/s", "cores": cb["cores"],
            "kind": "oracle",
            "sample": f"fp64 oracle backward of the leading {cb['n']}x{cb['n']} block of one "
                      f"head ({cb['flops'] / 1e9:.1f} GFLOP in {cb['seconds']:.2f} s)"}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ GPU arm --
def pipelined_e2e(h2d, run, d2h, E, stream):
    """E end-to-end steps, each copying its inputs from pinned host memory to one
    of two device buffer sets (h2d: [(host, (dev_a, dev_b)), ...]), running
    run(b) on `stream` for buffer set b, and copying its outputs back (d2h:
    [((dev_a, dev_b), host), ...]). The copies in and the copies out each have
    their own stream, so step i+1's inputs travel while step i computes and
    step i-1's outputs come back; events keep a buffer set from being refilled
    before its outputs are out. Returns the ms per step (CUDA events, the
    first copy in to the last copy out, divided by E)."""
    import torch
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    e_in = [torch.cuda.Event() for _ in range(2)]
    e_run = [torch.cuda.Event() for _ in range(2)]
    e_free = [torch.cuda.Event() for _ in range(2)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(s_in)
    for i in range(E):
        b = i & 1
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(e_free[b])
            for host, devs in h2d:
                devs[b].copy_(host, non_blocking=True)
            e_in[b].record(s_in)
        stream.wait_event(e_in[b])
        run(b)
        e_run[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(e_run[b])
            for devs, host in d2h:
                host.copy_(devs[b], non_blocking=True)
            e_free[b].record(s_out)
    t1.record(s_out)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / E


def _maybe_batch(w, batch):
    import dataclasses
    return dataclasses.replace(w, B=batch) if batch else w


def _peaks_note(pk):
    return "of measured" if pk["source"] == "measured" else "of fallback"


def prefill_roofline(w, ms, pk, traffic=None):
    a = prefill_flops(w) / (ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": a, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
            "frac": a / pk["bf16_tflops"], "frac_of_sustained": a / pk["bf16_tflops_sustained"],
            "traffic": traffic, "algorithmic_bytes": prefill_bytes(w),
            "algorithmic_flops": prefill_flops(w), "ms": ms, "note": _peaks_note(pk)}


def prefill_cpu_baseline(w, budget_s):
    cb = oracle_prefill_sample(budget_s, max_heads=min(4, w.H), w=w)
    return {"value": cb["flops"] / cb["seconds"] / 1e12, "unit": "TFLOP/s", "cores": cb["cores"],
            "kind": "oracle",
            "sample": (f"fp64 oracle, {cb['rows']} evenly spaced query rows of each of "
                       f"{cb['heads']} heads of {w.name} ({cb['flops'] / 1e9:.2f} GFLOP in "
                       f"{cb['seconds']:.2f} s)")}


def time_prefill_workload(ea, w, K, warmup, dev, stream, local, cpu_budget):
    """One more prefill workload of the default line, timed on its own after
    the step: K calls of attn_fwd (cold L2 where the inputs fit in it, with the
    hot figure alongside), its roofline and the oracle on a bounded sample."""
    import torch
    q, k, v = make_workload(w, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    sp = stream.cuda_stream
    args_c = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.H,
              w.Nq, w.Nkv, w.d, int(w.causal), w.scale, sp)

    def step():
        rc = ea.lib.attn_fwd(*args_c)
        if rc != 0:
            raise RuntimeError(f"attn_fwd ({w.name}): {ea.attn_strerror(rc)}")

    flush = L2Flusher([q, k, v, o, lse], dev, False)
    for _ in range(warmup):
        step()
    if ea.attn_status() != 0:
        raise RuntimeError(f"device status reported an error during {w.name} warm-up")
    _, call_ms, clk, hot_ms = timed_calls(step, K, flush, stream, 1, local)
    if ea.attn_status() != 0:
        raise RuntimeError(f"device status reported an error timing {w.name}")
    pk = peaks()
    out = {"config": {"B": w.B, "H": w.H, "N": w.Nq, "d": w.d, "causal": w.causal,
                      "seed": w.seed, "l2": flush.note},
           "ms": call_ms, "value": prefill_flops(w) / (call_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
           "roofline": dict(prefill_roofline(w, call_ms, pk,
                                             recorded_traffic().get(("attn_fwd_sm100", w.name))),
                            kernel="attn_fwd_sm100"),
           "clocks": clk.summary(max_mhz_default=1965.0), "gpu_launches": K}
    if hot_ms is not None:
        out["hot"] = {"ms": hot_ms, "value": prefill_flops(w) / (hot_ms * 1e-3) / 1e12,
                      "unit": "TFLOP/s", "frac": prefill_flops(w) / (hot_ms * 1e-3) / 1e12
                      / pk["bf16_tflops"], "note": "back to back, L2 not flushed"}
    if cpu_budget > 0:
        out["cpu_baseline"] = prefill_cpu_baseline(w, cpu_budget)
    del q, k, v, o, lse
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    """The default line: one step = prefill_8k forward + decode_32k split-KV
    decode (partials + merge), plus, in the same run at one GPU, the other
    workloads (tiny, gpt2_1k, prefill_16k) timed on their own.

    With N GPUs (torchrun) the job grows with N (weak scaling): the prefill
    batch has N entries, one per GPU (its heads partitioned over the ranks by
    batch entry); the decode sequence has N x 32768 keys, one 32768-key shard
    per GPU, whose partials are all-gathered (NCCL) and merged on every GPU
    with attn_lse_merge_gathered."""
    import torch
    import torch.distributed as dist

    import exact_io_aware_70_b200 as ea
    from exact_io_aware_70_b200.sharding import max_over_ranks

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    L = ea.lib

    import dataclasses
    paged = args.workload == "decode_32k_paged"
    if args.workload == "step":
        pw, dw = PREFILL, DECODE
    elif args.workload in ("prefill_8k", "prefill_16k", "gpt2_1k", "tiny"):
        pw, dw = WORKLOADS[args.workload], None
    elif paged:
        from seeded_inputs import PAGED_DECODE as PD
        pw = None
        dw = dataclasses.replace(DECODE, name=PD["name"], B=PD["B"], H=PD["H"], Nkv=PD["seq_len"],
                                 d=PD["d"], num_splits=PD["num_splits"], seed=PD["seed"])
    else:
        pw, dw = None, WORKLOADS[args.workload]
    pw = _maybe_batch(pw, args.batch) if pw else None
    dw = _maybe_batch(dw, args.batch) if dw else None

    # ---- inputs resident in HBM; each rank draws its own slice of the job
    kernels = []        # (name, launch, is_ours)
    if pw:
        pw_r = rank_slice(pw, rank)
        q, k, v = make_workload(pw_r, device="cuda")
        o = torch.empty_like(q)
        lse = torch.empty((pw.B, pw.H, pw.Nq), dtype=torch.float32, device=dev)

        def launch_prefill():
            return L.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), pw.B, pw.H, pw.Nq, pw.Nkv, pw.d, int(pw.causal),
                              pw.scale, sp)
        kernels.append(("attn_fwd_sm100", launch_prefill, True))
    if dw:
        S = dw.num_splits
        dw_r = rank_slice(dw, rank)
        if paged:
            from seeded_inputs import PAGED_DECODE as PD, make_paged_cache
            dq, dk, dv, dtable, dlens = make_paged_cache(dw.B, dw.H, [dw.Nkv] * dw.B, dw.d,
                                                         PD["page_size"], dw_r.seed, device="cuda")
            if ws > 1:
                # the query row is the same on every rank (the base seed's first draw, which
                # does not depend on the cache size); the cache is the rank's shard
                dq = make_paged_cache(dw.B, dw.H, [1] * dw.B, dw.d, PD["page_size"],
                                      dw.seed, device="cuda")[0]
        else:
            dq, dk, dv = make_workload(dw_r, device="cuda")
            if ws > 1:
                # the query rows are the same on every rank (the base seed's first draw,
                # which does not depend on the key count); the keys are the rank's shard
                dq = make_qkv(dw.B, dw.H, 1, 1, dw.d, dw.seed, device="cuda")[0]
        do = torch.empty_like(dq)
        dlse = torch.empty((dw.B, dw.H, 1), dtype=torch.float32, device=dev)
        work = torch.empty(ea.attn_decode_workspace_bytes(dw.B, dw.H, dw.d, S), dtype=torch.uint8,
                           device=dev)
        o_bytes = ((dw.B * dw.H * S * dw.d * 4 + 255) // 256) * 256
        if ws > 1:
            # this rank's partials, and the buffers the all-gather fills (rank r at [r])
            po = torch.empty((dw.B, dw.H, S, dw.d), dtype=torch.float32, device=dev)
            pl = torch.empty((dw.B, dw.H, S), dtype=torch.float32, device=dev)
            og = torch.empty((ws, dw.B, dw.H, S, dw.d), dtype=torch.float32, device=dev)
            lg = torch.empty((ws, dw.B, dw.H, S), dtype=torch.float32, device=dev)
            o_part, lse_part = po.data_ptr(), pl.data_ptr()
        else:
            o_part, lse_part = work.data_ptr(), work.data_ptr() + o_bytes
        if paged:
            npages, ps = dk.shape[0], PD["page_size"]

            def launch_partials():
                return L.attn_decode_paged_partials(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                                    dtable.data_ptr(), dlens.data_ptr(), o_part,
                                                    lse_part, dw.B, dw.H, dw.d, ps,
                                                    dtable.shape[1], npages, dw.scale, S, sp)
        else:
            def launch_partials():
                return L.attn_decode_partials(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), o_part,
                                              lse_part, dw.B, dw.H, dw.Nkv, dw.d, dw.scale, S, sp)
        kernels.append(("attn_decode_partials", launch_partials, True))
        if ws > 1:
            def launch_gather():
                dist.all_gather_into_tensor(og, po)
                dist.all_gather_into_tensor(lg, pl)
                return 0

            def launch_merge():
                return L.attn_lse_merge_gathered(og.data_ptr(), lg.data_ptr(), do.data_ptr(),
                                                 dlse.data_ptr(), ws, dw.B, dw.H, S, dw.d, sp)
            kernels.append(("nccl_all_gather", launch_gather, False))
        else:
            def launch_merge():
                return L.attn_lse_merge(o_part, lse_part, do.data_ptr(), dlse.data_ptr(), dw.B,
                                        dw.H, S, dw.d, sp)
        kernels.append(("attn_lse_merge", launch_merge, True))
    torch.cuda.synchronize()
    resident = ([q, k, v, o, lse] if pw else []) + ([dq, dk, dv, do, dlse, work] if dw else [])
    if dw and paged:
        resident += [dtable, dlens]
    flush = L2Flusher(resident, dev, bool(args.batch))

    def step(evs=None):
        for i, (name, fn, _) in enumerate(kernels):
            if evs is not None:
                evs[i].record(stream)
            rc = fn()
            if rc != 0:
                raise RuntimeError(f"{name}: {ea.attn_strerror(rc)}")
        if evs is not None:
            evs[len(kernels)].record(stream)

    for _ in range(args.warmup):
        step()
    if ea.attn_status() != 0:
        raise RuntimeError("device status reported an error during warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(kernels) + 1)]
          for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        for s_ in range(K):
            flush()
            step(ev[s_])
        t_end.record(stream)
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
    if ea.attn_status() != 0:
        raise RuntimeError("device status reported an error in the timed region")
    total_ms = t_start.elapsed_time(t_end)
    per_kernel_ms = [statistics.mean(ev[s_][i].elapsed_time(ev[s_][i + 1]) for s_ in range(K))
                     for i in range(len(kernels))]
    hot_kernel_ms = []
    if flush.active:
        # the same kernels back to back, L2 not flushed
        for s_ in range(K):
            step(ev[s_])
        torch.cuda.synchronize()
        if ea.attn_status() != 0:
            raise RuntimeError("device status reported an error in the hot region")
        hot_kernel_ms = [statistics.mean(ev[s_][i].elapsed_time(ev[s_][i + 1]) for s_ in range(K))
                         for i in range(len(kernels))]
    vals = max_over_ranks([total_ms] + per_kernel_ms + hot_kernel_ms, device=dev)
    total_ms, per_kernel_ms = vals[0], vals[1:1 + len(kernels)]
    hot_kernel_ms = vals[1 + len(kernels):]
    kms = dict(zip([n for n, _, _ in kernels], per_kernel_ms))
    hot_kms = dict(zip([n for n, _, _ in kernels], hot_kernel_ms))

    # ---- e2e: the same work through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e:
        h2d = d2h = 0
        if pw:
            hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
            ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
            hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
            h2d += sum(t.numel() * t.element_size() for t in (hq, hk, hv))
            d2h += sum(t.numel() * t.element_size() for t in (ho, hl))
        if dw:
            hdq, hdk, hdv = (t.cpu().pin_memory() for t in (dq, dk, dv))
            hdo = torch.empty(do.shape, dtype=do.dtype, pin_memory=True)
            hdl = torch.empty(dlse.shape, dtype=dlse.dtype, pin_memory=True)
            h2d += sum(t.numel() * t.element_size() for t in (hdq, hdk, hdv))
            d2h += sum(t.numel() * t.element_size() for t in (hdo, hdl))

        # a second device buffer set, so that one step's copies overlap another's kernels
        E = max(4, min(K, 6))
        acc = []
        if pw:
            q2, k2, v2, o2 = (torch.empty_like(t) for t in (q, k, v, o))
            lse2 = torch.empty_like(lse)
            pset = [(q, k, v, o, lse), (q2, k2, v2, o2, lse2)]

            def run_prefill(b):
                Q, Kt, V, O, Ls = pset[b]
                ea.attn_fwd(Q, Kt, V, O, Ls, pw.causal, pw.scale)

            pipelined_e2e([(hq, (q, q2)), (hk, (k, k2)), (hv, (v, v2))], run_prefill,
                          [((o, o2), ho), ((lse, lse2), hl)], 2, stream)   # warm-up
            acc.append(pipelined_e2e([(hq, (q, q2)), (hk, (k, k2)), (hv, (v, v2))], run_prefill,
                                     [((o, o2), ho), ((lse, lse2), hl)], E, stream))
            del q2, k2, v2, o2, lse2, pset
        if dw:
            dq2, dk2, dv2, do2 = (torch.empty_like(t) for t in (dq, dk, dv, do))
            dlse2 = torch.empty_like(dlse)
            dset = [(dq, dk, dv, do, dlse), (dq2, dk2, dv2, do2, dlse2)]

            def run_decode(b):
                Q, Kt, V, O, Ls = dset[b]
                if ws > 1:
                    # this rank's shard through the public API, then the exchange and the merge
                    if paged:
                        ea.attn_decode_paged_partials(Q, Kt, V, dtable, dlens, po, pl, dw.scale, S)
                    else:
                        ea.attn_decode_partials(Q, Kt, V, po, pl, dw.scale, S)
                    launch_gather()
                    ea.attn_lse_merge_gathered(og, lg, O, Ls)
                elif paged:
                    ea.attn_decode_paged(Q, Kt, V, dtable, dlens, O, Ls, dw.scale, S, work)
                else:
                    ea.attn_decode_splitkv(Q, Kt, V, O, Ls, dw.scale, S, work)

            dh2d = [(hdq, (dq, dq2)), (hdk, (dk, dk2)), (hdv, (dv, dv2))]
            dd2h = [((do, do2), hdo), ((dlse, dlse2), hdl)]
            pipelined_e2e(dh2d, run_decode, dd2h, 2, stream)   # warm-up
            acc.append(pipelined_e2e(dh2d, run_decode, dd2h, E, stream))
            del dq2, dk2, dv2, do2, dlse2, dset
        acc = max_over_ranks(acc, device=dev)
        if ea.attn_status() != 0:
            raise RuntimeError("device status reported an error in the e2e region")
        e2e = {"h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": sum(acc),
               "steps": E,
               "path": "pinned host -> copy (own stream) -> attn_fwd / attn_decode_splitkv "
                       "(launching stream) -> copy back (own stream), every step; two device "
                       "buffer sets, so one step's copies overlap the neighbouring steps' "
                       "kernels; CUDA events from the first copy in to the last copy out"}
        if pw:
            e2e["value"] = ws * prefill_flops(pw) / (acc[0] * 1e-3) / 1e12
            e2e["unit"] = "TFLOP/s"
        if dw:
            dec = {"value": ws * decode_kv_bytes(dw) / (acc[-1] * 1e-3) / 1e9, "unit": "GB/s"}
            if pw:
                e2e["decode"] = dec
            else:
                e2e.update(dec)

    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    pk = peaks()
    traffic = recorded_traffic()
    step_ms = sum(per_kernel_ms)
    roof = {}
    if pw:
        roof["attn_fwd_sm100"] = dict(prefill_roofline(pw, kms["attn_fwd_sm100"], pk,
                                                       traffic.get(("attn_fwd_sm100", pw.name))),
                                      share=kms["attn_fwd_sm100"] / step_ms)
    if dw:
        mbytes = merge_bytes(dw) * ws
        for name, nbytes in (("attn_decode_partials", decode_partial_bytes(dw)),
                             ("attn_lse_merge", mbytes)):
            t = kms[name]
            a = nbytes / (t * 1e-3) / 1e9
            roof[name] = {"bound": "hbm", "achieved": a, "peak": pk["hbm_gbs"], "unit": "GB/s",
                          "frac": a / pk["hbm_gbs"], "traffic": traffic.get((name, dw.name)),
                          "algorithmic_bytes": nbytes, "ms": t, "share": t / step_ms,
                          "note": _peaks_note(pk)}
    dominant = max(roof, key=lambda n: roof[n]["ms"])
    dom = dict(roof[dominant], kernel=dominant)
    if ws > 1:
        par = []
        if pw:
            par.append(f"prefill: heads partitioned, one {pw.B}x{pw.H}-head batch slice per GPU")
        if dw:
            par.append(f"decode: KV sequence split, one {dw.Nkv}-key shard per GPU, partials "
                       "all-gathered (NCCL) and merged on every GPU")
        parallelism = f"{ws} GPUs; " + "; ".join(par)
    else:
        parallelism = "1 GPU"
    cfg = {"workload": "prefill_8k + decode_32k" if args.workload == "step" else args.workload,
           "l2": flush.note, "parallelism": parallelism}
    line = {"metric": METRIC}
    if pw:
        pf = kms["attn_fwd_sm100"]
        cfg["prefill"] = {"B": pw.B * ws, "H": pw.H, "N": pw.Nq, "d": pw.d, "causal": pw.causal,
                          "flop_per_step": ws * prefill_flops(pw)}
        line.update(value=ws * prefill_flops(pw) / (pf * 1e-3) / 1e12, unit="TFLOP/s")
        line["prefill"] = {"value": line["value"], "unit": "TFLOP/s", "ms": pf,
                           "frac_of_bf16_peak": roof["attn_fwd_sm100"]["frac"]}
    if dw:
        dnames = ["attn_decode_partials", "attn_lse_merge"] + (["nccl_all_gather"] if ws > 1 else [])
        dms = sum(kms[n] for n in dnames)
        cfg["decode"] = {"B": dw.B, "H": dw.H, "Nkv": dw.Nkv * ws, "d": dw.d,
                         "splits": dw.num_splits * ws, "kv_bytes_per_step": ws * decode_kv_bytes(dw)}
        dgbs = decode_kv_bytes(dw) / (dms * 1e-3) / 1e9
        line["decode"] = {"value": ws * dgbs, "unit": "GB/s", "ms": dms,
                          "frac_of_hbm_peak": dgbs / pk["hbm_gbs"]}
        if ws > 1:
            line["decode"]["all_gather_ms"] = kms["nccl_all_gather"]
        if not pw:
            line.update(value=ws * dgbs, unit="GB/s")
    line.update({
        "n_gpus": ws, "steps": K, "warmup": args.warmup, "ms_per_step": total_ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": cfg, "roofline": dom, "roofline_kernels": roof,
        "peaks": dict(pk, note=_peaks_note(pk)),
        "clocks": clk.summary(max_mhz_default=1965.0),
        "gpu_launches": sum(1 for _, _, ours in kernels if ours) * K, "e2e": e2e,
    })
    if hot_kms:
        hot = {"ms": sum(hot_kms.values()), "note": "the same kernels back to back, L2 not flushed"}
        if pw:
            hot.update(value=ws * prefill_flops(pw) / (hot_kms["attn_fwd_sm100"] * 1e-3) / 1e12,
                       unit="TFLOP/s")
        else:
            hot.update(value=ws * decode_kv_bytes(dw) / (hot["ms"] * 1e-3) / 1e9, unit="GB/s")
        line["hot"] = hot
    cb = None
    if ws == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(args.cpu_budget)
        line["cpu_baseline"] = cb
    if ws == 1 and args.workload == "step" and not args.no_workloads:
        # the five workloads, each with its own roofline and oracle baseline
        wl = {}
        for name in ("tiny", "gpt2_1k"):
            wl[name] = time_prefill_workload(ea, WORKLOADS[name], K, args.warmup, dev, stream,
                                             local, 0 if args.no_cpu_baseline else 2.0)
        wl["prefill_8k"] = {
            "config": {"B": pw.B, "H": pw.H, "N": pw.Nq, "d": pw.d, "causal": pw.causal,
                       "seed": pw.seed, "l2": flush.note},
            "ms": kms["attn_fwd_sm100"], "value": line["prefill"]["value"], "unit": "TFLOP/s",
            "roofline": dict(roof["attn_fwd_sm100"], kernel="attn_fwd_sm100"),
            "note": "timed inside the step (after the 8.6 GB decode of the previous step)"}
        if cb:
            wl["prefill_8k"]["cpu_baseline"] = {k_: cb[k_] for k_ in
                                                ("value", "unit", "cores", "kind", "sample")}
        wl["prefill_16k"] = time_prefill_workload(ea, WORKLOADS["prefill_16k"], max(3, K // 2),
                                                  args.warmup, dev, stream, local,
                                                  0 if args.no_cpu_baseline else 2.0)
        wl["decode_32k"] = {
            "config": {"B": dw.B, "H": dw.H, "Nkv": dw.Nkv, "d": dw.d, "splits": dw.num_splits,
                       "seed": dw.seed, "l2": flush.note},
            "ms": line["decode"]["ms"], "value": line["decode"]["value"], "unit": "GB/s",
            "roofline": dict(roof["attn_decode_partials"], kernel="attn_decode_partials"),
            "merge_roofline": dict(roof["attn_lse_merge"], kernel="attn_lse_merge"),
            "frac_of_hbm_peak": line["decode"]["frac_of_hbm_peak"],
            "note": "partials + merge, timed inside the step"}
        if cb:
            wl["decode_32k"]["cpu_baseline"] = dict(cb["decode"], cores=cb["cores"],
                                                    kind="oracle", sample=cb["decode_sample"])
        line["workloads"] = wl
        line["gpu_launches"] += sum(w_["gpu_launches"] for w_ in wl.values()
                                    if "gpu_launches" in w_)
    if ws == 1 and pw is PREFILL and not args.no_naive:
        line["naive_comparison"] = naive_comparison(dev, kms["attn_fwd_sm100"])
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="step",
                    choices=["step", "prefill_8k", "prefill_16k", "gpt2_1k", "tiny", "decode_32k",
                             "decode_32k_paged", "prefill_8k_bwd", "prefill_16k_bwd",
                             "gpt2_1k_bwd", "prefill_8k_fp8", "prefill_16k_fp8", "gpt2_1k_fp8"],
                    help="step = prefill_8k + decode_32k (the default bench line); "
                         "*_bwd = the backward pass of that prefill workload; "
                         "*_fp8 = its forward pass on e4m3 inputs")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the batch size (small profiling captures only)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="default line only: skip timing tiny, gpt2_1k and prefill_16k")
    ap.add_argument("--no-naive", action="store_true",
                    help="skip the naive materialising attention comparison")
    ap.add_argument("--deterministic", action="store_true",
                    help="*_bwd workloads: time attn_bwd_deterministic (fixed-point dQ)")
    ap.add_argument("--cpu-budget", type=float, default=8.0,
                    help="seconds of oracle work for the CPU baseline")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.workload.endswith("_bwd"):
        return run_bwd(args)
    if args.workload.endswith("_fp8"):
        return run_fp8(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
