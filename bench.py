#!/usr/bin/env python
"""Benchmark: CSA2 decode layer step at 128K tokens of context (FULL mode).

Workload "decode_128k_full": batch 32, one query token each, N = 32768 FP4
main-KV entries of dim 512 (128K tokens at 4:1 compression), 64 bf16 query
heads, indexer 64 heads x 128 with integer E4M3 values, top-2048, lengths
uniform in [16384, 32768]. One step = one pass of the whole hot path over the
batch: indexer scores -> top-K -> gather + FP4 dequant + sparse attention (+
split combine). The FP4 cache is built once before timing (a cache is built
when tokens arrive, not per step). Inputs are resident in HBM; L2 is flushed
between timed steps (a 256 MiB write, then a 256 MiB read so that the flush's
dirty lines are written back there), outside the timed events.

Prints one JSON line. With --impl reference it times the CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "CSA2 decode layer-steps/s at 128K ctx; achieved HBM GB/s vs 8 TB/s peak"
UNIT = "layer-steps/s"
DEFAULT_WORKLOAD = "decode_128k_full"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_workload(w, rank: int):
    """Weak scaling: every rank gets its own batch of sequences (its own seed)."""
    return w if rank == 0 else w.replace(seed=w.seed + 1000 * rank)


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value (every rank takes part; NCCL on GPUs, gloo on CPU)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def profiled_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    when the kernel's source has changed since the counters were taken."""
    import hashlib
    import re
    if kernel != "attn":
        return None
    src = os.path.join(ROOT, "fp4_kv_cache_step_b200", "csrc", "attn_tc.cu")
    prof = os.path.join(ROOT, "profiles", "decode_128k_step_kernels.md")
    try:
        text = open(prof).read()
        sha = hashlib.sha1(open(src, "rb").read()).hexdigest()
        m_sha = re.search(r"attn_tc\.cu sha1 at capture: ([0-9a-f]{40})", text)
        m_b = re.search(r"= ([0-9,]+) bytes", text)
        if m_sha and m_b and m_sha.group(1) == sha:
            return int(m_b.group(1).replace(",", ""))
    except OSError:
        pass
    return None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# --------------------------------------------------------------- algorithmic bytes
def algorithmic_bytes(w, nvalid: np.ndarray, topk: np.ndarray) -> dict:
    """Bytes each kernel must move at least, from the realised lengths and the
    selected indices (distinct 64-entry scale blocks per sequence)."""
    rows = w.B * w.Tq
    nv = nvalid.reshape(-1).astype(np.int64)
    tk = topk.reshape(rows, w.K)
    sel = (tk >= 0).sum(axis=1).astype(np.int64)
    blocks = np.array([np.unique(r[r >= 0] // 64).size for r in tk], np.int64)
    idx_k = int(nv.sum()) * w.Di
    idx_qw = rows * (w.Hi * w.Di + 4 * w.Hi)
    scores = int(nv.sum()) * 4
    kv_rows = int(sel.sum()) * (w.D // 2)
    scale_rows = int(blocks.sum()) * w.D
    q_out = 2 * rows * w.Hq * w.D * 2
    idx = rows * w.K * 4
    return {
        "score": idx_k + idx_qw + scores,
        "topk": scores + idx,
        "attn": kv_rows + scale_rows + q_out + idx,
        # the 16-channel layout: codes and their own scales in one row per entry
        "attn_g16": int(sel.sum()) * (w.D // 2 + w.D // 16) + q_out + idx,
        "step": idx_k + idx_qw + kv_rows + scale_rows + q_out,
        "flops_score": int(nv.sum()) * w.Hi * w.Di * 2,
        "flops_attn": int(sel.sum()) * w.Hq * w.D * 4,
    }


# --------------------------------------------------------------- clocks
class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons through NVML
    from a background thread while the timed region runs."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.dev, self.period = device_index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None

    def _loop(self, handle, nv):
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(handle) \
                    if hasattr(nv, "nvmlDeviceGetCurrentClocksEventReasons") \
                    else nv.nvmlDeviceGetCurrentClocksThrottleReasons(handle)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            cuda_vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = self.dev
            if cuda_vis:
                ids = [x for x in cuda_vis.split(",") if x.strip()]
                if self.dev < len(ids) and ids[self.dev].strip().isdigit():
                    idx = int(ids[self.dev])
            handle = nv.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._loop, args=(handle, nv), daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"],
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    from fp4_kv_cache_step_b200 import build as libbuild
    from fp4_kv_cache_step_b200 import csa2
    from fp4_kv_cache_step_b200 import workloads as wl
    from fp4_kv_cache_step_b200.runner import DeviceWorkload

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    if rank == 0:
        libbuild.build()
    if world > 1:
        dist.barrier()
    csa2.load()

    w = rank_workload(wl.WORKLOADS[args.workload], rank)
    dw = DeviceWorkload(w, dev)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush_rd = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)

    def flush_l2(i):
        # write 256 MiB (evicts every line of the step's data), then read another
        # 256 MiB so that the dirty flush lines are written back here, outside
        # the timed events, not by the next step's first kernel
        flush.fill_(i & 0xff)
        flush_rd.max()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- warm-up
    for _ in range(args.warmup):
        dw.step()
    csa2.check_device_errors()

    # ---- timed steps (device events on the launching stream)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier()
    with ClockSampler(dev.index) as clk:
        for i in range(args.steps):
            flush_l2(i)
            ev[i][0].record(stream)
            dw.step()
            ev[i][1].record(stream)
        barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    csa2.check_device_errors()
    max_total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = max_total_ms / args.steps
    value = world * args.steps / (max_total_ms / 1e3)

    # ---- per-kernel timing: the same kernels through the individual calls
    nsplit_ws = csa2.load().csa2_sparse_attn_workspace_bytes(w.B, w.Tq, w.Hq, w.D, w.K)
    kern = {"score": [], "topk": [], "attn": [], "block_pool": []}
    # the hierarchical indexer's blockwise pool (2048 blocks of 8), as a FULL
    # decoder layer emits it right after its top-K, from the same scores
    pool_out = torch.empty((w.B, w.Tq, 2048 * 8), dtype=torch.int32, device=dev)
    pool_ws = torch.empty(max(int(csa2.load().csa2_block_pool_workspace_bytes(
        w.B, w.Tq, w.N, 8, 2048)), 256), dtype=torch.uint8, device=dev)
    scores = torch.empty((w.B, w.Tq, w.N), dtype=torch.float32, device=dev)
    ws = torch.empty(max(int(nsplit_ws), 256), dtype=torch.uint8, device=dev)
    out = torch.empty_like(dw.out[0])
    lse = torch.empty_like(dw.lse[0])
    for i in range(args.warmup + args.steps):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        flush_l2(i)
        evs[0].record(stream)
        csa2.csa2_index_score(dw.idx_q[0], dw.idx_w[0], dw.idx_k, nvalid=dw.nvalid, out=scores)
        evs[1].record(stream)
        csa2.csa2_topk(scores, w.K, nvalid=dw.nvalid, out=dw.topk)
        evs[2].record(stream)
        e_pool = torch.cuda.Event(enable_timing=True)
        csa2.csa2_block_pool(scores, dw.nvalid, 2048, 8, out=pool_out, workspace=pool_ws)
        e_pool.record(stream)
        flush_l2(i)
        evs[3].record(stream)
        csa2.csa2_sparse_attn(dw.q[0], dw.kv_packed, dw.kv_scale, dw.topk, w.softmax_scale,
                              out=out, lse=lse, workspace=ws)
        e4 = torch.cuda.Event(enable_timing=True)
        e4.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            kern["score"].append(evs[0].elapsed_time(evs[1]))
            kern["topk"].append(evs[1].elapsed_time(evs[2]))
            kern["attn"].append(evs[3].elapsed_time(e4))
            kern["block_pool"].append(evs[2].elapsed_time(e_pool))
    kern_us = {k: 1e3 * statistics.mean(v) for k, v in kern.items()}

    nvalid = wl.nvalid(w)
    ab = algorithmic_bytes(w, nvalid, dw.topk.cpu().numpy())
    hbm_peak, tf_peak, peak_kind = measured_peaks()
    dom = max(("score", "attn", "topk"), key=lambda k: kern_us[k])
    if dom == "attn" and args.attn_bound == "tensor":
        achieved = ab["flops_attn"] / (kern_us["attn"] * 1e-6) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tf_peak, "unit": "TFLOP/s",
                "frac": achieved / tf_peak}
    else:
        achieved = ab[dom] / (kern_us[dom] * 1e-6) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak}
    traffic = args.traffic if args.traffic is not None else profiled_traffic(dom)
    roof.update({"kernel": dom, "peak_source": peak_kind + " (MEASURED_PEAKS.json)"
                 if peak_kind == "measured" else "fallback", "traffic": traffic})

    # ---- end to end through the C ABI with pinned host buffers
    g16 = g16_attention(args, w, dw, csa2, torch, flush_l2, stream, ws, ab, hbm_peak)

    e2e = run_e2e(args, w, dw, flush, csa2, torch)

    step_gbs = ab["step"] / (ms_per_step * 1e-3) / 1e9
    launches_per_step = 3 + (1 if nsplit_ws > 0 else 0)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Tq": w.Tq, "N": w.N, "D": w.D, "Hq": w.Hq,
                   "Hi": w.Hi, "Di": w.Di, "K": w.K, "context_tokens": 4 * w.N,
                   "kv_format": "E2M1 + E4M3 scale per channel per 64 entries",
                   "arith": "indexer e4m3 x e4m3 -> f32; attention f16 x f16 -> f32; out bf16",
                   "l2": "flushed between timed steps (256 MiB write, then a 256 MiB read so the "
                         "flush's dirty lines are written back outside the timed events)",
                   "parallelism": "dp%d (independent batches per GPU)" % world},
        "step_algorithmic_bytes": ab["step"],
        "step_gbs": step_gbs, "step_frac_of_8tbs": step_gbs / NOMINAL_HBM_GBS,
        "step_frac_of_measured_hbm": step_gbs / hbm_peak,
        "query_tokens_per_s": value * w.B * w.Tq,
        "kernel_us": kern_us,
        "roofline": roof,
        "attn_kv_g16": g16,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_sample_rows)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def g16_attention(args, w, dw, csa2, torch, flush_l2, stream, ws, ab, hbm_peak):
    """The attention kernel over the pages' own FP4 layout (one E4M3 scale per
    16 channels of an entry, 288-byte rows): the step's cache dequantised and
    re-quantised into that layout, the same queries and top-K, timed like the
    per-kernel times (L2 flushed before each call, device events)."""
    kv = csa2.fp4_kv_unpack(dw.kv_packed, dw.kv_scale)
    rows = csa2.fp4_kv_pack_g16(kv)
    del kv
    out = torch.empty_like(dw.out[0])
    lse = torch.empty_like(dw.lse[0])
    times = []
    for i in range(args.warmup + args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush_l2(i)
        e0.record(stream)
        csa2.csa2_sparse_attn_g16(dw.q[0], rows, dw.topk, w.softmax_scale, out=out, lse=lse,
                                  workspace=ws)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    csa2.check_device_errors()
    us = 1e3 * statistics.mean(times)
    gbs = ab["attn_g16"] / (us * 1e-6) / 1e9
    return {"layout": "E2M1 + E4M3 scale per 16 channels of an entry (288 B rows)",
            "attn_us": us, "algorithmic_bytes": ab["attn_g16"], "gbs": gbs,
            "frac_of_measured_hbm": gbs / hbm_peak,
            "cache": "the step's block-scaled cache dequantised and re-quantised per 16 channels"}


def run_e2e(args, w, dw, flush, csa2, torch):
    """The metric through the public call, end to end: every step copies its
    query-side inputs (queries, indexer queries and weights, lengths) from pinned
    host memory, runs csa2_layer_step, and copies the attention output and lse
    back to pinned host memory. The FP4 cache and the indexer keys stay resident
    (they are the cache). Steps are issued round-robin on three streams with their
    own buffers and their own copy of the cache, as a serving loop over several
    sequences' caches would, so one step's copies overlap another's kernels; the
    value is steps / elapsed device time from the first timed step's start to the
    last one's end."""
    from fp4_kv_cache_step_b200 import workloads as wl
    nslot = 3
    dev = dw.idx_k.device
    host_in = {
        "q": torch.from_numpy(wl.q(w, 0).view(np.int16)).view(torch.bfloat16).pin_memory(),
        "idx_q": torch.from_numpy(wl.idx_q(w, 0)).pin_memory(),
        "idx_w": torch.from_numpy(wl.idx_w(w, 0)).pin_memory(),
        "nvalid": torch.from_numpy(wl.nvalid(w)).pin_memory(),
    }
    slots = []
    for si in range(nslot):
        d = {k: torch.empty_like(t, device=dev) for k, t in host_in.items()}
        # each slot attends over its own copy of the cache, so consecutive steps
        # stream different 100 MB key sets and L2 cannot carry one into the next
        kvp = dw.kv_packed if si == 0 else dw.kv_packed.clone()
        kvs = dw.kv_scale if si == 0 else dw.kv_scale.clone()
        ik = dw.idx_k if si == 0 else dw.idx_k.clone()
        d["topk"] = torch.full_like(dw.topk, -1)
        d["out"] = torch.empty_like(dw.out[0])
        d["lse"] = torch.empty_like(dw.lse[0])
        d["host_out"] = torch.empty(d["out"].shape, dtype=torch.bfloat16).pin_memory()
        d["host_lse"] = torch.empty(d["lse"].shape, dtype=torch.float32).pin_memory()
        d["shared"] = csa2.Csa2Shared(kvp, kvs, ik, d["topk"], None)
        d["args"] = csa2.layer_args(d["q"], d["nvalid"], d["out"], w.K, w.softmax_scale,
                                    idx_q=d["idx_q"], idx_w=d["idx_w"], lse=d["lse"], N=w.N)
        need = csa2.layer_step_workspace_bytes(wl.FULL, d["args"], d["shared"])
        d["ws"] = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        d["stream"] = torch.cuda.Stream(device=dev)
        slots.append(d)
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = slots[0]["host_out"].numel() * 2 + slots[0]["host_lse"].numel() * 4

    def one_step(d):
        with torch.cuda.stream(d["stream"]):
            for k, t in host_in.items():
                d[k].copy_(t, non_blocking=True)
            csa2.csa2_layer_step(wl.FULL, d["args"], d["shared"], d["ws"])
            d["host_out"].copy_(d["out"], non_blocking=True)
            d["host_lse"].copy_(d["lse"], non_blocking=True)

    for i in range(args.warmup):
        one_step(slots[i % nslot])
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    start.record(torch.cuda.current_stream())
    for d in slots:
        d["stream"].wait_event(start)
    for i in range(args.steps):
        one_step(slots[i % nslot])
    ends = []
    for d in slots:
        e = torch.cuda.Event(enable_timing=True)
        e.record(d["stream"])
        ends.append(e)
    torch.cuda.synchronize()
    ms = max(start.elapsed_time(e) for e in ends) / args.steps
    return {"value": 1e3 / ms, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "streams": nslot,
            "l2": "not flushed: the three slots' caches (3 x 410 MB) are read in turn, so "
                  "no step finds the previous step's keys in L2"}


# --------------------------------------------------------------- CPU oracle
def oracle_layer_steps(w, rows):
    """Time the oracle's FULL layer step on the given batch rows (cache build
    excluded). Returns seconds."""
    import oracle
    from fp4_kv_cache_step_b200 import workloads as wl
    nv_all = wl.nvalid(w)
    total = 0.0
    for b in rows:
        packed, sc = oracle.fp4_kv_pack(wl.kv(w, rows=[b]))
        ik = wl.idx_k(w, rows=[b])
        q = wl.q(w, 0, rows=[b])
        iq = wl.idx_q(w, 0, rows=[b])
        iw = wl.idx_w(w, 0, rows=[b])
        topk = np.full((1, w.Tq, w.K), -1, np.int32)
        t0 = time.perf_counter()
        oracle.layer_step(oracle.MODE_FULL, q, iq, iw, ik, packed, sc, nv_all[b:b + 1], w.K,
                          w.softmax_scale, topk)
        total += time.perf_counter() - t0
    return total


def cpu_baseline(w, nrows):
    import oracle
    oracle.build()
    rows = list(range(min(nrows, w.B)))
    secs = oracle_layer_steps(w, rows)
    per_step = secs * w.B / len(rows)
    return {"value": 1.0 / per_step, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": "%d of %d sequences of one FULL layer step (score + top-K + attention, "
                      "cache build excluded), single-threaded fp64; scaled to a %d-sequence "
                      "layer step" % (len(rows), w.B, w.B)}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    sys.path.insert(0, ROOT)
    from fp4_kv_cache_step_b200 import workloads as wl
    import oracle
    oracle.build()
    w = wl.WORKLOADS[args.workload]
    for i in range(args.warmup):
        oracle_layer_steps(w, [i % w.B])
    secs = [oracle_layer_steps(w, [i % w.B]) for i in range(args.steps)]
    per_step = statistics.mean(secs) * w.B
    value = 1.0 / per_step
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "Tq": w.Tq, "N": w.N, "D": w.D, "Hq": w.Hq,
                       "Hi": w.Hi, "Di": w.Di, "K": w.K, "context_tokens": 4 * w.N,
                       "parallelism": "none (CPU oracle, rank 0)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": "each step: one sequence of the %d-sequence FULL layer "
                                       "step, scaled by %d; single-threaded fp64" % (w.B, w.B)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_stack(args):
    """One decode step of the model's own CSA2 layers (workloads.production_stack:
    three encoder groups [FULL + 5 REUSE] over caches of T/2 entries, the
    decoder's [FULL + 3 REUSE] + 4 x [REINDEX + 3 REUSE] over a cache of T
    entries with the blockwise pool; top-512, indexer 32 x 128), timed with
    device events over whole steps, L2 flushed between steps. One GPU."""
    import torch

    from fp4_kv_cache_step_b200 import csa2
    from fp4_kv_cache_step_b200 import workloads as wl
    from fp4_kv_cache_step_b200.runner import DeviceStack

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    csa2.load()
    st = wl.production_stack(args.context, args.batch)
    ds = DeviceStack(st, dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush_rd = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)
    for _ in range(args.warmup):
        ds.step()
    torch.cuda.synchronize()
    csa2.check_device_errors()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(dev.index) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xff)
            flush_rd.max()
            ev[i][0].record(stream)
            ds.step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    csa2.check_device_errors()
    ms = [a.elapsed_time(b) for a, b in ev]
    ms_per_step = sum(ms) / len(ms)
    nlayers = len(st.layers)
    modes = [st.segments[s].modes[l] for s, l in st.layers]
    launches = sum({"FULL": 3, "REINDEX": 3, "REUSE": 1}[m] for m in modes)
    launches += 3                                      # the decoder FULL's blockwise pool
    print(json.dumps({
        "metric": "CSA2 stack decode steps/s (the model's 38 CSA2 layers)",
        "value": 1e3 / ms_per_step, "unit": "stack-steps/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "production_stack", "context_tokens": args.context,
                   "B": args.batch, "csa2_layers": nlayers, "swa_only_layers": st.swa_only,
                   "encoder_entries": args.context // 2, "decoder_entries": args.context,
                   "K": wl.PROD_K, "Hi": wl.PROD_HI, "Di": wl.PROD_DI, "Hq": wl.PROD_HQ,
                   "pool": "%d blocks of %d" % (wl.PROD_POOL_BLOCKS, wl.PROD_POOL_BLOCK),
                   "modes": {m: modes.count(m) for m in ("FULL", "REINDEX", "REUSE")},
                   "l2": "flushed between timed steps"},
        "per_layer_us": 1e3 * ms_per_step / nlayers,
        "query_tokens_per_s": args.batch * 1e3 / ms_per_step,
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="workload name (fp4_kv_cache_step_b200.workloads.WORKLOADS)")
    ap.add_argument("--cpu-sample-rows", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--attn-bound", default="tensor", choices=["tensor", "hbm"])
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per launch of the dominant kernel, if captured")
    ap.add_argument("--stack", default=None, choices=["production"],
                    help="time the model's 38 CSA2 layers (one GPU) instead of the headline step")
    ap.add_argument("--context", type=int, default=131072, help="--stack: context in tokens")
    ap.add_argument("--batch", type=int, default=4, help="--stack: sequences")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.stack is not None and args.impl == "ours":
        run_stack(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
