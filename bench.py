#!/usr/bin/env python
"""Benchmark of the CSA2 layer step over an FP4 main KV cache.

Default workload "decode_128k_full": batch 32, one query token each, N = 32768
FP4 main-KV entries of dim 512 (128K tokens at 4:1 compression), 64 bf16 query
heads, indexer 64 heads x 128 with integer E4M3 values, top-2048, lengths
uniform in [16384, 32768]. One step = one pass of the whole hot path over the
batch: indexer scores -> top-K -> gather + FP4 dequant + sparse attention. The
FP4 cache is built once before timing (a cache is built when tokens arrive, not
per step). Inputs are resident in HBM; L2 is flushed between timed steps (a
256 MiB write, then a 256 MiB read so the flush's dirty lines are written back
there), outside the timed events.

The other workloads (--workload NAME, see fp4_kv_cache_step_b200.workloads)
print their own line: the tiny decode, the 4-layer FULL/REINDEX/REUSE/REUSE
stack (per layer and per stack), the 1M-token hierarchical pair (FULL emitting
a top-8192 pool, REINDEX inside it) and the 4096-query prefill chunk (whose
indexer is reported against the FP8 tensor peak). --stack production times the
model's own 38 CSA2 layers.

Prints one JSON line. With --impl reference it times the CPU oracle on the same
workload instead (the oracle is the only other implementation: the pages print
no code).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import json
import math
import os
import platform
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
FP8_OVER_BF16 = 2.0           # nominal dense ratio (4.5 / 2.25 PFLOP/s)
DTYPE = "e4m3 x e4m3 and f16 x f16 tensor-core products, f32 accumulation (FP4/E4M3 storage, bf16 out)"
CSRC = os.path.join(ROOT, "fp4_kv_cache_step_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "kernel_traffic.json")

# the sources each timed kernel is built from (its captured counters hold while they are unchanged)
KERNEL_SOURCES = {
    "score": ("score_tc.cu", "sm100.cuh", "common.cuh"),
    "topk": ("topk.cu", "common.cuh"),
    "attn": ("attn_tc.cu", "attn.cu", "sm100.cuh", "common.cuh"),
    "block_pool": ("pool.cu", "topk.cu", "common.cuh"),
}
# the kernels' names as ncu lists them (regular expressions)
KERNEL_NAMES = {
    "score": r"index_score",
    "topk": r"topk_reg_kernel<\d+, \d+, [01], 0>|topk_cluster_kernel|topk_kernel<",
    "attn": r"sparse_attn_tc_kernel",
    "block_pool": r"topk_reg_kernel<\d+, \d+, [01], 8>|block_(max|expand)_kernel",
}


def workload_metric(w):
    """(metric, unit) of a workload's line: one 'step' is one pass of its whole
    mode schedule over its batch."""
    if w.name in ("decode_128k_full",):
        return METRIC, UNIT
    if w.name == "tiny_decode_full":
        return "CSA2 decode layer-steps/s, tiny decode (B=1, N=4096)", UNIT
    if w.name == "stack_full_reindex_reuse_reuse":
        return "CSA2 4-layer stack steps/s (FULL, REINDEX, REUSE, REUSE; B=16, N=16384)", \
            "stack-steps/s"
    if w.name == "hier_1m_full_pool_reindex":
        return "CSA2 hierarchical steps/s at 1M tokens (FULL + top-8192 pool, REINDEX in pool)", \
            "hier-steps/s"
    if w.name == "prefill_chunk_4096_full":
        return "CSA2 prefill-chunk layer-steps/s (4096 queries over 65536 entries)", UNIT
    return "CSA2 %s steps/s" % w.name, "steps/s"


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


def sources_sha1(kernel: str) -> str:
    h = hashlib.sha1()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(kernel: str, workload: str, units: float):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    record (profiles/kernel_traffic.json), or (None, why) when there is no
    capture of the kernel's current sources. A capture on a smaller case of the
    same kernel is scaled by the units processed (valid keys for the scorer,
    selected entries for the attention)."""
    try:
        with open(TRAFFIC_FILE) as f:
            recs = json.load(f)["captures"]
    except (OSError, ValueError, KeyError):
        return None, "no ncu record"
    sha = sources_sha1(kernel)
    best = None
    for r in recs:
        if r.get("kernel") != kernel or r.get("sources_sha1") != sha:
            continue
        if r.get("workload") == workload:
            return float(r["dram_bytes_per_launch"]), "ncu capture of this workload"
        if best is None and r.get("units"):
            best = r                     # the first capture that can be scaled
    if best is not None:
        return float(best["dram_bytes_per_launch"]) * units / float(best["units"]), \
            "ncu capture of %s scaled by units (%s)" % (best["workload"], best.get("unit_kind"))
    if any(r.get("kernel") == kernel and r.get("sources_sha1") == sha for r in recs):
        return None, ("no ncu capture of this workload (the kernel's other captures carry "
                      "no unit count to scale by)")
    return None, "sources changed since the last ncu capture"


_NCU_SCALE = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "nsecond": 1e-3,
              "usecond": 1.0, "msecond": 1e3, "second": 1e6, "ns": 1e-3, "us": 1.0,
              "ms": 1e3, "s": 1e6, "KB": 1e3, "MB": 1e6, "GB": 1e9, "B": 1.0}


def record_ncu(csv_path: str, kernel: str, workload: str, command: str, units=None,
               unit_kind=None, out_path: str = TRAFFIC_FILE) -> dict:
    """Turn one ncu capture (--csv with dram__bytes_read.sum, dram__bytes_write.sum
    and gpu__time_duration.sum) into the per-launch record that the roofline's
    `traffic` reads: the launches of `kernel` in the file, their mean DRAM bytes
    and duration, the sha1 of the kernel's sources now, the workload and the
    command that made the capture. Replaces the record of the same kernel and
    workload in `out_path`."""
    import csv
    import re
    pat = re.compile(KERNEL_NAMES[kernel])
    per = {}
    with open(csv_path, newline="") as f:
        lines = [l for l in f if l.startswith('"')]       # ncu's own log lines are not CSV
    for row in csv.DictReader(lines):
        if not pat.search(row.get("Kernel Name", "")):
            continue
        name = row["Metric Name"]
        if name not in ("dram__bytes_read.sum", "dram__bytes_write.sum", "gpu__time_duration.sum"):
            continue
        v = float(row["Metric Value"].replace(",", "")) * _NCU_SCALE.get(row["Metric Unit"], 1.0)
        per.setdefault(row["ID"], {})[name] = v
    launches = [m for m in per.values() if len(m) == 3]
    if not launches:
        raise SystemExit("no complete %s launch in %s" % (kernel, csv_path))
    n = len(launches)
    rec = {"kernel": kernel, "sources_sha1": sources_sha1(kernel), "workload": workload,
           "launches": n,
           "dram_read_bytes_per_launch": sum(m["dram__bytes_read.sum"] for m in launches) / n,
           "dram_write_bytes_per_launch": sum(m["dram__bytes_write.sum"] for m in launches) / n,
           "duration_us_under_ncu": sum(m["gpu__time_duration.sum"] for m in launches) / n,
           "command": command}
    rec["dram_bytes_per_launch"] = rec["dram_read_bytes_per_launch"] + \
        rec["dram_write_bytes_per_launch"]
    if units is not None:
        rec["units"], rec["unit_kind"] = float(units), unit_kind
    try:
        with open(out_path) as f:
            doc = json.load(f)
    except (OSError, ValueError):
        doc = {}
    doc.setdefault("about", "DRAM bytes per launch of each timed kernel from ncu (cold "
                            "caches, serialised launches), with the sha1 of the kernel's sources "
                            "when captured; written by bench.py --record-ncu")
    caps = [r for r in doc.get("captures", [])
            if not (r.get("kernel") == kernel and r.get("workload") == workload)]
    doc["captures"] = caps + [rec]
    with open(out_path, "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")
    return rec


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured (MEASURED_PEAKS.json)"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def fp8_matmul_peak_live(dev, n: int = 8192, reps: int = 10) -> float:
    """Dense E4M3 GEMM throughput of torch._scaled_mm (cuBLASLt) on this GPU,
    best of `reps`, TFLOP/s: context for the FP8 roofline of the prefill indexer."""
    import torch
    a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device=dev, dtype=torch.float32)
    for _ in range(3):
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


# --------------------------------------------------------------- algorithmic bytes
def layer_accounting(w, mode: str, nvalid: np.ndarray, topk: np.ndarray, cand=None,
                     pooled: bool = False, emit_pool: bool = False) -> dict:
    """Bytes (and flops) each kernel of one layer must move at least, from the
    realised lengths and selections: the scorer reads every visible key (or the
    pool's keys) and the indexer query, and writes one score per key; the top-K
    reads the scores and writes K ids; the attention reads the selected packed
    rows, each distinct 64-entry scale row once, the queries and the ids, and
    writes the outputs. 'metric' is what the step must bring from HBM: keys,
    indexer queries, selected rows, scale rows, queries and outputs (scores and
    ids are intermediates)."""
    rows = w.B * w.Tq
    tk = topk.reshape(rows, w.K)
    sel = int((tk >= 0).sum())
    blocks = int(sum(np.unique(r[r >= 0] // 64).size for r in tk))
    q_out = 2 * rows * w.Hq * w.D * 2
    idx = rows * w.K * 4
    attn = sel * (w.D // 2) + blocks * w.D + q_out + idx
    acc = {"attn": attn, "attn_flops": sel * w.Hq * w.D * 4, "selected": sel,
           "scale_blocks": blocks, "score": 0, "score_flops": 0, "topk": 0, "keys": 0,
           "metric": sel * (w.D // 2) + blocks * w.D + q_out}
    if mode == "REUSE":
        return acc
    idx_qw = rows * (w.Hi * w.Di + 4 * w.Hi)
    if pooled:
        c = cand.reshape(rows, -1)
        keys = int((c >= 0).sum())
        acc["score"] = keys * (w.Di + 4) + c.size * 4 + idx_qw
        acc["topk"] = keys * 4 + c.size * 4 + idx
    else:
        nv = np.minimum(nvalid.reshape(w.B, w.Tq).astype(np.int64), w.N)
        keys = int(nv.sum())                       # (query, visible entry) pairs scored
        # every query of a sequence scores the same keys: each is read once
        uniq = int(nv.max(axis=1).sum())
        acc["score"] = uniq * w.Di + keys * 4 + idx_qw
        acc["topk"] = keys * 4 + idx + (rows * w.C * 4 if emit_pool else 0)
        acc["metric"] += uniq * w.Di + idx_qw
        acc["keys"] = keys
        acc["score_flops"] = keys * w.Hi * w.Di * 2
        return acc
    acc["keys"] = keys
    acc["score_flops"] = keys * w.Hi * w.Di * 2
    acc["metric"] += keys * w.Di + idx_qw
    return acc


def roofline(kernel: str, acc: dict, us: float, peaks: dict, fp8_peak: float) -> dict:
    """The kernel against whichever roofline bounds it: HBM bytes at the measured
    copy rate, or tensor-core flops at the measured peak of its dtype (the
    scorer is E4M3: the bf16 peak times the nominal FP8/bf16 ratio; attention is
    f16, at the bf16 peak)."""
    byts = acc[kernel]
    flops = acc.get(kernel + "_flops", 0)
    t_hbm = byts / (peaks["hbm_gbs"] * 1e9)
    tpeak = fp8_peak if kernel == "score" else peaks["bf16_tflops"]
    t_tc = flops / (tpeak * 1e12) if flops else 0.0
    if t_tc > t_hbm:
        ach = flops / (us * 1e-6) / 1e12
        r = {"bound": "tensor", "achieved": ach, "peak": tpeak, "unit": "TFLOP/s",
             "frac": ach / tpeak}
    else:
        ach = byts / (us * 1e-6) / 1e9
        r = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": ach / peaks["hbm_gbs"]}
    r.update({"kernel": kernel, "us": us, "algorithmic_bytes": byts, "flops": flops,
              "hbm_frac": byts / (us * 1e-6) / 1e9 / peaks["hbm_gbs"]})
    return r


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
class L2Flush:
    """Writes 256 MiB (evicting every line of the step's data), then reads
    another 256 MiB so that the dirty flush lines are written back here,
    outside the timed events, not by the next step's first kernel. Then the
    GPU spins for about 300 us, so that the host has queued everything the
    timed region launches before its first event fires (the events then see
    device time only, no gap while the host is still launching)."""

    def __init__(self, torch, dev):
        self.torch = torch
        self.w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)

    def __call__(self, i: int):
        self.w.fill_(i & 0xff)
        self.r.max()
        self.torch.cuda._sleep(600000)


def _mode_flags(w, mode):
    pooled = mode == "REINDEX" and w.C > 0
    emit = mode == "FULL" and w.C > 0
    return pooled, emit


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
    metric, unit = workload_metric(w)
    dw = DeviceWorkload(w, dev)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    flush_l2 = L2Flush(torch, dev)

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

    # ---- per layer (events between the layers of a step; L2 flushed between steps only,
    # so a REINDEX layer may find the FULL layer's keys in L2, as it would in the model)
    nl = len(w.modes)
    layer_ms = [[] for _ in range(nl)]
    for i in range(args.warmup + args.steps):
        flush_l2(i)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(nl + 1)]
        evs[0].record(stream)
        for l in range(nl):
            dw.step([l])
            evs[l + 1].record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            for l in range(nl):
                layer_ms[l].append(evs[l].elapsed_time(evs[l + 1]))
    # the selections each layer used (for the byte counts)
    dw.step(snapshot_topk=True)
    torch.cuda.synchronize()
    csa2.check_device_errors()
    nvalid = wl.nvalid(w)
    cand_host = dw.cand.cpu().numpy() if dw.cand is not None else None
    accs = []
    for l, mode in enumerate(w.modes):
        pooled, emit = _mode_flags(w, mode)
        accs.append(layer_accounting(w, mode, nvalid, dw.topk_per_layer[l].cpu().numpy(),
                                     cand_host, pooled=pooled, emit_pool=emit))
    step_bytes = sum(a["metric"] for a in accs)

    # ---- per kernel: the first layer's kernels through the individual calls, L2
    # flushed before each (the scorer and the top-K run back to back, as in a step)
    peaks = measured_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    kern_us = per_kernel_times(args, w, dw, csa2, torch, flush_l2, stream)
    acc0 = accs[0]
    rl = {k: roofline(k, acc0, kern_us[k], peaks, fp8_peak)
          for k in ("score", "topk", "attn") if k in kern_us and acc0[k] > 0}
    dom = max(rl, key=lambda k: kern_us[k])
    roof = dict(rl[dom])
    units = acc0["selected"] if dom == "attn" else acc0["keys"]
    traffic, traffic_note = profiled_traffic(dom, w.name, units)
    roof.update({"peak_source": peaks["source"] + (" x %.0f (nominal FP8/bf16)" % FP8_OVER_BF16
                                                  if roof["bound"] == "tensor" and dom == "score"
                                                  else ""),
                 "traffic": traffic, "traffic_source": traffic_note})

    line = {
        "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": DTYPE, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Tq": w.Tq, "N": w.N, "D": w.D, "Hq": w.Hq,
                   "Hi": w.Hi, "Di": w.Di, "K": w.K, "C": w.C, "modes": list(w.modes),
                   "context_tokens": 4 * w.N,
                   "kv_format": "E2M1 + E4M3 scale per channel per 64 entries",
                   "l2": "flushed between timed steps (256 MiB write, then a 256 MiB read so the "
                         "flush's dirty lines are written back outside the timed events)",
                   "parallelism": "dp%d (independent batches per GPU)" % world},
        "step_algorithmic_bytes": step_bytes,
        "step_gbs": step_bytes / (ms_per_step * 1e-3) / 1e9,
    }
    line["step_frac_of_8tbs"] = line["step_gbs"] / NOMINAL_HBM_GBS
    line["step_frac_of_measured_hbm"] = line["step_gbs"] / peaks["hbm_gbs"]
    line["query_tokens_per_s"] = value * w.B * w.Tq
    line["per_layer"] = [{"mode": m, "us": 1e3 * statistics.mean(layer_ms[l]),
                          "algorithmic_bytes": accs[l]["metric"],
                          "gbs": accs[l]["metric"] / (statistics.mean(layer_ms[l]) * 1e-3) / 1e9}
                         for l, m in enumerate(w.modes)]
    line["kernel_us"] = kern_us
    line["roofline"] = roof
    line["kernel_rooflines"] = {}
    for k, v in rl.items():
        kr = {kk: v[kk] for kk in ("bound", "achieved", "unit", "frac", "hbm_frac",
                                   "algorithmic_bytes")}
        kr["traffic"], kr["traffic_source"] = profiled_traffic(
            k, w.name, acc0["selected"] if k == "attn" else acc0["keys"])
        line["kernel_rooflines"][k] = kr
    if w.name == DEFAULT_WORKLOAD:
        line["attn_kv_g16"] = g16_attention(args, w, dw, csa2, torch, flush_l2, stream, acc0,
                                            peaks)
        line["attn_kv_swa"] = swa_attention(args, w, dw, csa2, wl, torch, flush_l2, stream,
                                            acc0, peaks, kern_us["attn"])
        if not args.no_prefill:
            line["prefill_indexer"] = prefill_indexer(args, dev, csa2, torch, flush_l2, stream,
                                                      peaks)
    if w.name == "prefill_chunk_4096_full":
        line["prefill_indexer"] = indexer_vs_fp8(kern_us["score"], acc0, peaks, dev)
    if not args.no_e2e:
        line["e2e"] = run_e2e(args, w, dw, csa2, torch)
    launches = sum({"FULL": 3, "REINDEX": 3, "REUSE": 1}[m] for m in w.modes)
    launches += sum(2 for m in w.modes if m == "FULL" and w.C and w.pool_block == 8)
    line["gpu_launches"] = launches * args.steps
    line["clocks"] = clk.summary()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_sample_rows)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def per_kernel_times(args, w, dw, csa2, torch, flush_l2, stream) -> dict:
    """Device time of each kernel of the workload's first layer, called one by
    one (events between them), averaged over the timed iterations."""
    mode = w.modes[0]
    dev = dw.idx_k.device
    out = torch.empty_like(dw.out[0])
    lse = torch.empty_like(dw.lse[0])
    ws_attn = csa2.load().csa2_sparse_attn_workspace_bytes(w.B, w.Tq, w.Hq, w.D, w.K)
    ws = torch.empty(max(int(ws_attn), 256), dtype=torch.uint8, device=dev)
    scores = torch.empty((w.B, w.Tq, w.N), dtype=torch.float32, device=dev) \
        if mode != "REUSE" else None
    topk = torch.empty_like(dw.topk)
    kern = {"score": [], "topk": [], "attn": []}
    if w.name == DEFAULT_WORKLOAD:
        kern["block_pool"] = []
        pool_out = torch.empty((w.B, w.Tq, 2048 * 8), dtype=torch.int32, device=dev)
        pool_ws = torch.empty(max(int(csa2.load().csa2_block_pool_workspace_bytes(
            w.B, w.Tq, w.N, 8, 2048)), 256), dtype=torch.uint8, device=dev)
    for i in range(args.warmup + args.steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        if mode != "REUSE":
            flush_l2(i)
            e[0].record(stream)
            csa2.csa2_index_score(dw.idx_q[0], dw.idx_w[0], dw.idx_k, nvalid=dw.nvalid,
                                  out=scores)
            e[1].record(stream)
            csa2.csa2_topk(scores, w.K, nvalid=dw.nvalid, out=topk)
            e[2].record(stream)
            if "block_pool" in kern:
                csa2.csa2_block_pool(scores, dw.nvalid, 2048, 8, out=pool_out, workspace=pool_ws)
                e[3].record(stream)
        else:
            topk.copy_(dw.topk)
        flush_l2(i)
        e[4].record(stream)
        csa2.csa2_sparse_attn(dw.q[0], dw.kv_packed, dw.kv_scale, topk, w.softmax_scale,
                              out=out, lse=lse, workspace=ws)
        e[5].record(stream)
        torch.cuda.synchronize()
        if i < args.warmup:
            continue
        if mode != "REUSE":
            kern["score"].append(e[0].elapsed_time(e[1]))
            kern["topk"].append(e[1].elapsed_time(e[2]))
            if "block_pool" in kern:
                kern["block_pool"].append(e[2].elapsed_time(e[3]))
        kern["attn"].append(e[4].elapsed_time(e[5]))
    csa2.check_device_errors()
    return {k: 1e3 * statistics.mean(v) for k, v in kern.items() if v}


def indexer_vs_fp8(score_us: float, acc: dict, peaks: dict, dev) -> dict:
    flops = acc["score_flops"]
    ach = flops / (score_us * 1e-6) / 1e12
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    r = {"kernel": "index_score_tc_kernel", "us": score_us, "flops": flops,
         "achieved_tflops": ach, "peak_tflops": fp8_peak,
         "peak_source": peaks["source"] + " bf16 x %.0f (nominal FP8/bf16)" % FP8_OVER_BF16,
         "frac": ach / fp8_peak,
         "flops_rule": "2 x Hi x Di per visible (query, entry) pair"}
    try:
        live = fp8_matmul_peak_live(dev)
        r["fp8_gemm_tflops_live"] = live
        r["frac_of_live_fp8_gemm"] = ach / live
        r["live_source"] = "torch._scaled_mm E4M3 8192^3 -> bf16, best of 10, this run"
    except Exception as ex:   # the live figure is context only
        r["fp8_gemm_tflops_live"] = None
        r["live_source"] = "unavailable: %s" % type(ex).__name__
    return r


def prefill_indexer(args, dev, csa2, torch, flush_l2, stream, peaks) -> dict:
    """The 4096-query prefill chunk's indexer alone (a dense E4M3 contraction of
    4096 x 65536 x 128 per head, causally masked), timed like the step kernels."""
    from fp4_kv_cache_step_b200 import workloads as wl
    w = wl.PREFILL_CHUNK
    idx_k = torch.from_numpy(wl.idx_k(w)).to(dev)
    idx_q = torch.from_numpy(wl.idx_q(w, 0)).to(dev)
    idx_w = torch.from_numpy(wl.idx_w(w, 0)).to(dev)
    nv = wl.nvalid(w)
    nvalid = torch.from_numpy(nv).to(dev)
    scores = torch.empty((w.B, w.Tq, w.N), dtype=torch.float32, device=dev)
    times = []
    for i in range(args.warmup + args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush_l2(i)
        e0.record(stream)
        csa2.csa2_index_score(idx_q, idx_w, idx_k, nvalid=nvalid, out=scores)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    csa2.check_device_errors()
    acc = {"score_flops": int(np.minimum(nv, w.N).astype(np.int64).sum()) * w.Hi * w.Di * 2}
    r = indexer_vs_fp8(1e3 * statistics.mean(times), acc, peaks, dev)
    r["workload"] = w.name
    del scores
    return r


def g16_attention(args, w, dw, csa2, torch, flush_l2, stream, acc, peaks):
    """The attention kernel over the pages' own FP4 layout (one E4M3 scale per
    16 channels of an entry, 288-byte rows): the step's cache dequantised and
    re-quantised into that layout, the same queries and top-K, timed like the
    per-kernel times (L2 flushed before each call, device events)."""
    kv = csa2.fp4_kv_unpack(dw.kv_packed, dw.kv_scale)
    rows = csa2.fp4_kv_pack_g16(kv)
    del kv
    out = torch.empty_like(dw.out[0])
    lse = torch.empty_like(dw.lse[0])
    need = csa2.load().csa2_sparse_attn_workspace_bytes(w.B, w.Tq, w.Hq, w.D, w.K)
    ws = torch.empty(max(int(need), 256), dtype=torch.uint8, device=rows.device)
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
    rows_q = w.B * w.Tq
    byts = acc["selected"] * (w.D // 2 + w.D // 16) + 2 * rows_q * w.Hq * w.D * 2 + rows_q * w.K * 4
    gbs = byts / (us * 1e-6) / 1e9
    return {"layout": "E2M1 + E4M3 scale per 16 channels of an entry (288 B rows)",
            "attn_us": us, "algorithmic_bytes": byts, "gbs": gbs,
            "frac_of_measured_hbm": gbs / peaks["hbm_gbs"],
            "cache": "the step's block-scaled cache dequantised and re-quantised per 16 channels"}


def swa_attention(args, w, dw, csa2, wl, torch, flush_l2, stream, acc, peaks, attn_us):
    """The attention kernel with the sliding-window branch: the step's queries,
    cache and top-K plus each row's full window of 128 E4M3 tokens, one
    softmax over both, timed like the per-kernel times (L2 flushed before each
    call, device events). The window adds 128 rows of 512 bytes per query row
    to the bytes read and 128 entries to each row's list."""
    swa = torch.from_numpy(wl.swa_kv(w)).to(dw.kv_packed.device)
    swa_n = torch.from_numpy(wl.swa_n(w)).to(dw.kv_packed.device)
    out = torch.empty_like(dw.out[0])
    lse = torch.empty_like(dw.lse[0])
    W = wl.SWA_WINDOW
    need = csa2.load().csa2_sparse_attn_workspace_bytes(w.B, w.Tq, w.Hq, w.D, w.K + W)
    ws = torch.empty(max(int(need), 256), dtype=torch.uint8, device=swa.device)
    times = []
    for i in range(args.warmup + args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush_l2(i)
        e0.record(stream)
        csa2.csa2_sparse_attn_swa(dw.q[0], dw.kv_packed, dw.kv_scale, dw.topk, swa, swa_n,
                                  w.softmax_scale, W=W, out=out, lse=lse, workspace=ws)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    csa2.check_device_errors()
    us = 1e3 * statistics.mean(times)
    rows_q = w.B * w.Tq
    win_tokens = int(np.minimum(wl.swa_n(w), W).sum())
    win_bytes = win_tokens * w.D
    byts = acc["attn"] + win_bytes
    flops = acc["attn_flops"] + win_tokens * w.Hq * w.D * 4
    gbs = byts / (us * 1e-6) / 1e9
    return {"window": W, "window_format": "E4M3, one 512-byte row per token, no scale",
            "combine": "one softmax over the selected rows and the window",
            "attn_us": us, "attn_us_without_window": attn_us,
            "window_tokens": win_tokens, "window_bytes": win_bytes,
            "algorithmic_bytes": byts, "flops": flops, "gbs": gbs,
            "frac_of_measured_hbm": gbs / peaks["hbm_gbs"],
            "tflops": flops / (us * 1e-6) / 1e12,
            "query_rows": rows_q}


def _pack_offsets(sizes, align=256):
    """Offsets that place byte blocks of the given sizes one after another at
    `align`-byte boundaries; returns (offsets, total bytes)."""
    offs, off = [], 0
    for n in sizes:
        offs.append(off)
        off += (n + align - 1) // align * align
    return offs, off


def _view(buf, off, dtype, shape, torch):
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    return buf[off:off + n].view(dtype).view(*shape)


def run_e2e(args, w, dw, csa2, torch):
    """The metric through the public call, end to end: every step copies its
    query-side inputs (attention queries, indexer queries and weights of every
    layer, lengths) from pinned host memory in one copy (the inputs sit at
    256-byte offsets of one pinned buffer), runs the workload's layers with
    csa2_layer_step, and copies every layer's attention output and lse back to
    pinned host memory in one copy (the layers write them into one device
    buffer). Consecutive steps go to three streams in turn (each with its own
    buffers and its own copy of the cache, so no step finds the previous step's
    data in L2), so that one step's copies overlap another's kernels, as a
    server would pipeline its requests. The FP4 cache and the indexer keys stay
    resident (they are the cache). value = steps / device time from the first
    timed step's start to the last one's end, across the streams."""
    from fp4_kv_cache_step_b200 import workloads as wl
    nslot = 3
    dev = dw.idx_k.device
    # host inputs: (name, array, torch dtype) packed into one pinned buffer
    ins = [("nvalid", wl.nvalid(w), torch.int32)]
    for l, mode in enumerate(w.modes):
        ins.append(("q%d" % l, wl.q(w, l), torch.bfloat16))
        if mode != "REUSE":
            ins.append(("idx_q%d" % l, wl.idx_q(w, l), torch.uint8))
            ins.append(("idx_w%d" % l, wl.idx_w(w, l), torch.float32))
    in_offs, h2d = _pack_offsets([a.nbytes for _, a, _ in ins])
    host_in = torch.empty(h2d, dtype=torch.uint8).pin_memory()
    for (_, a, _), off in zip(ins, in_offs):
        host_in[off:off + a.nbytes] = torch.from_numpy(np.ascontiguousarray(a).view(np.uint8)
                                                       .reshape(-1))
    # device outputs: every layer's out (bf16) and lse (f32), packed the same way
    out_shapes = []
    for l in range(len(w.modes)):
        out_shapes.append((torch.bfloat16, tuple(dw.out[l].shape)))
        out_shapes.append((torch.float32, tuple(dw.lse[l].shape)))
    out_offs, d2h = _pack_offsets([int(np.prod(sh)) * (2 if dt == torch.bfloat16 else 4)
                                   for dt, sh in out_shapes])
    slots = []
    for si in range(nslot):
        d = {"in": torch.empty(h2d, dtype=torch.uint8, device=dev),
             "outbuf": torch.empty(d2h, dtype=torch.uint8, device=dev),
             "host_out": torch.empty(d2h, dtype=torch.uint8).pin_memory()}
        t = {name: _view(d["in"], off, dt, a.shape, torch)
             for (name, a, dt), off in zip(ins, in_offs)}
        outs = [_view(d["outbuf"], off, dt, sh, torch)
                for (dt, sh), off in zip(out_shapes, out_offs)]
        kvp = dw.kv_packed if si == 0 else dw.kv_packed.clone()
        kvs = dw.kv_scale if si == 0 else dw.kv_scale.clone()
        ik = dw.idx_k if si == 0 else dw.idx_k.clone()
        d["topk"] = torch.full_like(dw.topk, -1)
        d["cand"] = torch.full_like(dw.cand, -1) if dw.cand is not None else None
        d["shared"] = csa2.Csa2Shared(kvp, kvs, ik, d["topk"], d["cand"])
        d["args"] = []
        need = 256
        for l, mode in enumerate(w.modes):
            pooled, emit = _mode_flags(w, mode)
            a = csa2.layer_args(t["q%d" % l], t["nvalid"], outs[2 * l], w.K, w.softmax_scale,
                                idx_q=t.get("idx_q%d" % l), idx_w=t.get("idx_w%d" % l),
                                lse=outs[2 * l + 1], N=w.N,
                                emit_pool=(0 if not emit else (2 if w.pool_block == 8 else 1)),
                                use_pool=pooled)
            d["args"].append(a)
            need = max(need, csa2.layer_step_workspace_bytes(mode, a, d["shared"]))
        d["ws"] = torch.empty(need, dtype=torch.uint8, device=dev)
        slots.append(d)

    def one_step(d):
        d["in"].copy_(host_in, non_blocking=True)
        for l, mode in enumerate(w.modes):
            csa2.csa2_layer_step(mode, d["args"][l], d["shared"], d["ws"])
        d["host_out"].copy_(d["outbuf"], non_blocking=True)

    base = torch.cuda.current_stream()
    streams = [torch.cuda.Stream(device=dev) for _ in range(nslot)]

    def run(n):
        for i in range(n):
            with torch.cuda.stream(streams[i % nslot]):
                one_step(slots[i % nslot])

    for st in streams:
        st.wait_stream(base)
    run(args.warmup)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(base)
    for st in streams:
        st.wait_event(start)
    run(args.steps)
    for st in streams:
        done = torch.cuda.Event()
        done.record(st)
        base.wait_event(done)
    end.record(base)
    torch.cuda.synchronize()
    csa2.check_device_errors()
    ms = start.elapsed_time(end) / args.steps
    _, unit = workload_metric(w)
    return {"value": 1e3 / ms, "unit": unit, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "streams": nslot,
            "copies_per_step": {"h2d": 1, "d2h": 1},
            "l2": "not flushed: three copies of the cache are read in turn"}


# --------------------------------------------------------------- CPU oracle
def cpu_info():
    model = platform.processor() or "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return model, os.cpu_count() or 1


def oracle_units(w, n: int):
    """Independent units of work of a workload for the oracle: (batch row, first
    query, end query). Decode workloads: whole sequences (one query each). The
    prefill chunk (one sequence of 4096 queries): single queries, n of them
    spread evenly over the chunk."""
    if w.Tq == 1:
        return [(b, 0, 1) for b in range(min(n, w.B))]
    n = max(1, min(n, w.B * w.Tq))
    step = w.B * w.Tq / n
    out = []
    for i in range(n):
        r = int(i * step)
        out.append((r // w.Tq, r % w.Tq, r % w.Tq + 1))
    return out


class OracleSequences:
    """The oracle's inputs for some units of a workload (see oracle_units; the
    FP4 cache packed by the oracle itself), prepared once; `step(units, threads)`
    runs the workload's mode schedule on them, one thread per unit (each unit is
    an independent problem; the oracle's calls release the interpreter lock)."""

    def __init__(self, w, units, threads):
        import oracle
        from fp4_kv_cache_step_b200 import workloads as wl
        oracle.build()
        self.w, self.oracle = w, oracle
        nv_all = wl.nvalid(w)
        # one small call first, on this thread (the oracle fills its E4M3 table once)
        oracle.fp4_kv_pack(np.zeros((1, 64, 64), np.float32))
        oracle.index_score(np.zeros((1, 1, 1, 16), np.uint8), np.ones((1, 1, 1), np.float32),
                           np.zeros((1, 64, 16), np.uint8), nvalid=np.full((1, 1), 64, np.int32))
        cache = {}

        def seq(b):
            if b not in cache:
                packed, sc = oracle.fp4_kv_pack(wl.kv(w, rows=[b]))
                cache[b] = (packed, sc, wl.idx_k(w, rows=[b]),
                            [(mode, wl.q(w, l, rows=[b]),
                              wl.idx_q(w, l, rows=[b]) if mode != "REUSE" else None,
                              wl.idx_w(w, l, rows=[b]) if mode != "REUSE" else None)
                             for l, mode in enumerate(w.modes)])
            return cache[b]

        with cf.ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(seq, sorted({u[0] for u in units})))

        def part(a, t0, t1):
            return None if a is None else np.ascontiguousarray(a[:, t0:t1])
        self.data = {}
        for (b, t0, t1) in units:
            packed, sc, ik, layers = cache[b]
            self.data[(b, t0, t1)] = {
                "packed": packed, "scale": sc, "idx_k": ik,
                "nvalid": np.ascontiguousarray(nv_all[b:b + 1, t0:t1]),
                "layers": [(m, part(q, t0, t1), part(iq, t0, t1), part(iw, t0, t1))
                           for m, q, iq, iw in layers]}

    def _one(self, u):
        o, w, d = self.oracle, self.w, self.data[u]
        tq = u[2] - u[1]
        topk = np.full((1, tq, w.K), -1, np.int32)
        cand = np.full((1, tq, w.C), -1, np.int32) if w.C else None
        modes = {"FULL": o.MODE_FULL, "REINDEX": o.MODE_REINDEX, "REUSE": o.MODE_REUSE}
        for mode, q, iq, iw in d["layers"]:
            pooled, _ = _mode_flags(w, mode)
            o.layer_step(modes[mode], q, iq, iw, d["idx_k"], d["packed"], d["scale"],
                         d["nvalid"], w.K, w.softmax_scale, topk, cand, w.C, use_pool=pooled)

    def step(self, units, threads) -> float:
        """Seconds for the given units, `threads` at a time."""
        t0 = time.perf_counter()
        if threads <= 1:
            for u in units:
                self._one(u)
        else:
            with cf.ThreadPoolExecutor(max_workers=threads) as ex:
                list(ex.map(self._one, units))
        return time.perf_counter() - t0


def cpu_baseline(w, nrows):
    """The oracle on the host cores: one thread on a sample of units, and one
    thread per unit over every core on the whole batch (or, for the largest
    workloads, as many units as there are cores), scaled to one step of the
    workload."""
    model, ncores = cpu_info()
    total = w.B * w.Tq
    big = w.name in ("prefill_chunk_4096_full", "hier_1m_full_pool_reindex")
    units_mt = oracle_units(w, min(total, ncores) if big else total)
    units_1 = units_mt[:max(1, min(nrows, len(units_mt)))]
    data = OracleSequences(w, units_mt, ncores)
    secs1 = data.step(units_1, 1)
    per_step1 = secs1 * total / len(units_1)
    threads = min(ncores, len(units_mt))
    secs_mt = data.step(units_mt, threads)
    per_step_mt = secs_mt * total / len(units_mt)
    _, unit = workload_metric(w)
    what = "queries" if w.Tq > 1 else "sequences"
    return {"value": 1.0 / per_step_mt, "unit": unit, "cores": threads, "kind": "oracle",
            "cpu_model": model, "host_cores": ncores,
            "sample": "%d of %d %s of one step of the workload's layers (cache build "
                      "excluded), fp64, one thread per unit on %d threads; scaled to the "
                      "whole step" % (len(units_mt), total, what, threads),
            "single_thread": {"value": 1.0 / per_step1, "cores": 1,
                              "sample": "%d of %d %s, one thread, scaled to the whole step"
                                        % (len(units_1), total, what)}}


def run_reference(args):
    """The oracle as the reference arm: every step is one whole step of the
    workload (all its sequences, one thread per sequence over the host's cores)
    when the host has the cores for it to end within about a second, else as
    many units as there are cores, scaled to the batch; ms_per_step is the
    measured time of what each step ran."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from fp4_kv_cache_step_b200 import workloads as wl
    name = getattr(args, "workload", DEFAULT_WORKLOAD)
    w = wl.WORKLOADS[name]
    metric, unit = workload_metric(w)
    model, ncores = cpu_info()
    total = w.B * w.Tq
    big = w.name in ("prefill_chunk_4096_full", "hier_1m_full_pool_reindex")
    n_units = min(total, ncores) if (big or ncores < total // 2) else total
    units = oracle_units(w, n_units)
    threads = min(ncores, len(units))
    data = OracleSequences(w, units, threads)
    for _ in range(args.warmup):
        data.step(units, threads)
    secs = [data.step(units, threads) for _ in range(args.steps)]
    step_s = statistics.mean(secs)
    value = len(units) / total / step_s
    what = "queries" if w.Tq > 1 else "sequences"
    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "Tq": w.Tq, "N": w.N, "D": w.D,
                       "Hq": w.Hq, "Hi": w.Hi, "Di": w.Di, "K": w.K, "C": w.C,
                       "modes": list(w.modes), "context_tokens": 4 * w.N,
                       "parallelism": "CPU oracle on rank 0, one thread per %s" % what[:-1]},
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                             "cpu_model": model, "host_cores": ncores,
                             "sample": "each step: %d of %d %s of the workload's step, fp64, "
                                       "%d threads; ms_per_step is that measured time"
                                       % (len(units), total, what, threads)},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    if len(units) != total:
        line["scaled_from"] = "%d of %d %s per step" % (len(units), total, what)
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
    flush_l2 = L2Flush(torch, dev)
    for _ in range(args.warmup):
        ds.step()
    torch.cuda.synchronize()
    csa2.check_device_errors()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(dev.index) as clk:
        for i in range(args.steps):
            flush_l2(i)
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
    launches += 2                                      # the decoder FULL's blockwise pool
    print(json.dumps({
        "metric": "CSA2 stack decode steps/s (the model's 38 CSA2 layers)",
        "value": 1e3 / ms_per_step, "unit": "stack-steps/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": DTYPE, "data": "synthetic",
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
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="workload name (fp4_kv_cache_step_b200.workloads.WORKLOADS)")
    ap.add_argument("--cpu-sample-rows", type=int, default=4,
                    help="sequences in the single-threaded oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill-chunk indexer figure of the default line")
    ap.add_argument("--stack", default=None, choices=["production"],
                    help="time the model's 38 CSA2 layers (one GPU) instead of the headline step")
    ap.add_argument("--context", type=int, default=131072, help="--stack: context in tokens")
    ap.add_argument("--batch", type=int, default=4, help="--stack: sequences")
    ap.add_argument("--record-ncu", default=None, metavar="CSV",
                    help="write the DRAM traffic of --kernel from an ncu CSV capture of "
                         "--workload into profiles/kernel_traffic.json (no GPU needed)")
    ap.add_argument("--kernel", default=None, choices=sorted(KERNEL_NAMES))
    ap.add_argument("--ncu-command", default="", help="--record-ncu: the capture's command")
    args = ap.parse_args()
    if args.record_ncu:
        rec = record_ncu(args.record_ncu, args.kernel, args.workload, args.ncu_command)
        print(json.dumps(rec))
        return
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
