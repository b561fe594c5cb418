"""Run a CSA2 layer stack on one GPU through the C ABI.

`DeviceWorkload` uploads a seeded workload (see workloads.py), builds the FP4
main KV with `fp4_kv_pack`, and runs the workload's mode schedule with
`csa2_layer_step`, the layers sharing one main KV, one indexer-key buffer and
the top-K / candidate-pool buffers ("The Three Modes Full Reindex And Reuse" in
"Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words"). All arithmetic
happens in the library's kernels.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import numpy as np
import torch

from . import csa2
from . import workloads as wl


def _dev(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device, non_blocking=False)


def _bf16_dev(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


class DeviceWorkload:
    def __init__(self, w: wl.Workload, device="cuda", keep_kv_f32: bool = False):
        self.w = w
        self.device = torch.device(device)
        B, N, D = w.B, w.N, w.D
        self.kv_packed = torch.empty((B, N, D // 2), dtype=torch.uint8, device=self.device)
        self.kv_scale = torch.empty((B, N // 64, D), dtype=torch.uint8, device=self.device)
        self.kv_f32 = None
        # pack one batch row at a time so the fp32 cache never has to be resident
        for b in range(B):
            row = _dev(wl.kv_row(w, b), self.device).unsqueeze(0)
            csa2.fp4_kv_pack(row, self.kv_packed[b:b + 1], self.kv_scale[b:b + 1])
            if keep_kv_f32:
                if self.kv_f32 is None:
                    self.kv_f32 = torch.empty((B, N, D), dtype=torch.float32, device=self.device)
                self.kv_f32[b].copy_(row[0])
        self.idx_k = _dev(wl.idx_k(w), self.device)
        self.nvalid = _dev(wl.nvalid(w), self.device)
        self.q: List[torch.Tensor] = []
        self.idx_q: List[Optional[torch.Tensor]] = []
        self.idx_w: List[Optional[torch.Tensor]] = []
        for layer, mode in enumerate(w.modes):
            self.q.append(_bf16_dev(wl.q(w, layer), self.device))
            if mode in (wl.FULL, wl.REINDEX):
                self.idx_q.append(_dev(wl.idx_q(w, layer), self.device))
                self.idx_w.append(_dev(wl.idx_w(w, layer), self.device))
            else:
                self.idx_q.append(None)
                self.idx_w.append(None)
        self.topk = torch.full((B, w.Tq, w.K), -1, dtype=torch.int32, device=self.device)
        self.cand = (torch.full((B, w.Tq, w.C), -1, dtype=torch.int32, device=self.device)
                     if w.C else None)
        self.shared = csa2.Csa2Shared(self.kv_packed, self.kv_scale, self.idx_k, self.topk,
                                      self.cand)
        self.out = [torch.empty((B, w.Tq, w.Hq, D), dtype=torch.bfloat16, device=self.device)
                    for _ in w.modes]
        self.lse = [torch.empty((B, w.Tq, w.Hq), dtype=torch.float32, device=self.device)
                    for _ in w.modes]
        self.args = []
        for layer, mode in enumerate(w.modes):
            self.args.append(csa2.layer_args(
                self.q[layer], self.nvalid, self.out[layer], w.K, w.softmax_scale,
                idx_q=self.idx_q[layer], idx_w=self.idx_w[layer], lse=self.lse[layer], N=N,
                emit_pool=(0 if mode != wl.FULL or w.C == 0 else
                           (2 if w.pool_block == 8 else 1)),
                use_pool=(mode == wl.REINDEX and w.C > 0)))
        need = max(csa2.layer_step_workspace_bytes(m, a, self.shared)
                   for m, a in zip(w.modes, self.args))
        self.workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
        self.topk_per_layer: List[Optional[torch.Tensor]] = [None] * len(w.modes)

    def step(self, layers: Optional[Sequence[int]] = None, snapshot_topk: bool = False):
        """Run the mode schedule once (all layers, or the given ones) on the
        current stream."""
        for layer in (range(len(self.w.modes)) if layers is None else layers):
            csa2.csa2_layer_step(self.w.modes[layer], self.args[layer], self.shared,
                                 self.workspace)
            if snapshot_topk:
                self.topk_per_layer[layer] = self.topk.clone()
        return self.out, self.lse


class DeviceStack:
    """The model's CSA2 layers (workloads.production_stack) on one GPU: one
    DeviceWorkload per cache-sharing segment (three encoder groups, the
    decoder), run in model order by `step()`."""

    def __init__(self, stack: wl.Stack, device="cuda"):
        self.stack = stack
        self.segments = [DeviceWorkload(w, device) for w in stack.segments]

    def step(self, snapshot_topk: bool = False):
        for seg, layer in self.stack.layers:
            self.segments[seg].step([layer], snapshot_topk=snapshot_topk)
        return [(d.out, d.lse) for d in self.segments]
