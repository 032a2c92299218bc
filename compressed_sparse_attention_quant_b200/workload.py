"""Device state of one synthetic decode workload: page table, lengths, the
paged caches of every KV owner (bulk-built through csa2_quant_kv_fp4), and
the per-layer step inputs, all resident in HBM. Used by the tests and the
benchmark; the values come from inputs.py."""
from __future__ import annotations

from typing import Dict, List

import torch

from . import inputs, lib
from .group import LayerGroup, StepGraph


class DeviceWorkload:
    def __init__(self, wl: inputs.Workload, device="cuda", pool_size=None):
        self.wl = wl
        self.device = device
        B, Sq = wl.batch, wl.q_tokens
        self.page_table = inputs.page_table(wl, device)
        self.seq_lens = inputs.seq_lens(wl, device)
        self.group = LayerGroup(wl.modes, B, Sq, wl.pages_per_seq, B * wl.pages_per_seq, wl.top_k, device,
                                pool_size=pool_size)
        lens = wl.lens()
        # Bulk build: positions [0, len_b - Sq) of each owner's cache.
        for owner, cache in self.group.caches.items():
            for b in range(B):
                t_end = lens[b] - Sq
                for t0, rows in inputs.kv_chunks(wl, owner, b, device, t_end=t_end):
                    n = rows.shape[0]
                    pos = torch.arange(t0, t0 + n, device=device)
                    slots = lib.slot_mapping(self.page_table, b, pos)
                    kid = inputs.kidx_rows(wl, owner, b, t0, t0 + n, device)
                    ksig = inputs.kidx_scale_rows(wl, owner, b, t0, t0 + n, device)
                    lib.quant_kv_fp4(rows.contiguous(), slots, cache, kid, ksig)
        # Per-step inputs.
        n_layers = len(wl.modes)
        self.q: List[torch.Tensor] = [inputs.attn_query(wl, li, device) for li in range(n_layers)]
        self.swa: List[torch.Tensor] = [inputs.swa_rows(wl, li, device) for li in range(n_layers)]
        self.q_idx: Dict[int, torch.Tensor] = {}
        self.w: Dict[int, torch.Tensor] = {}
        for li, m in enumerate(wl.modes):
            if m in ("F", "R"):
                self.q_idx[li] = inputs.idx_query(wl, li, device)
                self.w[li] = inputs.idx_weights(wl, li, device)
        # The Sq newest tokens every Full layer appends in the step.
        self.append: Dict[int, tuple] = {}
        for li, m in enumerate(wl.modes):
            if m != "F":
                continue
            xs, sl, ks, ss = [], [], [], []
            for b in range(B):
                pos = torch.arange(lens[b] - Sq, lens[b])
                xs.append(inputs.kv_rows(wl, li, b, pos, device))
                sl.append(lib.slot_mapping(self.page_table, b, pos.to(device)))
                ks.append(inputs.kidx_rows(wl, li, b, lens[b] - Sq, lens[b], device))
                ss.append(inputs.kidx_scale_rows(wl, li, b, lens[b] - Sq, lens[b], device))
            self.append[li] = (torch.cat(xs).contiguous(), torch.cat(sl).contiguous(),
                               torch.cat(ks).contiguous(), torch.cat(ss).contiguous())

    def step(self) -> None:
        self.group.step(self.page_table, self.seq_lens, self.q, self.swa, self.q_idx, self.w, self.append)

    def capture(self) -> StepGraph:
        """The step as a CUDA graph over this workload's resident tensors."""
        return StepGraph(self.group, self.page_table, self.seq_lens, self.q, self.swa, self.q_idx, self.w,
                         self.append)

    # ------------------------------------------------------------ accounting
    def algorithmic_bytes(self) -> Dict[str, float]:
        """Bytes one step must move (per the workload's layer plan), counting the
        distinct FP4 entries each layer reads as k per query token."""
        wl = self.wl
        lens = wl.lens()
        B, Sq, k = wl.batch, wl.q_tokens, wl.top_k
        out = {"indexer": 0.0, "attention": 0.0, "append": 0.0, "topk_io": 0.0}
        for m in wl.modes:
            if m in ("F", "R"):
                out["indexer"] += sum(68.0 * t for t in lens) + 272.0 * B * Sq
                out["topk_io"] += 4.0 * k * B * Sq
            if m == "F":
                out["append"] += 1544.0 * B * Sq
            out["attention"] += B * Sq * (324.0 * k + 18432.0 + 36928.0 + 4.0 * k) + B * 1152.0 * (127 + Sq)
        out["total"] = sum(out.values())
        return out
