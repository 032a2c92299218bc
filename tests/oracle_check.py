"""Oracle expectations for a DeviceWorkload, computed on the CPU from the very
same synthetic inputs (generated on the GPU by inputs.py, copied to the host).

For large contexts only the rows the oracle needs are quantized: the indexer
keys of positions 0..pos, and the KV latent rows of the selected positions
(the oracle's own top-k), which the oracle then attends to through a compact
cache with re-mapped indices (an exact re-indexing of the same computation).
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, Tuple

import numpy as np
import torch

import oracle
from compressed_sparse_attention_quant_b200 import inputs

SCALE = 1.0 / math.sqrt(576)


class OracleRun:
    def __init__(self, dw, seqs: Iterable[int], queries: Iterable[int] = None):
        self.dw = dw
        self.wl = dw.wl
        self.seqs = list(seqs)
        self.queries = list(range(self.wl.q_tokens)) if queries is None else list(queries)
        self.own, self.src = oracle.plan(self.wl.modes)
        self._kidx: Dict[Tuple[int, int], np.ndarray] = {}
        self.out: Dict[int, Dict[Tuple[int, int], dict]] = {i: {} for i in range(len(self.wl.modes))}
        self._run()

    def kidx(self, owner: int, b: int) -> Tuple[np.ndarray, np.ndarray]:
        key = (owner, b)
        if key not in self._kidx:
            T = self.wl.lens()[b]
            k = inputs.kidx_rows(self.wl, owner, b, 0, T, self.dw.device).cpu().numpy()
            s = inputs.kidx_scale_rows(self.wl, owner, b, 0, T, self.dw.device).cpu().numpy()
            self._kidx[key] = (k, s)
        return self._kidx[key]

    def _run(self):
        wl, dev = self.wl, self.dw.device
        Sq = wl.q_tokens
        for li, mode in enumerate(wl.modes):
            owner = self.own[li]
            for b in self.seqs:
                T = wl.lens()[b]
                q = oracle.bf16_bits(self.dw.q[li][b])
                swa = oracle.bf16_bits(self.dw.swa[li][b])
                for j in self.queries:
                    pos = T - Sq + j
                    if mode in ("F", "R"):
                        k_all, s_all = self.kidx(owner, b)
                        qi = self.dw.q_idx[li][b, j].cpu().numpy()
                        w = self.dw.w[li][b, j].cpu().numpy()
                        sc = oracle.indexer_scores(qi, w, k_all[:pos + 1], s_all[:pos + 1])
                        idx = oracle.topk(sc, pos + 1, wl.top_k)
                    else:
                        idx = self.out[self.src[li]][(b, j)]["idx"]
                    o, lse = attend(self.dw, owner, b, j, q[j], swa, idx)
                    self.out[li][(b, j)] = {"idx": idx, "o": o, "lse": lse}


def attend(dw, owner: int, b: int, j: int, q_bits, swa_bits, idx):
    """Oracle attention of query j of sequence b over the owner's cache."""
    wl = dw.wl
    T, Sq, W = wl.lens()[b], wl.q_tokens, inputs.WINDOW
    valid = idx[idx >= 0]
    rows = inputs.kv_rows(wl, owner, b, torch.from_numpy(valid.astype(np.int64)), dw.device)
    codes, scales = oracle.quant_fp4(oracle.bf16_bits(rows))
    compact = np.where(idx >= 0, np.cumsum(idx >= 0) - 1, -1).astype(np.int32)
    first = T - (W + Sq - 1)
    rws = [r for r in range(j, j + W) if first + r >= 0]
    swa = swa_bits[rws] if rws else np.zeros((0, 576), np.uint16)
    return oracle.sparse_attn(q_bits, codes, scales, compact, swa, SCALE)


def assert_attn_close(o_gpu: np.ndarray, lse_gpu: np.ndarray, o_ref: np.ndarray, lse_ref: np.ndarray,
                      what: str = ""):
    """The parity bar for attention: max-abs 2e-3 and relative L2 1e-3."""
    err = np.abs(o_gpu.astype(np.float64) - o_ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(o_ref))
    rel = float(np.linalg.norm(o_gpu - o_ref)) / denom if denom > 0 else float(np.linalg.norm(o_gpu))
    assert max_abs <= 2e-3, f"{what}: max-abs {max_abs:.3e} > 2e-3"
    assert rel <= 1e-3, f"{what}: rel-L2 {rel:.3e} > 1e-3"
    fin = np.isfinite(lse_ref)
    np.testing.assert_array_equal(np.isfinite(lse_gpu), fin, err_msg=what)
    if fin.any():
        assert float(np.abs(lse_gpu[fin] - lse_ref[fin]).max()) <= 2e-3, f"{what}: lse"
    return max_abs, rel
