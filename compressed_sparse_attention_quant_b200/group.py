"""Host-side bookkeeping of a group of CSA2 layers: static modes, KV owners
and index aliases. Page "DeepSeek V4 1-Flash 架构拆解…" (blog.zulogic.cn),
section 3: a Full layer is the physical cache owner of the compressed global
KV, the indexer K / scale and the top-K metadata; Reindex and Reuse layers
consume them. Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai),
architecture part 2: main KV and indexer keys are shared and top-K indices are
reused across layers.

No device work happens here beyond calling the library: a Reuse layer's index
tensor IS its source layer's tensor (same storage, no copy), and every layer
of an owner reads that owner's PagedCache.

With pool_size set (the hierarchical sparse indexer, neodrop.ai architecture
part 2), a Full layer keeps its top-pool_size positions as a candidate pool
and takes its own top-k inside it. A Reindex layer then scores only its KV
owner's pool instead of the whole context.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import torch

from . import lib

DEFAULT_SCALE = 1.0 / math.sqrt(lib.DIM)


class LayerGroup:
    def __init__(self, modes: Sequence[str], batch: int, q_tokens: int, max_pages: int,
                 num_pages: int, top_k: int, device="cuda", softmax_scale: float = DEFAULT_SCALE,
                 pool_size: Optional[int] = None):
        self.modes = tuple(modes)
        self.kv_owner, self.index_src = lib.plan(self.modes)
        self.B, self.Sq, self.k = batch, q_tokens, top_k
        self.max_pages, self.num_pages = max_pages, num_pages
        self.scale = softmax_scale
        self.device = device
        self.caches: Dict[int, lib.PagedCache] = {o: lib.PagedCache(num_pages, device)
                                                  for o in sorted(set(self.kv_owner))}
        self._index: Dict[int, torch.Tensor] = {
            i: torch.full((batch, q_tokens, top_k), -1, dtype=torch.int32, device=device)
            for i, m in enumerate(self.modes) if m in ("F", "R")}
        n = len(self.modes)
        self.out = [torch.empty(batch, q_tokens, lib.HEADS, lib.DIM, dtype=torch.float32, device=device)
                    for _ in range(n)]
        self.lse = [torch.empty(batch, q_tokens, lib.HEADS, dtype=torch.float32, device=device)
                    for _ in range(n)]
        self.pool_size = pool_size
        if pool_size is not None and pool_size < top_k:
            raise ValueError(f"pool_size {pool_size} must be at least top_k {top_k}")
        self._pool: Dict[int, torch.Tensor] = {} if pool_size is None else {
            i: torch.full((batch, q_tokens, pool_size), -1, dtype=torch.int32, device=device)
            for i, m in enumerate(self.modes) if m == "F"}
        self.ws_idx = lib.workspace(lib.indexer_topk_workspace_bytes(batch, q_tokens, max_pages, top_k), device)
        self.ws_att = lib.workspace(lib.sparse_attn_workspace_bytes(batch, q_tokens, top_k), device)

    def index(self, layer: int) -> torch.Tensor:
        """The top-k index tensor layer `layer` attends with (an alias for Reuse)."""
        return self._index[self.index_src[layer]]

    def cache(self, layer: int) -> lib.PagedCache:
        return self.caches[self.kv_owner[layer]]

    def pool(self, layer: int) -> torch.Tensor:
        """The candidate pool a layer's selection reads (its KV owner's), when pool_size is set."""
        return self._pool[self.kv_owner[layer]]

    def step(self, page_table: torch.Tensor, seq_lens: torch.Tensor, q: List[torch.Tensor],
             swa: List[torch.Tensor], q_idx: Dict[int, torch.Tensor], w: Dict[int, torch.Tensor],
             append: Optional[Dict[int, tuple]] = None, out: Optional[List[torch.Tensor]] = None,
             lse: Optional[List[torch.Tensor]] = None) -> None:
        """One decode step over every layer of the group, on the current stream.

        q[l], swa[l]: layer l's attention query and window rows.
        q_idx[l], w[l]: indexer query and head weights of Full / Reindex layers.
        append[l] = (x_new [n,576] bf16, slots [n] int32, kidx_new [n,64] u8,
                     ksig_new [n] f32): the new tokens a Full layer writes into
                     its cache before it indexes (None: cache already holds them).
        out[l], lse[l]: where layer l writes its output (default self.out, self.lse).
        """
        out = self.out if out is None else out
        lse = self.lse if lse is None else lse
        for li, mode in enumerate(self.modes):
            cache = self.cache(li)
            if mode == "F" and append is not None and li in append:
                x_new, slots, kidx_new, ksig_new = append[li]
                lib.quant_kv_fp4(x_new, slots, cache, kidx_new, ksig_new)
            if mode in ("F", "R") and self.pool_size is not None:
                if mode == "F":
                    lib.indexer_topk(q_idx[li], w[li], cache, page_table, seq_lens, self.pool_size,
                                     out=self._pool[li], ws=self.ws_idx)
                lib.indexer_pool_topk(q_idx[li], w[li], cache, page_table, seq_lens, self.pool(li), self.k,
                                      out=self._index[li])
            elif mode in ("F", "R"):
                lib.indexer_topk(q_idx[li], w[li], cache, page_table, seq_lens, self.k,
                                 out=self._index[li], ws=self.ws_idx)
            lib.sparse_attn_decode(q[li], cache, page_table, seq_lens, self.index(li), swa[li], self.scale,
                                   out=out[li], lse=lse[li], ws=self.ws_att)


class StepGraph:
    """One decode step of a LayerGroup captured once as a CUDA graph and then
    replayed with a single launch: the same library kernels in the same order,
    the programmatic-dependent-launch overlap between consecutive kernels kept
    as graph edges, and no host work per kernel. The graph reads and writes the
    tensors given at capture time, so a caller refreshes those in place between
    replays (new query rows, new tokens to append, new page-table entries).

    The first eager step runs before the capture so that the library's one-time
    device set-up does not happen while the stream is being captured.
    """

    def __init__(self, group: LayerGroup, *step_args, **step_kwargs):
        group.step(*step_args, **step_kwargs)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        n0 = lib.launch_count()
        # thread-local capture: other threads (a process group's watchdog) may
        # keep querying the device while this one captures
        with torch.cuda.graph(self.graph, capture_error_mode="thread_local"):
            group.step(*step_args, **step_kwargs)
        self.launches = lib.launch_count() - n0          # library kernels per replay

    def replay(self) -> None:
        """Enqueue the captured step on the current stream."""
        self.graph.replay()
