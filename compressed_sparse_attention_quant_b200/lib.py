"""Thin Python binding of the C ABI in include/csa2.h (argument marshalling
only: every step of the decode path runs in the library's CUDA kernels).

Tensors are torch tensors on the current CUDA device; calls are enqueued on
torch's current stream. A non-OK status raises Csa2Error. The library must
be built (see _build.py); importing this module fails loudly otherwise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

from . import _build

HEADS, DIM, IDX_HEADS, IDX_DIM, WINDOW, PAGE = 16, 576, 4, 64, 128, 64
FP4_BYTES, SCALE_BYTES, KIDX_PAGE_BYTES = 288, 36, 4096
MODES = {"F": 0, "R": 1, "U": 2}

STATUS = {0: "CSA2_OK", 1: "CSA2_ERR_INVALID_ARG", 2: "CSA2_ERR_UNSUPPORTED", 3: "CSA2_ERR_CUDA",
          4: "CSA2_ERR_BAD_PLAN", 5: "CSA2_ERR_TIMEOUT", 6: "CSA2_ERR_DEVICE_BOUNDS",
          7: "CSA2_ERR_WORKSPACE", 8: "CSA2_ERR_ALIGNMENT"}

# Every function include/csa2.h declares (checked by the CPU test suite).
EXPORTS = ("csa2_quant_kv_fp4", "csa2_quant_indexer_fp8", "csa2_indexer_topk_workspace_bytes",
           "csa2_indexer_topk", "csa2_indexer_pool_topk", "csa2_sparse_attn_workspace_bytes", "csa2_sparse_attn_decode",
           "csa2_sparse_attn_decode_noalloc", "csa2_indexer_topk_scores", "csa2_topk_merge", "csa2_lse_merge",
           "csa2_swa_replay_attn",
           "csa2_plan",
           "csa2_last_device_error", "csa2_status_string", "csa2_launch_count")


class Csa2Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


class _Cache(ctypes.Structure):
    _fields_ = [("kv_fp4", ctypes.c_void_p), ("kv_scale", ctypes.c_void_p), ("kidx", ctypes.c_void_p),
                ("kidx_scale", ctypes.c_void_p), ("num_pages", ctypes.c_int64)]


_vp, _i32, _i64, _sz, _f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_cp = ctypes.POINTER(_Cache)
_ip = ctypes.POINTER(ctypes.c_int)


def _load():
    path = _build.LIB
    if not os.path.exists(path):
        raise ImportError(f"CSA2 CUDA library not built: {path} is missing (run __graft_entry__.build())")
    L = ctypes.CDLL(path)
    sig = {
        "csa2_quant_kv_fp4": (_i32, [_vp, _i64, _i32, _vp, _vp, _vp, _cp, _vp]),
        "csa2_quant_indexer_fp8": (_i32, [_vp, _i64, _i32, _vp, _vp, _vp]),
        "csa2_indexer_topk_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32]),
        "csa2_indexer_topk": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _cp, _vp, _i32, _vp, _i32, _vp,
                                     _vp, _sz, _vp]),
        "csa2_indexer_pool_topk": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _cp, _vp, _i32, _vp, _vp, _i32, _i32,
                                          _vp, _vp]),
        "csa2_sparse_attn_workspace_bytes": (_sz, [_i32, _i32, _i32]),
        "csa2_sparse_attn_decode": (_i32, [_vp, _i32, _i32, _i32, _i32, _cp, _vp, _i32, _vp, _vp, _i32,
                                           _vp, _i32, _f32, _vp, _vp, _vp, _sz, _vp]),
        "csa2_sparse_attn_decode_noalloc": (_i32, [_vp, _i32, _i32, _i32, _i32, _cp, _vp, _i32, _vp, _vp,
                                                   _i32, _vp, _i32, _f32, _vp, _vp, _vp]),
        "csa2_indexer_topk_scores": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _cp, _vp, _i32, _vp, _i32, _vp,
                                            _vp, _vp, _sz, _vp]),
        "csa2_topk_merge": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
        "csa2_lse_merge": (_i32, [_vp, _vp, _i32, _i32, _vp, _vp, _vp]),
        "csa2_swa_replay_attn": (_i32, [_vp, _i32, _i32, _i32, _i32, _vp, _i32, _vp, _f32, _vp, _vp, _vp]),
        "csa2_plan": (_i32, [_ip, _i32, _ip, _ip]),
        "csa2_last_device_error": (_i32, [_vp]),
        "csa2_status_string": (ctypes.c_char_p, [_i32]),
        "csa2_launch_count": (ctypes.c_uint64, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


_L = _load()


def library_path() -> str:
    return _build.LIB


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(fn: str, rc: int):
    if rc != 0:
        raise Csa2Error(fn, rc)


def _req(t: torch.Tensor, dtype, name: str, shape=None):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


class PagedCache:
    """The paged global cache of one KV owner (caller-owned device memory)."""

    def __init__(self, num_pages: int, device="cuda"):
        self.num_pages = int(num_pages)
        self.kv_fp4 = torch.zeros(num_pages, PAGE, FP4_BYTES, dtype=torch.uint8, device=device)
        self.kv_scale = torch.zeros(num_pages, PAGE, SCALE_BYTES, dtype=torch.uint8, device=device)
        self.kidx = torch.zeros(num_pages, KIDX_PAGE_BYTES, dtype=torch.uint8, device=device)
        self.kidx_scale = torch.zeros(num_pages, PAGE, dtype=torch.float32, device=device)
        self.desc = _Cache(self.kv_fp4.data_ptr(), self.kv_scale.data_ptr(), self.kidx.data_ptr(),
                           self.kidx_scale.data_ptr(), self.num_pages)

    def kidx_logical(self) -> torch.Tensor:
        """Indexer keys as [num_pages, 64 tokens, 64 channels] (undoes the
        8x16-byte core-matrix order documented in csa2.h)."""
        v = self.kidx.view(self.num_pages, 8, 4, 8, 16)       # [page][t/8][c/16][t%8][c%16]
        return v.permute(0, 1, 3, 2, 4).reshape(self.num_pages, PAGE, IDX_DIM)


def slot_mapping(page_table: torch.Tensor, b: int, positions: torch.Tensor) -> torch.Tensor:
    """Physical slot ids (page * 64 + row) of sequence b's positions."""
    pos = positions.to(torch.int64)
    return (page_table[b].to(torch.int64)[pos // PAGE] * PAGE + pos % PAGE).to(torch.int32)


def quant_kv_fp4(x: torch.Tensor, slots: torch.Tensor, cache: PagedCache,
                 kidx_in: Optional[torch.Tensor] = None, kidx_scale_in: Optional[torch.Tensor] = None):
    n = x.shape[0]
    _req(x, torch.bfloat16, "x", (n, DIM))
    _req(slots, torch.int32, "slot_mapping", (n,))
    if kidx_in is not None:
        _req(kidx_in, torch.uint8, "kidx_in", (n, IDX_DIM))
        _req(kidx_scale_in, torch.float32, "kidx_scale_in", (n,))
    rc = _L.csa2_quant_kv_fp4(_ptr(x), n, DIM, _ptr(slots), _ptr(kidx_in), _ptr(kidx_scale_in),
                              ctypes.byref(cache.desc), _stream())
    _check("csa2_quant_kv_fp4", rc)


def quant_indexer_fp8(x: torch.Tensor, codes: Optional[torch.Tensor] = None,
                      sigma: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """bf16 rows of 64 channels -> (E4M3FN codes uint8 [..., 64], sigma f32 [...])."""
    if x.shape[-1] != IDX_DIM:
        raise ValueError(f"x: last dimension must be {IDX_DIM}, got {tuple(x.shape)}")
    lead = tuple(x.shape[:-1])
    n = 1
    for d in lead:
        n *= int(d)
    _req(x, torch.bfloat16, "x")
    if codes is None:
        codes = torch.empty(*lead, IDX_DIM, dtype=torch.uint8, device=x.device)
    if sigma is None:
        sigma = torch.empty(*lead, dtype=torch.float32, device=x.device)
    _req(codes, torch.uint8, "codes", lead + (IDX_DIM,))
    _req(sigma, torch.float32, "sigma", lead)
    rc = _L.csa2_quant_indexer_fp8(_ptr(x), n, IDX_DIM, _ptr(codes), _ptr(sigma), _stream())
    _check("csa2_quant_indexer_fp8", rc)
    return codes, sigma


def indexer_topk_workspace_bytes(B: int, Sq: int, max_pages: int, k: int) -> int:
    return int(_L.csa2_indexer_topk_workspace_bytes(B, Sq, max_pages, k))


def sparse_attn_workspace_bytes(B: int, Sq: int, k: int) -> int:
    return int(_L.csa2_sparse_attn_workspace_bytes(B, Sq, k))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def indexer_topk(q_idx: torch.Tensor, w: torch.Tensor, cache: PagedCache, page_table: torch.Tensor,
                 seq_lens: torch.Tensor, k: int, out: Optional[torch.Tensor] = None,
                 ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    B, Sq = q_idx.shape[0], q_idx.shape[1]
    max_pages = page_table.shape[1]
    _req(q_idx, torch.uint8, "q_idx", (B, Sq, IDX_HEADS, IDX_DIM))
    _req(w, torch.float32, "w", (B, Sq, IDX_HEADS))
    _req(page_table, torch.int32, "page_table", (B, max_pages))
    _req(seq_lens, torch.int32, "seq_lens", (B,))
    if out is None:
        out = torch.empty(B, Sq, k, dtype=torch.int32, device=q_idx.device)
    _req(out, torch.int32, "out_idx", (B, Sq, k))
    need = indexer_topk_workspace_bytes(B, Sq, max_pages, k)
    if ws is None:
        ws = workspace(need, q_idx.device)
    rc = _L.csa2_indexer_topk(_ptr(q_idx), _ptr(w), B, Sq, IDX_HEADS, IDX_DIM, ctypes.byref(cache.desc),
                              _ptr(page_table), max_pages, _ptr(seq_lens), k, _ptr(out), _ptr(ws),
                              ws.numel() * ws.element_size(), _stream())
    _check("csa2_indexer_topk", rc)
    return out


def indexer_topk_scores(q_idx: torch.Tensor, w: torch.Tensor, cache: PagedCache, page_table: torch.Tensor,
                        seq_lens: torch.Tensor, k: int, out: Optional[torch.Tensor] = None,
                        scores: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None
                        ) -> Tuple[torch.Tensor, torch.Tensor]:
    """indexer_topk that also returns the selected entries' fp32 scores (-inf for -1)."""
    B, Sq = q_idx.shape[0], q_idx.shape[1]
    max_pages = page_table.shape[1]
    _req(q_idx, torch.uint8, "q_idx", (B, Sq, IDX_HEADS, IDX_DIM))
    _req(w, torch.float32, "w", (B, Sq, IDX_HEADS))
    _req(page_table, torch.int32, "page_table", (B, max_pages))
    _req(seq_lens, torch.int32, "seq_lens", (B,))
    if out is None:
        out = torch.empty(B, Sq, k, dtype=torch.int32, device=q_idx.device)
    if scores is None:
        scores = torch.empty(B, Sq, k, dtype=torch.float32, device=q_idx.device)
    _req(out, torch.int32, "out_idx", (B, Sq, k))
    _req(scores, torch.float32, "out_scores", (B, Sq, k))
    if ws is None:
        ws = workspace(indexer_topk_workspace_bytes(B, Sq, max_pages, k), q_idx.device)
    rc = _L.csa2_indexer_topk_scores(_ptr(q_idx), _ptr(w), B, Sq, IDX_HEADS, IDX_DIM, ctypes.byref(cache.desc),
                                     _ptr(page_table), max_pages, _ptr(seq_lens), k, _ptr(out), _ptr(scores),
                                     _ptr(ws), ws.numel() * ws.element_size(), _stream())
    _check("csa2_indexer_topk_scores", rc)
    return out, scores


def topk_merge(cand_scores: torch.Tensor, cand_idx: torch.Tensor, k: int, shard_lo: int = 0, shard_hi: int = 0,
               out: Optional[torch.Tensor] = None, out_local: Optional[torch.Tensor] = None,
               want_global: bool = True, want_local: bool = False):
    """Global top-k from G shards' candidates [G, R, k_shard] (scores, global
    positions). Returns (global [R, k] or None, local [R, k] or None)."""
    G, R, ks = cand_idx.shape
    _req(cand_scores, torch.float32, "cand_scores", (G, R, ks))
    _req(cand_idx, torch.int32, "cand_idx", (G, R, ks))
    if want_global and out is None:
        out = torch.empty(R, k, dtype=torch.int32, device=cand_idx.device)
    if want_local and out_local is None:
        out_local = torch.empty(R, k, dtype=torch.int32, device=cand_idx.device)
    for t, name in ((out, "out_idx"), (out_local, "out_local")):
        if t is not None:
            _req(t, torch.int32, name, (R, k))
    rc = _L.csa2_topk_merge(_ptr(cand_scores), _ptr(cand_idx), G, R, ks, k, int(shard_lo), int(shard_hi),
                            _ptr(out), _ptr(out_local), _stream())
    _check("csa2_topk_merge", rc)
    return out, out_local


def lse_merge(o_parts: torch.Tensor, lse_parts: torch.Tensor, out: Optional[torch.Tensor] = None,
              lse: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One softmax over disjoint key sets: o_parts [P, R, 16, 576], lse_parts [P, R, 16]."""
    P, R = o_parts.shape[0], o_parts.shape[1]
    _req(o_parts, torch.float32, "o_parts", (P, R, HEADS, DIM))
    _req(lse_parts, torch.float32, "lse_parts", (P, R, HEADS))
    if out is None:
        out = torch.empty(R, HEADS, DIM, dtype=torch.float32, device=o_parts.device)
    if lse is None:
        lse = torch.empty(R, HEADS, dtype=torch.float32, device=o_parts.device)
    _req(out, torch.float32, "out", (R, HEADS, DIM))
    _req(lse, torch.float32, "lse", (R, HEADS))
    rc = _L.csa2_lse_merge(_ptr(o_parts), _ptr(lse_parts), P, R, _ptr(out), _ptr(lse), _stream())
    _check("csa2_lse_merge", rc)
    return out, lse


def swa_replay_attn(q: torch.Tensor, swa: torch.Tensor, seq_lens: torch.Tensor, softmax_scale: float,
                    out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None
                    ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Window attention of L consecutive queries per sequence: q [B, L, 16, 576]
    bf16, swa [B, 128 + L - 1, 576] bf16 -> (out [B, L, 16, 576], lse [B, L, 16])."""
    B, L = q.shape[0], q.shape[1]
    _req(q, torch.bfloat16, "q", (B, L, HEADS, DIM))
    _req(swa, torch.bfloat16, "swa", (B, WINDOW + L - 1, DIM))
    _req(seq_lens, torch.int32, "seq_lens", (B,))
    if out is None:
        out = torch.empty(B, L, HEADS, DIM, dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(B, L, HEADS, dtype=torch.float32, device=q.device)
    _req(out, torch.float32, "out", (B, L, HEADS, DIM))
    _req(lse, torch.float32, "lse", (B, L, HEADS))
    rc = _L.csa2_swa_replay_attn(_ptr(q), B, L, HEADS, DIM, _ptr(swa), WINDOW, _ptr(seq_lens),
                                 float(softmax_scale), _ptr(out), _ptr(lse), _stream())
    _check("csa2_swa_replay_attn", rc)
    return out, lse


def indexer_scores_in_workspace(ws: torch.Tensor, B: int, Sq: int, max_pages: int) -> torch.Tensor:
    """The fp32 scores a completed csa2_indexer_topk call leaves at the start
    of its workspace, as a view [B, Sq, 64 * max_pages] (csa2.h: entries after
    a query's position are unspecified)."""
    n = B * Sq * PAGE * max_pages
    return ws[:4 * n].view(torch.float32).view(B, Sq, PAGE * max_pages)


def indexer_pool_topk(q_idx: torch.Tensor, w: torch.Tensor, cache: PagedCache, page_table: torch.Tensor,
                      seq_lens: torch.Tensor, pool: torch.Tensor, k: int,
                      out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Top-k of each query row's candidate pool [B, Sq, C] (ascending token indices, -1 skipped)."""
    B, Sq = q_idx.shape[0], q_idx.shape[1]
    max_pages = page_table.shape[1]
    C = pool.shape[2]
    _req(q_idx, torch.uint8, "q_idx", (B, Sq, IDX_HEADS, IDX_DIM))
    _req(w, torch.float32, "w", (B, Sq, IDX_HEADS))
    _req(page_table, torch.int32, "page_table", (B, max_pages))
    _req(seq_lens, torch.int32, "seq_lens", (B,))
    _req(pool, torch.int32, "pool", (B, Sq, C))
    if out is None:
        out = torch.empty(B, Sq, k, dtype=torch.int32, device=q_idx.device)
    _req(out, torch.int32, "out_idx", (B, Sq, k))
    rc = _L.csa2_indexer_pool_topk(_ptr(q_idx), _ptr(w), B, Sq, IDX_HEADS, IDX_DIM, ctypes.byref(cache.desc),
                                   _ptr(page_table), max_pages, _ptr(seq_lens), _ptr(pool), C, k, _ptr(out),
                                   _stream())
    _check("csa2_indexer_pool_topk", rc)
    return out


def sparse_attn_decode(q: torch.Tensor, cache: PagedCache, page_table: torch.Tensor,
                       seq_lens: torch.Tensor, topk_idx: Optional[torch.Tensor], swa: Optional[torch.Tensor],
                       softmax_scale: float, out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None
                       ) -> Tuple[torch.Tensor, torch.Tensor]:
    """swa None: no window rows (W = 0, a context-parallel shard without the newest tokens)."""
    B, Sq = q.shape[0], q.shape[1]
    max_pages = page_table.shape[1]
    _req(q, torch.bfloat16, "q", (B, Sq, HEADS, DIM))
    _req(page_table, torch.int32, "page_table", (B, max_pages))
    _req(seq_lens, torch.int32, "seq_lens", (B,))
    k = 0 if topk_idx is None else topk_idx.shape[2]
    if topk_idx is not None:
        _req(topk_idx, torch.int32, "topk_idx", (B, Sq, k))
    if swa is not None:
        _req(swa, torch.bfloat16, "swa", (B, WINDOW + Sq - 1, DIM))
    if out is None:
        out = torch.empty(B, Sq, HEADS, DIM, dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(B, Sq, HEADS, dtype=torch.float32, device=q.device)
    _req(out, torch.float32, "out", (B, Sq, HEADS, DIM))
    _req(lse, torch.float32, "lse", (B, Sq, HEADS))
    need = sparse_attn_workspace_bytes(B, Sq, k)
    if ws is None:
        ws = workspace(need, q.device)
    rc = _L.csa2_sparse_attn_decode(_ptr(q), B, Sq, HEADS, DIM, ctypes.byref(cache.desc), _ptr(page_table),
                                    max_pages, _ptr(seq_lens), _ptr(topk_idx), k, _ptr(swa),
                                    WINDOW if swa is not None else 0,
                                    float(softmax_scale), _ptr(out), _ptr(lse), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream())
    _check("csa2_sparse_attn_decode", rc)
    return out, lse


NOALLOC_SCRATCH_BYTES = 32 << 20


def sparse_attn_decode_noalloc(q: torch.Tensor, cache: PagedCache, page_table: torch.Tensor,
                               seq_lens: torch.Tensor, topk_idx: Optional[torch.Tensor], swa: torch.Tensor,
                               softmax_scale: float, out: torch.Tensor, lse: torch.Tensor) -> None:
    """sparse_attn_decode without a workspace: the library's own device
    scratch holds the split partials (see csa2_sparse_attn_decode_noalloc in
    csa2.h). The caller passes the output buffers; nothing is allocated."""
    B, Sq = q.shape[0], q.shape[1]
    max_pages = page_table.shape[1]
    _req(q, torch.bfloat16, "q", (B, Sq, HEADS, DIM))
    _req(page_table, torch.int32, "page_table", (B, max_pages))
    _req(seq_lens, torch.int32, "seq_lens", (B,))
    k = 0 if topk_idx is None else topk_idx.shape[2]
    if topk_idx is not None:
        _req(topk_idx, torch.int32, "topk_idx", (B, Sq, k))
    _req(swa, torch.bfloat16, "swa", (B, WINDOW + Sq - 1, DIM))
    _req(out, torch.float32, "out", (B, Sq, HEADS, DIM))
    _req(lse, torch.float32, "lse", (B, Sq, HEADS))
    rc = _L.csa2_sparse_attn_decode_noalloc(_ptr(q), B, Sq, HEADS, DIM, ctypes.byref(cache.desc),
                                            _ptr(page_table), max_pages, _ptr(seq_lens), _ptr(topk_idx), k,
                                            _ptr(swa), WINDOW, float(softmax_scale), _ptr(out), _ptr(lse),
                                            _stream())
    _check("csa2_sparse_attn_decode_noalloc", rc)


def plan(modes: Sequence[str]) -> Tuple[list, list]:
    n = len(modes)
    m = (ctypes.c_int * n)(*[MODES[x] for x in modes])
    own = (ctypes.c_int * n)()
    src = (ctypes.c_int * n)()
    _check("csa2_plan", _L.csa2_plan(m, n, own, src))
    return list(own), list(src)


def last_device_error() -> int:
    """Synchronises the current stream and returns (and clears) the device status."""
    return int(_L.csa2_last_device_error(_stream()))


def status_string(s: int) -> str:
    return _L.csa2_status_string(int(s)).decode()


def launch_count() -> int:
    return int(_L.csa2_launch_count())
