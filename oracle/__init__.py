"""CPU oracle for the CSA2 FP4 sparse-decode path (TEST INFRASTRUCTURE).

Plain single-threaded C (csa2_oracle.c, fp64 and exact integers) wrapped with
ctypes and numpy. Only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline leg may import this package; the product library never does, and
this package never imports the product library.

Citation tags ([INF], [NEO], [ZUL]) are defined in csa2_oracle.h.

Parity status: every function below is pinned by tests/test_oracle_pins.py
against format definitions, brute force or library routines, except the
indexer formula itself (the pages print none; "parity unpinned" for the
choice of formula, while its arithmetic is pinned by brute force) and the
choice of V = K (the pages never split the 576 channels; unpinned reading).
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Sequence, Tuple

import numpy as np

from . import build as _build

_lib = None
_openmp = False


def use_all_cores(on: bool = True) -> None:
    """Load the OpenMP build of the same C source (bit-identical results; its
    independent outer loops run on every host core). For timing the oracle
    only; must be chosen before the first oracle call of the process."""
    global _openmp
    if _lib is not None and on != _openmp:
        raise RuntimeError("oracle library already loaded")
    _openmp = on


_nthreads = None


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def set_threads(n: int) -> None:
    """Threads of the OpenMP build's parallel loops (the test build ignores it)."""
    global _nthreads
    if _openmp:
        lib().omp_set_num_threads(int(n))       # libgomp, reached through the library's handle
        _nthreads = int(n)


def threads() -> int:
    """Threads the loaded oracle runs its parallel loops on (1 for the test build)."""
    if not _openmp:
        return 1
    return _nthreads if _nthreads is not None else host_cores()

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i32p = ctypes.POINTER(ctypes.c_int32)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_intp = ctypes.POINTER(ctypes.c_int)


def lib():
    global _lib
    if _lib is None:
        path = _build.build(openmp=_openmp)
        L = ctypes.CDLL(path)
        L.orc_bf16_value.restype = ctypes.c_double
        L.orc_bf16_value.argtypes = [ctypes.c_uint16]
        L.orc_e2m1_value.restype = ctypes.c_double
        L.orc_e2m1_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_group_scale.restype = ctypes.c_uint8
        L.orc_group_scale.argtypes = [ctypes.c_double]
        L.orc_e2m1_code.restype = ctypes.c_uint8
        L.orc_e2m1_code.argtypes = [ctypes.c_double, ctypes.c_double]
        L.orc_group_scale_n.restype = None
        L.orc_group_scale_n.argtypes = [_f64p, ctypes.c_int64, _u8p]
        L.orc_e2m1_code_n.restype = None
        L.orc_e2m1_code_n.argtypes = [_f64p, _f64p, ctypes.c_int64, _u8p]
        L.orc_quant_fp4.restype = None
        L.orc_quant_fp4.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int, _u8p, _u8p]
        L.orc_dequant_fp4.restype = None
        L.orc_dequant_fp4.argtypes = [_u8p, _u8p, ctypes.c_int64, ctypes.c_int, _f64p]
        L.orc_e4m3_code_quotient.restype = ctypes.c_uint8
        L.orc_e4m3_code_quotient.argtypes = [ctypes.c_double, ctypes.c_float]
        L.orc_quant_index_fp8.restype = None
        L.orc_quant_index_fp8.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int, _u8p, _f32p]
        L.orc_indexer_scores.restype = None
        L.orc_indexer_scores.argtypes = [_u8p, _f32p, ctypes.c_int, ctypes.c_int, _u8p, _f32p,
                                         ctypes.c_int64, ctypes.c_int, _f64p]
        L.orc_topk.restype = ctypes.c_int
        L.orc_topk.argtypes = [_f64p, ctypes.c_int64, ctypes.c_int, _i32p]
        L.orc_pool_topk.restype = ctypes.c_int
        L.orc_pool_topk.argtypes = [_f64p, _i32p, ctypes.c_int, ctypes.c_int, _i32p]
        L.orc_sparse_attn.restype = None
        L.orc_sparse_attn.argtypes = [_u16p, ctypes.c_int, ctypes.c_int, _u8p, _u8p,
                                      ctypes.c_int64, _i32p, ctypes.c_int, _u16p, ctypes.c_int,
                                      ctypes.c_double, _f64p, _f64p]
        L.orc_plan.restype = ctypes.c_int
        L.orc_plan.argtypes = [_intp, ctypes.c_int, _intp, _intp]
        _lib = L
    return _lib


def _p(a: np.ndarray, t):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(t)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


# ---------------------------------------------------------------- formats
def bf16_value(bits: int) -> float:
    return lib().orc_bf16_value(int(bits))


def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(int(code))


def e4m3_value(byte: int) -> float:
    return lib().orc_e4m3_value(int(byte))


def group_scale(amax: float) -> int:
    return int(lib().orc_group_scale(float(amax)))


def e2m1_code(x: float, s: float) -> int:
    return int(lib().orc_e2m1_code(float(x), float(s)))


def group_scale_n(amax) -> np.ndarray:
    a = _c(amax, np.float64).ravel()
    out = np.zeros(a.shape, np.uint8)
    lib().orc_group_scale_n(_p(a, _f64p), a.size, _p(out, _u8p))
    return out


def e2m1_code_n(x, s) -> np.ndarray:
    x, s = np.broadcast_arrays(np.asarray(x, np.float64), np.asarray(s, np.float64))
    x = _c(x, np.float64).ravel()
    s = _c(s, np.float64).ravel()
    out = np.zeros(x.shape, np.uint8)
    lib().orc_e2m1_code_n(_p(x, _f64p), _p(s, _f64p), x.size, _p(out, _u8p))
    return out


# ---------------------------------------------------------------- quantizer
def quant_fp4(x_bf16_bits) -> Tuple[np.ndarray, np.ndarray]:
    """x: uint16 bf16 bits [n, dim] -> (codes uint8 [n, dim/2], scales uint8 [n, dim/16])."""
    x = _c(x_bf16_bits, np.uint16)
    n, dim = x.shape
    codes = np.zeros((n, dim // 2), np.uint8)
    scales = np.zeros((n, dim // 16), np.uint8)
    lib().orc_quant_fp4(_p(x, _u16p), n, dim, _p(codes, _u8p), _p(scales, _u8p))
    return codes, scales


def dequant_fp4(codes, scales) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    n = codes.shape[0]
    dim = codes.shape[1] * 2
    out = np.zeros((n, dim), np.float64)
    lib().orc_dequant_fp4(_p(codes, _u8p), _p(scales, _u8p), n, dim, _p(out, _f64p))
    return out


# ---------------------------------------------------------------- indexer FP8 quantiser
def e4m3_code_quotient(x: float, sigma: float) -> int:
    """E4M3FN code nearest to the exact quotient x / sigma (x passed as a C
    double, sigma > 0 as a C float)."""
    return int(lib().orc_e4m3_code_quotient(float(x), float(sigma)))


def quant_index_fp8(x_bf16_bits) -> Tuple[np.ndarray, np.ndarray]:
    """x: uint16 bf16 bits [n, dim] -> (codes uint8 [n, dim] E4M3FN, sigma f32 [n])."""
    x = _c(x_bf16_bits, np.uint16)
    n, dim = x.shape
    codes = np.zeros((n, dim), np.uint8)
    sigma = np.zeros(n, np.float32)
    lib().orc_quant_index_fp8(_p(x, _u16p), n, dim, _p(codes, _u8p), _p(sigma, _f32p))
    return codes, sigma


# ---------------------------------------------------------------- indexer
def indexer_scores(q, w, k, sigma, relu: bool = True) -> np.ndarray:
    """q uint8 [HI, DI], w f32 [HI], k uint8 [n, DI], sigma f32 [n] -> f64 [n]."""
    q = _c(q, np.uint8)
    w = _c(w, np.float32)
    k = _c(k, np.uint8)
    sigma = _c(sigma, np.float32)
    n = k.shape[0]
    out = np.zeros(n, np.float64)
    lib().orc_indexer_scores(_p(q, _u8p), _p(w, _f32p), q.shape[0], q.shape[1], _p(k, _u8p),
                             _p(sigma, _f32p), n, 1 if relu else 0, _p(out, _f64p))
    return out


def topk(scores, n_valid: int, k: int) -> np.ndarray:
    s = _c(scores, np.float64)
    out = np.full(max(k, 0), -1, np.int32)
    if k > 0:
        lib().orc_topk(_p(s, _f64p), int(n_valid), int(k), _p(out, _i32p))
    return out


def pool_topk(scores, pool, k: int) -> np.ndarray:
    """Top-k of a candidate pool: scores f64 [n], pool int32 token indices [n] (-1 skipped)."""
    s = _c(scores, np.float64)
    p = _c(pool, np.int32)
    out = np.full(max(k, 0), -1, np.int32)
    if k > 0:
        lib().orc_pool_topk(_p(s, _f64p), _p(p, _i32p), len(p), int(k), _p(out, _i32p))
    return out


def pool_reindex(q, w, kidx, ksig, pool, k: int) -> np.ndarray:
    """A Reindex layer under the hierarchical sparse indexer: score only the
    pool's tokens (kidx uint8 [T, DI], ksig f32 [T] of the owner's cache) with
    this layer's q, w, then take the pool top-k."""
    pool = _c(pool, np.int32)
    valid = pool[pool >= 0]
    s = indexer_scores(q, w, kidx[valid], ksig[valid]) if len(valid) else np.zeros(0)
    return pool_topk(s, valid, k)


# ---------------------------------------------------------------- context-parallel merges
def merge_topk_candidates(scores: Sequence[np.ndarray], idx: Sequence[np.ndarray], k: int) -> np.ndarray:
    """Global top-k from per-shard candidate lists (scores f64, global token
    indices int32, -1 entries skipped): the k best of their union by (score
    desc, token index asc), ascending, -1 padded. Each shard's own top-k holds
    every one of its positions that belongs to the global top-k, so this is
    the top-k of the whole context (plan of the scope table's multi-GPU part)."""
    s = np.concatenate([np.asarray(x, np.float64) for x in scores]) if scores else np.zeros(0)
    p = np.concatenate([np.asarray(x, np.int32) for x in idx]) if idx else np.zeros(0, np.int32)
    return pool_topk(s, p, k)


def lse_merge(outs: Sequence[np.ndarray], lses: Sequence[np.ndarray]) -> Tuple[np.ndarray, np.ndarray]:
    """One softmax over the union of disjoint key sets from per-shard
    results: o = sum_r exp(lse_r - L) o_r, lse = L = log sum_r exp(lse_r)
    (a shard with no key has lse = -inf and weight 0). fp64."""
    o = np.stack([np.asarray(x, np.float64) for x in outs])       # [G, H, D]
    l = np.stack([np.asarray(x, np.float64) for x in lses])       # [G, H]
    m = l.max(axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    wts = np.where(np.isfinite(l), np.exp(l - m_safe[None]), 0.0)
    tot = wts.sum(axis=0)
    out = np.where(tot[:, None] > 0, (wts[:, :, None] * o).sum(axis=0) / np.where(tot > 0, tot, 1.0)[:, None], 0.0)
    lse = np.where(tot > 0, m_safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    return out, lse


# ---------------------------------------------------------------- attention
def sparse_attn(q_bits, codes, scales, idx, swa_bits, softmax_scale: float
                ) -> Tuple[np.ndarray, np.ndarray]:
    """One query token: q uint16 [H, D]; cache codes/scales of one sequence;
    idx int32 [k]; swa uint16 [n_swa, D] -> (o f64 [H, D], lse f64 [H])."""
    q = _c(q_bits, np.uint16)
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    idx = _c(idx, np.int32)
    swa = _c(swa_bits, np.uint16).reshape(-1, q.shape[1])
    h, d = q.shape
    o = np.zeros((h, d), np.float64)
    lse = np.zeros(h, np.float64)
    lib().orc_sparse_attn(_p(q, _u16p), h, d, _p(codes, _u8p), _p(scales, _u8p), codes.shape[0],
                          _p(idx, _i32p), len(idx), _p(swa, _u16p), swa.shape[0],
                          float(softmax_scale), _p(o, _f64p), _p(lse, _f64p))
    return o, lse


# ---------------------------------------------------------------- modes
MODE_CODE = {"F": 0, "R": 1, "U": 2}


def plan(modes: Sequence[str]) -> Tuple[List[int], List[int]]:
    """Per layer (kv_owner, index_src); raises ValueError on an invalid plan."""
    n = len(modes)
    m = (ctypes.c_int * n)(*[MODE_CODE[x] for x in modes])
    own = (ctypes.c_int * n)()
    src = (ctypes.c_int * n)()
    rc = lib().orc_plan(m, n, own, src)
    if rc != 0:
        raise ValueError(f"invalid plan: layer {-1 - rc} has no Full layer before it")
    return list(own), list(src)


# ---------------------------------------------------------------- one decode step
def bf16_bits(t) -> np.ndarray:
    """torch bf16 tensor (any device) -> numpy uint16 bits."""
    import torch
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def decode_group(q_tokens: int, modes: Sequence[str], seqs: Sequence[int], lens: Sequence[int],
                 owner_cache: Dict[int, Dict[int, dict]], layer_in: Dict[int, dict], top_k: int,
                 softmax_scale: float, queries: Sequence[int] = None,
                 pool_size: int = None) -> Dict[int, dict]:
    """Run the whole layer group for the given sequences and query tokens.

    owner_cache[owner][b] = {"codes": [T,288], "scales": [T,36], "kidx": [T,64],
                             "ksig": [T]} (the owner's cache, logical order)
    layer_in[layer][b] = {"q": uint16 [Sq,16,576], "swa": uint16 [W+Sq-1,576],
                          "qidx": uint8 [Sq,4,64], "w": f32 [Sq,4]} (qidx/w for F, R)
    Returns out[layer][(b, j)] = {"idx": int32 [k], "o": f64 [16,576], "lse": f64 [16]}.
    pool_size: when given, each Full layer also keeps its top-pool_size positions
    as the candidate pool ("pool" in its output), and a Reindex layer scores only
    its KV owner's pool (hierarchical sparse indexer).
    """
    own, src = plan(modes)
    queries = range(q_tokens) if queries is None else queries
    out: Dict[int, dict] = {i: {} for i in range(len(modes))}
    W = layer_in[0][seqs[0]]["swa"].shape[0] - q_tokens + 1
    for li, mode in enumerate(modes):
        for b in seqs:
            T = lens[b]
            cache = owner_cache[own[li]][b]
            for j in queries:
                pos = T - q_tokens + j
                pool = None
                if mode == "R" and pool_size is not None:
                    idx = pool_reindex(layer_in[li][b]["qidx"][j], layer_in[li][b]["w"][j], cache["kidx"],
                                       cache["ksig"], out[own[li]][(b, j)]["pool"], top_k)
                elif mode in ("F", "R"):
                    s = indexer_scores(layer_in[li][b]["qidx"][j], layer_in[li][b]["w"][j],
                                       cache["kidx"][:pos + 1], cache["ksig"][:pos + 1])
                    idx = topk(s, pos + 1, top_k)
                    if mode == "F" and pool_size is not None:
                        pool = topk(s, pos + 1, pool_size)
                else:
                    idx = out[src[li]][(b, j)]["idx"]
                # SWA rows j .. j+W-1 hold positions pos-W+1 .. pos; skip negatives.
                first_pos = T - (W + q_tokens - 1)
                rows = [r for r in range(j, j + W) if first_pos + r >= 0]
                swa = layer_in[li][b]["swa"][rows] if rows else np.zeros((0, 576), np.uint16)
                o, lse = sparse_attn(layer_in[li][b]["q"][j], cache["codes"], cache["scales"],
                                     idx, swa, softmax_scale)
                out[li][(b, j)] = {"idx": idx, "o": o, "lse": lse}
                if pool is not None:
                    out[li][(b, j)]["pool"] = pool
    return out
