"""LayerGroup host wiring (CPU): which library call each layer makes and which
buffers it passes, with and without the candidate pool. The device calls are
replaced by recorders; the plan comes from the real library's csa2_plan."""
import pytest
import torch

from compressed_sparse_attention_quant_b200 import group, lib


class _Cache:
    def __init__(self, num_pages, device="cpu"):
        self.num_pages = num_pages


@pytest.fixture
def rec(monkeypatch):
    calls = []
    monkeypatch.setattr(lib, "PagedCache", _Cache)
    monkeypatch.setattr(lib, "workspace", lambda n, device="cpu": torch.empty(max(int(n), 256), dtype=torch.uint8))
    monkeypatch.setattr(lib, "sparse_attn_workspace_bytes", lambda B, Sq, k: 1024)
    monkeypatch.setattr(lib, "indexer_topk",
                        lambda q, w, cache, pt, sl, k, out=None, ws=None: calls.append(("topk", q, cache, k, out)))
    monkeypatch.setattr(lib, "indexer_pool_topk",
                        lambda q, w, cache, pt, sl, pool, k, out=None: calls.append(("pool", q, cache, pool, k, out)))
    monkeypatch.setattr(lib, "sparse_attn_decode",
                        lambda q, cache, pt, sl, idx, swa, scale, out=None, lse=None, ws=None:
                        calls.append(("attn", q, cache, idx)))
    monkeypatch.setattr(lib, "quant_kv_fp4", lambda *a, **k: calls.append(("quant",)))
    return calls


def _inputs(n):
    q = [torch.full((1,), float(i)) for i in range(n)]
    q_idx = {i: torch.full((1,), float(10 + i)) for i in range(n)}
    w = {i: torch.ones(1) for i in range(n)}
    return q, q_idx, w


def test_pool_wiring_full_reindex_reuse(rec):
    modes = ("F", "R", "U", "R", "F", "R")
    g = group.LayerGroup(modes, 2, 1, 4, 8, top_k=4, device="cpu", pool_size=16)
    q, q_idx, w = _inputs(len(modes))
    g.step(None, None, q, [None] * len(modes), q_idx, w)
    kinds = [c[0] for c in rec]
    assert kinds == ["topk", "pool", "attn", "pool", "attn", "attn", "pool", "attn",
                     "topk", "pool", "attn", "pool", "attn"]
    # Full layer 0: its top-16 pool, then its top-4 inside that pool
    assert rec[0][3] == 16 and rec[0][4] is g._pool[0]
    assert rec[1][1] is q_idx[0] and rec[1][3] is g._pool[0] and rec[1][4] == 4 and rec[1][5] is g._index[0]
    # Reindex layers read their KV owner's pool with their own query
    assert rec[3][1] is q_idx[1] and rec[3][3] is g._pool[0] and rec[3][5] is g._index[1]
    assert rec[6][1] is q_idx[3] and rec[6][3] is g._pool[0]
    assert rec[9][1] is q_idx[4] and rec[9][3] is g._pool[4] and rec[11][3] is g._pool[4]
    assert rec[11][2] is g.caches[4]
    # Reuse attends with the Full layer's index tensor (alias, no copy)
    assert rec[5][3] is g._index[0]


def test_without_pool_every_indexing_layer_scans(rec):
    modes = ("F", "R", "U")
    g = group.LayerGroup(modes, 2, 1, 4, 8, top_k=4, device="cpu")
    q, q_idx, w = _inputs(3)
    g.step(None, None, q, [None] * 3, q_idx, w)
    assert [c[0] for c in rec] == ["topk", "attn", "topk", "attn", "attn"]
    assert rec[0][3] == 4 and rec[2][1] is q_idx[1] and rec[2][4] is g._index[1]


def test_pool_must_hold_top_k(rec):
    with pytest.raises(ValueError):
        group.LayerGroup(("F", "R"), 1, 1, 4, 8, top_k=64, device="cpu", pool_size=32)


def test_step_graph_runs_one_eager_step_then_captures_one(rec, monkeypatch):
    """StepGraph (CPU, CUDA graph API replaced by recorders): one eager step
    first (library set-up outside the capture), then exactly one step inside a
    thread-local capture; the launches counted during the capture are the
    kernels per replay, and replay() only replays the graph."""
    events = []
    counter = {"n": 0}

    class _Graph:
        def replay(self):
            events.append("replay")

    class _Capture:
        def __init__(self, graph, capture_error_mode="global"):
            events.append(("capture", capture_error_mode))

        def __enter__(self):
            events.append("enter")

        def __exit__(self, *exc):
            events.append("exit")
            return False

    def counting(kind):
        def f(*a, **k):
            counter["n"] += 3 if kind == "topk" else 2
            rec.append((kind,))
            events.append(kind)
        return f

    monkeypatch.setattr(torch.cuda, "CUDAGraph", _Graph)
    monkeypatch.setattr(torch.cuda, "graph", _Capture)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: events.append("sync"))
    monkeypatch.setattr(lib, "launch_count", lambda: counter["n"])
    monkeypatch.setattr(lib, "indexer_topk", counting("topk"))
    monkeypatch.setattr(lib, "sparse_attn_decode", counting("attn"))

    modes = ("F", "U")
    g = group.LayerGroup(modes, 2, 1, 4, 8, top_k=4, device="cpu")
    q, q_idx, w = _inputs(len(modes))
    sg = group.StepGraph(g, None, None, q, [None] * len(modes), q_idx, w)
    # eager step, sync, capture (thread-local) of one step
    assert events == ["topk", "attn", "attn", "sync", ("capture", "thread_local"), "enter",
                      "topk", "attn", "attn", "exit"]
    assert sg.launches == 3 + 2 + 2
    events.clear()
    sg.replay()
    assert events == ["replay"]
