"""The N > 1 host path on CPU: two gloo ranks run the replica logic the
benchmark uses under torchrun (independent replicas with their own seeds,
timings reduced to the maximum over ranks, whole-job throughput, rank 0
alone reports). The decode path itself has no exchange step, so no
collective is on the data path; only the timing scalars are reduced."""
import datetime
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

WORLD = 2


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, port: int, out):
    import torch.distributed as dist

    from compressed_sparse_attention_quant_b200 import inputs, replicas

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        wl = inputs.small_workload("multirank", 2, 1, [300, 200], 32, modes=("F",))
        wr = replicas.replica_workload(wl, rank)
        q = inputs.attn_query(wr, 0, "cpu")
        kid = inputs.kidx_rows(wr, 0, 0, 0, 64, "cpu")
        sample = (float(q.float().sum()), int(kid.to(torch.int32).sum()))
        shapes = (tuple(q.shape), tuple(kid.shape))
        # per-rank device times (step, indexer, end to end) that differ by rank
        mx = replicas.max_over_ranks([1.0 + rank, 10.0 - rank, 5.0 + 0.5 * rank], dist)
        value = replicas.job_throughput(wl.batch * wl.q_tokens, WORLD, mx[0])
        out.put((rank, wr.seed, sample, shapes, mx, value, replicas.reports(rank)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_run_independent_replicas():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, out)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank did not finish"
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(out.get(timeout=10) for _ in range(WORLD))
    (r0, s0, x0, sh0, m0, v0, p0), (r1, s1, x1, sh1, m1, v1, p1) = res
    assert (r0, r1) == (0, 1)
    assert s0 != s1 and x0 != x1              # independent replicas: own seeds, different data
    assert sh0 == sh1                         # same per-rank shapes (weak scaling)
    assert m0 == m1 == [2.0, 10.0, 5.5]       # every rank sees the maximum over ranks
    assert v0 == v1 == pytest.approx(2 * WORLD / 2e-3)
    assert (p0, p1) == (True, False)          # rank 0 alone reports


def test_replica_of_rank0_is_the_workload():
    from compressed_sparse_attention_quant_b200 import inputs, replicas
    wl = inputs.WORKLOADS["decode_b64_t128k"]
    assert replicas.replica_workload(wl, 0) is wl
    r3 = replicas.replica_workload(wl, 3)
    assert r3.seed == wl.seed + 3 * replicas.SEED_STRIDE and r3.batch == wl.batch and r3.context == wl.context
    assert replicas.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
