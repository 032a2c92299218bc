"""Context-parallel decode (one long sequence split over ranks): the
exchange of compressed_sparse_attention_quant_b200.context_parallel on two
gloo ranks on CPU, with the per-shard steps done by the oracle, against the
unsharded oracle: top-k indices bit-exact, attention equal to fp64 rounding.
The kernels of the same steps are checked on one GPU by
tests/test_gpu_context_parallel.py."""
import math
import os

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SCALE = 1.0 / math.sqrt(576)
LENS = [1500, 1333]
K = 96


def make_inputs():
    """Integer indexer inputs, FP4 cache codes and window rows for 2 sequences (CPU)."""
    import oracle
    g = torch.Generator().manual_seed(3)
    B, T = len(LENS), max(LENS)
    kidx = torch.randint(-8, 9, (B, T, 64), generator=g).float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    qidx = torch.randint(-8, 9, (B, 1, 4, 64), generator=g).float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    w = torch.tensor([0.25, 0.5, 1.0, 2.0])[torch.randint(0, 4, (B, 1, 4), generator=g)].numpy().astype(np.float32)
    kv = oracle.bf16_bits(torch.randn(B * T, 576, generator=g).to(torch.bfloat16)).reshape(B, T, 576)
    codes, scales = oracle.quant_fp4(kv.reshape(-1, 576))
    q = oracle.bf16_bits(torch.randn(B, 1, 16, 576, generator=g).to(torch.bfloat16))
    swa = oracle.bf16_bits(torch.randn(B, 128, 576, generator=g).to(torch.bfloat16))
    return kidx, qidx, w, codes.reshape(B, T, 288), scales.reshape(B, T, 36), q, swa


class OracleOps:
    """The per-shard steps of context_parallel.decode_step done by the oracle
    on the shard's own positions (CPU tensors in and out)."""

    def __init__(self, data, g, G):
        import oracle
        from compressed_sparse_attention_quant_b200 import context_parallel as cp
        self.o = oracle
        self.kidx, self.qidx, self.w, self.codes, self.scales, self.q, self.swa = data
        self.lo, self.hi = cp.shard_bounds(max(LENS), G, g)
        self.last = g == G - 1

    def local_candidates(self, shard, q_idx, w):
        sc = np.full((len(LENS), K), -np.inf, np.float32)
        gi = np.full((len(LENS), K), -1, np.int32)
        for b, T in enumerate(LENS):
            n = min(T, self.hi) - self.lo
            s = self.o.indexer_scores(self.qidx[b, 0], self.w[b, 0], self.kidx[b, self.lo:self.lo + n],
                                      np.ones(n, np.float32))
            idx = self.o.topk(s, n, K)
            sc[b] = np.where(idx >= 0, s[np.maximum(idx, 0)], -np.inf)
            gi[b] = np.where(idx >= 0, idx + self.lo, -1)
        return torch.from_numpy(sc), torch.from_numpy(gi)

    def own_entries(self, shard, all_scores, all_idx):
        out = np.full((len(LENS), K), -1, np.int32)
        for b in range(len(LENS)):
            glob = self.o.merge_topk_candidates([x[b].numpy().astype(np.float64) for x in all_scores],
                                                [x[b].numpy() for x in all_idx], K)
            out[b] = np.where((glob >= self.lo) & (glob < self.hi), glob - self.lo, -1)
        return torch.from_numpy(out)

    def attend(self, shard, q, swa, local_idx):
        o = np.zeros((len(LENS), 16, 576))
        l = np.zeros((len(LENS), 16))
        for b, T in enumerate(LENS):
            n = min(T, self.hi) - self.lo
            rows = self.swa[b] if self.last else np.zeros((0, 576), np.uint16)
            o[b], l[b] = self.o.sparse_attn(self.q[b, 0], self.codes[b, self.lo:self.lo + n],
                                            self.scales[b, self.lo:self.lo + n], local_idx[b].numpy(), rows, SCALE)
        return torch.from_numpy(o), torch.from_numpy(l)

    def combine(self, all_o, all_lse):
        o = np.zeros((len(LENS), 16, 576))
        l = np.zeros((len(LENS), 16))
        for b in range(len(LENS)):
            o[b], l[b] = self.o.lse_merge([x[b].numpy() for x in all_o], [x[b].numpy() for x in all_lse])
        return torch.from_numpy(o), torch.from_numpy(l)


def _rank(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from compressed_sparse_attention_quant_b200 import context_parallel as cp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        data = make_inputs()
        ops = OracleOps(data, rank, world)
        shard = cp.Shard(rank, world, ops.lo, ops.hi, torch.zeros(1, 1, dtype=torch.int32),
                         torch.zeros(1, dtype=torch.int32))
        o, l = cp.decode_step(shard, ops, None, None, None, None, cp.dist_all_gather())
        q.put((rank, o.numpy(), l.numpy()))
    except Exception as e:                      # report instead of leaving the parent waiting
        q.put((rank, repr(e), None))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_the_unsharded_oracle():
    import socket
    import oracle
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, o, l = q.get(timeout=180)
        assert l is not None, f"rank {r}: {o}"
        res[r] = (o, l)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    kidx, qidx, w, codes, scales, qb, swa = make_inputs()
    for b, T in enumerate(LENS):
        s = oracle.indexer_scores(qidx[b, 0], w[b, 0], kidx[b, :T], np.ones(T, np.float32))
        idx = oracle.topk(s, T, K)
        o_ref, l_ref = oracle.sparse_attn(qb[b, 0], codes[b, :T], scales[b, :T], idx, swa[b], SCALE)
        for r in range(2):                      # every rank ends with the whole result
            np.testing.assert_allclose(res[r][0][b], o_ref, rtol=0, atol=1e-12)
            np.testing.assert_allclose(res[r][1][b], l_ref, rtol=0, atol=1e-12)
