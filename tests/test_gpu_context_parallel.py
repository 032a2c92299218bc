"""Context-parallel decode kernels on one GPU: the candidate merge
(csa2_topk_merge) against oracle.merge_topk_candidates on tie-heavy scores,
the LSE merge (csa2_lse_merge) against oracle.lse_merge, and the 1M-context
workload split over 2 logical shards (sliced page tables over one cache)
against the unsharded oracle: global top-k bit-exact, attention within
max-abs 2e-3 / rel-L2 1e-3."""
import math

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_attention_quant_b200 import inputs
from oracle_check import OracleRun, assert_attn_close

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(576)


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from compressed_sparse_attention_quant_b200 import lib as L
    return L


@pytest.mark.parametrize("G,ks,k", [(2, 64, 64), (4, 300, 250), (8, 2048, 2048)])
def test_topk_merge_matches_oracle(lib, G, ks, k):
    rng = np.random.default_rng(G * 1000 + ks)
    R = 5
    span = 100000
    sc = np.zeros((G, R, ks), np.float32)
    gi = np.full((G, R, ks), -1, np.int32)
    for g in range(G):
        for r in range(R):
            n = ks if (g + r) % 3 else ks // 2                       # some lists -1 padded
            pos = np.sort(rng.choice(span, n, replace=False)).astype(np.int32) + g * span
            gi[g, r, :n] = pos
            sc[g, r, :n] = rng.integers(0, 40, n).astype(np.float32) / 4      # heavy ties
            sc[g, r, n:] = -np.inf
    lo, hi = span, 2 * span
    out, local = lib.topk_merge(torch.from_numpy(sc).cuda(), torch.from_numpy(gi).cuda(), k, lo, hi,
                                want_global=True, want_local=True)
    assert lib.last_device_error() == 0
    out, local = out.cpu().numpy(), local.cpu().numpy()
    for r in range(R):
        want = oracle.merge_topk_candidates([sc[g, r].astype(np.float64) for g in range(G)],
                                            [gi[g, r] for g in range(G)], k)
        np.testing.assert_array_equal(out[r], want, err_msg=f"row {r}")
        np.testing.assert_array_equal(local[r], np.where((want >= lo) & (want < hi), want - lo, -1))


def test_lse_merge_matches_oracle(lib):
    rng = np.random.default_rng(3)
    P, R = 3, 4
    o = rng.standard_normal((P, R, 16, 576)).astype(np.float32)
    lse = (rng.standard_normal((P, R, 16)) * 5).astype(np.float32)
    lse[1, 2, :] = -np.inf                                            # an empty part
    lse[:, 3, 5] = -np.inf                                            # no key at all for one head
    out, l = lib.lse_merge(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda())
    out, l = out.cpu().numpy(), l.cpu().numpy()
    for r in range(R):
        ro, rl = oracle.lse_merge([o[p, r].astype(np.float64) for p in range(P)],
                                  [lse[p, r].astype(np.float64) for p in range(P)])
        np.testing.assert_allclose(out[r], ro, rtol=0, atol=2e-6)
        np.testing.assert_array_equal(np.isfinite(l[r]), np.isfinite(rl))
        fin = np.isfinite(rl)
        np.testing.assert_allclose(l[r][fin], rl[fin], rtol=0, atol=2e-5)


@pytest.mark.slow
def test_long_context_on_two_logical_shards(lib):
    from compressed_sparse_attention_quant_b200 import context_parallel as cp
    from compressed_sparse_attention_quant_b200 import workload
    wl = inputs.WORKLOADS["long_b4_t1m"]
    dw = workload.DeviceWorkload(wl)
    dw.step()                                        # the unsharded step (also appends the new token)
    g = dw.group
    shards = [cp.make_shard(dw.page_table, dw.seq_lens, 2, s) for s in range(2)]
    ops_for = lambda s: cp.GpuOps(lib, g.cache(0), wl.top_k, SCALE)     # noqa: E731
    # global top-k of the merge, per shard view
    cands = [ops_for(s).local_candidates(s, dw.q_idx[0], dw.w[0]) for s in shards]
    glob, _ = lib.topk_merge(torch.stack([c[0] for c in cands]), torch.stack([c[1] for c in cands]), wl.top_k)
    o, lse = cp.decode_step_in_process(shards, ops_for, dw.q[0], dw.q_idx[0], dw.w[0], dw.swa[0])
    assert lib.last_device_error() == 0
    ref = OracleRun(dw, range(wl.batch))
    glob = glob.cpu().numpy()
    o, lse = o.cpu().numpy(), lse.cpu().numpy()
    idx_unsharded = g.index(0).cpu().numpy()
    for b in range(wl.batch):
        r = ref.out[0][(b, 0)]
        np.testing.assert_array_equal(glob[b], r["idx"], err_msg=f"b {b}")
        np.testing.assert_array_equal(glob[b], idx_unsharded[b, 0])
        assert_attn_close(o[b], lse[b], r["o"], r["lse"], f"sharded b {b}")
