"""Candidate-pool top-k (hierarchical sparse indexer) against the oracle:
indices bit-exact. The pool is the Full layer's top-C from
csa2_indexer_topk; a Reindex layer's query selects inside it."""
import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_attention_quant_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from compressed_sparse_attention_quant_b200 import lib, workload
    return lib, workload


def _keys(wl, dw, b):
    T = wl.lens()[b]
    return (inputs.kidx_rows(wl, 0, b, 0, T, dw.device).cpu().numpy(),
            inputs.kidx_scale_rows(wl, 0, b, 0, T, dw.device).cpu().numpy())


@pytest.mark.parametrize("C,k", [(64, 40), (700, 300), (4096, 1000)])
def test_pool_topk_matches_oracle(mods, C, k):
    lib, workload = mods
    wl = inputs.small_workload(f"pool{C}", 3, 2, [9000, 2500, 500], k, modes=("F", "R"), seed=C)
    dw = workload.DeviceWorkload(wl)
    dw.step()
    g = dw.group
    cache = g.cache(0)
    pool = lib.indexer_topk(dw.q_idx[0], dw.w[0], cache, dw.page_table, dw.seq_lens, C)
    out_r = lib.indexer_pool_topk(dw.q_idx[1], dw.w[1], cache, dw.page_table, dw.seq_lens, pool, k)
    out_f = lib.indexer_pool_topk(dw.q_idx[0], dw.w[0], cache, dw.page_table, dw.seq_lens, pool, k)
    assert lib.last_device_error() == 0
    pool_h, out_r, out_f = pool.cpu().numpy(), out_r.cpu().numpy(), out_f.cpu().numpy()
    full_idx = g.index(0).cpu().numpy()
    for b in range(3):
        kid, ks = _keys(wl, dw, b)
        for j in range(2):
            want = oracle.pool_reindex(dw.q_idx[1][b, j].cpu().numpy(), dw.w[1][b, j].cpu().numpy(), kid, ks,
                                       pool_h[b, j], k)
            np.testing.assert_array_equal(out_r[b, j], want, err_msg=f"b {b} j {j}")
            # the Full layer's own query over its own pool gives its top-k
            np.testing.assert_array_equal(out_f[b, j], full_idx[b, j], err_msg=f"full b {b} j {j}")


def test_pool_topk_ties_and_padding(mods):
    """A zero query makes every pool score 0: the k lowest pool tokens win.
    Rows whose pool holds fewer than k valid entries are -1 padded."""
    lib, workload = mods
    wl = inputs.small_workload("poolties", 2, 1, [3000, 90], 64, modes=("F", "R"), seed=3)
    dw = workload.DeviceWorkload(wl)
    dw.step()
    cache = dw.group.cache(0)
    pool = lib.indexer_topk(dw.q_idx[0], dw.w[0], cache, dw.page_table, dw.seq_lens, 200)
    q0 = torch.zeros_like(dw.q_idx[1])
    out = lib.indexer_pool_topk(q0, dw.w[1], cache, dw.page_table, dw.seq_lens, pool, 120).cpu().numpy()
    assert lib.last_device_error() == 0
    p = pool.cpu().numpy()
    np.testing.assert_array_equal(out[0, 0], p[0, 0][:120])
    valid = p[1, 0][p[1, 0] >= 0]
    assert len(valid) == 90
    np.testing.assert_array_equal(out[1, 0][:90], valid)
    assert np.all(out[1, 0][90:] == -1)
