"""Indexer scores element by element, and the paths into and around the
indexer, against the oracle:
  * integer E4M3 inputs (sigma = 1, and power-of-two sigma): every score of
    every position up to the query equals the oracle's fp64 score exactly,
    and the top-k indices are bit-exact;
  * bf16 keys and queries quantised by csa2_quant_indexer_fp8, appended by
    csa2_quant_kv_fp4 and scored by csa2_indexer_topk: codes and sigma
    bit-exact, scores within the stated fp32 bound, the selection exactly the
    top-k of the scores as computed, and valid against the exact scores;
  * the hierarchical sparse indexer through LayerGroup(pool_size) on a
    Full -> Reindex -> Reuse group against oracle.decode_group(pool_size);
  * a pool with 4 query tokens (causal bound per query)."""
import math

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_attention_quant_b200 import inputs
from oracle_check import assert_attn_close

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(576)
# Bound on |computed - exact| of a score whose inputs are not small integers:
# a relative 2^-12 of sum_h w_h * sigma_t * sum_c |q_hc * k_tc| (the FP8 dot
# products accumulate in fp32 in the tensor core; the bound leaves room for
# an accumulator narrower than binary32, and the epilogue adds 6 roundings).
SCORE_REL_BOUND = 2.0 ** -12


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from compressed_sparse_attention_quant_b200 import lib as L
    return L


def build_cache(lib, kidx: np.ndarray, ksig: np.ndarray, lens, seed=0):
    """A paged cache holding indexer keys kidx [B, T, 64] (E4M3 bytes) and
    scales ksig [B, T] at a random page placement; KV latent zero."""
    B, Tm = kidx.shape[0], kidx.shape[1]
    mp = -(-Tm // 64)
    g = torch.Generator().manual_seed(seed)
    pt = torch.randperm(B * mp, generator=g).view(B, mp).to(torch.int32).cuda()
    cache = lib.PagedCache(B * mp)
    for b in range(B):
        T = lens[b]
        pos = torch.arange(T, device="cuda")
        slots = lib.slot_mapping(pt, b, pos)
        x = torch.zeros(T, 576, dtype=torch.bfloat16, device="cuda")
        lib.quant_kv_fp4(x, slots, cache, torch.from_numpy(np.ascontiguousarray(kidx[b, :T])).cuda(),
                         torch.from_numpy(np.ascontiguousarray(ksig[b, :T])).cuda())
    return cache, pt, torch.tensor(lens, dtype=torch.int32, device="cuda")


def small_int_e4m3(rng, shape):
    v = rng.integers(-8, 9, shape).astype(np.float32)
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def run_indexer(lib, q, w, cache, pt, lens_t, k):
    B, Sq = q.shape[0], q.shape[1]
    mp = pt.shape[1]
    ws = lib.workspace(lib.indexer_topk_workspace_bytes(B, Sq, mp, k))
    out = lib.indexer_topk(torch.from_numpy(q).cuda(), torch.from_numpy(w).cuda(), cache, pt, lens_t, k, ws=ws)
    assert lib.last_device_error() == 0
    sc = lib.indexer_scores_in_workspace(ws, B, Sq, mp).cpu().numpy().astype(np.float64)
    return out.cpu().numpy(), sc


@pytest.mark.parametrize("pow2_sigma", [False, True], ids=["sigma1", "sigma_pow2"])
def test_integer_scores_exact_elementwise(lib, pow2_sigma):
    rng = np.random.default_rng(7 + pow2_sigma)
    B, Sq, lens, k = 3, 2, [5000, 1300, 70], 300
    T = max(lens)
    kidx = small_int_e4m3(rng, (B, T, 64))
    ksig = (np.exp2(rng.integers(-3, 4, (B, T))) if pow2_sigma else np.ones((B, T))).astype(np.float32)
    q = small_int_e4m3(rng, (B, Sq, 4, 64))
    w = np.array([0.25, 0.5, 1.0, 2.0], np.float32)[rng.integers(0, 4, (B, Sq, 4))]
    cache, pt, lens_t = build_cache(lib, kidx, ksig, lens, seed=1)
    idx, sc = run_indexer(lib, q, w, cache, pt, lens_t, k)
    n_neg = 0
    for b in range(B):
        for j in range(Sq):
            pos = lens[b] - Sq + j
            want = oracle.indexer_scores(q[b, j], w[b, j], kidx[b, :pos + 1], ksig[b, :pos + 1])
            np.testing.assert_array_equal(sc[b, j, :pos + 1], want, err_msg=f"scores b {b} j {j}")
            np.testing.assert_array_equal(idx[b, j], oracle.topk(want, pos + 1, k), err_msg=f"idx b {b} j {j}")
            n_neg += int((oracle.indexer_scores(q[b, j], w[b, j], kidx[b, :pos + 1], ksig[b, :pos + 1],
                                                relu=False) < 0).sum())
    assert n_neg > 0                        # the ReLU was exercised


def test_fp8_quantised_inputs_through_the_indexer(lib):
    """bf16 -> csa2_quant_indexer_fp8 -> csa2_quant_kv_fp4 -> csa2_indexer_topk."""
    rng = np.random.default_rng(21)
    B, Sq, lens, k = 2, 2, [4000, 1500], 256
    T = max(lens)
    kx = (rng.standard_normal((B, T, 64)) * np.exp2(rng.uniform(-3, 3, (B, T, 1)))).astype(np.float32)
    qx = rng.standard_normal((B, Sq, 4, 64)).astype(np.float32)
    kb = torch.from_numpy(kx).to(torch.bfloat16)
    qb = torch.from_numpy(qx).to(torch.bfloat16)
    kc, ks = lib.quant_indexer_fp8(kb.cuda())
    qc, qs = lib.quant_indexer_fp8(qb.cuda())
    assert lib.last_device_error() == 0
    kc, ks, qc, qs = kc.cpu().numpy(), ks.cpu().numpy(), qc.cpu().numpy(), qs.cpu().numpy()
    rkc, rks = oracle.quant_index_fp8(oracle.bf16_bits(kb).reshape(-1, 64))
    rqc, rqs = oracle.quant_index_fp8(oracle.bf16_bits(qb).reshape(-1, 64))
    np.testing.assert_array_equal(kc.reshape(-1, 64), rkc)
    np.testing.assert_array_equal(ks.reshape(-1).view(np.uint32), rks.view(np.uint32))
    np.testing.assert_array_equal(qc.reshape(-1, 64), rqc)
    np.testing.assert_array_equal(qs.reshape(-1).view(np.uint32), rqs.view(np.uint32))
    w = np.array([0.25, 0.5, 1.0, 2.0], np.float32)[rng.integers(0, 4, (B, Sq, 4))]
    w_eff = (w * qs).astype(np.float32)                   # the query scale folds into the head weight
    cache, pt, lens_t = build_cache(lib, kc, ks, lens, seed=2)
    idx, sc = run_indexer(lib, qc, w_eff, cache, pt, lens_t, k)
    ev = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    worst = 0.0
    for b in range(B):
        for j in range(Sq):
            pos = lens[b] - Sq + j
            exact = oracle.indexer_scores(qc[b, j], w_eff[b, j], kc[b, :pos + 1], ks[b, :pos + 1])
            mag = np.abs(ev[kc[b, :pos + 1]]) @ np.abs(ev[qc[b, j]]).T          # [t, h] sum_c |q k|
            bound = SCORE_REL_BOUND * (mag * w_eff[b, j][None, :]).sum(axis=1) * ks[b, :pos + 1]
            got = sc[b, j, :pos + 1]
            err = np.abs(got - exact)
            assert np.all(err <= bound), f"b {b} j {j}: score error {err.max():.3e}"
            worst = max(worst, float((err / np.maximum(bound / SCORE_REL_BOUND, 1e-300)).max()))
            # the selection is exactly the top-k of the scores as computed
            np.testing.assert_array_equal(idx[b, j], oracle.topk(got, pos + 1, k), err_msg=f"b {b} j {j}")
            # and valid against the exact scores: sure winners in, sure losers out
            theta = np.sort(exact)[::-1][k - 1]
            band = 2 * bound.max()
            sel = np.zeros(pos + 1, bool)
            sel[idx[b, j]] = True
            assert np.all(sel[exact > theta + band]) and np.all(exact[sel] >= theta - band)
    print(f"worst relative score error: {worst:.3e} (bound {SCORE_REL_BOUND:.3e})")


def test_layer_group_with_candidate_pool_matches_oracle(lib):
    from compressed_sparse_attention_quant_b200 import workload
    wl = inputs.small_workload("poolgroup", 3, 2, [3000, 1700, 600], 96, modes=("F", "R", "U"), seed=31)
    C = 400
    dw = workload.DeviceWorkload(wl, pool_size=C)
    dw.step()
    assert lib.last_device_error() == 0
    own, _ = oracle.plan(wl.modes)
    owner_cache, layer_in = {}, {}
    for o in set(own):
        owner_cache[o] = {}
        for b in range(wl.batch):
            T = wl.lens()[b]
            # the inputs are drawn on the device the workload was built on
            kv = torch.cat([r for _, r in inputs.kv_chunks(wl, o, b, dw.device)])
            codes, scales = oracle.quant_fp4(oracle.bf16_bits(kv[:T]))
            owner_cache[o][b] = {"codes": codes, "scales": scales,
                                 "kidx": inputs.kidx_rows(wl, o, b, 0, T, dw.device).cpu().numpy(),
                                 "ksig": inputs.kidx_scale_rows(wl, o, b, 0, T, dw.device).cpu().numpy()}
    for li, m in enumerate(wl.modes):
        layer_in[li] = {}
        for b in range(wl.batch):
            d = {"q": oracle.bf16_bits(dw.q[li][b]), "swa": oracle.bf16_bits(dw.swa[li][b])}
            if m in ("F", "R"):
                d["qidx"] = dw.q_idx[li][b].cpu().numpy()
                d["w"] = dw.w[li][b].cpu().numpy()
            layer_in[li][b] = d
    ref = oracle.decode_group(wl.q_tokens, wl.modes, list(range(wl.batch)), wl.lens(), owner_cache, layer_in,
                              wl.top_k, SCALE, pool_size=C)
    g = dw.group
    pool0 = g.pool(0).cpu().numpy()
    for li in range(len(wl.modes)):
        idx = g.index(li).cpu().numpy()
        o, lse = g.out[li].cpu().numpy(), g.lse[li].cpu().numpy()
        for b in range(wl.batch):
            for j in range(wl.q_tokens):
                r = ref[li][(b, j)]
                if li == 0:
                    np.testing.assert_array_equal(pool0[b, j], r["pool"], err_msg=f"pool b {b} j {j}")
                np.testing.assert_array_equal(idx[b, j], r["idx"], err_msg=f"layer {li} b {b} j {j}")
                assert_attn_close(o[b, j], lse[b, j], r["o"], r["lse"], f"layer {li} b {b} j {j}")


def test_pool_with_four_query_tokens_is_causal_per_query(lib):
    """Sq = 4: each query's pool is its own Full top-C, and an entry after a
    query's position (planted in a copy of the pool) is flagged and skipped."""
    from compressed_sparse_attention_quant_b200 import workload
    wl = inputs.small_workload("pool_sq4", 2, 4, [2200, 900], 100, modes=("F", "R"), seed=41)
    dw = workload.DeviceWorkload(wl)
    dw.step()
    cache = dw.group.cache(0)
    pool = lib.indexer_topk(dw.q_idx[0], dw.w[0], cache, dw.page_table, dw.seq_lens, 500)
    out = lib.indexer_pool_topk(dw.q_idx[1], dw.w[1], cache, dw.page_table, dw.seq_lens, pool, 100)
    assert lib.last_device_error() == 0
    ph, oh = pool.cpu().numpy(), out.cpu().numpy()
    for b in range(2):
        T = wl.lens()[b]
        kid = inputs.kidx_rows(wl, 0, b, 0, T, dw.device).cpu().numpy()
        ks = inputs.kidx_scale_rows(wl, 0, b, 0, T, dw.device).cpu().numpy()
        for j in range(4):
            assert ph[b, j].max() <= T - 4 + j
            want = oracle.pool_reindex(dw.q_idx[1][b, j].cpu().numpy(), dw.w[1][b, j].cpu().numpy(), kid, ks,
                                       ph[b, j], 100)
            np.testing.assert_array_equal(oh[b, j], want, err_msg=f"b {b} j {j}")
    # query 0 of sequence 0 is at T - 4: the future position T - 1 is out of range
    bad = pool.clone()
    T0 = wl.lens()[0]
    bad[0, 0, -1] = T0 - 1
    bad[0, 0] = torch.sort(bad[0, 0]).values
    out2 = lib.indexer_pool_topk(dw.q_idx[1], dw.w[1], cache, dw.page_table, dw.seq_lens, bad, 100)
    assert lib.last_device_error() == 6                     # CSA2_ERR_DEVICE_BOUNDS
    assert (out2[0, 0] == T0 - 1).sum().item() == 0
