"""K2-K5 and the layer modes against the oracle, on small ragged workloads that
span several pages, CTAs and tiles with ragged tails: top-k indices
bit-exact, attention within max-abs 2e-3 / relative L2 1e-3."""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_attention_quant_b200 import inputs
from oracle_check import OracleRun, assert_attn_close, attend

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(576)


@pytest.fixture(scope="module")
def mods():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from compressed_sparse_attention_quant_b200 import lib, workload
    return lib, workload


SMALL = [
    # name, B, Sq, lens, k, modes
    ("one_seq", 1, 1, [4096], 512, ("F",)),
    ("ragged_b4", 4, 1, [5000, 3333, 129, 70], 300, ("F",)),
    ("ragged_sq4", 3, 4, [2500, 1000, 600], 256, ("F", "U", "R", "U")),
    ("many_chunks", 2, 1, [20000, 9000], 1000, ("F", "R", "U")),
    ("k_exceeds_len", 3, 2, [40, 90, 200], 128, ("F", "R")),
    ("tiny", 2, 1, [1, 64], 8, ("F", "U")),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_decode_group_matches_oracle(mods, case):
    lib, workload = mods
    name, B, Sq, lens, k, modes = case
    wl = inputs.small_workload(name, B, Sq, lens, k, modes=modes, random_pages=True, seed=zlib.crc32(name.encode()) % 1000)
    dw = workload.DeviceWorkload(wl)
    dw.step()
    assert lib.last_device_error() == 0
    ref = OracleRun(dw, range(B))
    for li, mode in enumerate(modes):
        idx = dw.group.index(li).cpu().numpy()
        o = dw.group.out[li].cpu().numpy()
        lse = dw.group.lse[li].cpu().numpy()
        for b in range(B):
            for j in range(Sq):
                r = ref.out[li][(b, j)]
                np.testing.assert_array_equal(idx[b, j], r["idx"], err_msg=f"layer {li} b {b} j {j}")
                assert_attn_close(o[b, j], lse[b, j], r["o"], r["lse"], f"{name} layer {li} b {b} j {j}")
    # Reuse layers alias their source's index tensor: same storage, no copy.
    own, src = lib.plan(modes)
    for li, m in enumerate(modes):
        if m == "U":
            assert dw.group.index(li).data_ptr() == dw.group.index(src[li]).data_ptr()


def test_topk_ties_go_to_lower_index(mods):
    """All-zero indexer query: every score is 0, so the top-k are 0..k-1. The
    28000-token rows are split over 2 CTAs of about 14000 positions, more equal
    scores than a CTA's candidate list holds, so they take the re-scan path."""
    lib, workload = mods
    wl = inputs.small_workload("ties", 3, 2, [28000, 3000, 777], 100, modes=("F",))
    dw = workload.DeviceWorkload(wl)
    dw.q_idx[0].zero_()
    dw.step()
    assert lib.last_device_error() == 0
    idx = dw.group.index(0).cpu().numpy()
    for b in range(3):
        for j in range(2):
            np.testing.assert_array_equal(idx[b, j], np.arange(100, dtype=np.int32))


def test_topk_heavy_ties_against_oracle(mods):
    """Indexer queries with a single non-zero channel: scores take few
    distinct values, so the threshold bin is crowded and many positions tie
    at the threshold key (tie ranking across the CTAs of a row); indices
    must match the oracle."""
    lib, workload = mods
    wl = inputs.small_workload("crowd", 3, 1, [30000, 6000, 2500], 700, modes=("F",), seed=5)
    dw = workload.DeviceWorkload(wl)
    dw.q_idx[0][:, :, :, 1:] = 0
    dw.step()
    assert lib.last_device_error() == 0
    ref = OracleRun(dw, range(3))
    idx = dw.group.index(0).cpu().numpy()
    for b in range(3):
        np.testing.assert_array_equal(idx[b, 0], ref.out[0][(b, 0)]["idx"], err_msg=f"b {b}")


def test_topk_negative_scores_against_oracle(mods):
    """Negative head weights make every score <= 0, so the threshold bin lies
    among negative keys (the selection's general key path, not the
    positive-bits shortcut); -0 and +0 scores must tie. Indices must match
    the oracle exactly."""
    lib, workload = mods
    wl = inputs.small_workload("negw", 3, 2, [9000, 4000, 700], 300, modes=("F",), seed=21)
    dw = workload.DeviceWorkload(wl)
    dw.w[0].neg_()
    dw.step()
    assert lib.last_device_error() == 0
    ref = OracleRun(dw, range(3))
    idx = dw.group.index(0).cpu().numpy()
    for b in range(3):
        for j in range(2):
            np.testing.assert_array_equal(idx[b, j], ref.out[0][(b, j)]["idx"], err_msg=f"b {b} j {j}")


def test_topk_rows_longer_than_one_window(mods):
    """80 query rows give one CTA per row, and rows longer than 2^17 positions
    are then covered in two rounds of windows; shorter rows in the same
    launch take one round. Sampled rows must match the oracle exactly."""
    lib, workload = mods
    lens = [140000 if b % 3 == 0 else (131100 if b % 3 == 1 else 5000) for b in range(80)]
    wl = inputs.small_workload("rounds", 80, 1, lens, 2048, modes=("F",), seed=11)
    dw = workload.DeviceWorkload(wl)
    dw.step()
    assert lib.last_device_error() == 0
    rows = [0, 1, 2, 39, 79]
    ref = OracleRun(dw, rows)
    idx = dw.group.index(0).cpu().numpy()
    for b in rows:
        np.testing.assert_array_equal(idx[b, 0], ref.out[0][(b, 0)]["idx"], err_msg=f"b {b}")


def test_topk_all_valid_when_k_covers_context(mods):
    """top-k = every position reduces the sparse attention to dense attention
    over all entries plus the window."""
    lib, workload = mods
    wl = inputs.small_workload("dense", 2, 1, [300, 150], 512, modes=("F",))
    dw = workload.DeviceWorkload(wl)
    dw.step()
    idx = dw.group.index(0).cpu().numpy()
    for b, T in enumerate(wl.lens()):
        np.testing.assert_array_equal(idx[b, 0, :T], np.arange(T))
        assert np.all(idx[b, 0, T:] == -1)
    ref = OracleRun(dw, range(2))
    for b in range(2):
        r = ref.out[0][(b, 0)]
        assert_attn_close(dw.group.out[0][b, 0].cpu().numpy(), dw.group.lse[0][b, 0].cpu().numpy(),
                          r["o"], r["lse"], f"dense b {b}")


def test_attention_window_only_and_padding(mods):
    """k = 0 (window only), and an index list with -1 holes."""
    lib, workload = mods
    wl = inputs.small_workload("win", 3, 2, [1000, 100, 5], 64, modes=("F",))
    dw = workload.DeviceWorkload(wl)
    dw.step()
    g = dw.group
    cache = g.cache(0)
    o0, l0 = lib.sparse_attn_decode(dw.q[0], cache, dw.page_table, dw.seq_lens, None, dw.swa[0], SCALE)
    holes = g.index(0).clone()
    holes[:, :, ::3] = -1
    o1, l1 = lib.sparse_attn_decode(dw.q[0], cache, dw.page_table, dw.seq_lens, holes, dw.swa[0], SCALE)
    assert lib.last_device_error() == 0
    for b in range(3):
        q = oracle.bf16_bits(dw.q[0][b])
        swa = oracle.bf16_bits(dw.swa[0][b])
        for j in range(2):
            ro, rl = attend(dw, 0, b, j, q[j], swa, np.zeros(0, np.int32))
            assert_attn_close(o0[b, j].cpu().numpy(), l0[b, j].cpu().numpy(), ro, rl, f"window b{b} j{j}")
            ro, rl = attend(dw, 0, b, j, q[j], swa, holes[b, j].cpu().numpy())
            assert_attn_close(o1[b, j].cpu().numpy(), l1[b, j].cpu().numpy(), ro, rl, f"holes b{b} j{j}")


def test_cache_bytes_match_oracle_quantizer(mods):
    """The bulk build and the step's append leave exactly the oracle's FP4
    bytes, scales and indexer keys in the pages."""
    lib, workload = mods
    wl = inputs.small_workload("bytes", 2, 2, [777, 200], 64, modes=("F",))
    dw = workload.DeviceWorkload(wl)
    dw.step()
    cache = dw.group.cache(0)
    for b, T in enumerate(wl.lens()):
        pos = torch.arange(T)
        slots = lib.slot_mapping(dw.page_table, b, pos.cuda()).long()
        kv = torch.cat([r for _, r in inputs.kv_chunks(wl, 0, b, "cuda")])
        rc, rs = oracle.quant_fp4(oracle.bf16_bits(kv))
        np.testing.assert_array_equal(cache.kv_fp4.view(-1, 288)[slots].cpu().numpy(), rc)
        np.testing.assert_array_equal(cache.kv_scale.view(-1, 36)[slots].cpu().numpy(), rs)
        kid = inputs.kidx_rows(wl, 0, b, 0, T, "cuda").cpu()
        assert torch.equal(cache.kidx_logical().reshape(-1, 64)[slots].cpu(), kid)


def test_bad_page_table_entry_sets_status_without_fault(mods):
    lib, workload = mods
    wl = inputs.small_workload("badpage", 2, 1, [500, 300], 64, modes=("F",))
    dw = workload.DeviceWorkload(wl)
    assert lib.last_device_error() == 0
    pt = dw.page_table.clone()
    pt[1, 2] = 10 ** 6
    g = dw.group
    lib.indexer_topk(dw.q_idx[0], dw.w[0], g.cache(0), pt, dw.seq_lens, 64)
    assert lib.last_device_error() == 6
    idx = g.index(0).clone()
    idx[1, 0, 0] = 150                                    # in page 2 of sequence 1
    lib.sparse_attn_decode(dw.q[0], g.cache(0), pt, dw.seq_lens, idx, dw.swa[0], SCALE)
    assert lib.last_device_error() == 6
    bad_len = torch.tensor([500, 10 ** 6], dtype=torch.int32, device="cuda")
    lib.indexer_topk(dw.q_idx[0], dw.w[0], g.cache(0), dw.page_table, bad_len, 64)
    assert lib.last_device_error() == 6
    torch.cuda.synchronize()


def test_argument_errors_are_reported_before_launch(mods):
    lib, workload = mods
    cache = lib.PagedCache(2)
    slots = torch.zeros(4, dtype=torch.int32, device="cuda")
    before = lib.launch_count()
    xm = torch.zeros(4 * 576 + 1, dtype=torch.bfloat16, device="cuda")[1:].view(4, 576)
    with pytest.raises(lib.Csa2Error) as e:
        lib.quant_kv_fp4(xm, slots, cache)
    assert e.value.status == 8                             # CSA2_ERR_ALIGNMENT
    q = torch.zeros(1, 1, 16, 576, dtype=torch.bfloat16, device="cuda")
    swa = torch.zeros(1, 128, 576, dtype=torch.bfloat16, device="cuda")
    pt = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    sl = torch.ones(1, dtype=torch.int32, device="cuda")
    if lib.sparse_attn_workspace_bytes(1, 1, 0) > 0:
        with pytest.raises(lib.Csa2Error) as e:
            lib.sparse_attn_decode(q, cache, pt, sl, None, swa, SCALE,
                                   ws=torch.empty(0, dtype=torch.uint8, device="cuda"))
        assert e.value.status == 7                         # CSA2_ERR_WORKSPACE
    qi = torch.zeros(1, 5, 4, 64, dtype=torch.uint8, device="cuda")
    w = torch.zeros(1, 5, 4, dtype=torch.float32, device="cuda")
    with pytest.raises(lib.Csa2Error) as e:
        lib.indexer_topk(qi, w, cache, pt, sl, 4)
    assert e.value.status == 2                             # CSA2_ERR_UNSUPPORTED (Sq > 4)
    assert lib.launch_count() == before


def _assert_scaled_close(o_gpu, lse_gpu, o_ref, lse_ref, what):
    """The attention bar for inputs far from unit scale: relative L2 1e-3, and
    max-abs 2e-3 times the output's magnitude (an absolute 2e-3 is below the
    fp32 resolution of outputs near 1e5); lse to 2e-3 relative to its size."""
    mag = max(1.0, float(np.abs(o_ref).max()))
    err = np.abs(o_gpu.astype(np.float64) - o_ref)
    rel = float(np.linalg.norm(o_gpu - o_ref)) / max(float(np.linalg.norm(o_ref)), 1e-300)
    assert float(err.max()) <= 2e-3 * mag, f"{what}: max-abs {err.max():.3e} (scale {mag:.3e})"
    assert rel <= 1e-3, f"{what}: rel-L2 {rel:.3e}"
    fin = np.isfinite(lse_ref)
    np.testing.assert_array_equal(np.isfinite(lse_gpu), fin, err_msg=what)
    if fin.any():
        tol = 2e-3 * np.maximum(1.0, np.abs(lse_ref[fin]))
        assert np.all(np.abs(lse_gpu[fin] - lse_ref[fin]) <= tol), f"{what}: lse"


@pytest.mark.parametrize("q_gain,w_gain", [(1e5, 1.0), (1.0, 1e5), (1e-6, 1.0), (1.0, 1e-6), (1e-6, 1e-6),
                                           (3e4, 3e4)],
                         ids=["q1e5", "win1e5", "q1e-6", "win1e-6", "both1e-6", "both3e4"])
def test_attention_inputs_outside_the_f16_range(mods, q_gain, w_gain):
    """Queries and window rows far outside f16's exact range (|x| > 65504 or
    < 2^-14) against the oracle: the kernel carries power-of-two exponents
    for them instead of narrowing to f16 directly."""
    lib, workload = mods
    wl = inputs.small_workload(f"range{q_gain}_{w_gain}", 2, 2, [900, 400], 64, modes=("F",), seed=9)
    dw = workload.DeviceWorkload(wl)
    dw.step()
    g = dw.group
    q = (dw.q[0].float() * q_gain).to(torch.bfloat16)
    swa = (dw.swa[0].float() * w_gain).to(torch.bfloat16)
    o, l = lib.sparse_attn_decode(q, g.cache(0), dw.page_table, dw.seq_lens, g.index(0), swa, SCALE)
    assert lib.last_device_error() == 0
    idx = g.index(0).cpu().numpy()
    for b in range(2):
        qb, sb = oracle.bf16_bits(q[b]), oracle.bf16_bits(swa[b])
        for j in range(2):
            ro, rl = attend(dw, 0, b, j, qb[j], sb, idx[b, j])
            _assert_scaled_close(o[b, j].cpu().numpy(), l[b, j].cpu().numpy(), ro, rl, f"b {b} j {j}")


def test_attention_index_after_the_query_is_flagged(mods):
    """Query j sits at position T - Sq + j; a selected index after it (a
    future draft token) is out of range: flagged and skipped."""
    lib, workload = mods
    wl = inputs.small_workload("causal", 1, 4, [600], 32, modes=("F",), seed=5)
    dw = workload.DeviceWorkload(wl)
    dw.step()
    g = dw.group
    idx = g.index(0).clone()
    T = wl.lens()[0]
    idx[0, 0, 0] = T - 1                                   # query 0 is at T - 4
    idx[0, 0] = torch.sort(idx[0, 0]).values
    o, l = lib.sparse_attn_decode(dw.q[0], g.cache(0), dw.page_table, dw.seq_lens, idx, dw.swa[0], SCALE)
    assert lib.last_device_error() == 6                    # CSA2_ERR_DEVICE_BOUNDS
    q = oracle.bf16_bits(dw.q[0][0])
    swa = oracle.bf16_bits(dw.swa[0][0])
    keep = idx[0, 0].cpu().numpy().copy()
    keep[keep > T - 4] = -1                                # the kernel skips the future entry
    ro, rl = attend(dw, 0, 0, 0, q[0], swa, keep)
    assert_attn_close(o[0, 0].cpu().numpy(), l[0, 0].cpu().numpy(), ro, rl, "query 0")
