"""K9, window attention of L consecutive queries (SWA bounded replay), against
the oracle's attention with no selected entries (k = 0): every query of
every sequence, at L = 1, 40, 128 and 1024, with short sequences (window rows
at negative positions skipped), a ragged last tile of queries, and window
values far outside f16's exact range."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle_check import assert_attn_close

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(576)
W = 128


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from compressed_sparse_attention_quant_b200 import lib as L
    return L


def _check(lib, L, lens, q_gain=1.0, w_gain=1.0, seed=0, sample=None):
    g = torch.Generator().manual_seed(seed)
    B = len(lens)
    q = (torch.randn(B, L, 16, 576, generator=g) * q_gain).to(torch.bfloat16)
    swa = (torch.randn(B, W + L - 1, 576, generator=g) * w_gain).to(torch.bfloat16)
    lens_t = torch.tensor(lens, dtype=torch.int32)
    o, lse = lib.swa_replay_attn(q.cuda(), swa.cuda(), lens_t.cuda(), SCALE)
    assert lib.last_device_error() == 0
    o, lse = o.cpu().numpy(), lse.cpu().numpy()
    qb, sb = oracle.bf16_bits(q), oracle.bf16_bits(swa)
    empty_c = np.zeros((0, 288), np.uint8)
    empty_s = np.zeros((0, 36), np.uint8)
    mag = max(1.0, w_gain)
    for b, T in enumerate(lens):
        first = T - (W + L - 1)
        js = range(L) if sample is None else sorted(set(list(range(min(L, 9))) + list(range(L - 9, L)) +
                                                         list(np.random.default_rng(b).choice(L, sample))))
        for j in js:
            rows = [r for r in range(j, j + W) if first + r >= 0]
            ro, rl = oracle.sparse_attn(qb[b, j], empty_c, empty_s, np.zeros(0, np.int32),
                                        sb[b][rows] if rows else np.zeros((0, 576), np.uint16), SCALE)
            if mag > 1.0:
                err = np.abs(o[b, j] - ro).max()
                rel = np.linalg.norm(o[b, j] - ro) / np.linalg.norm(ro)
                assert err <= 2e-3 * mag and rel <= 1e-3, f"b {b} j {j}: {err:.3e} {rel:.3e}"
            else:
                assert_attn_close(o[b, j], lse[b, j], ro, rl, f"L {L} b {b} j {j}")


def test_replay_single_query(lib):
    _check(lib, 1, [500, 129, 1], seed=1)


def test_replay_40_queries_ragged_tile(lib):
    _check(lib, 40, [1000, 60, 40], seed=2)


def test_replay_128_queries_short_sequence(lib):
    _check(lib, 128, [128, 300], seed=3)


def test_replay_1024_queries(lib):
    _check(lib, 1024, [5000], seed=4, sample=120)


def test_replay_window_values_outside_f16_range(lib):
    _check(lib, 40, [900], w_gain=1e5, seed=5)
    _check(lib, 40, [900], w_gain=1e-6, seed=6)


def test_replay_matches_decode_entry_point_with_no_selection(lib):
    """The same computation through csa2_sparse_attn_decode (k = 0, Sq = L)."""
    from compressed_sparse_attention_quant_b200 import lib as L_
    g = torch.Generator().manual_seed(7)
    B, L = 2, 24
    q = torch.randn(B, L, 16, 576, generator=g).to(torch.bfloat16).cuda()
    swa = torch.randn(B, W + L - 1, 576, generator=g).to(torch.bfloat16).cuda()
    lens = torch.tensor([700, 200], dtype=torch.int32).cuda()
    o1, l1 = lib.swa_replay_attn(q, swa, lens, SCALE)
    cache = L_.PagedCache(B * 11)
    pt = torch.arange(B * 11, dtype=torch.int32).view(B, 11).cuda()
    o2, l2 = lib.sparse_attn_decode(q, cache, pt, lens, None, swa, SCALE)
    assert lib.last_device_error() == 0
    np.testing.assert_allclose(o1.cpu().numpy(), o2.cpu().numpy(), rtol=0, atol=2e-3)
    np.testing.assert_allclose(l1.cpu().numpy(), l2.cpu().numpy(), rtol=0, atol=2e-3)
