"""Pins of the CPU oracle to things other than itself (CPU only).

What pins each oracle function:
  e2m1_value      format definition via a golden fixture of the pages' format
                  (tests/golden/pages_constants.txt) + sign symmetry
  e4m3_value      torch's float8_e4m3fn decode of all 256 bytes (library)
  group_scale     exhaustive over every finite bf16 amax: exact-integer
                  brute-force nearest search, and torch's RNE fp8 cast
  e2m1_code       exhaustive over every finite bf16 x and every positive
                  finite E4M3 scale: brute-force argmin of |x - s*m|
  quant_fp4       group/nibble layout against a composition written here from
                  the pinned pieces; error bound; idempotence; bytes per token
  e4m3_code_quotient  with sigma = 1: torch's RNE float8_e4m3fn cast
                  (library) and a brute-force nearest search over every finite
                  bf16 value in range and every E4M3 midpoint with its
                  binary32 neighbours; saturation; canonical +0
  quant_index_fp8 sigma: the binary32 value nearest amax / 448, checked in
                  exact rationals against its neighbours; codes: an
                  exact-rational brute force over all 127 grid values on
                  wide-magnitude rows and on rows where the binary32 quotient
                  lands on an E4M3 midpoint that the exact quotient misses
                  (where the two roundings differ); idempotence on E4M3-grid
                  rows; power-of-two equivariance; half-step error bound;
                  zero rows
  indexer_scores  one-hot head weights reduce to an integer matmul (numpy);
                  linearity in w; ReLU placement with negative sigma; q = 0.
                  The formula itself is a reading (parity unpinned).
  topk            numpy lexsort on tie-heavy inputs; rank-count brute force;
                  k >= n; padding
  pool_topk       rank-count brute force on tie-heavy pools; pool order
                  invariance; -1 entries; a pool of exactly k; the Full
                  layer's own pool under its own scores gives its top-k
  pool_reindex    a pool holding every valid position reduces to the full
  (decode_group)  scan (topk); the pool is the Full layer's top-C
  merge_topk_candidates  per-shard top-k lists merged = the unsharded top-k
                  (tie-heavy scores, 2 to 8 shards)
  lse_merge       attention split over shards and merged = one softmax over
                  the union; an empty shard contributes nothing
  sparse_attn     top-k covering every entry = dense attention computed with
                  torch's scaled_dot_product_attention in fp64 (library);
                  single key; equal logits; k = 0 (window only); no keys;
                  -1 entries; index order invariance
  plan            golden plans from the pages' mode table
  decode_group    Reuse carries the Full layer's indices unchanged; window of
                  128 rows per query (golden constant)
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from compressed_sparse_attention_quant_b200 import inputs
from conftest import golden, read_kv_fixture
from fp8_cases import double_rounding_rows

CONST = read_kv_fixture("pages_constants.txt")


def all_finite_bf16_bits():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32)
    keep = np.isfinite(vals)
    return bits[keep], vals[keep].astype(np.float64)


def e4m3_finite_values():
    """All 256 E4M3FN bytes decoded by torch (library), NaN where undefined."""
    b = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return b.view(torch.float8_e4m3fn).to(torch.float64).numpy()


# ------------------------------------------------------------------ formats
def test_e2m1_magnitudes_match_pages_fixture():
    mags = [float(x) for x in CONST["e2m1_magnitudes"].split()]
    assert len(mags) == 8
    for code in range(8):
        assert oracle.e2m1_value(code) == mags[code]
        v = oracle.e2m1_value(code | 8)
        assert v == -mags[code] and math.copysign(1.0, v) == -1.0


def test_e4m3_decode_matches_torch_all_bytes():
    ref = e4m3_finite_values()
    for b in range(256):
        got = oracle.e4m3_value(b)
        if math.isnan(ref[b]):
            assert math.isnan(got)
        else:
            assert got == ref[b], b
    assert max(v for v in ref if not math.isnan(v)) == 448.0


# ------------------------------------------------------------------ scale rule
def test_group_scale_exhaustive_against_bruteforce():
    _, vals = all_finite_bf16_bits()
    amax = np.unique(np.abs(vals))
    got = oracle.group_scale_n(amax)

    # brute force: nearest of the 127 finite non-negative E4M3 values to
    # amax/6, distance |6v - amax| compared exactly in integers (scaled by
    # 2^16; exact for amax in [2^-9, 2^12)), ties to the even byte.
    ev = e4m3_finite_values()[:127]                   # bytes 0x00..0x7E
    ok = (amax >= 2.0 ** -9) & (amax < 2.0 ** 12)
    a_int = (amax[ok] * 2 ** 16).astype(np.int64)
    assert np.all(a_int.astype(np.float64) == amax[ok] * 2 ** 16)
    v_int = (6 * ev * 2 ** 16).astype(np.int64)
    dist = np.abs(v_int[None, :] - a_int[:, None])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # among equal distances prefer the even byte (even mantissa)
    even_pref = np.where(cand & (np.arange(127) % 2 == 0)[None, :], 1, 0)
    pick = np.where(even_pref.any(axis=1), even_pref.argmax(axis=1), cand.argmax(axis=1))
    np.testing.assert_array_equal(got[ok], pick.astype(np.uint8))

    # below 2^-9: amax/6 < 2^-9/6 < 2^-10 (half the smallest subnormal) -> 0
    assert np.all(got[amax < 2.0 ** -9] == 0)
    # at or above 6*448 the nearest value saturates to 448 (byte 0x7E)
    assert np.all(got[amax >= 2688.0] == 0x7E)


def test_group_scale_matches_torch_rne_cast():
    _, vals = all_finite_bf16_bits()
    amax = np.unique(np.abs(vals))
    amax = amax[amax / 6 <= 448.0]
    t = torch.from_numpy(amax / 6.0).to(torch.float32)   # exact side argued in the oracle
    ref = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.group_scale_n(amax), ref)


# ------------------------------------------------------------------ indexer FP8 quantiser
def e4m3_nearest_bruteforce(r: np.ndarray) -> np.ndarray:
    """Nearest finite E4M3FN byte to each binary32 value (fp64 distances are
    exact here), ties to the even byte, saturating, canonical +0."""
    ev = e4m3_finite_values()[:127]                  # 0x00 .. 0x7E, ascending
    a = np.minimum(np.abs(r.astype(np.float64)), 448.0)
    dist = np.abs(ev[None, :] - a[:, None])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    even = cand & (np.arange(127) % 2 == 0)[None, :]
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1)).astype(np.uint8)
    return np.where((r < 0) & (pick != 0), pick | 0x80, pick).astype(np.uint8)


def test_e4m3_code_quotient_sigma_one_against_torch_cast_and_bruteforce():
    """With sigma = 1 the quotient is x itself: every finite bf16 value in
    range and every E4M3 midpoint with its binary32 neighbours against
    torch's RNE float8_e4m3fn cast (library) and the brute-force nearest
    search; saturation; canonical +0."""
    _, vals = all_finite_bf16_bits()
    ev = e4m3_finite_values()[:127]
    mids = ((ev[:-1] + ev[1:]) / 2).astype(np.float32)          # exact: at most 5 significant bits
    assert np.all(mids.astype(np.float64) == (ev[:-1] + ev[1:]) / 2)
    up = np.nextafter(mids, np.float32(np.inf))
    down = np.nextafter(mids, np.float32(0))
    r = np.concatenate([vals[np.abs(vals) <= 448].astype(np.float32), mids, up, down, -mids, -up, -down])
    got = np.array([oracle.e4m3_code_quotient(float(x), 1.0) for x in r], np.uint8)
    ref = torch.from_numpy(r).to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()
    ref[(ref & 0x7F) == 0] = 0                                    # canonical +0
    np.testing.assert_array_equal(got, ref)
    np.testing.assert_array_equal(got, e4m3_nearest_bruteforce(r))
    # saturation above the largest finite value, both signs
    for x in (448.5, 464.0, 1e6, 3.0e38):
        assert oracle.e4m3_code_quotient(x, 1.0) == 0x7E and oracle.e4m3_code_quotient(-x, 1.0) == 0xFE


def bf16_rows(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


E4M3_GRID = [Fraction(float(v)) for v in e4m3_finite_values()[:127]]   # codes 0x00 .. 0x7E, ascending


def exact_nearest_e4m3(x: float, sigma: float) -> int:
    """Brute force in exact rationals: the E4M3FN byte whose value is nearest
    to x / sigma over all 127 non-negative grid values (ties to the even
    byte, saturating at 448, canonical +0). Independent of the oracle's
    midpoint comparisons and of any binary32 quotient."""
    r = abs(Fraction(x) / Fraction(sigma))
    best_d, best_i = None, 0
    for i, v in enumerate(E4M3_GRID):
        d = abs(r - v)
        if best_d is None or d < best_d or (d == best_d and i % 2 == 0):
            best_d, best_i = d, i
    if best_i == 0:
        return 0
    return best_i | 0x80 if x < 0 else best_i


def binary32_nearest(q: Fraction) -> np.float32:
    """The binary32 value nearest to a positive rational q (ties to even),
    found by comparing the candidates around float(q) exactly."""
    c = np.float32(float(q))
    cands = [np.nextafter(c, np.float32(0)), c, np.nextafter(c, np.float32(np.inf))]
    best = min(cands, key=lambda f: (abs(Fraction(float(f)) - q), int(np.array(f).view(np.uint32)) & 1))
    return np.float32(best)


def test_quant_index_fp8_sigma_is_the_nearest_binary32():
    """sigma is the binary32 value nearest to amax / 448, checked in exact
    rationals against its neighbours (not by repeating the division)."""
    rng = np.random.default_rng(10)
    x = rng.standard_normal((400, 64)) * np.exp2(rng.integers(-120, 120, (400, 1)))
    x[0] = 0.0
    x[1, 3] = 1e-39                                               # a bf16 subnormal maximum
    bits = bf16_rows(x)
    _, sigma = oracle.quant_index_fp8(bits)
    amax = np.abs(bits_to_f32(bits)).max(axis=1)
    assert sigma[0] == 0.0
    for a, s in zip(amax[1:], sigma[1:]):
        assert s == binary32_nearest(Fraction(float(a)) / 448), (a, s)


def test_quant_index_fp8_codes_against_exact_bruteforce():
    """Codes against the exact-rational brute force on wide-magnitude rows,
    zero / subnormal / near-maximum rows, and the double-rounding rows."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((40, 64)) * np.exp2(rng.integers(-60, 60, (40, 1)))
    x[0] = 0.0
    x[1] = -0.0
    x[2] = 0.0
    x[2, 17] = -3.0e-38                                           # one tiny non-zero channel
    x[3] = rng.standard_normal(64) * 1e-39                        # bf16 subnormals
    x[4, :] = 3.3e38                                              # near the bf16 maximum
    x[4, ::2] *= -1
    bits = np.concatenate([bf16_rows(x), double_rounding_rows(12, seed=1)])
    codes, sigma = oracle.quant_index_fp8(bits)
    xv = bits_to_f32(bits)
    assert sigma[0] == 0 and sigma[1] == 0 and np.all(codes[:2] == 0)
    for r in range(len(bits)):
        if sigma[r] == 0:
            continue
        want = [exact_nearest_e4m3(float(v), float(sigma[r])) for v in xv[r]]
        np.testing.assert_array_equal(codes[r], np.array(want, np.uint8), err_msg=f"row {r}")


def test_quant_index_fp8_rounds_the_exact_quotient_not_the_binary32_one():
    """On the double-rounding rows the oracle's codes differ from rounding
    the binary32 quotient (torch's RNE cast of numpy's binary32 division) in
    some channels, and agree with the exact brute force in all of them."""
    bits = double_rounding_rows(20, seed=2)
    codes, sigma = oracle.quant_index_fp8(bits)
    xv = bits_to_f32(bits)
    q32 = xv / sigma[:, None]                                      # numpy binary32 division (library)
    via32 = torch.from_numpy(np.ascontiguousarray(q32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    via32 = np.where((via32 & 0x7F) == 0, 0, via32)
    assert np.count_nonzero(via32 != codes) > 0
    diff = np.argwhere(via32 != codes)
    for r, c in diff[:200]:
        assert codes[r, c] == exact_nearest_e4m3(float(xv[r, c]), float(sigma[r]))


def test_quant_index_fp8_idempotent_on_grid_rows():
    rng = np.random.default_rng(12)
    ev = e4m3_finite_values()
    b = rng.integers(0, 0x7F, (50, 64)).astype(np.uint8) | (rng.integers(0, 2, (50, 64)) * 0x80).astype(np.uint8)
    b[:, 5] = 0x7E                                                # row maximum 448 -> sigma = 1
    x = ev[b]
    bits = bf16_rows(x)
    assert np.all(bits_to_f32(bits).astype(np.float64) == x)    # E4M3 values are exact in bf16
    codes, sigma = oracle.quant_index_fp8(bits)
    assert np.all(sigma == 1.0)
    want = np.where((b & 0x7F) == 0, 0, b).astype(np.uint8)
    np.testing.assert_array_equal(codes, want)


def test_quant_index_fp8_power_of_two_equivariance_and_error_bound():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((100, 64)).astype(np.float32)
    bits = bf16_rows(x)
    codes, sigma = oracle.quant_index_fp8(bits)
    xv = bits_to_f32(bits).astype(np.float64)
    for k in (-40, -9, 9, 40):
        c2, s2 = oracle.quant_index_fp8(bf16_rows(xv * 2.0 ** k))
        np.testing.assert_array_equal(c2, codes)
        np.testing.assert_array_equal(s2.astype(np.float64), sigma.astype(np.float64) * 2.0 ** k)
    ev = e4m3_finite_values()
    deq = np.where(codes >= 0x80, -ev[codes & 0x7F], ev[codes & 0x7F]) * sigma[:, None].astype(np.float64)
    r = np.abs(xv) / sigma[:, None]
    e = np.floor(np.log2(np.maximum(r, 2.0 ** -6)))
    half_step = np.exp2(e - 4)                                    # half the E4M3 step at r (2^-10 below 2^-6)
    # one rounding of the exact quotient: within half a grid step (fp64 slack only)
    assert np.all(np.abs(xv - deq) <= sigma[:, None] * half_step * (1 + 2.0 ** -40))


# ------------------------------------------------------------------ codes
def test_e2m1_code_exhaustive_against_argmin():
    _, xs = all_finite_bf16_bits()
    ev = e4m3_finite_values()
    scales = ev[1:127]                                 # every positive finite scale
    mags = np.array([float(x) for x in CONST["e2m1_magnitudes"].split()])
    x = np.repeat(xs, len(scales))
    s = np.tile(scales, len(xs))
    got = oracle.e2m1_code_n(x, s)
    # Brute force: argmin over the 8 magnitudes of | |x| - s*m |, ties to the
    # even code. A distance is trusted only where fp64 computed it exactly
    # (TwoSum error term zero); every pair whose distances are not all exact
    # has |x| and 6s so far apart that the answer is the saturated code or 0.
    ref = np.empty_like(got)
    checked = np.zeros(len(x), bool)
    step = 1 << 21
    for i in range(0, len(x), step):
        ax = np.abs(x[i:i + step])[:, None]
        b = -(s[i:i + step, None] * mags[None, :])
        t = ax + b
        bb = t - ax
        err = (ax - (t - bb)) + (b - bb)
        exact = np.all(err == 0, axis=1)
        d = np.abs(t)
        best = d.min(axis=1, keepdims=True)
        cand = d == best
        even = cand & (np.arange(8) % 2 == 0)[None, :]
        code = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
        sat = ax[:, 0] > 6 * s[i:i + step]
        code = np.where(exact, code, np.where(sat, 7, 0))
        tiny = ax[:, 0] < 0.25 * s[i:i + step]
        assert np.all(exact | sat | tiny)
        neg = (x[i:i + step] < 0) & (code != 0)
        ref[i:i + step] = (code | (neg * 8)).astype(np.uint8)
        checked[i:i + step] = exact | sat | tiny
    assert checked.all()
    np.testing.assert_array_equal(got, ref)


def test_e2m1_code_zero_scale_and_canonical_zero():
    assert oracle.e2m1_code(5.0, 0.0) == 0
    assert oracle.e2m1_code(-0.0, 1.0) == 0
    assert oracle.e2m1_code(-0.2, 1.0) == 0         # rounds to 0: canonical +0
    assert oracle.e2m1_code(-0.3, 1.0) == 0x9       # -0.5
    assert oracle.e2m1_code(1e30, 1.0) == 0x7       # saturates at 6


# ------------------------------------------------------------------ quantizer
def _compose_quant(x_bits):
    """Quantize via the pinned pieces, with grouping and packing written here."""
    vals = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    n, d = vals.shape
    g = vals.reshape(n, d // 16, 16)
    amax = np.abs(g).max(axis=2)
    sb = oracle.group_scale_n(amax).reshape(n, d // 16)
    s = np.vectorize(oracle.e4m3_value)(sb)
    codes = oracle.e2m1_code_n(g, np.repeat(s[:, :, None], 16, axis=2)).reshape(n, d)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, sb


def test_quant_fp4_layout_matches_composition():
    wl = inputs.small_workload("q", 1, 1, [300], 16)
    x = torch.cat([r for _, r in inputs.kv_chunks(wl, 0, 0, "cpu")])
    bits = oracle.bf16_bits(x)
    codes, scales = oracle.quant_fp4(bits)
    ref_codes, ref_scales = _compose_quant(bits)
    np.testing.assert_array_equal(scales, ref_scales)
    np.testing.assert_array_equal(codes, ref_codes)


def test_quant_fp4_bytes_per_token():
    d = inputs.DIM
    codes, scales = oracle.quant_fp4(np.zeros((3, d), np.uint16))
    assert codes.shape == (3, d // 2) and scales.shape == (3, d // 16)
    assert codes.shape[1] + scales.shape[1] == 324          # 288 data + 36 scales
    assert int(CONST["scale_group_channels"]) * scales.shape[1] == d


def test_quant_fp4_error_bound():
    rng = np.random.default_rng(0)
    mag = np.exp(rng.uniform(-9, 7, (400, 1)))
    x = torch.from_numpy(rng.standard_normal((400, 576)) * mag).to(torch.bfloat16)
    codes, scales = oracle.quant_fp4(oracle.bf16_bits(x))
    xh = oracle.dequant_fp4(codes, scales)
    xv = x.to(torch.float64).numpy()
    s = np.repeat(np.vectorize(oracle.e4m3_value)(scales), 16, axis=1)
    amax = np.repeat(np.abs(xv).reshape(400, 36, 16).max(2), 16, axis=1)
    err = np.abs(xv - xh)
    # normal E4M3 scales (relative rounding of the scale <= 1/16)
    normal = (s >= 2.0 ** -6) & (amax <= 6 * 448)
    assert normal.mean() > 0.5 and (s == 0).any() and (amax > 6 * 448).any()
    assert np.all(err[normal] <= s[normal])                  # half of the top step (4 -> 6)
    # subnormal scales: the step 2^-9 bounds the scale error, amax <= s*6 + 3*2^-9
    sub = (s > 0) & (s < 2.0 ** -6)
    assert sub.any() and np.all(err[sub] <= np.maximum(s[sub], amax[sub] - 6 * s[sub]))
    small = normal & (np.abs(xv) < 2 * s)
    assert np.all(err[small] <= s[small] / 4)                # half of the 0.5 step
    # scale underflow: amax/6 at or below half the smallest subnormal -> all codes 0
    under = s == 0
    assert np.all(amax[under] <= 6 * 2.0 ** -10) and np.all(xh[under] == 0)
    # saturation: the scale is 448 and magnitudes clamp to 6 * 448
    sat = amax > 6 * 464
    assert np.all(s[sat] == 448) and np.all(np.abs(xh[sat]) <= 6 * 448)


def test_quant_fp4_idempotent_when_group_max_code_is_six():
    rng = np.random.default_rng(1)
    n = 64
    codes = rng.integers(0, 16, (n, 576)).astype(np.uint8)
    codes[:, ::16] = 7 | (rng.integers(0, 2, (n, 36)) * 8)  # each group holds +-6
    sbytes = rng.integers(1, 127, (n, 36)).astype(np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    xh = oracle.dequant_fp4(packed, sbytes)
    x = torch.from_numpy(xh).to(torch.bfloat16)
    assert np.all(x.to(torch.float64).numpy() == xh)         # values are exact in bf16
    c2, s2 = oracle.quant_fp4(oracle.bf16_bits(x))
    canon = np.where((codes & 7) == 0, 0, codes)             # -0 is stored as +0
    np.testing.assert_array_equal(s2, sbytes)
    np.testing.assert_array_equal(c2, (canon[:, 0::2] | (canon[:, 1::2] << 4)).astype(np.uint8))


# ------------------------------------------------------------------ indexer
def _int_e4m3(v):
    return torch.tensor(v, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_indexer_one_hot_weights_reduce_to_integer_matmul():
    rng = np.random.default_rng(2)
    qi = rng.integers(-8, 9, (4, 64))
    ki = rng.integers(-8, 9, (50, 64))
    q, k = _int_e4m3(qi), _int_e4m3(ki)
    sig = np.ones(50, np.float32)
    dots = ki @ qi.T                                         # numpy integer matmul [50, 4]
    for h in range(4):
        w = np.zeros(4, np.float32)
        w[h] = 1.0
        s = oracle.indexer_scores(q, w, k, sig)
        np.testing.assert_array_equal(s, np.maximum(dots[:, h], 0).astype(np.float64))
        s_norelu = oracle.indexer_scores(q, w, k, sig, relu=False)
        np.testing.assert_array_equal(s_norelu, dots[:, h].astype(np.float64))


def test_indexer_linear_in_weights_and_relu_inside_sigma():
    rng = np.random.default_rng(3)
    q = _int_e4m3(rng.integers(-8, 9, (4, 64)))
    k = _int_e4m3(rng.integers(-8, 9, (40, 64)))
    w1 = np.array([0.25, 0.5, 1.0, 2.0], np.float32)
    w2 = np.array([2.0, 1.0, 0.5, 0.25], np.float32)
    sig = np.ones(40, np.float32)
    s1 = oracle.indexer_scores(q, w1, k, sig)
    s2 = oracle.indexer_scores(q, w2, k, sig)
    s12 = oracle.indexer_scores(q, w1 + w2, k, sig)
    np.testing.assert_array_equal(s12, s1 + s2)
    # negative sigma flips which heads pass the ReLU: relu(sigma * dot)
    neg = -np.ones(40, np.float32)
    sn = oracle.indexer_scores(q, w1, k, neg)
    dots = (np.vectorize(oracle.e4m3_value)(k) @ np.vectorize(oracle.e4m3_value)(q).T)
    np.testing.assert_array_equal(sn, (np.maximum(-dots, 0) * w1[None, :]).sum(1))
    assert np.all(oracle.indexer_scores(np.zeros((4, 64), np.uint8), w1, k, sig) == 0)


# ------------------------------------------------------------------ top-k
def test_topk_matches_lexsort_with_heavy_ties():
    rng = np.random.default_rng(4)
    for n, k in [(100, 7), (1000, 64), (333, 333), (50, 200), (2000, 1)]:
        s = rng.integers(0, 6, n).astype(np.float64) * 0.25
        got = oracle.topk(s, n, k)
        if n <= k:
            np.testing.assert_array_equal(got, np.r_[np.arange(n), -np.ones(k - n)].astype(np.int32))
            continue
        order = np.lexsort((np.arange(n), -s))[:k]           # primary -s, secondary index
        np.testing.assert_array_equal(got, np.sort(order).astype(np.int32))


def test_topk_rank_count_bruteforce_and_negative_zero():
    s = np.array([0.0, -0.0, 1.5, -2.0, 1.5, 0.0, -0.0, 3.0])
    for k in range(1, 8):
        sel = []
        for t in range(len(s)):
            rank = sum(1 for u in range(len(s)) if s[u] > s[t] or (s[u] == s[t] and u < t))
            if rank < k:
                sel.append(t)
        np.testing.assert_array_equal(oracle.topk(s, len(s), k), np.array(sel, np.int32))


def test_topk_only_first_n_valid_entries():
    s = np.array([1.0, 2.0, 3.0, 100.0, 200.0])
    np.testing.assert_array_equal(oracle.topk(s, 3, 2), [1, 2])


# ------------------------------------------------------------------ attention
def _rand_case(seed, n_cache=40, n_swa=7):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(16, 576, generator=g).to(torch.bfloat16)
    kv = (torch.randn(n_cache, 576, generator=g) * 2).to(torch.bfloat16)
    swa = torch.randn(n_swa, 576, generator=g).to(torch.bfloat16)
    codes, scales = oracle.quant_fp4(oracle.bf16_bits(kv))
    return q, codes, scales, swa


def _sdpa(q64, keys64, scale):
    o = F.scaled_dot_product_attention(q64[None, :, None, :], keys64[None, None].expand(1, 16, -1, -1),
                                       keys64[None, None].expand(1, 16, -1, -1), scale=scale)
    logits = (q64 @ keys64.T) * scale
    return o[0, :, 0, :].numpy(), torch.logsumexp(logits, dim=1).numpy()


def test_attn_topk_all_entries_is_dense_attention():
    q, codes, scales, swa = _rand_case(5)
    scale = 1 / math.sqrt(576)
    idx = np.arange(40, dtype=np.int32)
    o, lse = oracle.sparse_attn(oracle.bf16_bits(q), codes, scales, idx, oracle.bf16_bits(swa), scale)
    keys = torch.cat([torch.from_numpy(oracle.dequant_fp4(codes, scales)), swa.to(torch.float64)])
    ro, rl = _sdpa(q.to(torch.float64), keys, scale)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_attn_window_only_when_no_index():
    q, codes, scales, swa = _rand_case(6)
    scale = 0.05
    o, lse = oracle.sparse_attn(oracle.bf16_bits(q), codes, scales, np.full(9, -1, np.int32),
                                oracle.bf16_bits(swa), scale)
    ro, rl = _sdpa(q.to(torch.float64), swa.to(torch.float64), scale)
    np.testing.assert_allclose(o, ro, atol=1e-12)
    np.testing.assert_allclose(lse, rl, atol=1e-12)


def test_attn_single_key_and_equal_logits_and_empty():
    q, codes, scales, swa = _rand_case(7)
    qb = oracle.bf16_bits(q)
    v = oracle.dequant_fp4(codes[5:6], scales[5:6])[0]
    o, lse = oracle.sparse_attn(qb, codes, scales, np.array([5], np.int32),
                                np.zeros((0, 576), np.uint16), 0.1)
    np.testing.assert_array_equal(o, np.tile(v, (16, 1)))
    np.testing.assert_allclose(lse, 0.1 * (q.to(torch.float64).numpy() @ v), rtol=1e-13)
    # q = 0: every logit is 0 -> mean of the values, lse = log(n)
    zq = np.zeros((16, 576), np.uint16)
    idx = np.array([1, 3, 3, 9], np.int32)
    o, lse = oracle.sparse_attn(zq, codes, scales, idx, oracle.bf16_bits(swa), 1.0)
    vals = np.concatenate([oracle.dequant_fp4(codes[idx], scales[idx]),
                           swa.to(torch.float64).numpy()])
    np.testing.assert_allclose(o, np.tile(vals.mean(0), (16, 1)), atol=1e-13)
    np.testing.assert_allclose(lse, math.log(len(vals)), rtol=1e-14)
    # no keys at all
    o, lse = oracle.sparse_attn(qb, codes, scales, np.full(3, -1, np.int32),
                                np.zeros((0, 576), np.uint16), 0.1)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_attn_skips_padding_and_ignores_index_order():
    q, codes, scales, swa = _rand_case(8)
    qb, sb = oracle.bf16_bits(q), oracle.bf16_bits(swa)
    a = oracle.sparse_attn(qb, codes, scales, np.array([2, 7, 11, 30], np.int32), sb, 0.04)
    b = oracle.sparse_attn(qb, codes, scales, np.array([30, -1, 11, 2, -1, 7], np.int32), sb, 0.04)
    np.testing.assert_allclose(a[0], b[0], atol=1e-14)
    np.testing.assert_allclose(a[1], b[1], atol=1e-14)


# ------------------------------------------------------------------ modes
def test_plan_matches_golden_mode_table():
    with open(golden("mode_plans.txt")) as f:
        rows = [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]
    for row in rows:
        parts = [p.strip() for p in row.split("|")]
        modes = parts[0].split()
        if parts[1] == "error":
            with pytest.raises(ValueError):
                oracle.plan(modes)
            continue
        own, src = oracle.plan(modes)
        assert own == [int(x) for x in parts[1].split()], row
        assert src == [int(x) for x in parts[2].split()], row


def _logical_inputs(wl):
    own, _ = oracle.plan(wl.modes)
    caches = {}
    for o in set(own):
        caches[o] = {}
        for b in range(wl.batch):
            T = wl.lens()[b]
            kv = torch.cat([r for _, r in inputs.kv_chunks(wl, o, b, "cpu")])
            codes, scales = oracle.quant_fp4(oracle.bf16_bits(kv))
            caches[o][b] = {"codes": codes, "scales": scales,
                            "kidx": inputs.kidx_rows(wl, o, b, 0, T, "cpu").numpy(),
                            "ksig": inputs.kidx_scale_rows(wl, o, b, 0, T, "cpu").numpy()}
    layers = {}
    for li in range(len(wl.modes)):
        q = inputs.attn_query(wl, li, "cpu")
        swa = inputs.swa_rows(wl, li, "cpu")
        qi = inputs.idx_query(wl, li, "cpu")
        w = inputs.idx_weights(wl, li, "cpu")
        layers[li] = {b: {"q": oracle.bf16_bits(q[b]), "swa": oracle.bf16_bits(swa[b]),
                          "qidx": qi[b].numpy(), "w": w[b].numpy()} for b in range(wl.batch)}
    return caches, layers


def test_decode_group_reuse_carries_full_indices_and_window_rows():
    wl = inputs.small_workload("g", 2, 2, [700, 150], 40, modes=("F", "R", "U"))
    caches, layers = _logical_inputs(wl)
    out = oracle.decode_group(wl.q_tokens, wl.modes, range(wl.batch), wl.lens(), caches, layers,
                              wl.top_k, 1 / math.sqrt(576))
    W = int(CONST["swa_window"])
    assert layers[0][0]["swa"].shape[0] == W + wl.q_tokens - 1
    for key in out[0]:
        assert out[2][key]["idx"].tobytes() == out[0][key]["idx"].tobytes()
        assert out[1][key]["idx"].tobytes() != out[0][key]["idx"].tobytes()
        b, j = key
        pos = wl.lens()[b] - wl.q_tokens + j
        assert out[0][key]["idx"].max() <= pos                # causal selection
    # the window of query j is rows j..j+W-1: a direct window-only call agrees
    b, j = 1, 1
    rows = layers[2][b]["swa"][j:j + W]
    o, lse = oracle.sparse_attn(layers[2][b]["q"][j], caches[0][b]["codes"], caches[0][b]["scales"],
                                out[0][(b, j)]["idx"], rows, 1 / math.sqrt(576))
    np.testing.assert_array_equal(o, out[2][(b, j)]["o"])


# ------------------------------------------------------------------ hierarchical sparse indexer
def test_pool_topk_rank_count_bruteforce_and_order_invariance():
    rng = np.random.default_rng(21)
    for trial in range(200):
        n = int(rng.integers(1, 40))
        k = int(rng.integers(1, 12))
        pool = rng.choice(5000, n, replace=False).astype(np.int32)
        s = rng.integers(-3, 4, n).astype(np.float64)          # heavy ties
        got = oracle.pool_topk(s, pool, k)
        # rank count: an entry is kept iff fewer than k entries beat it by
        # (score desc, token index asc)
        beats = (s[None, :] > s[:, None]) | ((s[None, :] == s[:, None]) & (pool[None, :] < pool[:, None]))
        keep = np.sort(pool[beats.sum(axis=1) < k])
        want = np.full(k, -1, np.int32)
        want[:len(keep)] = keep
        np.testing.assert_array_equal(got, want)
        perm = rng.permutation(n)
        np.testing.assert_array_equal(oracle.pool_topk(s[perm], pool[perm], k), got)
        holes = np.concatenate([pool, -np.ones(3, np.int32)])
        np.testing.assert_array_equal(oracle.pool_topk(np.concatenate([s, [9.0, 9.0, 9.0]]), holes, k), got)
    # a pool of exactly k entries is returned whole, sorted
    pool = np.array([40, 3, 17, 8], np.int32)
    np.testing.assert_array_equal(oracle.pool_topk([0.1, 0.9, 0.5, 0.2], pool, 4), np.sort(pool))


def test_full_layer_pool_is_consistent_with_its_topk():
    rng = np.random.default_rng(22)
    s = rng.integers(0, 50, 3000).astype(np.float64)
    for k, C in ((16, 64), (100, 100), (7, 2999)):
        pool = oracle.topk(s, 3000, C)
        np.testing.assert_array_equal(oracle.pool_topk(s[pool], pool, k), oracle.topk(s, 3000, k))


def test_pool_reindex_with_every_position_is_the_full_scan():
    wl = inputs.small_workload("pool", 2, 2, [700, 150], 40, modes=("F", "R", "U"))
    caches, layers = _logical_inputs(wl)
    scale = 1 / math.sqrt(576)
    plain = oracle.decode_group(wl.q_tokens, wl.modes, range(wl.batch), wl.lens(), caches, layers, wl.top_k, scale)
    big = oracle.decode_group(wl.q_tokens, wl.modes, range(wl.batch), wl.lens(), caches, layers, wl.top_k, scale,
                              pool_size=1000)
    small = oracle.decode_group(wl.q_tokens, wl.modes, range(wl.batch), wl.lens(), caches, layers, wl.top_k, scale,
                                pool_size=64)
    for key in plain[0]:
        # a pool holding every valid position reduces to the full scan
        np.testing.assert_array_equal(big[1][key]["idx"], plain[1][key]["idx"])
        np.testing.assert_array_equal(big[1][key]["o"], plain[1][key]["o"])
        # with a smaller pool the Reindex layer picks only pool members,
        # the Full layer and its Reuse consumer are unchanged
        pool = small[0][key]["pool"]
        sel = small[1][key]["idx"]
        assert set(sel[sel >= 0]) <= set(pool[pool >= 0])
        np.testing.assert_array_equal(small[0][key]["idx"], plain[0][key]["idx"])
        np.testing.assert_array_equal(small[2][key]["idx"], plain[2][key]["idx"])
        b, j = key
        pos = wl.lens()[b] - wl.q_tokens + j
        # the pool is the Full layer's top-64 under its own scores
        sc = oracle.indexer_scores(layers[0][b]["qidx"][j], layers[0][b]["w"][j],
                                   caches[0][b]["kidx"][:pos + 1], caches[0][b]["ksig"][:pos + 1])
        np.testing.assert_array_equal(pool, oracle.topk(sc, pos + 1, 64))


# ------------------------------------------------------------------ replay (window-only, many query tokens)
def test_window_only_queries_are_banded_causal_attention():
    """L query tokens with no selected entries, each over its 128 window rows
    (rows j .. j+127 of a [127 + L]-row window tensor; rows at negative
    positions skipped), equal banded causal attention computed by torch's
    scaled_dot_product_attention in fp64 with a band mask (library)."""
    g = torch.Generator().manual_seed(31)
    W, L = 128, 40
    scale = 1 / math.sqrt(576)
    q = torch.randn(L, 16, 576, generator=g).to(torch.bfloat16)
    rows = torch.randn(W + L - 1, 576, generator=g).to(torch.bfloat16)
    empty = np.zeros((0, 288), np.uint8), np.zeros((0, 36), np.uint8)
    for T in (W + L - 1, 60):                       # full window, and a short sequence
        first = T - (W + L - 1)                     # position of window row 0
        q64 = q.to(torch.float64).transpose(0, 1)   # [16, L, 576]
        kv64 = rows.to(torch.float64)
        r = torch.arange(W + L - 1)
        j = torch.arange(L)[:, None]
        band = (r[None, :] >= j) & (r[None, :] <= j + W - 1) & (first + r[None, :] >= 0)
        ro = F.scaled_dot_product_attention(q64, kv64[None], kv64[None], attn_mask=band[None], scale=scale)
        for jj in (0, 17, L - 1):
            sel = [x for x in range(jj, jj + W) if first + x >= 0]
            o, lse = oracle.sparse_attn(oracle.bf16_bits(q[jj]), *empty, np.zeros(0, np.int32),
                                        oracle.bf16_bits(rows)[sel], scale)
            np.testing.assert_allclose(o, ro[:, jj].numpy(), rtol=0, atol=1e-12)
            logits = (q64[:, jj] @ kv64[band[jj]].T) * scale
            np.testing.assert_allclose(lse, torch.logsumexp(logits, dim=-1).numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------------------------ context-parallel merges
def test_sharded_topk_merge_equals_unsharded_topk():
    """Each of G shards takes the top-k of its own contiguous positions; the
    merge of their candidate lists equals the top-k of the whole context
    (heavy ties included, so the tie rule must survive the merge)."""
    rng = np.random.default_rng(41)
    for G, n, k in ((2, 3000, 100), (4, 1001, 257), (8, 640, 640), (3, 50, 80)):
        s = rng.integers(0, 20, n).astype(np.float64)
        want = oracle.topk(s, n, k)
        bounds = np.linspace(0, n, G + 1).astype(int)
        cs, ci = [], []
        for r in range(G):
            t0, t1 = bounds[r], bounds[r + 1]
            loc = oracle.topk(s[t0:t1], t1 - t0, k)
            loc = loc[loc >= 0]
            cs.append(s[t0 + loc])
            ci.append((t0 + loc).astype(np.int32))
        np.testing.assert_array_equal(oracle.merge_topk_candidates(cs, ci, k), want)


def test_sharded_attention_lse_merge_equals_one_softmax():
    """Attention over the selected entries split between shards (the window
    on the last shard), merged by LSE, equals one softmax over all of them;
    a shard with no key contributes nothing."""
    q, codes, scales, swa = _rand_case(43, n_cache=40, n_swa=7)
    scale = 1 / math.sqrt(576)
    qb, wb = oracle.bf16_bits(q), oracle.bf16_bits(swa)
    idx = np.arange(40, dtype=np.int32)
    o_all, lse_all = oracle.sparse_attn(qb, codes, scales, idx, wb, scale)
    no_rows = np.zeros((0, 576), np.uint16)
    parts = [(idx[:13], no_rows), (np.zeros(0, np.int32), no_rows), (idx[13:], wb)]
    res = [oracle.sparse_attn(qb, codes, scales, i, rows, scale) for i, rows in parts]
    assert np.all(np.isneginf(res[1][1]))
    o, lse = oracle.lse_merge([r[0] for r in res], [r[1] for r in res])
    np.testing.assert_allclose(o, o_all, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_all, rtol=0, atol=1e-12)
    o0, l0 = oracle.lse_merge([res[1][0]], [res[1][1]])
    assert np.all(o0 == 0) and np.all(np.isneginf(l0))
