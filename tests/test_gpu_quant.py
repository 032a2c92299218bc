"""K1 (FP4 quantize + append) against the oracle: bit-exact bytes."""
import numpy as np
import pytest
import torch

import oracle
from fp8_cases import double_rounding_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from compressed_sparse_attention_quant_b200 import lib as L
    return L


def _bf16_from_bits(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)


def _quant_through_cache(lib, x_bits: np.ndarray, seed=0):
    """Quantize rows via the kernel into randomly placed slots; read them back."""
    n = x_bits.shape[0]
    pages = (n + 63) // 64 + 3
    cache = lib.PagedCache(pages)
    g = torch.Generator().manual_seed(seed)
    slots = torch.randperm(pages * 64, generator=g)[:n].to(torch.int32).cuda()
    x = _bf16_from_bits(x_bits).cuda()
    lib.quant_kv_fp4(x, slots, cache)
    assert lib.last_device_error() == 0
    fp4 = cache.kv_fp4.view(-1, 288)[slots.long()].cpu().numpy()
    sc = cache.kv_scale.view(-1, 36)[slots.long()].cpu().numpy()
    return fp4, sc


def test_quant_random_rows_bit_exact(lib):
    rng = np.random.default_rng(0)
    mag = np.exp(rng.uniform(-12, 10, (3000, 1)))
    x = torch.from_numpy(rng.standard_normal((3000, 576)) * mag).to(torch.bfloat16)
    bits = oracle.bf16_bits(x)
    fp4, sc = _quant_through_cache(lib, bits)
    rc, rs = oracle.quant_fp4(bits)
    np.testing.assert_array_equal(sc, rs)
    np.testing.assert_array_equal(fp4, rc)


def test_quant_every_value_under_every_scale(lib):
    """Every finite bf16 magnitude x <= 6s under every positive E4M3 scale s
    (group max pinned to 6s), both signs, plus ties on every midpoint."""
    e4m3 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    allv = (allbits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    rows = []
    rng = np.random.default_rng(1)
    for sb in range(1, 127):
        s = e4m3[sb]
        A = 6 * s                                       # exact in bf16 (<= 6 significant bits)
        vals = allbits[np.isfinite(allv) & (np.abs(allv) <= A)]
        mids = s * np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
        midbits = oracle.bf16_bits(torch.from_numpy(np.r_[mids, -mids]).to(torch.bfloat16))
        vals = np.r_[vals, midbits]
        if len(vals) > 15 * 40:
            vals = rng.choice(vals, 15 * 40, replace=False)
        pad = (-len(vals)) % 15
        vals = np.r_[vals, np.zeros(pad, np.uint16)].reshape(-1, 15)
        head = oracle.bf16_bits(torch.full((len(vals), 1), A, dtype=torch.float64).to(torch.bfloat16))
        rows.append(np.concatenate([head, vals], axis=1))   # one 16-channel group per row
    groups = np.concatenate(rows)
    pad = (-len(groups)) % 36
    groups = np.concatenate([groups, np.zeros((pad, 16), np.uint16)])
    x_bits = groups.reshape(-1, 576)
    fp4, sc = _quant_through_cache(lib, x_bits, seed=2)
    rc, rs = oracle.quant_fp4(x_bits)
    np.testing.assert_array_equal(sc, rs)
    np.testing.assert_array_equal(fp4, rc)


def test_quant_scale_boundaries(lib):
    """Group maxima on both sides of every E4M3 midpoint times 6 and of the
    underflow / saturation limits."""
    e4m3 = torch.arange(127, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mids = np.r_[(e4m3[:-1] + e4m3[1:]) / 2, 2.0 ** -10, 448.0, 464.0, 500.0]
    amax = torch.from_numpy(6 * mids).to(torch.bfloat16)
    up = torch.nextafter(amax.float(), torch.tensor(1e30)).to(torch.bfloat16)
    cand = torch.cat([amax, up, amax * 1.0078125, amax * 0.9921875]).to(torch.bfloat16)
    cand = torch.cat([cand, torch.tensor([0.0, -0.0, 3e38, -3e38, 1e-40], dtype=torch.bfloat16)])
    bits = oracle.bf16_bits(cand)
    groups = np.zeros((len(bits), 16), np.uint16)
    groups[:, 3] = bits
    pad = (-len(groups)) % 36
    x_bits = np.concatenate([groups, np.zeros((pad, 16), np.uint16)]).reshape(-1, 576)
    fp4, sc = _quant_through_cache(lib, x_bits, seed=3)
    rc, rs = oracle.quant_fp4(x_bits)
    np.testing.assert_array_equal(sc, rs)
    np.testing.assert_array_equal(fp4, rc)


def test_quant_appends_indexer_key_and_skips_negative_slots(lib):
    n = 200
    cache = lib.PagedCache(8)
    g = torch.Generator().manual_seed(4)
    slots = torch.randperm(8 * 64, generator=g)[:n].to(torch.int32)
    slots[::7] = -1
    x = torch.randn(n, 576, generator=g).to(torch.bfloat16).cuda()
    kid = torch.randint(0, 256, (n, 64), generator=g, dtype=torch.int32).to(torch.uint8).cuda()
    ks = torch.rand(n, generator=g).cuda()
    lib.quant_kv_fp4(x, slots.cuda(), cache, kid, ks)
    assert lib.last_device_error() == 0
    live = slots >= 0
    sl = slots[live].long()
    logical = cache.kidx_logical().reshape(-1, 64)
    assert torch.equal(logical[sl].cpu(), kid.cpu()[live])
    assert torch.equal(cache.kidx_scale.view(-1)[sl].cpu(), ks.cpu()[live])
    written = torch.zeros(8 * 64, dtype=torch.bool)
    written[sl] = True
    assert torch.all(cache.kv_scale.view(-1, 36)[~written.cuda()] == 0)


def test_quant_out_of_range_slot_sets_device_status(lib):
    cache = lib.PagedCache(2)
    x = torch.randn(4, 576).to(torch.bfloat16).cuda()
    slots = torch.tensor([0, 1, 128, 5], dtype=torch.int32).cuda()   # 128 >= 2 pages * 64
    lib.quant_kv_fp4(x, slots, cache)
    assert lib.last_device_error() == 6            # CSA2_ERR_DEVICE_BOUNDS
    assert lib.last_device_error() == 0            # cleared by the read
    assert torch.any(cache.kv_scale.view(-1, 36)[0] != 0)


# ------------------------------------------------------------------ K1b: indexer FP8 quantiser
def _index_rows(rng, n):
    """Wide-magnitude rows plus the rows where a rounding decision is close:
    zero rows, bf16 subnormals, near the bf16 maximum, E4M3 midpoints (ties)
    and their bf16 neighbours under sigma = 1, and rows whose binary32
    quotient x / sigma lands exactly on an E4M3 midpoint that the exact
    quotient misses."""
    x = rng.standard_normal((n, 64)) * np.exp2(rng.integers(-60, 60, (n, 1)))
    x[0] = 0.0
    x[1] = -0.0
    x[2] = rng.standard_normal(64) * 1e-39
    x[3, :] = 3.3e38
    x[3, 1::2] *= -1
    x[4] = 0.0
    x[4, 63] = -2.0e-38
    ev = torch.arange(127, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mids = (ev[:-1] + ev[1:]) / 2
    rows = []
    for k in range(0, len(mids), 63):
        r = np.zeros(64)
        r[0] = 448.0
        m = mids[k:k + 63]
        r[1:1 + len(m)] = m * np.where(np.arange(len(m)) % 2 == 0, 1, -1)
        rows.append(r)
    x[5:5 + len(rows)] = np.array(rows)
    bits = oracle.bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
    # bf16 neighbours of the midpoint rows (one ulp up and down, same row maximum)
    nb = bits[5:5 + len(rows)].copy()
    up, down = nb.copy(), nb.copy()
    up[:, 1:] += (nb[:, 1:] & 0x7FFF) != 0
    down[:, 1:] -= (nb[:, 1:] & 0x7FFF) != 0
    special = 5 + len(rows)
    # the close-call rows first, so that a caller taking the first n rows keeps them
    return np.concatenate([bits[:special], up, down, double_rounding_rows(40, seed=n), bits[special:]])


@pytest.mark.parametrize("n", [1, 37, 75813])
def test_quant_indexer_fp8_bit_exact(lib, n):
    """Codes and sigma bit-exact against the oracle; 75813 rows run the
    grid-stride loop twice per thread with a ragged tail."""
    rng = np.random.default_rng(n)
    bits = _index_rows(rng, max(n, 16))[:n] if n >= 16 else oracle.bf16_bits(
        torch.from_numpy(rng.standard_normal((n, 64))).to(torch.bfloat16))
    x = _bf16_from_bits(bits).cuda()
    codes, sigma = lib.quant_indexer_fp8(x)
    assert lib.last_device_error() == 0
    rc, rs = oracle.quant_index_fp8(bits)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(sigma.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def test_quant_indexer_fp8_feeds_the_cache_and_indexer(lib):
    """Quantised keys go through K1's indexer-key path unchanged, and an empty
    call is a no-op."""
    rng = np.random.default_rng(5)
    bits = oracle.bf16_bits(torch.from_numpy(rng.standard_normal((200, 64))).to(torch.bfloat16))
    kc, ks = lib.quant_indexer_fp8(_bf16_from_bits(bits).cuda())
    cache = lib.PagedCache(4)
    slots = torch.arange(200, dtype=torch.int32, device="cuda")
    xkv = torch.zeros(200, 576, dtype=torch.bfloat16, device="cuda")
    lib.quant_kv_fp4(xkv, slots, cache, kc, ks)
    assert lib.last_device_error() == 0
    got = cache.kidx_logical().reshape(-1, 64)[:200].cpu().numpy()
    np.testing.assert_array_equal(got, kc.cpu().numpy())
    np.testing.assert_array_equal(cache.kidx_scale.reshape(-1)[:200].cpu().numpy(), ks.cpu().numpy())
    e = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    c0, s0 = lib.quant_indexer_fp8(e)
    assert c0.shape == (0, 64) and s0.shape == (0,)
