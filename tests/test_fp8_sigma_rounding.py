"""The FP8 indexer quantiser computes sigma = RN(amax / 448) without a
division: q0 = RN(amax * r) with r = RN(1/448), then one fma correction
q1 = RN(q0 + RN(amax - q0 * 448) * r) (each fma rounded once). This pins that
the correction equals the correctly rounded quotient for every finite,
non-negative bf16 amax (the only inputs the kernel gives it), with exact
rational arithmetic for every rounding step (binary32, subnormals included)."""
import math
import struct
from fractions import Fraction as F


def rn32(x: F) -> F:
    """Binary32 round-to-nearest-even of an exact rational (no overflow here)."""
    if x == 0:
        return F(0)
    s = -1 if x < 0 else 1
    a = abs(x)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while F(2) ** e > a:
        e -= 1
    while F(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)                             # subnormals share the quantum 2^-149
    q = F(2) ** (e - 23)
    n = a / q
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > F(1, 2) or (rem == F(1, 2) and fl % 2 == 1):
        fl += 1
    return s * fl * q


def bf16(bits: int) -> F:
    return F(struct.unpack("<f", struct.pack("<I", bits << 16))[0])


def test_rn32_helper_matches_numpy_on_samples():
    import numpy as np
    rng = np.random.default_rng(3)
    for v in rng.standard_normal(2000) * 10.0 ** rng.integers(-40, 38, 2000):
        assert rn32(F(float(v))) == F(float(np.float32(v)))


def test_sigma_fma_correction_is_the_correctly_rounded_quotient_for_every_bf16():
    r = rn32(F(1, 448))
    bad = []
    for bits in range(0, 0x7F80):                # +0 .. largest finite bf16
        a = bf16(bits)
        q0 = rn32(a * r)
        e = rn32(a - q0 * 448)
        q1 = rn32(q0 + e * r)
        if q1 != rn32(a / 448):
            bad.append(bits)
    assert not bad, [hex(b) for b in bad[:10]]
