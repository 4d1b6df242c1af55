"""Pins for the oracle's number formats and ExpCast (CPU only).

Each check compares the oracle with something other than itself: torch's
float8_e4m3fn / bfloat16 conversions (library routines), exact rational
arithmetic (fractions), the identity the ExpCast page prints, or the error
bounds that follow from the E4M3 format.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))


def test_e4m3_decode_all_codes_match_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ours = orc.e4m3_value(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zero is kept
    assert np.signbit(ours[0x80]) and not np.signbit(ours[0x00])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def _random_f32(rng, n, lo_exp=-20, hi_exp=9):
    mant = rng.integers(0, 1 << 23, n, dtype=np.uint32)
    ex = rng.integers(127 + lo_exp, 127 + hi_exp, n, dtype=np.uint32)
    sign = rng.integers(0, 2, n, dtype=np.uint32) << 31
    return (sign | (ex << 23) | mant).view(np.float32)


def test_e4m3_encode_matches_torch_rne(orc):
    rng = np.random.default_rng(1)
    x = _random_f32(rng, 1 << 21)
    # all midpoints between adjacent codes, where ties-to-even decides
    vals = orc.e4m3_value(np.arange(0, 0x7F, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1000)])
    x = x[np.abs(x) < 464]          # torch does not saturate; above 464 it gives NaN
    ours = orc.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_saturates_to_448():
    import oracle as orc
    x = np.array([448, 464, 465, 480, 1e6, np.inf, -470, -np.inf], np.float32)
    assert orc.e4m3_encode(x).tolist() == [0x7E] * 6 + [0xFE] * 2


def test_bf16_round_matches_torch(orc):
    rng = np.random.default_rng(2)
    x = _random_f32(rng, 1 << 20, -60, 60)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.bf16_round(x), ref)


def test_expcast_identity_golden(orc):
    """byte = 8*log2(v) + 56 exactly where the mantissa field is zero."""
    rows = [ln.split() for ln in open(os.path.join(HERE, "golden", "expcast_identity.txt"))
            if ln.strip() and not ln.startswith("#")]
    for b, v in rows:
        assert orc.e4m3_value(np.uint8(int(b))) == float(Fraction(v))
    # and for every other normal code the identity is only approximate
    codes = np.arange(8, 127, dtype=np.uint8)
    approx = 8 * np.log2(orc.e4m3_value(codes)) + 56
    assert np.all(np.abs(approx - codes) < 1.0)
    assert np.all((approx == codes) == (codes % 8 == 0))


def test_expcast_fma_single_rounding_exact_rational(orc):
    """The byte is the nearest integer of the binary32-rounded fused product-sum."""
    rng = np.random.default_rng(3)
    n = 4000
    acc = (rng.standard_normal(n) * 3000).astype(np.float32)
    alpha = (rng.uniform(0.001, 0.2, n)).astype(np.float32)
    c = (rng.integers(-400, 130, n)).astype(np.float32)
    got = orc.expcast(acc, alpha, c)
    for i in range(n):
        exact = Fraction(float(acc[i])) * Fraction(float(alpha[i])) + Fraction(float(c[i]))
        v32 = float(np.float32(_round_to_f32(exact)))
        r = _rne_int(Fraction(v32))
        want = 0 if r <= 0 else min(r, 126)
        assert got[i] == want, (acc[i], alpha[i], c[i])


def _round_to_f32(q: Fraction) -> float:
    """Round an exact rational to the nearest binary32 (ties to even)."""
    if q == 0:
        return 0.0
    f = float(q)                       # nearest double
    a = np.float32(f)
    # fix double rounding: pick between the two binary32 neighbours of q
    lo = np.float32(a) if Fraction(float(a)) <= q else np.nextafter(a, np.float32(-np.inf))
    hi = np.nextafter(lo, np.float32(np.inf))
    dl, dh = q - Fraction(float(lo)), Fraction(float(hi)) - q
    if dl < dh:
        return float(lo)
    if dh < dl:
        return float(hi)
    return float(lo) if (lo.view(np.uint32) & 1) == 0 else float(hi)


def _rne_int(q: Fraction) -> int:
    fl = q.numerator // q.denominator
    rem = q - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def test_expcast_error_bounds_and_grid_position(orc):
    """Decoded byte vs the true 2^((v-56)/8): within the piecewise-linear bound
    (1+f)/2^f <= 1.0615 times the rounding factor 2^(+-1/16), and in the
    normal range it is the nearest E4M3 code or the next one up."""
    v = np.linspace(7.6, 126.4, 2_000_001).astype(np.float32)
    b = orc.expcast(v, 1.0, 0.0)
    val = orc.e4m3_value(b)
    true = 2.0 ** ((v.astype(np.float64) - 56) / 8)
    m = b >= 8
    rel = val[m] / true[m]
    lo, hi = 2 ** (-1 / 16), 2 ** (1 / 16) * (1 / np.log(2)) / 2 ** (1 / np.log(2) - 1)
    assert rel.min() >= lo - 1e-12 and rel.max() <= hi + 1e-12
    assert rel.min() < lo + 1e-4 and rel.max() > hi - 1e-3   # bounds are attained
    near = orc.e4m3_encode(true.astype(np.float32))
    mm = m & (near >= 8)
    off = b[mm].astype(int) - near[mm].astype(int)
    assert set(np.unique(off).tolist()) <= {0, 1}


def test_expcast_clamp_and_special_values(orc):
    acc = np.array([1e30, -1e30, 0.0, -0.0, np.nan, 130.0, 126.6, 0.49, 0.5, 1.5, 2.5], np.float32)
    got = orc.expcast(acc, 1.0, 0.0).tolist()
    assert got == [126, 0, 0, 0, 0, 126, 126, 0, 0, 2, 2]


def test_kappa_folds_log2e_and_byte_units(orc):
    s = np.float32(1 / np.sqrt(128))
    assert orc.kappa(s) == np.float32(8 * np.log2(np.e) * np.float64(s))
    # the scale ln2/8 makes one byte unit exactly one nat*8*log2e = 1
    assert orc.kappa(np.float32(np.log(2) / 8)) == np.float32(1.0)


def test_repair_count_matches_workloads(orc):
    assert [orc.repair_count(0.005, n) for n in (1024, 4256, 16544, 32928, 75600)] == \
        [6, 22, 83, 165, 378]
    assert orc.repair_count(0.0, 1000) == 0 and orc.repair_count(0.5, 3) == 2
