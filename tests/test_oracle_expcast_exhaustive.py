"""Exhaustive pin of the oracle's ExpCast over the whole score range.

Page "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58× sem
retreinamento", section "ExpCast-FP8: eliminando o gargalo do softmax": the
probability byte is written from the log-domain score by one fused
multiply-add, because an E4M3 byte read as an integer is close to
8*log2(v) + 56.

Every binary32 score acc with acc*alpha in [-(c+1), 0] is swept (about 1.1e9
inputs per case): the scores that can reach a nonzero byte when the frame
offset is c. Two cases: alpha = 1, c = C = 120 (the score is the byte-unit
value itself), and a non-power-of-two alpha with c = 112 (a frame one binade
above the running maximum), so that the fused product's rounding is
exercised. For each input the independent checker (tests/expcast_pin.c)
computes the probability t = 2^((acc*alpha + c - 56)/8) with exp2 and its
nearest E4M3 value; the oracle's byte must decode to that value or to the
next code up wherever the byte is a normal code, and decoded/t must lie in
[2^(-h/8), 2^(h/8) * max_f (1+f)/2^f] with h = 1/2 + 2^-18: half a byte of
integer rounding plus half a binary32 ulp of the fused sum (below 128 its ulp
is at most 2^-17; that part of the bound is attained, at sums that round
onto a half-integer). Along each sweep the bytes must move
monotonically, and every point where the byte changes is checked with exact
rational arithmetic (the binary32 rounding of acc*alpha + c, then the
nearest integer with ties to even): together these fix every byte of the
range.
"""
import ctypes
import math
import os
import subprocess
from fractions import Fraction

import numpy as np
import pytest

from test_oracle_formats import _rne_int, _round_to_f32

HERE = os.path.dirname(os.path.abspath(__file__))
CHUNK = 1 << 26


class PinStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_longlong) for n in ("n_normal", "n_equal", "n_next", "n_bad", "n_ambiguous",
                                                 "n_nonmono", "n_trans")] + \
               [("min_ratio", ctypes.c_double), ("max_ratio", ctypes.c_double)]


@pytest.fixture(scope="module")
def pin(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("pin") / "libexpcast_pin.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fopenmp",
                           os.path.join(HERE, "expcast_pin.c"), "-o", out, "-lm"])
    L = ctypes.CDLL(out)
    P = ctypes.c_void_p
    L.pin_expcast_run.argtypes = [P, ctypes.c_uint32, ctypes.c_longlong, ctypes.c_int, ctypes.c_double,
                                  ctypes.c_double, ctypes.c_int, ctypes.POINTER(PinStats), P, P, P,
                                  ctypes.c_longlong]
    return L


def _f32_bits(x: float) -> int:
    return int(np.float32(x).view(np.uint32))


def _exact_byte(acc: float, alpha: float, c: float) -> int:
    """The byte by exact rational arithmetic: binary32 rounding of acc*alpha + c, nearest integer (ties to
    even), clamped to [0, 126]."""
    q = Fraction(acc) * Fraction(alpha) + Fraction(c)
    r = _rne_int(Fraction(_round_to_f32(q)))
    return 0 if r <= 0 else min(r, 126)


def _sweep(orc, pin, alpha: float, c: float):
    """All binary32 acc <= 0 with acc*alpha >= -(c+1): magnitudes by bit pattern from +0 upwards."""
    alpha = float(np.float32(alpha))
    last = _f32_bits(float(np.float32((c + 1.0) / alpha)))
    while float(np.float32(np.uint32(last).view(np.float32))) * alpha < c + 1.0:
        last += 1
    n_total = last + 1
    st = PinStats(0, 0, 0, 0, 0, 0, 0, np.inf, -np.inf)
    cap = 4096
    t_bits = np.zeros(cap, np.int64)
    t_from = np.zeros(cap, np.int32)
    t_to = np.zeros(cap, np.int32)
    prev = -1
    first_byte = None
    for lo in range(0, n_total, CHUNK):
        n = min(CHUNK, n_total - lo)
        b = orc.expcast_bits(lo, n, True, alpha, c)
        if first_byte is None:
            first_byte = int(b[0])
        pin.pin_expcast_run(b.ctypes.data, lo, n, 1, alpha, float(c), prev, ctypes.byref(st),
                            t_bits.ctypes.data, t_from.ctypes.data, t_to.ctypes.data, cap)
        prev = int(b[-1])
    k = min(st.n_trans, cap)
    return st, n_total, first_byte, prev, list(zip(t_bits[:k].tolist(), t_from[:k].tolist(), t_to[:k].tolist()))


def _neg_f32(bits: int) -> float:
    return -float(np.uint32(bits).view(np.float32))


PL_MAX = (1 / math.log(2)) / 2 ** (1 / math.log(2) - 1)   # max over f in [0,1] of (1+f)/2^f


@pytest.mark.parametrize("alpha,c", [(1.0, 120.0), (0.0553709, 112.0)])
def test_expcast_exhaustive_over_score_range(orc, pin, alpha, c):
    alpha32 = float(np.float32(alpha))
    st, n_total, first_byte, last_byte, trans = _sweep(orc, pin, alpha32, c)
    assert n_total > 1_000_000_000
    # the normal-code range: nearest E4M3 of the true probability or the next code up
    assert st.n_bad == 0 and st.n_ambiguous == 0, (st.n_bad, st.n_ambiguous)
    assert st.n_normal > 0.9 * n_total
    # binary32 inputs crowd towards acc = 0 (the row maximum, an exact power of two), so most of them
    # take the nearest code; the next code up still occurs millions of times
    assert st.n_equal + st.n_next == st.n_normal and st.n_next > 1_000_000
    h = 0.5 + 2.0 ** -18
    lo, hi = 2 ** (-h / 8), 2 ** (h / 8) * PL_MAX
    assert lo - 1e-12 <= st.min_ratio and st.max_ratio <= hi + 1e-12, (st.min_ratio, st.max_ratio)
    assert st.min_ratio < lo + 1e-3 and st.max_ratio > hi - 1e-3   # both bounds are approached
    # monotone, one step at a time, from byte c at acc = -0 down to 0 at the far end
    assert st.n_nonmono == 0
    assert first_byte == int(c) and last_byte == 0
    assert st.n_trans == int(c) and [t[1] - t[2] for t in trans] == [1] * int(c)
    # every change point, exactly: the last input with the old byte and the first with the new one
    for bits, before, after in trans:
        assert _exact_byte(_neg_f32(bits), alpha32, c) == after
        assert _exact_byte(_neg_f32(bits - 1), alpha32, c) == before
