"""Pins for the oracle's NVFP4-residual variant (CPU only).

Page "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58× sem
retreinamento": "V-Smooth: corrigindo outliers de valor", item Demean (the
residual in NVFP4 for the 4-bit kernel) and "ExpCast-FP8: eliminando o
gargalo do softmax" (ExpCast is 8-bit only: the 4-bit kernel takes its
probabilities from an exp2 softmax).

What pins it, none of it the oracle's own formulas retyped:
- the E2M1 format against a library (ml_dtypes' float4_e2m1fn, round to
  nearest even) for every code and a dense set of binary32 inputs;
- the probability and value quantizers against properties the NVFP4 format
  fixes (the block maximum takes the top code, the rounding error is within
  half a grid step, scaling by a power of two commutes with quantization, an
  input already on the grid is reproduced exactly);
- the whole 4-bit attention against exact softmax attention in a lossless
  case, where every probability and every value residual is on the NVFP4 grid
  (frame changes, a ragged last tile and a partial scale block included), and
  against an un-tiled evaluation on random inputs.
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

from bit_attention_diffusion_b200 import synth

E2M1_LIB = ml_dtypes.float4_e2m1fn
E4M3_LIB = ml_dtypes.float8_e4m3fn


# ---------------------------------------------------------------- E2M1
def test_e2m1_decode_all_codes_match_library(orc):
    lib_vals = np.arange(16, dtype=np.uint8).view(E2M1_LIB).astype(np.float64)
    ours = orc.e2m1_value(np.arange(16, dtype=np.uint8))
    assert np.array_equal(ours, lib_vals)
    assert np.array_equal(np.signbit(ours), np.signbit(lib_vals))


def test_e2m1_encode_matches_library_rne(orc):
    rng = np.random.default_rng(3)
    grid = np.arange(-8 * 4096, 8 * 4096 + 1, dtype=np.float64) / 4096.0   # every multiple of 2^-12 in [-8, 8]
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0], np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(10))])
    rand = (rng.standard_normal(200000) * np.exp2(rng.uniform(-12, 6, 200000))).astype(np.float32)
    big = np.array([6.0, 6.5, 8.0, 1e3, 3e38, -6.5, -1e3, 0.0, -0.0, 1e-40, -1e-40], np.float32)
    x = np.concatenate([grid.astype(np.float32), near, -near, rand, big])
    ours = orc.e2m1_encode(x)
    want = x.astype(E2M1_LIB).view(np.uint8)
    bad = np.nonzero(ours != want)[0]
    assert bad.size == 0, (x[bad[:5]], ours[bad[:5]], want[bad[:5]])


# ---------------------------------------------------------------- probabilities
def _p_blocks(rng, nblk, lo=-14.0):
    """Blocks of 16 exponents x <= 0 whose maximum lies in [lo, 0]."""
    x = rng.uniform(-6.0, 0.0, (nblk, 16)).astype(np.float32)
    top = rng.uniform(lo, 0.0, (nblk, 1)).astype(np.float32)
    return (x - x.max(1, keepdims=True) + top).astype(np.float32)


def test_p_block_maximum_takes_the_top_code(orc):
    """With a normal block scale the block maximum maps to 6 within the scale's
    rounding (448 a / sf in [1/(1+1/16), 1/(1-1/16)]), and 6 x that is above 5."""
    rng = np.random.default_rng(7)
    for x in _p_blocks(rng, 400):
        codes, sfc = orc.nvfp4_p_block(x)
        assert codes[int(np.argmax(x))] == 7
        assert 0 < sfc < 0x7F


def test_p_block_error_within_half_a_grid_step(orc):
    rng = np.random.default_rng(8)
    for x in _p_blocks(rng, 300, lo=-20.0):
        codes, sfc = orc.nvfp4_p_block(x)
        sfv = float(orc.e4m3_value(np.array([sfc], np.uint8))[0])
        p = np.exp2(x.astype(np.float64))
        if sfv == 0.0:
            assert np.all(codes == 0)
            continue
        q = p * 2688.0 / sfv                     # the exact scaled value
        got = orc.e2m1_value(codes)
        half = np.where(q < 2.0, 0.25, np.where(q < 4.0, 0.5, 1.0))
        # the multiplier is 2688/sf rounded once to binary32: allow its relative
        # rounding; past 7 (a subnormal scale rounded far down) the code saturates
        sat = q >= 7.0
        assert np.all(got[sat] == 6.0)
        assert np.all(np.abs(got - q)[~sat] <= (half + q * 2.0 ** -23)[~sat]), (x, codes, sfc)
        assert np.all(codes < 8)                  # probabilities are never negative


def test_p_block_matches_library_roundings(orc):
    """The scale and the codes from library conversions (ml_dtypes E4M3 and
    E2M1, round to nearest even) applied to the same binary32 steps."""
    rng = np.random.default_rng(9)
    for x in _p_blocks(rng, 300, lo=-24.0):
        n = int(rng.integers(1, 17))
        xs = x[:n]
        p = np.exp2(xs.astype(np.float64)).astype(np.float32)
        a = p.max()
        sf = np.array([a * np.float32(448.0)], np.float32).astype(E4M3_LIB)
        sfv = np.float32(sf.astype(np.float64)[0])
        rcp = np.float32(0.0) if sfv == 0 else np.float32(np.float32(2688.0) / sfv)
        want = (p * rcp).astype(np.float32).astype(E2M1_LIB).view(np.uint8)
        codes, sfc = orc.nvfp4_p_block(xs)
        assert sfc == int(sf.view(np.uint8)[0])
        assert np.array_equal(codes, want)


# ---------------------------------------------------------------- values
def _v_case(seed, N=300, d=128, outlier=True):
    wl = synth.custom(1, 1, N, seed=seed)
    x = synth.make_inputs(wl)
    v = x["v"][0, 0].copy()
    if outlier:
        vf = synth.bf16_bits_to_f32(v)
        vf[5, 17] = 40.0
        vf[200, 3] = -25.0
        v = synth.f32_to_bf16_bits(vf)
    rng = np.random.default_rng(seed)
    perm = rng.permutation(N).astype(np.int32)
    return v, perm


def _deq(orc, vq):
    N = vq["codes"].shape[0]
    sf = orc.e4m3_value(vq["sfc"])[np.arange(N) // 16]
    return orc.e2m1_value(vq["codes"]) * sf * vq["vscale"].astype(np.float64)


def test_quant_v4_error_within_half_a_grid_step(orc):
    v, perm = _v_case(40)
    vq = orc.quant_v4_head(v, perm, demean=True, R=0)
    N = v.shape[0]
    vf = synth.bf16_bits_to_f32(v)[perm].astype(np.float64)
    mu = orc.bf16_value(vq["vmean"]).astype(np.float64)[np.arange(N) // 128]
    r = (vf - mu).astype(np.float32).astype(np.float64)
    g = vq["vscale"].astype(np.float64)
    # g is the least power of two with amax <= 2688 g
    amax = np.abs(r).max(0)
    assert np.all(amax <= 2688 * g) and np.all(amax > 1344 * g)
    assert np.all(np.log2(g) == np.round(np.log2(g)))
    sfv = orc.e4m3_value(vq["sfc"])[np.arange(N) // 16]
    err = np.abs(r - _deq(orc, vq))
    # half of the top grid step (2) in scaled units, plus the clip of a scale rounded down
    assert np.all(err <= sfv * g * 1.0 + 1e-30)
    # the per-token error the repair ranks by is the channel sum of squares
    assert np.allclose(vq["err"], ((r - _deq(orc, vq)) ** 2).sum(1), rtol=1e-5, atol=0)


def test_quant_v4_commutes_with_power_of_two_scaling(orc):
    v, perm = _v_case(41)
    vf = synth.bf16_bits_to_f32(v)
    v4 = synth.f32_to_bf16_bits(vf * 4.0)
    R = 3
    a = orc.quant_v4_head(v, perm, demean=True, R=R)
    b = orc.quant_v4_head(v4, perm, demean=True, R=R)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["sfc"], b["sfc"])
    assert np.array_equal(b["vscale"], a["vscale"] * 4)
    assert np.array_equal(orc.bf16_value(b["vmean"]), orc.bf16_value(a["vmean"]) * 4)
    assert np.array_equal(b["err"], a["err"] * 16)
    assert np.array_equal(a["rep_idx"], b["rep_idx"])
    assert np.array_equal(orc.bf16_value(b["rep_delta"]), orc.bf16_value(a["rep_delta"]) * 4)


def test_quant_v4_matches_library_roundings(orc):
    """Block scales and codes from library conversions (ml_dtypes E4M3 and
    E2M1, round to nearest even) applied to the same binary32 steps: the
    scaled block maximum over 6, and the scaled residual times the rounded
    reciprocal of the block scale."""
    v, perm = _v_case(42, N=260)
    vq = orc.quant_v4_head(v, perm, demean=True, R=0)
    N = v.shape[0]
    vf = synth.bf16_bits_to_f32(v)[perm]
    mu = orc.bf16_value(vq["vmean"])[np.arange(N) // 128].astype(np.float32)
    x = ((vf - mu).astype(np.float32) / vq["vscale"]).astype(np.float32)   # exact: g is a power of two
    for jb in range((N + 15) // 16):
        xb = x[16 * jb:16 * jb + 16]
        b = np.abs(xb).max(0).astype(np.float32)
        sf = (b / np.float32(6.0)).astype(np.float32).astype(E4M3_LIB)
        assert np.array_equal(sf.view(np.uint8), vq["sfc"][jb])
        sfv = sf.astype(np.float32)
        with np.errstate(divide="ignore"):
            rcp = np.where(sfv == 0, np.float32(0), (np.float32(1.0) / sfv).astype(np.float32)).astype(np.float32)
        want = (xb * rcp).astype(np.float32).astype(E2M1_LIB).view(np.uint8)
        want = np.where(sfv == 0, 0, want)
        assert np.array_equal(vq["codes"][16 * jb:16 * jb + 16], want), jb


# ---------------------------------------------------------------- lossless case
def _lossless_case(seed, N=300, d=128):
    """Scores on multiples of 8 byte units (kappa = 1), so every probability
    is a power of two, and within every block of 16 keys and every row the
    scores span at most two steps: 2688 p / sf is 6, 3 or 1.5, all on the
    E2M1 grid. V residuals are E2M1 values times a per-block scale that is an
    E4M3 value times g = 2^-4, each block holding a +/-6 element, in +/- pairs
    inside each 128-token block so that the block means are exact. Two tokens
    are 1/4 of a grid step off (the repair list)."""
    rng = np.random.default_rng(seed)
    scale = np.float32(np.log(2) / 8)
    perm = rng.permutation(N).astype(np.int32)
    # Q: channel 0 the amax marker (448 -> scale 1), channel 10 reads the boost,
    # one of channels 2..9 per row at 2
    q = np.zeros((N, d), np.float32)
    q[:, 0] = 448.0
    q[:, 10] = 1.0
    q[np.arange(N), rng.integers(2, 10, N)] = 2.0
    # K (permuted order): channel 1 the marker, channels 2..9 in {0, -4, -8}:
    # scores in {0, -8, -16}; the 16 keys at permuted positions 256..271 get a
    # +16 boost, so the running maximum (and the frame) moves in tile 2
    kp = np.zeros((N, d), np.float32)
    kp[:, 1] = 448.0
    kp[:, 2:10] = rng.choice([0.0, -4.0, -8.0], (N, 8))
    kp[256:272, 10] = 16.0
    # V (permuted order)
    grid = np.array([0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])

    def blocks(n16, scales):
        r = rng.choice(grid, (n16, 16, d)) * rng.choice([-1.0, 1.0], (n16, 16, d))
        slot = rng.integers(0, 16, (n16, d))
        for b in range(n16):
            r[b, slot[b], np.arange(d)] = 6.0 * rng.choice([-1.0, 1.0], d)
        return r * scales[:, None, :] / 16.0

    vp = np.zeros((N, d), np.float64)
    mus = [np.zeros(d)] + [rng.integers(-3, 4, d) / 2.0 for _ in range(2)]
    # tile 0: block [0, 16) has scale 448 on every channel and the channel amax
    # marker +/-168 = 6 * 448 / 16 at positions 2 / 66
    sc0 = rng.choice([1.0, 2.0, 4.0], (4, d))
    sc0[0] = 448.0
    h = blocks(4, sc0).reshape(64, d)
    h[2] = 168.0
    vp[0:64], vp[64:128] = h, -h
    # tile 1: four scaled blocks and their negations; the repair tokens at
    # permuted positions 133 and 197 sit at 4.25 grid units on every channel
    sc1 = rng.choice([1.0, 2.0, 4.0], (4, d))
    h = blocks(4, sc1).reshape(64, d)
    h[5] = 4.25 * sc1[0] / 16.0
    h[6] = -6.0 * sc1[0] / 16.0     # the block keeps a +/-6 element
    vp[128:192], vp[192:256] = mus[1] + h, mus[1] - h
    # tile 2 (44 tokens): blocks [256, 272) and [272, 288) paired, the partial
    # block [288, 300) without residual
    sc2 = rng.choice([1.0, 2.0, 4.0], (1, d))
    h = blocks(1, sc2).reshape(16, d)
    vp[256:272], vp[272:288] = mus[2] + h, mus[2] - h
    vp[288:300] = mus[2]
    vp = vp.astype(np.float32)
    for name, arr in (("q", q), ("kp", kp), ("vp", vp)):
        assert np.array_equal(synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(arr)), arr), name
    k = np.empty_like(kp)
    k[perm] = kp
    v = np.empty_like(vp)
    v[perm] = vp
    return (synth.f32_to_bf16_bits(q), synth.f32_to_bf16_bits(k), synth.f32_to_bf16_bits(v), perm, scale)


@pytest.mark.parametrize("seed", [50, 51, 52])
def test_lossless_case_reduces_to_exact_attention(orc, seed):
    q, k, v, perm, scale = _lossless_case(seed)
    flags = orc.FLAG_VSMOOTH | orc.FLAG_REPAIR | orc.FLAG_VFMT_NVFP4
    r = orc.vc_attention_head(q, k, v, flags=flags, rho=0.005, softmax_scale=scale, perm=perm)
    vq = r["vq"]
    assert r["R"] == 2
    assert set(np.nonzero(vq["err"])[0].tolist()) == {133, 197}
    assert vq["rep_idx"].tolist() == [133, 197]
    assert np.all(vq["vscale"] == 2.0 ** -4)
    assert np.all(r["qk"]["sq"] == 1.0) and np.all(r["qk"]["sk"] == 1.0)
    # the boost moved every row's frame from 0 to 16
    assert np.all(r["F"] == 16.0)
    ex = orc.exact_attention_head(q, k, v, softmax_scale=scale)
    rel = np.abs(r["out"] - ex).max() / np.abs(ex).max()
    assert rel < 1e-8, rel       # the softmax scale ln2/8 rounded to binary32 leaves ~1e-9
    r2 = orc.vc_attention_head(q, k, v, flags=flags & ~orc.FLAG_REPAIR, softmax_scale=scale, perm=perm)
    rel2 = np.abs(r2["out"] - ex).max() / np.abs(ex).max()
    assert rel2 > 1e3 * rel and rel2 > 1e-6


def test_lossless_case_demean_off_still_exact_without_repair_tokens(orc):
    """Without the demean the residual is the value itself: the marker block
    still fixes g, and the block means (multiples of 1/2) must then be carried
    by the codes, which puts some values off the grid; the method is then
    within NVFP4 error of exact attention, and with demean on it is exact."""
    q, k, v, perm, scale = _lossless_case(53)
    on = orc.vc_attention_head(q, k, v, flags=orc.FLAG_VSMOOTH | orc.FLAG_VFMT_NVFP4, softmax_scale=scale,
                               perm=perm)
    off = orc.vc_attention_head(q, k, v, flags=orc.FLAG_VFMT_NVFP4, softmax_scale=scale, perm=perm)
    ex = orc.exact_attention_head(q, k, v, softmax_scale=scale)
    e_on = np.abs(on["out"] - ex).max() / np.abs(ex).max()
    e_off = np.abs(off["out"] - ex).max() / np.abs(ex).max()
    assert e_off > 100 * e_on


# ---------------------------------------------------------------- online vs un-tiled
def _fma32(a, b, c) -> np.float32:
    """fmaf: the exact a*b + c rounded once to binary32 (ties to even)."""
    q = Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c))
    if q == 0:
        return np.float32(0.0)
    f = np.float32(float(q))
    lo = f if Fraction(float(f)) <= q else np.nextafter(f, np.float32(-np.inf))
    hi = np.nextafter(lo, np.float32(np.inf))
    dl, dh = q - Fraction(float(lo)), Fraction(float(hi)) - q
    if dl != dh:
        return lo if dl < dh else hi
    return lo if (lo.view(np.uint32) & 1) == 0 else hi


def _direct_global_frame4(orc, pro, N, rows, scale, qd_all=None, kd_all=None):
    """Every tile's probabilities quantized against its own frame F_t (by the
    pinned block quantizer), all contributions scaled once to the final frame.
    qd_all / kd_all: the score operands (default: the E4M3 decode of q8 / k8)."""
    qk, vq = pro["qk"], pro["vq"]
    kap = np.float32(orc.kappa(scale))
    Nb = (N + 127) // 128
    kd = orc.e4m3_value(qk["k8"][:N]) if kd_all is None else kd_all
    vd = _deq(orc, vq)
    mu = orc.bf16_value(vq["vmean"]).astype(np.float64)
    tile = np.arange(N) // 128
    out = []
    for i in rows:
        qd = orc.e4m3_value(qk["q8"][i]) if qd_all is None else qd_all[i]
        acc = (kd @ qd).astype(np.float32)
        alpha = ((np.float32(qk["sq"][i // 128]) * qk["sk"]).astype(np.float32) * kap).astype(np.float32)
        u = (acc * alpha[tile]).astype(np.float32)
        run = np.maximum.accumulate(np.array([u[tile == t].max() for t in range(Nb)], np.float32))
        Ft = (8 * np.ceil(run * np.float32(0.125))).astype(np.float32)
        P = np.zeros(N)
        for b0 in range(0, N, 16):
            b1 = min(N, b0 + 16, (b0 // 128 + 1) * 128)
            t = b0 // 128
            x = np.array([_fma32(acc[j], alpha[t] * np.float32(0.125), -Ft[t] * np.float32(0.125))
                          for j in range(b0, b1)], np.float32)
            codes, sfc = orc.nvfp4_p_block(x)
            P[b0:b1] = orc.e2m1_value(codes) * orc.e4m3_value(np.array([sfc], np.uint8))[0]
        P *= 2.0 ** ((Ft[tile].astype(np.float64) - Ft[-1]) / 8)
        lt = np.array([P[tile == t].sum() for t in range(Nb)])
        num = P @ vd + lt @ mu
        ridx = vq["rep_idx"]
        if ridx.size:
            xr = np.array([_fma32(acc[j], alpha[tile[j]] * np.float32(0.125), -Ft[-1] * np.float32(0.125))
                           for j in ridx], np.float32)
            Pr = orc.bf16_value(orc.bf16_round((np.exp2(xr.astype(np.float64)).astype(np.float32)
                                                * np.float32(2688.0)).astype(np.float32)))
            num = num + Pr.astype(np.float64) @ orc.bf16_value(vq["rep_delta"]).astype(np.float64)
        out.append(num / P.sum())
    return np.array(out)


def test_online_rescaling_equals_global_frame_form(orc):
    wl = synth.custom(1, 1, 700, seed=33)
    x = synth.make_inputs(wl)
    q, k, v = x["q"][0, 0], x["k"][0, 0], x["v"][0, 0]
    rows = np.array([0, 1, 127, 128, 300, 699], np.int32)
    r = orc.vc_attention_head(q, k, v, rows=rows, flags=orc.FLAGS_DEFAULT | orc.FLAG_VFMT_NVFP4)
    assert r["R"] == 4
    want = _direct_global_frame4(orc, r, 700, rows, orc.DEFAULT_SCALE)
    assert np.allclose(r["out"], want, rtol=1e-9, atol=1e-12)


def test_random_inputs_error_band_vs_exact(orc):
    """On i.i.d. Gaussian inputs the 4-bit variant sits near the NVFP4 noise
    floor, well above the 8-bit path's."""
    wl, x = synth.make_by_name("tiny_b1h2n1024")
    q, k, v = x["q"][0, 0], x["k"][0, 0], x["v"][0, 0]
    rows = np.arange(0, 1024, 7, dtype=np.int32)
    ex = orc.exact_attention_head(q, k, v, rows=rows)
    r4 = orc.vc_attention_head(q, k, v, rows=rows, flags=orc.FLAGS_DEFAULT | orc.FLAG_VFMT_NVFP4)
    r8 = orc.vc_attention_head(q, k, v, rows=rows)
    e4 = np.linalg.norm(r4["out"] - ex) / np.linalg.norm(ex)
    e8 = np.linalg.norm(r8["out"] - ex) / np.linalg.norm(ex)
    assert e8 < e4 < 0.5, (e4, e8)


# ---------------------------------------------------------------- full 4-bit path (Q and K in NVFP4 too)
def test_quant_qk4_matches_library_roundings(orc):
    """Per 128-row block g = the least power of two with amax <= 2688 g; per
    row and 16 channels the scale E4M3(fl(b/g)/6) and codes
    E2M1(fl(fl(x/g) * fl(1/sf))), from ml_dtypes roundings of the same
    binary32 steps; K' = K - channel mean, rows through the permutation."""
    x = synth.make_inputs(synth.custom(1, 1, 300, seed=61))
    q, k = x["q"][0, 0], x["k"][0, 0]
    perm = np.random.default_rng(61).permutation(300).astype(np.int32)
    o = orc.quant_qk4_head(q, k, perm, ksmooth=True)
    kf = synth.bf16_bits_to_f32(k).astype(np.float64)
    kbar = (kf.sum(0) / 300).astype(np.float32)
    assert np.array_equal(o["kbar"], kbar)
    for name, X, codes, sfc, g in (("q", synth.bf16_bits_to_f32(q), o["qcodes"], o["qsfc"], o["qg"]),
                                   ("k", (synth.bf16_bits_to_f32(k)[perm] - kbar).astype(np.float32), o["kcodes"],
                                    o["ksfc"], o["kg"])):
        for t in range(3):
            blk = X[128 * t:128 * t + 128]
            amax = np.abs(blk).max()
            assert amax <= 2688 * g[t] and amax > 1344 * g[t] and np.log2(g[t]) == np.round(np.log2(g[t])), name
            xs = (blk / g[t]).astype(np.float32)                      # exact: g is a power of two
            b = np.abs(xs.reshape(-1, 8, 16)).max(2).astype(np.float32)
            sf = (b / np.float32(6.0)).astype(np.float32).astype(E4M3_LIB)
            assert np.array_equal(sf.view(np.uint8), sfc[128 * t:128 * t + len(blk)]), (name, t)
            sfv = sf.astype(np.float32)
            with np.errstate(divide="ignore"):
                rcp = np.where(sfv == 0, np.float32(0), (np.float32(1.0) / sfv).astype(np.float32)).astype(np.float32)
            want = (xs.reshape(-1, 8, 16) * rcp[:, :, None]).astype(np.float32).astype(E2M1_LIB).view(np.uint8)
            want = np.where(sfv[:, :, None] == 0, 0, want).reshape(-1, 128)
            assert np.array_equal(codes[128 * t:128 * t + len(blk)], want), (name, t)
    # padding rows of the ragged last block are zero
    assert np.all(o["qcodes"][300:] == 0) and np.all(o["ksfc"][300:] == 0)


def _lossless_case_qk4(seed, N=300, d=128):
    """The a10 lossless values and permutation, with Q and K on the NVFP4 grid:
    channel block 16..31 carries everything. Q: channel 16 = 3 on every row
    (the block maximum: g_q = 2^-9, scale 256), one of channels 17..23 = 2,
    channel 24 = 1. K: channel 25 = 24 on every key (g_k = 2^-6, scale 256),
    channels 17..23 in {0, -4, -8}, channel 24 = 16 on the keys at permuted
    positions 256..271. Scores q.k lie in {0, -8, -16} (+16 for the boosted
    keys): multiples of 8 byte units at kappa = 1."""
    _, _, v, perm, scale = _lossless_case(seed, N, d)
    rng = np.random.default_rng(seed + 1000)
    q = np.zeros((N, d), np.float32)
    q[:, 16] = 3.0
    q[:, 24] = 1.0
    q[np.arange(N), rng.integers(17, 24, N)] = 2.0
    kp = np.zeros((N, d), np.float32)
    kp[:, 25] = 24.0
    kp[:, 17:24] = rng.choice([0.0, -4.0, -8.0], (N, 7))
    kp[256:272, 24] = 16.0
    k = np.empty_like(kp)
    k[perm] = kp
    return synth.f32_to_bf16_bits(q), synth.f32_to_bf16_bits(k), v, perm, scale


@pytest.mark.parametrize("seed", [70, 71])
def test_full_4bit_lossless_case_reduces_to_exact_attention(orc, seed):
    q, k, v, perm, scale = _lossless_case_qk4(seed)
    flags = orc.FLAG_VSMOOTH | orc.FLAG_REPAIR | orc.FLAG_VFMT_NVFP4 | orc.FLAG_QK_NVFP4
    r = orc.vc_attention_head(q, k, v, flags=flags, rho=0.005, softmax_scale=scale, perm=perm)
    qk = r["qk"]
    assert np.all(qk["qg"] == 2.0 ** -9) and np.all(qk["kg"] == 2.0 ** -6)
    # the scores' block: scale 256 on every row; the other blocks are empty
    assert np.all(qk["qsfc"][:300, 1] == 0x78) and np.all(qk["ksfc"][:300, 1] == 0x78)   # E4M3 256
    assert np.all(qk["qsfc"][:300, [0, 2, 3, 4, 5, 6, 7]] == 0)
    assert np.all(r["F"] == 16.0)
    ex = orc.exact_attention_head(q, k, v, softmax_scale=scale)
    rel = np.abs(r["out"] - ex).max() / np.abs(ex).max()
    assert rel < 1e-8, rel
    # a score off the grid (one key's channel 17 at -5: between -4 and -6)
    # breaks it
    kb = synth.bf16_bits_to_f32(k)
    kb[perm[10], 17] = -5.0
    r2 = orc.vc_attention_head(q, synth.f32_to_bf16_bits(kb), v, flags=flags, softmax_scale=scale, perm=perm)
    ex2 = orc.exact_attention_head(q, synth.f32_to_bf16_bits(kb), v, softmax_scale=scale)
    assert np.abs(r2["out"] - ex2).max() / np.abs(ex2).max() > 1e3 * rel


def test_full_4bit_online_rescaling_equals_global_frame_form(orc):
    """Random inputs: the online 4-bit path equals an un-tiled evaluation that
    takes the scores from the dequantized NVFP4 Q and K, quantizes each tile's
    probabilities against its own frame and scales everything once."""
    wl = synth.custom(1, 1, 400, seed=35)
    x = synth.make_inputs(wl)
    q, k, v = x["q"][0, 0], x["k"][0, 0], x["v"][0, 0]
    rows = np.array([0, 5, 127, 128, 399], np.int32)
    flags = orc.FLAGS_DEFAULT | orc.FLAG_VFMT_NVFP4 | orc.FLAG_QK_NVFP4
    r = orc.vc_attention_head(q, k, v, rows=rows, flags=flags)
    qk = r["qk"]
    N = 400
    qd = orc.e2m1_value(qk["qcodes"][:N]) * orc.e4m3_value(qk["qsfc"][:N]).repeat(16, axis=1)
    kd = orc.e2m1_value(qk["kcodes"][:N]) * orc.e4m3_value(qk["ksfc"][:N]).repeat(16, axis=1)
    # the FP8-path helper with the NVFP4 operands and global scales in place of
    # the E4M3 decode and block scales
    pro = {"qk": {"q8": None, "sq": qk["qg"], "k8": None, "sk": qk["kg"]}, "vq": r["vq"]}
    want = _direct_global_frame4(orc, pro, N, rows, orc.DEFAULT_SCALE, qd_all=qd, kd_all=kd)
    assert np.allclose(r["out"], want, rtol=1e-9, atol=1e-12)
