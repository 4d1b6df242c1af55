"""Pins for the oracle's attention forward (CPU only).

The strongest pin is a closed form: when every quantization step is lossless
(codes exactly on the E4M3 grid, block means and residuals exact) and every
score lands on a byte whose mantissa field is zero (where the ExpCast identity
is exact), the method must reduce to exact softmax attention, whatever the
joint K/V permutation, with frame changes across tiles, a ragged last tile,
and repair tokens whose residual error is corrected exactly. A dropped restore
term, a wrong rescale, a wrong tile index or a transposed operand each break it.
"""
import numpy as np
import pytest

from bit_attention_diffusion_b200 import synth


def _exact_case(orc, seed, N=300):
    rng = np.random.default_rng(seed)
    d = 128
    assert N % 2 == 0
    half = N // 2
    scale = np.float32(np.log(2) / 8)
    assert orc.kappa(scale) == 1.0
    perm = rng.permutation(N).astype(np.int32)
    # Q: channel 0 is the per-block amax marker (448 -> scale 1); channels 2..9
    # carry the scores with 3 entries in {-2, 2}; channel 10 reads the boost.
    q = np.zeros((N, d), np.float32)
    q[:, 0] = 448.0
    q[:, 10] = 1.0
    for i in range(N):
        ch = rng.choice(np.arange(2, 10), 3, replace=False)
        q[i, ch] = rng.choice([-2.0, 2.0], 3)
    # K: channel 1 is the amax marker (+/-448), channels 2..9 in {-4, 0, 4};
    # token j + N/2 is the negation of token j so every channel mean is 0.
    # A +16 boost on channel 10 for a few keys placed in later tiles raises the
    # row maximum there, so the frame must change (their partners get -16).
    k = np.zeros((N, d), np.float32)
    k[:half, 1] = 448.0
    k[:half, 2:10] = rng.choice([-4.0, 0.0, 4.0], (half, 8))
    boost = set()
    for p in (130, 200, 260, 290):
        j = int(perm[p])
        if j in boost or (j + half) % N in boost:
            continue
        boost.add(j)
    for j in boost:
        jj = j if j < half else j - half
        k[jj, 10] = 16.0 if jj == j else -16.0
    k[half:] = -k[:half]
    # V in permuted order: per block t a mean mu_t (multiples of 1/4, |mu| <= 3.25),
    # residuals in +/- pairs on the E4M3 grid with scale 2^-3.
    vp = np.zeros((N, d), np.float32)
    Nb = (N + 127) // 128
    grid = np.array([0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    for t in range(Nb):
        p0, p1 = t * 128, min(N, t * 128 + 128)
        hc = (p1 - p0) // 2
        mu = rng.integers(-13, 14, d) / 4.0
        r = rng.choice(grid, (hc, d)) * rng.choice([-1, 1], (hc, d))
        vp[p0:p1] = mu + np.concatenate([r, -r], 0)
    mu0 = vp[0:128].mean(0)
    # channel amax marker: a +/-56 pair in block 0 (56 = 448 * 2^-3 for every channel)
    vp[2], vp[66] = mu0 + 56.0, mu0 - 56.0
    # the two repair tokens: residual 0.515625 = 4.125 * 2^-3 is off the grid by 2^-6
    vp[5], vp[69] = mu0 + 0.515625, mu0 - 0.515625
    for name, arr in (("q", q), ("k", k), ("vp", vp)):
        assert np.array_equal(synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(arr)), arr), name
    v = np.empty_like(vp)
    v[perm] = vp
    return (synth.f32_to_bf16_bits(q), synth.f32_to_bf16_bits(k), synth.f32_to_bf16_bits(v),
            perm, scale)


@pytest.mark.parametrize("seed", [20, 21, 22])
def test_lossless_case_reduces_to_exact_attention(orc, seed):
    q, k, v, perm, scale = _exact_case(orc, seed)
    flags = orc.FLAG_VSMOOTH | orc.FLAG_REPAIR | orc.FLAG_KSMOOTH
    r = orc.vc_attention_head(q, k, v, flags=flags, rho=0.005, softmax_scale=scale, perm=perm)
    # the case is lossless except for the two repair tokens
    vq = r["vq"]
    assert r["R"] == 2
    nz = np.nonzero(vq["err"])[0]
    assert set(nz.tolist()) == {5, 69} and vq["rep_idx"].tolist() == [5, 69]
    assert np.all(r["qk"]["sq"] == 1.0) and np.all(r["qk"]["sk"] == 1.0)
    assert np.all(r["qk"]["kbar"] == 0.0)
    assert np.all(vq["vscale"] == 0.125)
    # frames changed across tiles for some rows (F_final > first tile's frame)
    ex = orc.exact_attention_head(q, k, v, softmax_scale=scale)
    rel = np.abs(r["out"] - ex).max() / np.abs(ex).max()
    assert rel < 1e-6, rel
    # and without repair the two tokens' grid error shows up
    r2 = orc.vc_attention_head(q, k, v, flags=flags & ~orc.FLAG_REPAIR, softmax_scale=scale,
                               perm=perm)
    rel2 = np.abs(r2["out"] - ex).max() / np.abs(ex).max()
    assert rel2 > 10 * rel


def test_lossless_case_is_permutation_invariant(orc):
    q, k, v, perm, scale = _exact_case(orc, 23)
    ex = orc.exact_attention_head(q, k, v, softmax_scale=scale)
    # exact attention itself is invariant under a joint K/V permutation
    rng = np.random.default_rng(5)
    p2 = rng.permutation(q.shape[0])
    ex2 = orc.exact_attention_head(q, k[p2], v[p2], softmax_scale=scale)
    assert np.allclose(ex, ex2, rtol=1e-12, atol=1e-12)


def test_frames_change_in_lossless_case(orc):
    q, k, v, perm, scale = _exact_case(orc, 24)
    flags = orc.FLAG_VSMOOTH | orc.FLAG_REPAIR | orc.FLAG_KSMOOTH
    r = orc.vc_attention_head(q, k, v, flags=flags, softmax_scale=scale, perm=perm)
    # first-tile frame per row vs final frame: some rows must have moved
    qk = r["qk"]
    qd = orc.e4m3_value(qk["q8"][:300])
    kd = orc.e4m3_value(qk["k8"][:128])
    first_max = (qd @ kd.T).max(1)
    F0 = 8 * np.ceil(first_max / 8)
    assert np.any(r["F"] > F0)


def _direct_global_frame(orc, pro, N, rows, scale, C=120):
    """Un-tiled evaluation: every tile's bytes against its own frame F_t, all
    contributions scaled once to the final frame (no online rescaling)."""
    qk, vq = pro["qk"], pro["vq"]
    kap = np.float32(orc.kappa(scale))
    Nb = (N + 127) // 128
    kd = orc.e4m3_value(qk["k8"][:N])
    vd = orc.e4m3_value(vq["v8"][:N]) * vq["vscale"].astype(np.float64)
    mu = orc.bf16_value(vq["vmean"]).astype(np.float64)
    out = []
    for i in rows:
        qd = orc.e4m3_value(qk["q8"][i])
        acc = (kd @ qd).astype(np.float32)
        tile = np.arange(N) // 128
        alpha = ((np.float32(qk["sq"][i // 128]) * qk["sk"]).astype(np.float32) * kap).astype(np.float32)
        u = (acc * alpha[tile]).astype(np.float32)
        tmax = np.array([u[tile == t].max() for t in range(Nb)], np.float32)
        run = np.maximum.accumulate(tmax)
        Ft = (8 * np.ceil(run * np.float32(0.125))).astype(np.float32)
        b = orc.expcast(acc, alpha[tile], (np.float32(C) - Ft[tile]).astype(np.float32))
        p = orc.e4m3_value(b) * 2.0 ** ((Ft[tile].astype(np.float64) - Ft[-1]) / 8)
        lt = np.array([p[tile == t].sum() for t in range(Nb)])
        num = p @ vd + lt @ mu
        ridx = vq["rep_idx"]
        if ridx.size:
            br = orc.expcast(acc[ridx], alpha[tile[ridx]], np.float32(C) - Ft[-1])
            num = num + orc.e4m3_value(br) @ orc.bf16_value(vq["rep_delta"]).astype(np.float64)
        out.append(num / p.sum())
    return np.array(out)


def test_online_rescaling_equals_global_frame_form(orc):
    wl = synth.custom(1, 1, 700, seed=31)
    x = synth.make_inputs(wl)
    q, k, v = x["q"][0, 0], x["k"][0, 0], x["v"][0, 0]
    rows = np.array([0, 1, 127, 128, 300, 699], np.int32)
    r = orc.vc_attention_head(q, k, v, rows=rows)
    want = _direct_global_frame(orc, r, 700, rows, orc.DEFAULT_SCALE)
    assert np.allclose(r["out"], want, rtol=1e-9, atol=1e-12)


def test_random_inputs_error_band_vs_exact(orc):
    """On i.i.d. Gaussian inputs the 8-bit path sits near the FP8 noise floor."""
    wl, x = synth.make_by_name("tiny_b1h2n1024")
    q, k, v = x["q"][0, 0], x["k"][0, 0], x["v"][0, 0]
    rows = np.arange(0, 1024, 7, dtype=np.int32)
    r = orc.vc_attention_head(q, k, v, rows=rows)
    ex = orc.exact_attention_head(q, k, v, rows=rows)
    rel = np.linalg.norm(r["out"] - ex) / np.linalg.norm(ex)
    assert 0.02 < rel < 0.09, rel


def test_exactv_diagnostic_equals_method_when_values_are_lossless(orc):
    """The value-term diagnostic keeps the method's bytes and swaps in exact
    values: in the lossless case (repair off, so the two off-grid tokens remain)
    it differs from the method only by those tokens' residual error."""
    q, k, v, perm, scale = _exact_case(orc, 25)
    flags = orc.FLAG_VSMOOTH | orc.FLAG_REPAIR | orc.FLAG_KSMOOTH
    r = orc.vc_attention_head(q, k, v, flags=flags, softmax_scale=scale, perm=perm)
    ev = orc.attn_exactv_rows(r["qk"], v, r["perm"], 300, r["rows"], softmax_scale=scale)
    assert np.allclose(ev, r["out"], rtol=1e-9, atol=1e-9)
    r2 = orc.vc_attention_head(q, k, v, flags=flags & ~orc.FLAG_REPAIR, softmax_scale=scale, perm=perm)
    assert not np.allclose(ev, r2["out"], rtol=1e-9, atol=1e-9)


@pytest.mark.parametrize("fmt", ["e4m3", "nvfp4", "nvfp4qk"])
def test_constant_values_are_reproduced_exactly(orc, fmt):
    """Every value token of a head is one bf16 vector: the block means are
    that vector and every residual is zero, so each output row is
    sum_t l_t * mu / sum_t l_t = mu whatever the scores (the restore through
    the row sums, in closed form); an all-zero head gives zeros. A dropped
    restore, a normalizer other than the decoded row sum, or frames applied
    to O and l differently break it. 300 tokens: three KV tiles, the last
    one ragged."""
    extra = {"e4m3": 0, "nvfp4": orc.FLAG_VFMT_NVFP4,
             "nvfp4qk": orc.FLAG_VFMT_NVFP4 | orc.FLAG_QK_NVFP4}[fmt]
    N = 300
    x = synth.make_inputs(synth.custom(1, 1, N, seed=905))
    row = x["v"][0, 0, 7].copy()
    assert (synth.bf16_bits_to_f32(row) != 0).all()
    for vrow in (row, np.zeros_like(row)):
        v = np.broadcast_to(vrow, (N, 128)).copy()
        r = orc.vc_attention_head(x["q"][0, 0], x["k"][0, 0], v, flags=orc.FLAGS_DEFAULT | extra)
        assert np.array_equal(orc.to_bf16_bits(r["out"]), np.broadcast_to(vrow, (N, 128)))


def test_dominant_key_rows_return_its_reconstructed_value(orc):
    """One key (token 1500, 2000 times the unit direction of the summed query
    rows) outscores every other key by more than 64 log2 units on many rows
    (exact scores; FP8 rounding of Q and K' moves them by a few units). That
    is far beyond the byte range (C = 120 byte units = 15 log2 units), so
    every later key's byte is 0. The earlier tiles, at most N keys of at most
    2^8.75 each, survive only scaled by about 2^-60 after the frame jump.
    Those rows' output is then the dominant token's reconstructed value
    mu_t + value(code) * s (+ its repair delta) to within 1e-9. This pins the
    clamp at 0, a frame jump of hundreds of byte units, and the value
    reconstruction of a single key."""
    N = 2000
    x = synth.make_inputs(synth.custom(1, 1, N, seed=880))
    q = orc.bf16_value(x["q"][0, 0]).astype(np.float64)
    u = q.sum(axis=0)
    kb = x["k"][0, 0].copy()
    kb[1500] = orc.to_bf16_bits(2000.0 * u / np.linalg.norm(u))
    k = orc.bf16_value(kb).astype(np.float64)
    s = q @ (k - k.mean(axis=0)).T / np.sqrt(128.0) * np.log2(np.e)
    gap = s[:, 1500] - np.delete(s, 1500, axis=1).max(axis=1)
    rows = np.nonzero(gap > 64.0)[0].astype(np.int32)
    assert rows.size > 100
    r = orc.vc_attention_head(x["q"][0, 0], kb, x["v"][0, 0], rows=rows)
    vq = r["vq"]
    pos = int(np.nonzero(r["perm"] == 1500)[0][0])  # its permuted position
    vhat = (orc.bf16_value(vq["vmean"][pos // 128]).astype(np.float64)
            + orc.e4m3_value(vq["v8"][pos]).astype(np.float64) * vq["vscale"].astype(np.float64))
    hit = np.nonzero(vq["rep_idx"] == pos)[0]
    if hit.size:
        vhat = vhat + orc.bf16_value(vq["rep_delta"][hit[0]]).astype(np.float64)
    assert np.allclose(r["out"], np.broadcast_to(vhat, r["out"].shape), rtol=1e-9, atol=1e-12)
