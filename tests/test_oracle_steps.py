"""Pins for the oracle's prologue steps: k-means grouping, the permutation,
Q/K quantization and V demean/quantize/repair (CPU only).

The checks use brute force on small inputs, library routines (numpy sorts),
closed forms (cluster means, planted clusters) and the error bounds implied by
round-to-nearest on the E4M3 grid.
"""
import numpy as np
import pytest

from bit_attention_diffusion_b200 import synth


def _bf16(rng, shape, scale=1.0):
    return synth.f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _e4m3_half_step(mag):
    """Half the E4M3 grid spacing at |value| = mag (normal: 2^(e-4); subnormal 2^-10)."""
    e = np.floor(np.log2(np.maximum(mag, 2.0 ** -6)))
    return 2.0 ** (e - 4)


# ---------------------------------------------------------------- k-means
def test_kmeans_labels_are_brute_force_argmin(orc):
    rng = np.random.default_rng(10)
    for N, k in [(37, 3), (200, 8), (256, 5)]:
        v = _bf16(rng, (N, 128))
        cent, lab = orc.kmeans_head(v, k, 2)
        x = orc.bf16_value(v).astype(np.float64)
        d2 = ((x[:, None, :] - cent[None, :, :].astype(np.float64)) ** 2).sum(-1)
        best = d2.argmin(1)
        srt = np.sort(d2, 1)
        clear = (srt[:, 1] - srt[:, 0]) > 1e-4 * srt[:, 0]
        assert np.array_equal(lab[clear], best[clear])
        # the chosen centroid is always within rounding of the minimum
        assert np.all(d2[np.arange(N), lab] <= srt[:, 0] * (1 + 1e-5))


def test_kmeans_objective_never_increases(orc):
    rng = np.random.default_rng(11)
    v = _bf16(rng, (500, 128))
    x = orc.bf16_value(v).astype(np.float64)
    objs = []
    for it in range(6):
        cent, lab = orc.kmeans_head(v, 8, it)
        objs.append(((x - cent[lab].astype(np.float64)) ** 2).sum())
    assert all(objs[i + 1] <= objs[i] * (1 + 1e-6) for i in range(len(objs) - 1)), objs


def test_kmeans_k1_is_mean_and_identity_perm(orc):
    rng = np.random.default_rng(12)
    v = _bf16(rng, (300, 128))
    cent, lab = orc.kmeans_head(v, 1, 3)
    assert np.all(lab == 0)
    mean = orc.bf16_value(v).astype(np.float64).mean(0).astype(np.float32)
    assert np.array_equal(cent[0], mean)
    assert np.array_equal(orc.stable_sort_labels(lab, 1), np.arange(300))


def test_kmeans_recovers_planted_clusters(orc):
    rng = np.random.default_rng(13)
    k, N = 4, 400
    centers = rng.standard_normal((k, 128)) * 20
    truth = rng.integers(0, k, N)
    truth[:k] = np.arange(k)  # every cluster present
    v = synth.f32_to_bf16_bits((centers[truth] + rng.standard_normal((N, 128)) * 0.1).astype(np.float32))
    # init picks tokens floor(j*N/k); put one token of each cluster there
    order = np.argsort(truth, kind="stable")
    v = v[order]
    truth = truth[order]
    cent, lab = orc.kmeans_head(v, k, 3)
    # same partition as the planted one
    for j in range(k):
        assert len(set(truth[lab == j].tolist())) == 1
    assert len(set(lab.tolist())) == k


def test_stable_sort_matches_numpy(orc):
    rng = np.random.default_rng(14)
    lab = rng.integers(0, 8, 5000).astype(np.int32)
    assert np.array_equal(orc.stable_sort_labels(lab, 8), np.argsort(lab, kind="stable"))


# ---------------------------------------------------------------- Q/K quantization
def test_quant_qk_error_bounds_and_smoothing(orc):
    rng = np.random.default_rng(15)
    N = 300
    q = _bf16(rng, (N, 128))
    kf = rng.standard_normal((N, 128)) + rng.standard_normal(128) * 1.4
    k = synth.f32_to_bf16_bits(kf.astype(np.float32))
    perm = rng.permutation(N).astype(np.int32)
    r = orc.quant_qk_head(q, k, perm, ksmooth=True)
    kx = orc.bf16_value(k).astype(np.float64)
    assert np.allclose(r["kbar"], kx.mean(0), rtol=1e-6, atol=1e-7)
    for name, src, rows in [("q", orc.bf16_value(q).astype(np.float64), np.arange(N)),
                            ("k", kx - r["kbar"].astype(np.float64), perm)]:
        codes, sc = r[name + "8"], r["s" + name]
        for t in range(3):
            p = np.arange(t * 128, min(N, t * 128 + 128))
            x = src[rows[p]]
            amax = np.abs(x).max()
            assert np.isclose(sc[t], amax / 448, rtol=1e-7)
            deq = orc.e4m3_value(codes[p]) * sc[t]
            err = np.abs(deq - x)
            assert np.all(err <= _e4m3_half_step(np.abs(x) / sc[t]) * sc[t] * (1 + 1e-6) + 1e-12)
            assert np.abs(orc.e4m3_value(codes[p])).max() == 448.0
        assert np.all(codes[N:] == 0)  # padding rows


# ---------------------------------------------------------------- V demean / quantize / repair
def _vq_case(orc, seed=16, N=300, demean=True, R=2):
    rng = np.random.default_rng(seed)
    vf = rng.standard_normal((N, 128)).astype(np.float32)
    vf[rng.integers(0, N, 3), rng.integers(0, 128, 3)] = 25.0
    v = synth.f32_to_bf16_bits(vf)
    perm = rng.permutation(N).astype(np.int32)
    return v, perm, orc.quant_v_head(v, perm, demean=demean, R=R)


def test_quant_v_block_means_and_residual_grid(orc):
    N = 300
    v, perm, r = _vq_case(orc, N=N)
    x = orc.bf16_value(v).astype(np.float64)[perm]
    mu = orc.bf16_value(r["vmean"]).astype(np.float64)
    for t in range(3):
        blk = x[t * 128:min(N, t * 128 + 128)]
        exact = blk.mean(0)
        # bf16 rounding of the block mean: within half a bf16 step (2^-8 relative)
        assert np.all(np.abs(mu[t] - exact) <= np.abs(exact) * 2.0 ** -8 + 1e-30)
    res = x - mu[np.arange(N) // 128]
    s = r["vscale"].astype(np.float64)
    # power-of-two scale: the least 2^e with amax <= 448 * 2^e
    amax = np.abs(res).max(0)
    assert np.all(np.log2(s) == np.round(np.log2(s)))
    assert np.all(amax <= 448 * s) and np.all(amax > 224 * s)
    deq = orc.e4m3_value(r["v8"][:N]) * s
    err = res - deq
    assert np.all(np.abs(err) <= _e4m3_half_step(np.abs(res) / s) * s * (1 + 1e-6))
    # per-token error sum (float32 accumulation: loose relative tolerance)
    assert np.allclose(r["err"], (err ** 2).sum(1), rtol=1e-5, atol=1e-12)
    assert np.all(r["v8"][N:] == 0)


def test_quant_v_demean_off_keeps_zero_mean(orc):
    v, perm, r = _vq_case(orc, demean=False)
    assert np.all(r["vmean"] == 0)


def test_repair_selection_matches_full_sort(orc):
    for seed, R in [(17, 2), (18, 7), (19, 40)]:
        v, perm, r = _vq_case(orc, seed=seed, R=R)
        e = r["err"]
        order = np.lexsort((np.arange(e.size), -e.astype(np.float64)))  # desc e, asc position
        want = np.sort(order[:R])
        assert np.array_equal(r["rep_idx"], want)
        # everything selected has error >= everything not selected
        rest = np.setdiff1d(np.arange(e.size), want)
        assert e[want].min() >= e[rest].max()


def test_repair_delta_restores_values(orc):
    N = 300
    v, perm, r = _vq_case(orc, N=N, R=10)
    x = orc.bf16_value(v).astype(np.float64)[perm]
    mu = orc.bf16_value(r["vmean"]).astype(np.float64)
    s = r["vscale"].astype(np.float64)
    idx = r["rep_idx"]
    vhat = mu[idx // 128] + orc.e4m3_value(r["v8"][idx]) * s + orc.bf16_value(r["rep_delta"])
    # after repair the value is within bf16 rounding of the residual error
    resid_err = x[idx] - mu[idx // 128] - orc.e4m3_value(r["v8"][idx]) * s
    assert np.all(np.abs(vhat - x[idx]) <= np.abs(resid_err) * 2.0 ** -8 + 1e-30)
    before = np.abs(resid_err).max()
    after = np.abs(vhat - x[idx]).max()
    assert after < before / 64


def test_kmeans_ties_go_to_lowest_cluster(orc):
    """With N < k the init repeats tokens, so centroids tie exactly: every
    token must take the lowest-numbered of its equal centroids."""
    rng = np.random.default_rng(19)
    v = _bf16(rng, (4, 128))
    cent, lab = orc.kmeans_head(v, 8, 3)
    assert lab.tolist() == [0, 2, 4, 6]
    assert np.array_equal(orc.stable_sort_labels(lab, 8), np.arange(4))


def test_quant_v_constant_channel_gets_unit_scale(orc):
    """A channel whose residuals are all zero (constant within every block)
    gets the power-of-two scale 1 and zero codes."""
    rng = np.random.default_rng(20)
    vf = rng.standard_normal((260, 128)).astype(np.float32)
    vf[:, 7] = 3.0
    v = synth.f32_to_bf16_bits(vf)
    r = orc.quant_v_head(v, np.arange(260, dtype=np.int32), demean=True, R=0)
    assert r["vscale"][7] == 1.0
    assert np.all(r["v8"][:, 7] == 0)
    assert np.all(orc.bf16_value(r["vmean"][:, 7]) == 3.0)


def test_kmeans_warm_start_chains_lloyd_iterations(orc):
    """Warm start (cross-step V-Smooth): starting from the centroids a cold run
    reached after i iterations and running m more gives exactly the cold run
    with i + m iterations (Lloyd is a deterministic map on the centroids); and
    starting from a fixed point changes nothing."""
    rng = np.random.default_rng(5)
    N, d, k = 600, 128, 5
    v = synth.f32_to_bf16_bits(rng.standard_normal((N, d)).astype(np.float32) + 3.0 * (rng.integers(0, k, N)[:, None]
                                                                                      == np.arange(d)[None, :] % k))
    c2, _ = orc.kmeans_head(v, k, 2)
    c5, l5 = orc.kmeans_head(v, k, 5)
    cw, lw = orc.kmeans_head(v, k, 3, init=c2)
    assert np.array_equal(cw.view(np.uint32), c5.view(np.uint32))
    assert np.array_equal(lw, l5)
    # run to a fixed point, then a warm start with one more iteration is the identity
    cf, lf = orc.kmeans_head(v, k, 30)
    cg, lg = orc.kmeans_head(v, k, 1, init=cf)
    assert np.array_equal(cg.view(np.uint32), cf.view(np.uint32)) and np.array_equal(lg, lf)
