"""GPU parity of the prologue steps, bit-exact against the oracle through the
C ABI: V-Smooth grouping (permutation + centroids), Q/K smoothing and
quantization, V demean + residual codes + scales + repair list."""
import numpy as np
import pytest

import oracle
from bit_attention_diffusion_b200 import synth, vcattn

from gpu_util import from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu

SHAPES = [(1, 2, 1024), (1, 3, 300), (2, 2, 129), (1, 1, 1), (1, 2, 7), (1, 2, 128), (1, 4, 4256)]


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a B200"
    from bit_attention_diffusion_b200 import build_lib
    build_lib.build()
    return torch


def _inputs(B, H, N, seed=0):
    wl = synth.custom(B, H, N, seed=1000 + 7 * N + seed)
    return synth.make_inputs(wl)


@pytest.mark.parametrize("B,H,N", SHAPES)
@pytest.mark.parametrize("k,iters", [(8, 3), (3, 1), (1, 2), (12, 2)])
def test_cluster_bit_exact(torch, B, H, N, k, iters):
    x = _inputs(B, H, N)
    p = vcattn.params(k=k, iters=iters)
    perm, cent = vcattn.cluster(to_dev_bf16(x["v"]), p)
    perm, cent = perm.cpu().numpy(), cent.cpu().numpy()
    for b in range(B):
        for h in range(H):
            c_o, lab_o = oracle.kmeans_head(x["v"][b, h], k, iters)
            assert np.array_equal(perm[b, h], oracle.stable_sort_labels(lab_o, k)), (b, h)
            assert np.array_equal(cent[b, h].view(np.uint32), c_o.view(np.uint32)), (b, h)


def _tie_inputs(N=600, seed=5):
    """V with exact and near ties for the first assignment (initial centroids
    are the tokens j*N/8: 0, 75, 150, ...): centroids 0 and 1 differ only in
    channel 0 (0 and 2); tokens 1-74 are token 0 with channel 0 = 1
    (equidistant: ties go to cluster 0), tokens 76-149 the same with channel
    0 one bf16 step above or below 1 (a gap far below the estimate's error
    bound); tokens 400-419 repeat cluster 3's initial centroid exactly."""
    x = _inputs(1, 2, N, seed=seed)
    v = synth.bf16_bits_to_f32(x["v"]).astype(np.float32)
    one_up, one_dn = np.float32(1.0078125), np.float32(0.99609375)   # bf16 neighbours of 1
    for h in range(2):
        base = v[0, h, 0].copy()
        base[0] = 0.0
        v[0, h, 0] = base
        v[0, h, N // 8] = base
        v[0, h, N // 8, 0] = 2.0
        v[0, h, 1:N // 8] = base
        v[0, h, 1:N // 8, 0] = 1.0
        v[0, h, N // 8 + 1:2 * N // 8] = base
        v[0, h, N // 8 + 1:N // 8 + 38, 0] = one_up
        v[0, h, N // 8 + 38:2 * N // 8, 0] = one_dn
        v[0, h, 400:420] = v[0, h, 3 * N // 8]
    x["v"] = synth.f32_to_bf16_bits(v)
    return x


@pytest.mark.parametrize("k,iters", [(8, 0), (8, 3), (5, 2)])
def test_cluster_ties_and_near_ties_bit_exact(torch, k, iters):
    """The clustering kernel labels by a certified estimate and falls back to
    the pinned distances where the estimate cannot decide: exact ties and
    near ties must come out as the oracle's (lowest cluster on a tie)."""
    x = _tie_inputs()
    p = vcattn.params(k=k, iters=iters)
    perm, cent = vcattn.cluster(to_dev_bf16(x["v"]), p)
    perm, cent = perm.cpu().numpy(), cent.cpu().numpy()
    for h in range(2):
        c_o, lab_o = oracle.kmeans_head(x["v"][0, h], k, iters)
        if iters == 0:
            assert np.all(lab_o[1:75] == 0) and np.all(lab_o[76:113] == 1) and np.all(lab_o[113:150] == 0)
        assert np.array_equal(perm[0, h], oracle.stable_sort_labels(lab_o, k)), h
        assert np.array_equal(cent[0, h].view(np.uint32), c_o.view(np.uint32)), h


@pytest.mark.parametrize("B,H,N", SHAPES)
@pytest.mark.parametrize("ksmooth", [True, False])
def test_quant_qk_bit_exact(torch, B, H, N, ksmooth):
    x = _inputs(B, H, N, seed=1)
    rng = np.random.default_rng(N)
    perm = np.stack([np.stack([rng.permutation(N) for _ in range(H)]) for _ in range(B)]).astype(np.int32)
    flags = vcattn.FLAGS_DEFAULT if ksmooth else (vcattn.VC_VSMOOTH | vcattn.VC_REPAIR)
    r = vcattn.quant_qk(to_dev_bf16(x["q"]), to_dev_bf16(x["k"]), torch.from_numpy(perm).cuda(),
                        vcattn.params(flags=flags))
    g = {k: v.cpu().numpy() for k, v in r.items()}
    for b in range(B):
        for h in range(H):
            o = oracle.quant_qk_head(x["q"][b, h], x["k"][b, h], perm[b, h], ksmooth=ksmooth)
            assert np.array_equal(g["q8"][b, h], o["q8"]), (b, h)
            assert np.array_equal(g["sq"][b, h], o["sq"]), (b, h)
            assert np.array_equal(g["k8"][b, h], o["k8"]), (b, h)
            assert np.array_equal(g["sk"][b, h], o["sk"]), (b, h)


@pytest.mark.parametrize("B,H,N", SHAPES)
@pytest.mark.parametrize("flags", [vcattn.FLAGS_DEFAULT, vcattn.VC_KSMOOTH | vcattn.VC_REPAIR,
                                   vcattn.VC_VSMOOTH | vcattn.VC_KSMOOTH])
def test_quant_v_bit_exact(torch, B, H, N, flags):
    x = _inputs(B, H, N, seed=2)
    rng = np.random.default_rng(N + 1)
    perm = np.stack([np.stack([rng.permutation(N) for _ in range(H)]) for _ in range(B)]).astype(np.int32)
    p = vcattn.params(flags=flags)
    R = vcattn.vc_attn_repair_count(N, p)
    r = vcattn.quant_v(to_dev_bf16(x["v"]), torch.from_numpy(perm).cuda(), p)
    v8 = r["v8"].cpu().numpy()
    vscale = r["vscale"].cpu().numpy()
    vmean = from_dev_bf16(r["vmean"])
    rep_idx = r["rep_idx"].cpu().numpy()
    rep_delta = from_dev_bf16(r["rep_delta"])
    for b in range(B):
        for h in range(H):
            o = oracle.quant_v_head(x["v"][b, h], perm[b, h], demean=bool(flags & vcattn.VC_VSMOOTH), R=R)
            assert np.array_equal(v8[b, h].T, o["v8"]), (b, h)
            assert np.array_equal(vscale[b, h], o["vscale"]), (b, h)
            assert np.array_equal(vmean[b, h], o["vmean"]), (b, h)
            if R:
                assert np.array_equal(rep_idx[b, h], o["rep_idx"]), (b, h)
                assert np.array_equal(rep_delta[b, h], o["rep_delta"]), (b, h)


def test_quant_v_ties_in_repair_take_lowest_positions(torch):
    """Constant-valued tokens give equal (zero) errors; the repair list must
    then be the lowest permuted positions, as the oracle's rule says."""
    B, H, N = 1, 1, 1000
    v = np.full((B, H, N, 128), synth.f32_to_bf16_bits(np.float32(0.5)), np.uint16)
    p = vcattn.params()
    r = vcattn.quant_v(to_dev_bf16(v), None, p)
    R = vcattn.vc_attn_repair_count(N, p)
    assert r["rep_idx"].cpu().numpy()[0, 0].tolist() == list(range(R))


@pytest.mark.parametrize("B,H,N", [(1, 2, 1024), (2, 1, 300)])
def test_cluster_warm_start_bit_exact(torch, B, H, N):
    """VC_WARMSTART: starting from given centroids matches the oracle started
    from the same centroids; and warm start from the 2-iteration centroids plus
    3 more iterations equals the cold 5-iteration result."""
    x = _inputs(B, H, N, seed=3)
    v = to_dev_bf16(x["v"])
    _, c2 = vcattn.cluster(v, vcattn.params(iters=2))
    perm_w, cent_w = vcattn.cluster(v, vcattn.params(iters=3), init=c2)
    perm_5, cent_5 = vcattn.cluster(v, vcattn.params(iters=5))
    assert torch.equal(perm_w, perm_5) and torch.equal(cent_w, cent_5)
    c2h, pw, cw = c2.cpu().numpy(), perm_w.cpu().numpy(), cent_w.cpu().numpy()
    for b in range(B):
        for h in range(H):
            c_o, lab_o = oracle.kmeans_head(x["v"][b, h], 8, 3, init=c2h[b, h])
            assert np.array_equal(pw[b, h], oracle.stable_sort_labels(lab_o, 8)), (b, h)
            assert np.array_equal(cw[b, h].view(np.uint32), c_o.view(np.uint32)), (b, h)
