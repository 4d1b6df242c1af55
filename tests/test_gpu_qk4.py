"""GPU parity of the full 4-bit path (VC_QK_NVFP4 with VC_VFMT_NVFP4) against the oracle.

Page "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58× sem
retreinamento": "Por que a atenção é o gargalo" (low-precision tensor cores
for both products) and "Benchmarks" (the 4-bit V-Smooth kernel against
SageAttention3): Q and K' in NVFP4 as well as P and the V residual.

- The Q/K quantization is byte work decided in binary32 on both sides: global
  scales, block-scale codes and E2M1 codes are compared bit for bit, in the
  tile-image layout the kernel reads.
- The attention output is compared with the oracle's (rounded the same way to
  bf16) at relative L2 <= 1e-3, as for the NVFP4-residual variant: the score
  is an exact sum of exact products rounded to binary32 by the tensor core (the
  oracle rounds its fp64 sum once), the kernel's 2^x is ex2.approx.
"""
import numpy as np
import pytest

import oracle
from bit_attention_diffusion_b200 import synth, vcattn

from gpu_util import bf16_vals, from_dev_bf16, rel_l2, to_dev_bf16

pytestmark = pytest.mark.gpu
TOL = 1e-3
FP4 = vcattn.VC_VFMT_NVFP4 | vcattn.VC_QK_NVFP4
IMG = 9216


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a B200"
    from bit_attention_diffusion_b200 import build_lib
    build_lib.build()
    return torch


def unpack_qk_images(buf, BH, N):
    """Q or K' tile images -> per head (codes [Nb*128, 128], scale codes [Nb*128, 8])."""
    Nb = (N + 127) // 128
    img = np.asarray(buf).reshape(-1)[:BH * Nb * IMG].reshape(BH, Nb, IMG)
    r = np.arange(128)[:, None]
    jb = np.arange(8)[None, :]
    sf_off = 512 * (jb // 4) + 16 * (r % 32) + 4 * (r // 32) + jb % 4           # [128 rows, 8 blocks]
    i = np.arange(64)[None, :]
    code_off = 1024 + 512 * (r // 8) + 64 * (r % 8) + 16 * ((i // 16) ^ ((r // 2) % 4)) + i % 16   # [128, 64]
    sfc = img[:, :, sf_off].reshape(BH, Nb * 128, 8)
    b = img[:, :, code_off]                                                      # [BH, Nb, 128 rows, 64]
    codes = np.empty((BH, Nb, 128, 128), np.uint8)
    codes[..., 0::2] = b & 15
    codes[..., 1::2] = b >> 4
    return codes.reshape(BH, Nb * 128, 128), sfc


SHAPES = [(1, 2, 1024), (1, 3, 300), (2, 2, 129), (1, 1, 1), (1, 2, 7), (1, 2, 4256)]


@pytest.mark.parametrize("B,H,N", SHAPES)
@pytest.mark.parametrize("ksmooth", [True, False])
def test_quant_qk4_bit_exact(torch, B, H, N, ksmooth):
    x = synth.make_inputs(synth.custom(B, H, N, seed=3100 + N))
    rng = np.random.default_rng(N + 17)
    perm = np.stack([np.stack([rng.permutation(N) for _ in range(H)]) for _ in range(B)]).astype(np.int32)
    flags = (vcattn.VC_KSMOOTH if ksmooth else 0) | FP4
    r = vcattn.quant_qk(to_dev_bf16(x["q"]), to_dev_bf16(x["k"]), torch.from_numpy(perm).cuda(),
                        vcattn.params(flags=flags))
    torch.cuda.synchronize()
    qc, qs = unpack_qk_images(r["q8"].cpu().numpy(), B * H, N)
    kc, ks = unpack_qk_images(r["k8"].cpu().numpy(), B * H, N)
    gq, gk = r["sq"].cpu().numpy(), r["sk"].cpu().numpy()
    for b in range(B):
        for h in range(H):
            o = oracle.quant_qk4_head(x["q"][b, h], x["k"][b, h], perm[b, h], ksmooth=ksmooth)
            bh = b * H + h
            assert np.array_equal(gq[b, h], o["qg"]), (b, h)
            assert np.array_equal(gk[b, h], o["kg"]), (b, h)
            assert np.array_equal(qs[bh], o["qsfc"]), (b, h)
            assert np.array_equal(ks[bh], o["ksfc"]), (b, h)
            assert np.array_equal(qc[bh], o["qcodes"]), (b, h)
            assert np.array_equal(kc[bh], o["kcodes"]), (b, h)


def test_quant_qk4_degenerate_blocks(torch):
    """An all-zero block (g = 1, every scale and code 0) and a block holding a
    single nonzero value, next to ordinary ones."""
    B, H, N = 1, 1, 400
    x = synth.make_inputs(synth.custom(B, H, N, seed=3190))
    q, k = x["q"].copy(), x["k"].copy()
    q[0, 0, 128:256] = 0
    k[0, 0, :] = x["k"][0, 0, :1]          # every row the same: K' = 0 after smoothing
    q[0, 0, 256:384] = 0
    q[0, 0, 300, 5] = 0x4040               # 3.0
    perm = np.arange(N, dtype=np.int32)[None, None]
    r = vcattn.quant_qk(to_dev_bf16(q), to_dev_bf16(k), torch.from_numpy(perm).cuda(),
                        vcattn.params(flags=vcattn.VC_KSMOOTH | FP4))
    torch.cuda.synchronize()
    qc, qs = unpack_qk_images(r["q8"].cpu().numpy(), 1, N)
    kc, ks = unpack_qk_images(r["k8"].cpu().numpy(), 1, N)
    o = oracle.quant_qk4_head(q[0, 0], k[0, 0], perm[0, 0], ksmooth=True)
    assert np.array_equal(r["sq"].cpu().numpy()[0, 0], o["qg"])
    assert np.array_equal(r["sk"].cpu().numpy()[0, 0], o["kg"])
    assert o["qg"][1] == 1.0 and not qc[0, 128:256].any() and not qs[0, 128:256].any()
    assert np.array_equal(qc[0], o["qcodes"]) and np.array_equal(qs[0], o["qsfc"])
    assert np.array_equal(kc[0], o["kcodes"]) and np.array_equal(ks[0], o["ksfc"])


def test_qk4_needs_the_nvfp4_residual(torch):
    q = to_dev_bf16(synth.make_inputs(synth.custom(1, 1, 64, seed=1))["q"])
    with pytest.raises(RuntimeError):
        vcattn.fwd(q, q, q, p=vcattn.params(flags=vcattn.FLAGS_DEFAULT | vcattn.VC_QK_NVFP4))


def _run(torch, x, p, perm=None):
    q, k, v = (to_dev_bf16(x[n]) for n in "qkv")
    pm = None if perm is None else torch.from_numpy(perm).cuda()
    out = vcattn.fwd(q, k, v, perm=pm, p=p)
    torch.cuda.synchronize()
    return from_dev_bf16(out)


def _compare(x, out_bits, heads, rows_fn, flags, **kw):
    num = den = 0.0
    worst = 0.0
    for (b, h) in heads:
        N = x["q"].shape[2]
        rows = rows_fn(N)
        r = oracle.vc_attention_head(x["q"][b, h], x["k"][b, h], x["v"][b, h], rows=rows, flags=flags, **kw)
        ref = bf16_vals(oracle.to_bf16_bits(r["out"]))
        got = bf16_vals(out_bits[b, h][rows])
        e = np.linalg.norm(got - ref) ** 2
        num += e
        den += np.linalg.norm(ref) ** 2
        worst = max(worst, float(np.sqrt(e / max(np.linalg.norm(ref) ** 2, 1e-300))))
    return float(np.sqrt(num / den)), worst


def _all_rows(N):
    return np.arange(N, dtype=np.int32)


def _sampled_rows(N, n=24, seed=0):
    rng = np.random.default_rng(seed + N)
    fixed = [0, 1, 127, 128, N - 1, N - 2, ((N - 1) // 128) * 128]
    rnd = rng.choice(N, size=min(n, N), replace=False).tolist()
    return np.array(sorted(set(r for r in fixed + rnd if 0 <= r < N)), dtype=np.int32)


SMALL = [(1, 2, 1024), (1, 2, 300), (1, 1, 129), (1, 1, 1), (1, 1, 128), (2, 3, 700), (1, 2, 4000)]


@pytest.mark.parametrize("B,H,N", SMALL)
def test_fwd44_matches_oracle_all_rows(torch, B, H, N):
    x = synth.make_inputs(synth.custom(B, H, N, seed=3300 + N))
    flags = vcattn.FLAGS_DEFAULT | FP4
    out = _run(torch, x, vcattn.params(flags=flags))
    heads = [(b, h) for b in range(B) for h in range(H)]
    rel, worst = _compare(x, out, heads, _all_rows, flags)
    assert rel <= TOL and worst <= TOL, (rel, worst)


@pytest.mark.parametrize("flags", [0, vcattn.VC_KSMOOTH | vcattn.VC_REPAIR, vcattn.VC_VSMOOTH | vcattn.VC_KSMOOTH,
                                   vcattn.VC_VSMOOTH | vcattn.VC_REPAIR])
def test_fwd44_flag_variants(torch, flags):
    B, H, N = 1, 2, 1000
    x = synth.make_inputs(synth.custom(B, H, N, seed=3400 + flags))
    out = _run(torch, x, vcattn.params(flags=flags | FP4))
    rel, worst = _compare(x, out, [(0, 0), (0, 1)], _all_rows, flags | FP4)
    assert rel <= TOL and worst <= TOL, (rel, worst)


def test_fwd44_other_parameters(torch):
    B, H, N = 1, 2, 900
    x = synth.make_inputs(synth.custom(B, H, N, seed=3477))
    p = vcattn.params(k=5, iters=2, rho=0.02, softmax_scale=0.05, flags=vcattn.FLAGS_DEFAULT | FP4)
    out = _run(torch, x, p)
    for h in range(H):
        r = oracle.vc_attention_head(x["q"][0, h], x["k"][0, h], x["v"][0, h], k=5, iters=2, rho=0.02,
                                     softmax_scale=0.05, flags=vcattn.FLAGS_DEFAULT | FP4)
        assert rel_l2(bf16_vals(out[0, h]), bf16_vals(oracle.to_bf16_bits(r["out"]))) <= TOL


def test_fwd44_lossless_case_equals_exact_attention(torch):
    """The oracle's closed-form pin of the full 4-bit path run on the GPU: Q,
    K', probabilities and value residuals on the NVFP4 grid, a ragged last
    tile and repaired tokens: the kernel reproduces exact attention to bf16
    rounding."""
    from test_oracle_nvfp4 import _lossless_case_qk4
    q, k, v, perm, scale = _lossless_case_qk4(57)
    x = {"q": q[None, None], "k": k[None, None], "v": v[None, None]}
    flags = vcattn.VC_VSMOOTH | vcattn.VC_REPAIR | FP4
    out = _run(torch, x, vcattn.params(softmax_scale=float(scale), flags=flags), perm=perm[None, None].copy())
    ex = oracle.exact_attention_head(q, k, v, softmax_scale=scale)
    got = bf16_vals(out[0, 0])
    assert rel_l2(got, ex) < 3e-3   # bf16 output rounding only
    assert np.mean(got == bf16_vals(oracle.to_bf16_bits(ex))) > 0.95


@pytest.mark.parametrize("N", [4097, 8300])
def test_fwd44_restore_chunk_boundaries(torch, N):
    x = synth.make_inputs(synth.custom(1, 2, N, seed=3600 + N))
    flags = vcattn.FLAGS_DEFAULT | FP4
    out = _run(torch, x, vcattn.params(flags=flags))
    rel, worst = _compare(x, out, [(0, 0), (0, 1)], lambda n: _sampled_rows(n, 48), flags)
    assert rel <= TOL and worst <= TOL, (rel, worst)


def test_fwd44_video_workload_sampled_rows(torch):
    """The 720p video workload (B=1, H=40, N=75600) at full size, default
    parameters plus the full 4-bit flags: sampled rows of the first and last head."""
    wl, x = synth.make_by_name("video720p_b1h40n75600")
    flags = vcattn.FLAGS_DEFAULT | FP4
    out = _run(torch, x, vcattn.params(flags=flags))
    rel, worst = _compare(x, out, [(0, 0), (0, 39)], lambda n: _sampled_rows(n, 8), flags)
    assert rel <= TOL and worst <= TOL, (rel, worst)
    assert np.isfinite(bf16_vals(out)).all()


def test_fwd44_vs_exact_attention_band(torch):
    """Against exact attention the full 4-bit path is noisier than the
    NVFP4-residual variant (QK^T in FP8), which is noisier than the 8-bit path."""
    wl, x = synth.make_by_name("image1024_b1h24n4256")
    out44 = _run(torch, x, vcattn.params(flags=vcattn.FLAGS_DEFAULT | FP4))
    out4 = _run(torch, x, vcattn.params(flags=vcattn.FLAGS_DEFAULT | vcattn.VC_VFMT_NVFP4))
    e44, e4 = [], []
    for h in (0, 11, 23):
        rows = _sampled_rows(wl.N, 48, seed=h)
        ex = oracle.exact_attention_head(x["q"][0, h], x["k"][0, h], x["v"][0, h], rows=rows)
        e44.append(rel_l2(bf16_vals(out44[0, h][rows]), ex))
        e4.append(rel_l2(bf16_vals(out4[0, h][rows]), ex))
    assert np.mean(e4) < np.mean(e44) and max(e44) < 0.6, (e44, e4)
