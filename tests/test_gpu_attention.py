"""GPU parity of the fused VC-Attention FP8 forward against the oracle.

Bar: relative L2 <= 1e-3 between the kernel's bf16 output and the
oracle's output rounded the same way (fp64 -> fp32 -> bf16), over the checked
rows of every head (each head on its own, and all heads together), on every
row for small and ragged shapes, in the launch configuration the bench times
(vc_attn_fwd with default parameters, clustering inside the call). The full
workload sizes are in test_gpu_fullsize.py.

Against exact fp64 attention the 8-bit path sits at the FP8 noise floor on
i.i.d. Gaussian inputs (about 5-6% relative L2, cosine ~0.998, the value the
oracle itself gives); those numbers are recorded and checked against a band.
The value-term error (same probability bytes, exact values) is where V-Smooth
and repair act: on the outlier channel they must lower it clearly.
"""
import numpy as np
import pytest

import oracle
from bit_attention_diffusion_b200 import synth, vcattn

from gpu_util import bf16_vals, cosine, from_dev_bf16, rel_l2, to_dev_bf16

pytestmark = pytest.mark.gpu
TOL = 1e-3


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a B200"
    from bit_attention_diffusion_b200 import build_lib
    build_lib.build()
    return torch


def _run_gpu(torch, x, p, perm=None):
    q, k, v = (to_dev_bf16(x[n]) for n in "qkv")
    pm = None if perm is None else torch.from_numpy(perm).cuda()
    out = vcattn.fwd(q, k, v, perm=pm, p=p)
    torch.cuda.synchronize()
    return from_dev_bf16(out)


def _compare(x, out_bits, heads, rows_fn, flags, perm=None):
    """rel-L2 of GPU vs oracle (both bf16) over the checked rows of the given heads."""
    num = den = 0.0
    worst = 0.0
    for (b, h) in heads:
        N = x["q"].shape[2]
        rows = rows_fn(N)
        pm = None if perm is None else perm[b, h]
        r = oracle.vc_attention_head(x["q"][b, h], x["k"][b, h], x["v"][b, h], rows=rows, flags=flags, perm=pm)
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
def test_fwd_matches_oracle_all_rows(torch, B, H, N):
    x = synth.make_inputs(synth.custom(B, H, N, seed=300 + N))
    out = _run_gpu(torch, x, vcattn.params())
    heads = [(b, h) for b in range(B) for h in range(H)]
    rel, worst = _compare(x, out, heads, _all_rows, oracle.FLAGS_DEFAULT)
    assert rel <= TOL and worst <= TOL, (rel, worst)


@pytest.mark.parametrize("flags", [oracle.FLAG_KSMOOTH, oracle.FLAG_KSMOOTH | oracle.FLAG_REPAIR,
                                   oracle.FLAG_VSMOOTH | oracle.FLAG_KSMOOTH, oracle.FLAG_VSMOOTH,
                                   oracle.FLAG_VSMOOTH | oracle.FLAG_REPAIR])
def test_fwd_flag_variants(torch, flags):
    B, H, N = 1, 2, 1000
    x = synth.make_inputs(synth.custom(B, H, N, seed=400 + flags))
    out = _run_gpu(torch, x, vcattn.params(flags=flags))
    rel, worst = _compare(x, out, [(0, 0), (0, 1)], _all_rows, flags)
    assert rel <= TOL and worst <= TOL, (rel, worst)


def test_fwd_other_parameters(torch):
    """k, iters, rho, C and the softmax scale reach the kernel unchanged."""
    B, H, N = 1, 2, 900
    x = synth.make_inputs(synth.custom(B, H, N, seed=77))
    p = vcattn.params(k=5, iters=2, rho=0.02, softmax_scale=0.05, expcast_bias=112)
    out = _run_gpu(torch, x, p)
    for h in range(H):
        r = oracle.vc_attention_head(x["q"][0, h], x["k"][0, h], x["v"][0, h], k=5, iters=2, rho=0.02,
                                     softmax_scale=0.05, C=112)
        ref = bf16_vals(oracle.to_bf16_bits(r["out"]))
        assert rel_l2(bf16_vals(out[0, h]), ref) <= TOL


def test_fwd_cached_permutation_gives_identical_output(torch):
    """Clustering once and passing the permutation back (later denoising steps)
    gives bit-identical output to clustering inside the call."""
    B, H, N = 1, 3, 2000
    x = synth.make_inputs(synth.custom(B, H, N, seed=91))
    q, k, v = (to_dev_bf16(x[n]) for n in "qkv")
    p = vcattn.params()
    perm, _ = vcattn.cluster(v, p)
    o1 = vcattn.fwd(q, k, v, perm=None, p=p)
    o2 = vcattn.fwd(q, k, v, perm=perm, p=p)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_fwd_lossless_case_equals_exact_attention(torch):
    """The closed-form pin of the oracle, run on the GPU: with every
    quantization step lossless and bytes on the exact part of the ExpCast map,
    the kernel must reproduce exact softmax attention (to bf16 output rounding)."""
    from test_oracle_attention import _exact_case
    q, k, v, perm, scale = _exact_case(oracle, 26)
    x = {"q": q[None, None], "k": k[None, None], "v": v[None, None]}
    out = _run_gpu(torch, x, vcattn.params(softmax_scale=float(scale)), perm=perm[None, None].copy())
    ex = oracle.exact_attention_head(q, k, v, softmax_scale=scale)
    got = bf16_vals(out[0, 0])
    assert rel_l2(got, ex) < 3e-3   # bf16 output rounding only
    ref = bf16_vals(oracle.to_bf16_bits(ex))
    assert np.mean(got == ref) > 0.95


@pytest.mark.parametrize("name,rows_per_head,heads", [
    ("tiny_b1h2n1024", None, [(0, 0), (0, 1)]),
])
def test_fwd_workloads_match_oracle(torch, name, rows_per_head, heads):
    """The tiny workload, every row, default parameters, clustering inside
    vc_attn_fwd (the call the bench times); the four larger workloads are
    checked at full size in test_gpu_fullsize.py."""
    wl, x = synth.make_by_name(name)
    out = _run_gpu(torch, x, vcattn.params())
    rows_fn = _all_rows if rows_per_head is None else (lambda N: _sampled_rows(N, rows_per_head))
    rel, worst = _compare(x, out, heads, rows_fn, oracle.FLAGS_DEFAULT)
    assert rel <= TOL and worst <= TOL, (rel, worst)
    # every row of every head is finite
    assert np.isfinite(bf16_vals(out)).all()


def test_fwd_vs_exact_attention_band(torch):
    """Accuracy against exact fp64 attention on the 1024^2-image workload
    (sampled rows): at the FP8 noise floor the oracle predicts."""
    wl, x = synth.make_by_name("image1024_b1h24n4256")
    out = _run_gpu(torch, x, vcattn.params())
    rels, coss = [], []
    for h in (0, 7, 15, 23):
        rows = _sampled_rows(wl.N, 64, seed=h)
        ex = oracle.exact_attention_head(x["q"][0, h], x["k"][0, h], x["v"][0, h], rows=rows)
        got = bf16_vals(out[0, h][rows])
        rels.append(rel_l2(got, ex))
        coss.append(cosine(got, ex))
    assert max(rels) < 0.08 and min(coss) > 0.996, (rels, coss)


def test_vsmooth_lowers_value_term_error_on_outlier_channel(torch):
    """Same inputs (0.5% outlier tokens, one channel per head), two variants
    of the same kernel: full method vs plain FP8 (no V-Smooth, no repair).
    The value-term error is measured against the oracle's exact-value output
    with the kernel's own probability bytes."""
    B, H, N = 1, 6, 2048
    x = synth.make_inputs(synth.custom(B, H, N, seed=11))
    acc = {"full": [0.0, 0.0], "plain": [0.0, 0.0]}
    for name, flags in (("full", oracle.FLAGS_DEFAULT), ("plain", oracle.FLAG_KSMOOTH)):
        out = _run_gpu(torch, x, vcattn.params(flags=flags))
        for h in range(H):
            ch = int(np.argmax(np.abs(bf16_vals(x["v"][0, h])).max(0)))
            pro = oracle.head_prologue(x["q"][0, h], x["k"][0, h], x["v"][0, h], flags=flags)
            ev = oracle.attn_exactv_rows(pro["qk"], x["v"][0, h], pro["perm"], N, _all_rows(N))
            e = bf16_vals(out[0, h]) - ev
            acc[name][0] += float((e[:, ch] ** 2).sum())
            acc[name][1] += float((ev[:, ch] ** 2).sum())
    full = np.sqrt(acc["full"][0] / acc["full"][1])
    plain = np.sqrt(acc["plain"][0] / acc["plain"][1])
    assert full < 0.75 * plain, (full, plain)


@pytest.mark.parametrize("N", [4097, 4200, 4224, 8300])
def test_fwd_restore_chunk_boundaries(torch, N):
    """KV-tile counts where the block-mean restore chunks (32 tiles each) end
    right at the last tile (two chunks restored after the loop) or one past it."""
    x = synth.make_inputs(synth.custom(1, 2, N, seed=600 + N))
    out = _run_gpu(torch, x, vcattn.params())
    rel, worst = _compare(x, out, [(0, 0), (0, 1)], lambda n: _sampled_rows(n, 48), oracle.FLAGS_DEFAULT)
    assert rel <= TOL and worst <= TOL, (rel, worst)


@pytest.mark.parametrize("groups", [1, 2, 7])
def test_fwd_host_equals_device_call(torch, groups):
    """vc_attn_fwd_host (host buffers, runs of heads, copies overlapped with
    compute) gives bit-identical output to vc_attn_fwd on device buffers;
    groups = 2 leaves a shorter last run (7 heads in runs of 4 and 3)."""
    B, H, N = 1, 7, 700
    x = synth.make_inputs(synth.custom(B, H, N, seed=800 + groups))
    q, k, v = (to_dev_bf16(x[n]) for n in "qkv")
    ref = vcattn.fwd(q, k, v, p=vcattn.params())
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hout = vcattn.fwd_host(hq, hk, hv, groups, p=vcattn.params())
    torch.cuda.synchronize()
    assert torch.equal(hout, ref.cpu())


@pytest.mark.parametrize("extra", ["VC_VFMT_NVFP4", "VC_QK_NVFP4", "VC_FUSED_PROLOGUE", "VC_KSMOOTH"])
def test_fwd_host_equals_device_call_variants(torch, extra):
    """The host-buffer entry point runs the same per-run pipeline for the
    4-bit variants and the one-launch prologue: bit-identical output to the
    device call with the same flags (B=2 so that runs cross a batch)."""
    flags = vcattn.FLAGS_DEFAULT | getattr(vcattn, extra)
    if extra == "VC_QK_NVFP4":
        flags |= vcattn.VC_VFMT_NVFP4
    if extra == "VC_KSMOOTH":
        flags = vcattn.VC_KSMOOTH
    p = vcattn.params(flags=flags)
    B, H, N = 2, 3, 900
    x = synth.make_inputs(synth.custom(B, H, N, seed=820 + len(extra)))
    q, k, v = (to_dev_bf16(x[n]) for n in "qkv")
    ref = vcattn.fwd(q, k, v, p=p)
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hout = vcattn.fwd_host(hq, hk, hv, 4, p=p)
    torch.cuda.synchronize()
    assert torch.equal(hout, ref.cpu())


@pytest.mark.parametrize("extra", ["", "VC_VFMT_NVFP4", "VC_QK_NVFP4"])
def test_fwd_constant_values_are_reproduced_exactly(torch, extra):
    """Every value token of a head is one bf16 vector (head 0: zeros). The
    block means are that vector and every residual, code and repair delta is
    zero, so each output row is sum_t l_t * mean / sum_t l_t: the vector
    itself, bit for bit in bf16 (the row sums' bf16 hi/lo split and fp32 sums
    leave a relative error near 1e-5, far below half a bf16 ulp). N = 4300:
    a ragged last tile, 34 KV tiles, two block-mean restore chunks."""
    flags = vcattn.FLAGS_DEFAULT
    if extra:
        flags |= vcattn.VC_VFMT_NVFP4
    if extra == "VC_QK_NVFP4":
        flags |= vcattn.VC_QK_NVFP4
    B, H, N = 1, 2, 4300
    x = synth.make_inputs(synth.custom(B, H, N, seed=850))
    row = x["v"][0, 1, 0].copy()
    assert (bf16_vals(row) != 0).all()
    x["v"][0, 0] = 0
    x["v"][0, 1] = row[None, :]
    out = _run_gpu(torch, x, vcattn.params(flags=flags))
    assert (out[0, 0] == 0).all()
    assert (out[0, 1] == row[None, :]).all()


def test_fwd_large_repair_budget(torch):
    """rho = 0.9: 270 of 300 tokens repaired, as many repair chunks (3) as KV
    tiles; every row against the oracle."""
    B, H, N = 1, 2, 300
    x = synth.make_inputs(synth.custom(B, H, N, seed=860))
    out = _run_gpu(torch, x, vcattn.params(rho=0.9))
    for h in range(H):
        r = oracle.vc_attention_head(x["q"][0, h], x["k"][0, h], x["v"][0, h], rho=0.9)
        ref = bf16_vals(oracle.to_bf16_bits(r["out"]))
        assert rel_l2(bf16_vals(out[0, h]), ref) <= TOL


@pytest.mark.parametrize("extra", ["", "VC_VFMT_NVFP4", "VC_QK_NVFP4"])
def test_fwd_dominant_key_moves_the_frame_past_fp32_range(torch, extra):
    """One key (position 1500, KV tile 11) is 2000 times the unit direction of
    the summed query rows. For about a third of the rows its log2-domain score
    lies more than 150 units above the earlier tiles' maximum, so the frame
    jumps by more than 1200 byte units at once and the rescale factor of
    everything accumulated so far is below fp32's range (the kernels flush it
    to zero); for about half the rows that key takes all the probability
    mass. Every row against the oracle."""
    flags = vcattn.FLAGS_DEFAULT
    if extra:
        flags |= vcattn.VC_VFMT_NVFP4
    if extra == "VC_QK_NVFP4":
        flags |= vcattn.VC_QK_NVFP4
    B, H, N = 1, 1, 2000
    x = synth.make_inputs(synth.custom(B, H, N, seed=880))
    u = bf16_vals(x["q"][0, 0]).sum(axis=0)
    x["k"][0, 0, 1500] = oracle.to_bf16_bits(2000.0 * u / np.linalg.norm(u))
    out = _run_gpu(torch, x, vcattn.params(flags=flags))
    r = oracle.vc_attention_head(x["q"][0, 0], x["k"][0, 0], x["v"][0, 0], flags=flags)
    ref = bf16_vals(oracle.to_bf16_bits(r["out"]))
    assert np.isfinite(bf16_vals(out[0, 0])).all()
    assert rel_l2(bf16_vals(out[0, 0]), ref) <= TOL
