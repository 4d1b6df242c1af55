"""GPU parity at the workloads' full sizes, through the C ABI.

Prologue, bit for bit: at N = 16544 (the 2048^2 image workload, 24 heads) and
N = 75600 (the 720p video workload, 40 heads) the clustering runs over every
head of the workload, so that the k-means block count per head, the
last-block reductions and the repair selection take the paths the bench
takes; on two heads each the permutation, the centroids, the Q/K codes and
scales, the V residual codes, scales and block means, the repair list and
its deltas must equal the oracle's.

Attention output, against the oracle (relative L2 <= 1e-3 on every checked
head, bf16 against bf16): every row of four heads of the 1024^2 and 2048^2
image workloads, and 512 seeded rows (with the first, last and tail-tile
rows) of two heads of the image-to-image and video workloads, in the launch
configuration the bench times (vc_attn_fwd, default parameters, clustering
inside the call).
"""
import numpy as np
import pytest

import oracle
from bit_attention_diffusion_b200 import synth, vcattn

from gpu_util import bf16_vals, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu
TOL = 1e-3


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a B200"
    from bit_attention_diffusion_b200 import build_lib
    build_lib.build()
    oracle.set_threads(0)
    return torch


def _rows(N, n, seed):
    rng = np.random.default_rng(seed + N)
    fixed = [0, 1, 127, 128, N - 1, N - 2, ((N - 1) // 128) * 128]
    rnd = rng.choice(N, size=min(n, N), replace=False).tolist()
    return np.array(sorted(set(r for r in fixed + rnd if 0 <= r < N)), dtype=np.int32)


@pytest.mark.parametrize("name,heads", [
    ("image2048_b1h24n16544", [(0, 0), (0, 23)]),
    ("video720p_b1h40n75600", [(0, 1), (0, 38)]),
])
def test_prologue_full_size_bit_exact(torch, name, heads):
    wl, x = synth.make_by_name(name)
    p = vcattn.params()
    q, k, v = (to_dev_bf16(x[n]) for n in "qkv")
    perm, cent = vcattn.cluster(v, p)
    qk = vcattn.quant_qk(q, k, perm, p)
    vq = vcattn.quant_v(v, perm, p)
    torch.cuda.synchronize()
    perm, cent = perm.cpu().numpy(), cent.cpu().numpy()
    g = {n: t.cpu().numpy() for n, t in qk.items()}
    v8 = vq["v8"].cpu().numpy()
    vscale = vq["vscale"].cpu().numpy()
    vmean = from_dev_bf16(vq["vmean"])
    rep_idx = vq["rep_idx"].cpu().numpy()
    rep_delta = from_dev_bf16(vq["rep_delta"])
    R = vcattn.vc_attn_repair_count(wl.N, p)
    assert R == oracle.repair_count(0.005, wl.N) > 0
    for b, h in heads:
        o = oracle.head_prologue(x["q"][b, h], x["k"][b, h], x["v"][b, h])
        assert np.array_equal(perm[b, h], o["perm"]), (b, h)
        assert np.array_equal(cent[b, h].view(np.uint32), o["cent"].view(np.uint32)), (b, h)
        for n in ("q8", "sq", "k8", "sk"):
            assert np.array_equal(g[n][b, h], o["qk"][n]), (n, b, h)
        assert np.array_equal(v8[b, h].T, o["vq"]["v8"]), (b, h)
        assert np.array_equal(vscale[b, h], o["vq"]["vscale"]), (b, h)
        assert np.array_equal(vmean[b, h], o["vq"]["vmean"]), (b, h)
        assert np.array_equal(rep_idx[b, h], o["vq"]["rep_idx"]), (b, h)
        assert np.array_equal(rep_delta[b, h], o["vq"]["rep_delta"]), (b, h)


@pytest.mark.parametrize("name,heads,nrows", [
    ("image1024_b1h24n4256", [(0, 0), (0, 7), (0, 16), (0, 23)], None),
    ("image2048_b1h24n16544", [(0, 0), (0, 9), (0, 14), (0, 23)], None),
    ("i2i2048_b2h24n32928", [(0, 5), (1, 17)], 512),
    ("video720p_b1h40n75600", [(0, 0), (0, 39)], 512),
])
def test_fwd_full_size_matches_oracle(torch, name, heads, nrows):
    wl, x = synth.make_by_name(name)
    q, k, v = (to_dev_bf16(x[n]) for n in "qkv")
    out = vcattn.fwd(q, k, v, p=vcattn.params())
    torch.cuda.synchronize()
    out = from_dev_bf16(out)
    assert np.isfinite(bf16_vals(out)).all()
    for b, h in heads:
        rows = np.arange(wl.N, dtype=np.int32) if nrows is None else _rows(wl.N, nrows, 31 * b + h)
        r = oracle.vc_attention_head(x["q"][b, h], x["k"][b, h], x["v"][b, h], rows=rows)
        ref = bf16_vals(oracle.to_bf16_bits(r["out"]))
        got = bf16_vals(out[b, h][rows])
        rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
        print(f"{name} head ({b},{h}) rows {rows.size}: rel-L2 {rel:.3e}")
        assert rel <= TOL, (b, h, rel)
