"""Accuracy against exact fp64 attention on all five workloads, and what
V-Smooth and repair change, measured through the C ABI.

For every workload (full size, default parameters, clustering inside the
call) and every path - the 8-bit path, the NVFP4-residual variant and the
full 4-bit path - the output on sampled rows of two heads (256 seeded rows
each plus the first, last and tail-tile rows) is compared with exact
softmax(QK^T/sqrt(d))V computed in float64 from the same bf16 inputs: relative
L2 and cosine over the sampled rows. Each path also runs without V-Smooth and
repair (flags = K smoothing only: no grouping, demean, restore or repair; the
same per-channel scales), and on the 8-bit path the value-term error alone is
measured (the kernel's output against the oracle's output with the same
probability bytes and exact values) on the outlier channel of each head and
over all channels.

The page "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58×
sem retreinamento" (section "Por que a atenção é o gargalo") attributes most
of the quantization error of 8-bit attention to the value term; the
synthetic Gaussian inputs put the FP8 probability rounding itself (E4M3 has a
relative step of 6-12%) at about 5% relative L2 on diffuse rows, so the
targets 3e-2 / 0.999 against exact attention are not expected to hold on
every workload, whatever the kernel. The test checks bands and writes the
table (stdout, and accuracy.json under $VC_REPORT_DIR when that is set).
"""
import json
import os

import numpy as np
import pytest

import oracle
from bit_attention_diffusion_b200 import synth, vcattn

from gpu_util import bf16_vals, cosine, from_dev_bf16, rel_l2, to_dev_bf16

pytestmark = pytest.mark.gpu

WORKLOADS = [("tiny_b1h2n1024", [(0, 0), (0, 1)]),
             ("image1024_b1h24n4256", [(0, 0), (0, 23)]),
             ("image2048_b1h24n16544", [(0, 0), (0, 23)]),
             ("i2i2048_b2h24n32928", [(0, 5), (1, 17)]),
             ("video720p_b1h40n75600", [(0, 0), (0, 39)])]
PATHS = {"fp8": 0, "nvfp4": vcattn.VC_VFMT_NVFP4, "nvfp4qk": vcattn.VC_VFMT_NVFP4 | vcattn.VC_QK_NVFP4}
# bands (not targets): the 8-bit path at the FP8 noise floor, the 4-bit paths at theirs
BANDS = {"fp8": (0.08, 0.996), "nvfp4": (0.25, 0.97), "nvfp4qk": (0.30, 0.95)}


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a B200"
    from bit_attention_diffusion_b200 import build_lib
    build_lib.build()
    oracle.set_threads(0)
    return torch


@pytest.fixture(scope="module")
def report():
    rows = []
    yield rows
    lines = ["| workload | path | rel-L2 vs exact | cosine | without V-Smooth+repair: rel-L2 | cosine | "
             "value-term error, outlier channel (with / without) | value-term error, all channels (with / without) |",
             "|---|---|---|---|---|---|---|---|"]
    for r in rows:
        vt = r.get("value_term")
        vt_o = f"{vt['outlier_with']:.4f} / {vt['outlier_without']:.4f}" if vt else "-"
        vt_a = f"{vt['all_with']:.4f} / {vt['all_without']:.4f}" if vt else "-"
        lines.append(f"| {r['workload']} | {r['path']} | {r['rel_l2']:.4f} | {r['cosine']:.5f} | "
                     f"{r['plain_rel_l2']:.4f} | {r['plain_cosine']:.5f} | {vt_o} | {vt_a} |")
    print("\n" + "\n".join(lines))
    out_dir = os.environ.get("VC_REPORT_DIR")
    if out_dir:
        os.makedirs(out_dir, exist_ok=True)
        with open(os.path.join(out_dir, "accuracy.json"), "w") as f:
            json.dump(rows, f, indent=1)
        with open(os.path.join(out_dir, "accuracy.md"), "w") as f:
            f.write("\n".join(lines) + "\n")


def _rows(N, seed):
    rng = np.random.default_rng(seed + N)
    fixed = [0, 1, 127, 128, N - 1, N - 2, ((N - 1) // 128) * 128]
    rnd = rng.choice(N, size=min(256, N), replace=False).tolist()
    return np.array(sorted(set(r for r in fixed + rnd if 0 <= r < N)), dtype=np.int32)


@pytest.mark.parametrize("name,heads", WORKLOADS)
def test_accuracy_against_exact_attention(torch, report, name, heads):
    wl, x = synth.make_by_name(name)
    q, k, v = (to_dev_bf16(x[n]) for n in "qkv")
    rows = {bh: _rows(wl.N, 17 * bh[0] + bh[1]) for bh in heads}
    exact = {(b, h): oracle.exact_attention_head(x["q"][b, h], x["k"][b, h], x["v"][b, h], rows=rows[(b, h)])
             for b, h in heads}
    for path, extra in PATHS.items():
        res = {}
        for tag, flags in (("with", vcattn.FLAGS_DEFAULT | extra), ("without", vcattn.VC_KSMOOTH | extra)):
            out = vcattn.fwd(q, k, v, p=vcattn.params(flags=flags))
            torch.cuda.synchronize()
            res[tag] = from_dev_bf16(out)
            del out
        got = {t: np.concatenate([bf16_vals(res[t][b, h][rows[(b, h)]]) for b, h in heads]) for t in res}
        ex = np.concatenate([exact[bh] for bh in heads])
        r = {"workload": name, "path": path, "rows": int(sum(rows[bh].size for bh in heads)),
             "heads": [list(bh) for bh in heads],
             "rel_l2": rel_l2(got["with"], ex), "cosine": cosine(got["with"], ex),
             "plain_rel_l2": rel_l2(got["without"], ex), "plain_cosine": cosine(got["without"], ex)}
        if path == "fp8":
            # value term: the kernel's output against the oracle's output with the same
            # probability bytes (the same flags' Q/K prologue) and exact values
            acc = {t: [0.0, 0.0, 0.0, 0.0] for t in ("with", "without")}
            for (b, h) in heads:
                vh = x["v"][b, h]
                ch = int(np.argmax(np.abs(bf16_vals(vh)).max(axis=0)))
                for tag, flags in (("with", vcattn.FLAGS_DEFAULT), ("without", vcattn.VC_KSMOOTH)):
                    pro = oracle.head_prologue(x["q"][b, h], x["k"][b, h], vh, flags=flags)
                    ev = oracle.attn_exactv_rows(pro["qk"], vh, pro["perm"], wl.N, rows[(b, h)])
                    e = bf16_vals(res[tag][b, h][rows[(b, h)]]) - ev
                    acc[tag][0] += float((e[:, ch] ** 2).sum())
                    acc[tag][1] += float((ev[:, ch] ** 2).sum())
                    acc[tag][2] += float((e ** 2).sum())
                    acc[tag][3] += float((ev ** 2).sum())
            r["value_term"] = {"outlier_with": np.sqrt(acc["with"][0] / acc["with"][1]),
                               "outlier_without": np.sqrt(acc["without"][0] / acc["without"][1]),
                               "all_with": np.sqrt(acc["with"][2] / acc["with"][3]),
                               "all_without": np.sqrt(acc["without"][2] / acc["without"][3])}
        report.append(r)
        print(name, path, {kk: vv for kk, vv in r.items() if kk not in ("heads",)})
        max_rel, min_cos = BANDS[path]
        assert r["rel_l2"] < max_rel and r["cosine"] > min_cos, r
