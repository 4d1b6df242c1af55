"""Cross-step V-Smooth on a synthetic denoising run (GPU).

The pages run the value grouping only in the first quarter of the denoising
steps and reuse it afterwards ([VCA] "V-Smooth", Group), and measure the
grouping by the share of block energy the demean removes. Here: value tensors
whose tokens belong to persistent groups in random sequence positions and
drift from step to step; the schedule clusters, warm-started, in the
first 25% of the steps and then reuses the permutation; every step is compared
with a cold clustering of that step. Printed numbers are the measurement
(run with -s); the asserts are loose bounds on it."""
import numpy as np
import pytest

from bit_attention_diffusion_b200 import synth, vcattn  # noqa: F401

from gpu_util import to_dev_bf16

pytestmark = pytest.mark.gpu


def _demean_energy(v: np.ndarray, perm: np.ndarray) -> float:
    """Share of ||V||^2 removed by subtracting 128-token block means in permuted order."""
    vp = v[perm]
    N = vp.shape[0]
    removed = 0.0
    for s in range(0, N, 128):
        blk = vp[s:s + 128]
        mu = blk.mean(axis=0)
        removed += blk.shape[0] * float(mu @ mu)
    return removed / float((vp * vp).sum())


def test_schedule_reuses_the_grouping_with_little_loss():
    import torch
    assert torch.cuda.is_available()
    from bit_attention_diffusion_b200 import build_lib
    build_lib.build()
    # tokens drawn from 8 persistent groups per head in random sequence
    # positions (group centres ~ N(0, 1) per channel, token noise N(0, 1)),
    # plus a step-to-step drift of every token and of every centre
    H, N, S, G = 4, 8192, 12, 8
    rng = np.random.default_rng(10)
    centres = rng.standard_normal((H, G, 128), dtype=np.float32)
    groups = rng.integers(0, G, (H, N))
    noise = rng.standard_normal((H, N, 128), dtype=np.float32)
    v = (np.take_along_axis(centres, groups[:, :, None], axis=1) + noise)[None]
    sched = vcattn.VSmoothSchedule(S, cluster_fraction=0.25)
    rows = []
    for s in range(S):
        if s > 0:
            centres = centres + np.float32(0.05) * rng.standard_normal(centres.shape, dtype=np.float32)
            noise = noise + np.float32(0.1) * rng.standard_normal(noise.shape, dtype=np.float32)
            v = (np.take_along_axis(centres, groups[:, :, None], axis=1) + noise)[None]
        bits = synth.f32_to_bf16_bits(v)
        vf = synth.bf16_bits_to_f32(bits)
        vd = to_dev_bf16(bits)
        perm_s = sched.perm(vd, s).cpu().numpy()
        perm_c, _ = vcattn.cluster(vd, vcattn.params())
        perm_c = perm_c.cpu().numpy()
        e_seq = np.mean([_demean_energy(vf[0, h], np.arange(N)) for h in range(H)])
        e_sched = np.mean([_demean_energy(vf[0, h], perm_s[0, h]) for h in range(H)])
        e_cold = np.mean([_demean_energy(vf[0, h], perm_c[0, h]) for h in range(H)])
        rows.append((s, sched.clusters_at(s), e_seq, e_sched, e_cold))
    print("\nstep clustered  energy removed: sequence order / schedule / cold clustering")
    for s, c, a, b, c0 in rows:
        print(f"{s:4d} {str(c):9s} {a:8.4f} {b:8.4f} {c0:8.4f}")
    for s, c, e_seq, e_sched, e_cold in rows:
        assert e_sched > e_seq                  # the grouping still helps after it stops being recomputed
        assert e_sched >= 0.8 * e_cold          # and loses little against reclustering every step

