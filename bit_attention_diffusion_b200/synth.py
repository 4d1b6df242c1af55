"""Seeded synthetic inputs shaped like the diffusion-transformer attention workloads.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests. It contains no arithmetic of the attention method itself: it draws
random numbers, places value outliers, and rounds fp32 draws to bf16 bit
patterns. Everything returned is a host numpy array of bf16 bit patterns
(``uint16``) laid out [B, H, N, 128], the same bytes for both sides.

Workloads. The pages measure on video/image DiTs (Wan2.2-T2V-A14B,
LongCat-Video, HunyuanVideo-1.5, MiniMax-H3, FLUX 3) whose activations are not
available; these generators stand in for them with the token counts the pages
give (4256 tokens for a 1024x1024 FLUX image with text, ~70k tokens for a 5 s
720p clip) and with the structure the method targets: per-channel key bias
(what Q/K smoothing removes) and value outliers confined to a few tokens whose
channel changes between heads (page "VC-Attention acelera atenção em modelos de
vídeo de IA…", section "V-Smooth: corrigindo outliers de valor").

Recipe (variances, not standard deviations, in N(mu, var)):
  * Q, K, V ~ N(0, 1) drawn in fp32, then rounded to bf16 (nearest-even).
  * K += a per-(b, h, channel) bias ~ N(0, 2).
  * V outliers: a set of tokens per (b, h); each gets one channel (fixed per
    (b, h)) overwritten with +/- magnitude.
  * video: a per-(b, h, channel) random walk over frames is added to V.
Seeds: seed = 1000 + workload index; sub-streams per tensor are fixed.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

D_HEAD = 128


@dataclass(frozen=True)
class Workload:
    """One synthetic attention problem: shapes plus the V-outlier recipe."""
    name: str
    B: int
    H: int
    N: int
    seed: int
    # outliers per (b,h): count, magnitude range, token range [lo, hi)
    n_outliers: int = 0
    out_mag: tuple = (20.0, 20.0)
    out_range: tuple | None = None      # None -> whole sequence
    out_channel_per_token: bool = False  # tiny case: each token its own channel
    frames: int = 0                      # >0: add a smooth per-frame drift to V
    drift_var0: float = 0.5
    drift_var_step: float = 0.5 / 21
    k_bias_var: float = 2.0
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs of one forward pass: 4*B*H*N^2*d (QK^T and PV)."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * D_HEAD


def _wl_table() -> dict:
    t = {}
    t["tiny_b1h2n1024"] = Workload(
        "tiny_b1h2n1024", 1, 2, 1024, 1000, n_outliers=4, out_mag=(20.0, 20.0),
        out_channel_per_token=True,
        note="tiny check: 4 outlier tokens per head, each its own channel set to +/-20")
    t["image1024_b1h24n4256"] = Workload(
        "image1024_b1h24n4256", 1, 24, 4256, 1001, n_outliers=(4256 * 5) // 1000,
        out_mag=(15.0, 30.0),
        note="1024^2 image DiT joint attention (160 text + 4096 image tokens)")
    t["image2048_b1h24n16544"] = Workload(
        "image2048_b1h24n16544", 1, 24, 16544, 1002, n_outliers=(16544 * 5) // 1000,
        out_mag=(15.0, 30.0),
        note="2048^2 image DiT joint attention (160 text + 16384 image tokens)")
    t["i2i2048_b2h24n32928"] = Workload(
        "i2i2048_b2h24n32928", 2, 24, 32928, 1003, n_outliers=32928 // 100,
        out_mag=(20.0, 40.0), out_range=(16544, 32928),
        note="image-to-image 2048^2 with one reference; CFG pair; outliers in reference half")
    t["video720p_b1h40n75600"] = Workload(
        "video720p_b1h40n75600", 1, 40, 75600, 1004, n_outliers=(75600 * 3) // 1000,
        out_mag=(15.0, 30.0), frames=21,
        note="720p video clip: 21 latent frames x 45 x 80 tokens, frame-major, per-frame drift")
    return t


WORKLOADS = _wl_table()
WORKLOAD_ORDER = list(WORKLOADS.keys())


def custom(B: int, H: int, N: int, seed: int = 7, outlier_frac: float = 0.005,
           out_mag=(15.0, 30.0), frames: int = 0) -> Workload:
    """A workload with arbitrary shape and the image-DiT recipe (parity sizes)."""
    return Workload(f"custom_b{B}h{H}n{N}", B, H, N, seed,
                    n_outliers=int(N * outlier_frac), out_mag=out_mag, frames=frames)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to the nearest bf16 (ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + r) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def make_inputs(wl: Workload) -> dict:
    """Draw Q, K, V for a workload. Returns dict(q, k, v) of uint16 [B,H,N,128]."""
    B, H, N, d = wl.B, wl.H, wl.N, D_HEAD
    ss = np.random.SeedSequence(wl.seed)
    gq, gk, gv, gb, go, gd = [np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(6)]

    q = gq.standard_normal((B, H, N, d), dtype=np.float32)
    qb = f32_to_bf16_bits(q)
    del q

    k = gk.standard_normal((B, H, N, d), dtype=np.float32)
    bias = (gb.standard_normal((B, H, 1, d), dtype=np.float32) * np.float32(np.sqrt(wl.k_bias_var)))
    k += bias
    kb = f32_to_bf16_bits(k)
    del k

    v = gv.standard_normal((B, H, N, d), dtype=np.float32)
    if wl.frames > 0:
        per = N // wl.frames
        steps = gd.standard_normal((B, H, wl.frames, d), dtype=np.float32)
        steps[:, :, 0] *= np.float32(np.sqrt(wl.drift_var0))
        steps[:, :, 1:] *= np.float32(np.sqrt(wl.drift_var_step))
        walk = np.cumsum(steps, axis=2, dtype=np.float32)
        for f in range(wl.frames):
            lo = f * per
            hi = N if f == wl.frames - 1 else lo + per
            v[:, :, lo:hi, :] += walk[:, :, f:f + 1, :]
    if wl.n_outliers > 0:
        lo, hi = wl.out_range if wl.out_range is not None else (0, N)
        lo, hi = max(0, lo), min(N, hi)
        cnt = min(wl.n_outliers, hi - lo)
        for b in range(B):
            for h in range(H):
                toks = go.choice(hi - lo, size=cnt, replace=False) + lo
                ch_head = int(go.integers(0, d))
                mags = go.uniform(wl.out_mag[0], wl.out_mag[1], size=cnt)
                signs = np.where(go.random(cnt) < 0.5, -1.0, 1.0)
                for i, tkn in enumerate(toks):
                    ch = int(go.integers(0, d)) if wl.out_channel_per_token else ch_head
                    v[b, h, tkn, ch] = np.float32(signs[i] * mags[i])
    vb = f32_to_bf16_bits(v)
    del v
    return {"q": qb, "k": kb, "v": vb}


def make_by_name(name: str) -> tuple[Workload, dict]:
    wl = WORKLOADS[name]
    return wl, make_inputs(wl)
