"""The one-launch prologue (VC_FUSED_PROLOGUE): vc_attn_fwd's clustering,
Q/K and V quantization and repair as one cooperative persistent kernel.

Every step computes what the separate kernels compute (each work item is one
of their blocks), so the output must be bit-identical to the default path's,
which the attention parity tests hold against the oracle; one case is also
checked against the oracle directly. The device status must report no
barrier timeout.
"""
import numpy as np
import pytest

import oracle
from bit_attention_diffusion_b200 import synth, vcattn

from gpu_util import bf16_vals, from_dev_bf16, rel_l2, to_dev_bf16

pytestmark = pytest.mark.gpu
FUSED = vcattn.VC_FUSED_PROLOGUE


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a B200"
    from bit_attention_diffusion_b200 import build_lib
    build_lib.build()
    return torch


def _pair(torch, x, p, perm=None):
    """(default path, one-launch prologue) outputs, and the device status after the latter."""
    q, k, v = (to_dev_bf16(x[n]) for n in "qkv")
    pm = None if perm is None else torch.from_numpy(perm).cuda()
    o1 = vcattn.fwd(q, k, v, perm=pm, p=p)
    pf = vcattn.params(k=p.k, iters=p.iters, rho=p.rho, softmax_scale=p.softmax_scale,
                       expcast_bias=p.expcast_bias, flags=p.flags | FUSED)
    B, H, N, _ = q.shape
    ws, nb = vcattn.workspace(B, H, N, pf)
    o2 = vcattn.fwd(q, k, v, perm=pm, p=pf, ws=ws)
    torch.cuda.synchronize()
    st = vcattn.vc_attn_device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return o1, o2, st


SHAPES = [(1, 2, 1024), (1, 3, 300), (2, 2, 129), (1, 1, 1), (1, 2, 7), (1, 4, 4256), (1, 2, 8300)]


@pytest.mark.parametrize("B,H,N", SHAPES)
def test_fused_prologue_bit_identical(torch, B, H, N):
    x = synth.make_inputs(synth.custom(B, H, N, seed=5100 + N))
    o1, o2, st = _pair(torch, x, vcattn.params())
    assert st == vcattn.VC_OK
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("flags", [vcattn.VC_KSMOOTH, vcattn.VC_VSMOOTH | vcattn.VC_REPAIR,
                                   vcattn.VC_VSMOOTH | vcattn.VC_KSMOOTH, 0])
def test_fused_prologue_flag_variants(torch, flags):
    x = synth.make_inputs(synth.custom(1, 2, 1000, seed=5200 + flags))
    o1, o2, st = _pair(torch, x, vcattn.params(flags=flags))
    assert st == vcattn.VC_OK
    assert torch.equal(o1, o2)


def test_fused_prologue_other_parameters_and_cached_permutation(torch):
    x = synth.make_inputs(synth.custom(1, 3, 2000, seed=5301))
    p = vcattn.params(k=5, iters=2, rho=0.02, softmax_scale=0.05)
    o1, o2, st = _pair(torch, x, p)
    assert st == vcattn.VC_OK and torch.equal(o1, o2)
    rng = np.random.default_rng(5302)
    perm = np.stack([rng.permutation(2000) for _ in range(3)])[None].astype(np.int32)
    o1, o2, st = _pair(torch, x, vcattn.params(), perm=perm)
    assert st == vcattn.VC_OK and torch.equal(o1, o2)


def test_fused_prologue_matches_oracle(torch):
    B, H, N = 1, 2, 1500
    x = synth.make_inputs(synth.custom(B, H, N, seed=5400))
    q, k, v = (to_dev_bf16(x[n]) for n in "qkv")
    out = from_dev_bf16(vcattn.fwd(q, k, v, p=vcattn.params(flags=vcattn.FLAGS_DEFAULT | FUSED)))
    for h in range(H):
        r = oracle.vc_attention_head(x["q"][0, h], x["k"][0, h], x["v"][0, h])
        assert rel_l2(bf16_vals(out[0, h]), bf16_vals(oracle.to_bf16_bits(r["out"]))) <= 1e-3


def test_fused_prologue_image_workload(torch):
    """The image workload (B=1, H=24, N=16544) at full size."""
    wl, x = synth.make_by_name("image2048_b1h24n16544")
    o1, o2, st = _pair(torch, x, vcattn.params())
    assert st == vcattn.VC_OK
    assert torch.equal(o1, o2)


def test_fused_prologue_ignored_where_it_does_not_apply(torch):
    """k > 8 and the 4-bit variants take the separate kernels: same output."""
    x = synth.make_inputs(synth.custom(1, 2, 700, seed=5500))
    for p in (vcattn.params(k=12), vcattn.params(flags=vcattn.FLAGS_DEFAULT | vcattn.VC_VFMT_NVFP4)):
        o1, o2, st = _pair(torch, x, p)
        assert st == vcattn.VC_OK and torch.equal(o1, o2)
