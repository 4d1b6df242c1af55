"""GPU check of the in-library BF16 comparator against exact fp64 attention.

Tolerance: P is rounded to bf16 before the PV product (2^-9 relative per
probability, averaging out over the row) and O is rounded to bf16 at the end
(rel-L2 ~ 2^-9/sqrt(3) ~ 1.1e-3); 4e-3 leaves room for the SFU exp2 and the
fp32 accumulation."""
import numpy as np
import pytest

import oracle
from bit_attention_diffusion_b200 import synth, vcattn

from gpu_util import bf16_vals, from_dev_bf16, rel_l2, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a B200"
    from bit_attention_diffusion_b200 import build_lib
    build_lib.build()
    return torch


@pytest.mark.parametrize("B,H,N", [(1, 2, 1024), (1, 1, 1), (1, 2, 300), (2, 2, 129), (1, 3, 4256)])
def test_ref_bf16_matches_exact_attention(torch, B, H, N):
    x = synth.make_inputs(synth.custom(B, H, N, seed=500 + N))
    out = vcattn.fwd_ref_bf16(*(to_dev_bf16(x[n]) for n in "qkv"))
    torch.cuda.synchronize()
    out = from_dev_bf16(out)
    for b in range(B):
        for h in range(H):
            rows = np.arange(N) if N <= 1024 else np.linspace(0, N - 1, 200).astype(int)
            ex = oracle.exact_attention_head(x["q"][b, h], x["k"][b, h], x["v"][b, h], rows=rows)
            assert rel_l2(bf16_vals(out[b, h][rows]), ex) < 4e-3, (b, h)


def test_ref_bf16_custom_scale_and_large_scores(torch):
    """A large softmax scale (peaked rows) exercises the lazy rescale."""
    B, H, N = 1, 2, 1500
    x = synth.make_inputs(synth.custom(B, H, N, seed=501))
    out = from_dev_bf16(vcattn.fwd_ref_bf16(*(to_dev_bf16(x[n]) for n in "qkv"), softmax_scale=0.6))
    for h in range(H):
        ex = oracle.exact_attention_head(x["q"][0, h], x["k"][0, h], x["v"][0, h], softmax_scale=0.6)
        assert rel_l2(bf16_vals(out[0, h]), ex) < 4e-3
