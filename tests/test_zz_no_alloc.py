"""The allocation-free clustering entry point, through the C ABI.

vc_attn_cluster_noalloc serves callers that cannot allocate device memory
where they cluster (a plugin whose host framework owns all allocations, a
deployment that forbids cudaMalloc after start-up, a path where an allocation
would synchronize the device): its scratch is a fixed array the library
reserves on each GPU. Its output must equal vc_attn_cluster's, call after
call, since every call reuses (and clears) the same array. This file sorts
last so a failure here comes after every other test has run; it also passes
alone in a fresh process.
"""
import numpy as np
import pytest

from bit_attention_diffusion_b200 import synth, vcattn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a B200"
    from bit_attention_diffusion_b200 import build_lib
    build_lib.build()
    return torch


def _dev_bf16(torch, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _noalloc(torch, v, p, init=None):
    B, H, N, d = (int(s) for s in v.shape)
    perm = torch.empty((B, H, N), dtype=torch.int32, device="cuda")
    if init is None:
        cent = torch.empty((B, H, p.k, 128), dtype=torch.float32, device="cuda")
    else:
        cent = init.clone()
        p = vcattn.VcParams(p.k, p.iters, p.rho, p.softmax_scale, p.expcast_bias, p.flags | vcattn.VC_WARMSTART)
    st = vcattn.vc_attn_cluster_noalloc(v.data_ptr(), B, H, N, d, p, perm.data_ptr(), cent.data_ptr(),
                                        torch.cuda.current_stream().cuda_stream)
    assert st == vcattn.VC_OK, vcattn.status_str(st)
    return perm, cent


def test_noalloc_cluster_matches_workspace_cluster_twice_in_a_row(torch):
    p = vcattn.params()
    cases = [synth.make_inputs(synth.custom(1, 3, 1500, seed=71)),
             synth.make_by_name("image1024_b1h24n4256")[1]]
    for x in cases:                      # two calls in a row on the shared scratch
        v = _dev_bf16(torch, x["v"])
        perm_ref, cent_ref = vcattn.cluster(v, p)
        perm, cent = _noalloc(torch, v, p)
        torch.cuda.synchronize()
        assert torch.equal(perm, perm_ref)
        assert torch.equal(cent.view(torch.int32), cent_ref.view(torch.int32))


def test_noalloc_more_clusters_and_warm_start_match_back_to_back(torch):
    """k = 16 (the general k-means kernel, its own shared-memory sizing) and a
    warm start from given centroids (VC_WARMSTART: the centroids are an input),
    run back to back on the shared array, each against vc_attn_cluster."""
    x = synth.make_inputs(synth.custom(1, 4, 3000, seed=73))
    v = _dev_bf16(torch, x["v"])
    p16 = vcattn.params(k=16, iters=2)
    perm_ref, cent_ref = vcattn.cluster(v, p16)
    perm, cent = _noalloc(torch, v, p16)
    torch.cuda.synchronize()
    assert torch.equal(perm, perm_ref) and torch.equal(cent.view(torch.int32), cent_ref.view(torch.int32))
    _, c2 = vcattn.cluster(v, vcattn.params(iters=2))
    p3 = vcattn.params(iters=3)
    perm_ref, cent_ref = vcattn.cluster(v, p3, init=c2)
    perm, cent = _noalloc(torch, v, p3, init=c2)
    torch.cuda.synchronize()
    assert torch.equal(perm, perm_ref) and torch.equal(cent.view(torch.int32), cent_ref.view(torch.int32))


def test_noalloc_video_workload_shape(torch):
    """The 720p video shape (B=1, H=40, N=75600: 3.0 M tokens) fits the array:
    equal to vc_attn_cluster, and head 0 equal to the oracle."""
    import oracle
    wl, x = synth.make_by_name("video720p_b1h40n75600")
    p = vcattn.params()
    v = _dev_bf16(torch, x["v"])
    perm_ref, cent_ref = vcattn.cluster(v, p)
    perm, cent = _noalloc(torch, v, p)
    torch.cuda.synchronize()
    assert torch.equal(perm, perm_ref) and torch.equal(cent.view(torch.int32), cent_ref.view(torch.int32))
    c_o, lab_o = oracle.kmeans_head(x["v"][0, 0], p.k, p.iters)
    assert np.array_equal(perm[0, 0].cpu().numpy(), oracle.stable_sort_labels(lab_o, p.k))
    assert np.array_equal(cent[0, 0].cpu().numpy().view(np.uint32), c_o.view(np.uint32))


def test_noalloc_rejects_shapes_beyond_its_scratch(torch):
    p = vcattn.params()
    assert vcattn.vc_attn_cluster_noalloc_max_bytes() == 32 << 20
    # 4 x 64 heads x 32768 tokens needs far more than 32 MiB: rejected before any launch
    st = vcattn.vc_attn_cluster_noalloc(1 << 20, 4, 64, 32768, 128, p, 1 << 20, 1 << 20, None)
    assert st == vcattn.VC_ERR_WORKSPACE
