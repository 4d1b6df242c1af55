"""CPU checks of the C-ABI boundary: the library loads, exports every function
include/vc_attn.h declares, and rejects bad arguments on the host before any
device work (these calls never reach a launch, so they run without a GPU)."""
import ctypes
import os
import re

import pytest

from bit_attention_diffusion_b200 import vcattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "vc_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(vc_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from bit_attention_diffusion_b200 import build_lib
    build_lib.build()
    return vcattn.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert "vc_attn_fwd" in names and "vc_attn_cluster" in names and "vc_attn_quant_v" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(vcattn.EXPORTED)


def test_defaults_and_status_strings(L):
    p = vcattn.params()
    assert (p.k, p.iters, p.expcast_bias, p.flags) == (8, 3, 120, 11)
    assert abs(p.rho - 0.005) < 1e-9
    assert vcattn.status_str(0) == "ok"
    assert "workspace" in vcattn.status_str(3)


def test_repair_count_and_workspace_size(L):
    p = vcattn.params()
    assert [vcattn.vc_attn_repair_count(n, p) for n in (1024, 4256, 16544, 32928, 75600)] == \
        [6, 22, 83, 165, 378]
    assert vcattn.vc_attn_repair_count(1000, vcattn.params(flags=vcattn.VC_VSMOOTH)) == 0
    ws = vcattn.vc_attn_workspace_bytes(1, 24, 16544, 128, p)
    # at least the quantized Q, K, V (one byte per element) plus the permutation
    assert ws >= 3 * 24 * 16640 * 128 + 24 * 16544 * 4
    assert vcattn.vc_attn_workspace_bytes(1, 1, 100, 64, p) == 0
    assert vcattn.vc_attn_workspace_bytes(1, 1, 0, 128, p) == 0


FAKE = 1 << 20  # a 256-aligned non-null address; never dereferenced in these calls


@pytest.mark.parametrize("case,status", [
    (dict(d=64), vcattn.VC_ERR_UNSUPPORTED),
    (dict(N=0), vcattn.VC_ERR_INVALID_ARG),
    (dict(B=0), vcattn.VC_ERR_INVALID_ARG),
    (dict(N=1 << 24, H=64), vcattn.VC_ERR_INVALID_ARG),      # B*H*Npad*d >= 2^31
    (dict(ws=0), vcattn.VC_ERR_INVALID_ARG),
    (dict(ws=FAKE + 16), vcattn.VC_ERR_INVALID_ARG),         # workspace not 256-aligned
    (dict(ws_bytes=1024), vcattn.VC_ERR_WORKSPACE),
    (dict(p=dict(k=0)), vcattn.VC_ERR_INVALID_ARG),
    (dict(p=dict(k=65)), vcattn.VC_ERR_INVALID_ARG),
    (dict(p=dict(rho=1.0)), vcattn.VC_ERR_INVALID_ARG),
    (dict(p=dict(rho=-0.1)), vcattn.VC_ERR_INVALID_ARG),
    (dict(p=dict(expcast_bias=127)), vcattn.VC_ERR_INVALID_ARG),
    (dict(p=dict(flags=4)), vcattn.VC_ERR_INVALID_ARG),
    (dict(p=dict(flags=256)), vcattn.VC_ERR_INVALID_ARG),
    (dict(p=dict(flags=vcattn.FLAGS_DEFAULT | vcattn.VC_QK_NVFP4)), vcattn.VC_ERR_INVALID_ARG),  # needs VFMT_NVFP4
    (dict(p=dict(softmax_scale=-1.0)), vcattn.VC_ERR_INVALID_ARG),
])
def test_fwd_rejects_bad_arguments_on_host(L, case, status):
    B, H, N, d = case.get("B", 1), case.get("H", 2), case.get("N", 256), case.get("d", 128)
    p = vcattn.params(**case.get("p", {}))
    ws = case.get("ws", FAKE)
    ws_bytes = case.get("ws_bytes", 1 << 40)
    st = vcattn.vc_attn_fwd(FAKE, FAKE, FAKE, B, H, N, d, None, p, FAKE, ws, ws_bytes, None)
    assert st == status


def test_ref_and_units_reject_bad_arguments_on_host(L):
    assert vcattn.vc_attn_fwd_ref_bf16(FAKE, FAKE, FAKE, 1, 1, 128, 96, 0.0, FAKE, None) == vcattn.VC_ERR_UNSUPPORTED
    assert vcattn.vc_attn_fwd_ref_bf16(FAKE + 8, FAKE, FAKE, 1, 1, 128, 128, 0.0, FAKE, None) == \
        vcattn.VC_ERR_INVALID_ARG
    assert vcattn.vc_attn_expcast(FAKE, FAKE, FAKE, 3, FAKE, None) == vcattn.VC_ERR_INVALID_ARG
    assert vcattn.vc_attn_e4m3_encode(None, 4, FAKE, None) == vcattn.VC_ERR_INVALID_ARG
    assert vcattn.vc_attn_wait_selftest(FAKE + 4, 100, None) == vcattn.VC_ERR_INVALID_ARG
    assert vcattn.vc_attn_device_status(None, None) == vcattn.VC_ERR_INVALID_ARG
    p = vcattn.params()
    assert vcattn.vc_attn_cluster(FAKE, 1, 1, 256, 128, p, None, None, FAKE, 1 << 40, None) == \
        vcattn.VC_ERR_INVALID_ARG
    assert vcattn.vc_attn_quant_v(FAKE, None, 1, 1, 256, 128, p, FAKE, FAKE, FAKE, None, None, FAKE, 1 << 40,
                                  None) == vcattn.VC_ERR_INVALID_ARG   # R > 0 needs rep_idx/rep_delta


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib
    mod = importlib.reload(vcattn)
    monkeypatch.setattr(mod, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(mod, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        mod.lib()
    importlib.reload(vcattn)


@pytest.mark.parametrize("case,status", [
    (dict(d=96), vcattn.VC_ERR_UNSUPPORTED),
    (dict(groups=0), vcattn.VC_ERR_INVALID_ARG),
    (dict(null_host=True), vcattn.VC_ERR_INVALID_ARG),
    (dict(dev_off=8), vcattn.VC_ERR_INVALID_ARG),                # device staging not 16-byte aligned
    (dict(ws_bytes=1024), vcattn.VC_ERR_WORKSPACE),             # smaller than one run of heads
])
def test_fwd_host_rejects_bad_arguments_on_host(L, case, status):
    p = vcattn.params()
    d = case.get("d", 128)
    host = 0 if case.get("null_host") else FAKE
    dev = FAKE + case.get("dev_off", 0)
    st = vcattn.vc_attn_fwd_host(host, FAKE, FAKE, 1, 4, 256, d, p, FAKE, dev, FAKE, FAKE, FAKE,
                                 case.get("groups", 2), FAKE, case.get("ws_bytes", 1 << 40), None)
    assert st == status


def test_fwd_host_workspace_is_sized_for_one_run_of_heads(L):
    """The workspace needed is the one for a run of ceil(B*H/groups) heads (here
    B*H = 6 in 2 runs of 3): one byte less is rejected before any device work."""
    p = vcattn.params()
    need = vcattn.vc_attn_workspace_bytes(1, 3, 256, 128, p)   # B*H = 6, groups = 2 -> runs of 3 heads
    st = vcattn.vc_attn_fwd_host(FAKE, FAKE, FAKE, 2, 3, 256, 128, p, FAKE, FAKE, FAKE, FAKE, FAKE, 2, FAKE,
                                 need - 1, None)
    assert st == vcattn.VC_ERR_WORKSPACE


def test_vsmooth_schedule_clusters_in_the_first_quarter(L):
    sched = vcattn.VSmoothSchedule(20, cluster_fraction=0.25)
    assert sched.last_cluster_step == 4
    sched._perm = object()   # as after a first clustering
    assert [sched.clusters_at(s) for s in range(7)] == [True] * 5 + [False] * 2


def test_noalloc_cluster_rejects_bad_arguments_on_host(L):
    """The allocation-free clustering entry point checks its arguments, and
    that the clustering scratch fits its fixed array, before touching a
    device."""
    p = vcattn.params()
    ok = (FAKE, 1, 2, 1024, 128, p, FAKE, FAKE, None)
    assert vcattn.vc_attn_cluster_noalloc_max_bytes() == 32 << 20
    for i, bad in ((0, None), (6, None), (7, None), (0, FAKE + 8), (6, FAKE + 4)):
        args = list(ok)
        args[i] = bad
        assert vcattn.vc_attn_cluster_noalloc(*args) == vcattn.VC_ERR_INVALID_ARG, (i, bad)
    assert vcattn.vc_attn_cluster_noalloc(FAKE, 1, 2, 1024, 64, p, FAKE, FAKE, None) == vcattn.VC_ERR_UNSUPPORTED
    assert vcattn.vc_attn_cluster_noalloc(FAKE, 1, 2, 1024, 128, vcattn.params(k=0), FAKE, FAKE, None) == \
        vcattn.VC_ERR_INVALID_ARG
    # about 7.8 M tokens fit at k = 8; 8.4 M do not
    assert vcattn.vc_attn_cluster_noalloc(FAKE, 4, 64, 32768, 128, p, FAKE, FAKE, None) == vcattn.VC_ERR_WORKSPACE
