"""Thin Python binding of libvcattn (include/vc_attn.h).

Argument marshalling only: every step of the method runs in the CUDA library.
The low-level functions carry the C names and take integers (device pointers,
sizes, a cudaStream_t as int) and return the integer status. The convenience
wrappers (``fwd``, ``cluster``, ``quant_qk``, ``quant_v``, ``fwd_ref_bf16``,
``expcast``, ``e4m3_encode``) take torch CUDA tensors, allocate the outputs and
the workspace with torch (the library itself never allocates), and raise
``VcError`` on a non-OK status.

There is no CPU fallback: loading fails with an error if ``libvcattn.so`` has
not been built (``python -m bit_attention_diffusion_b200.build_lib``).
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvcattn.so")

VC_OK, VC_ERR_INVALID_ARG, VC_ERR_UNSUPPORTED, VC_ERR_WORKSPACE, VC_ERR_CUDA, VC_ERR_TIMEOUT = range(6)
VC_VSMOOTH, VC_REPAIR, VC_KSMOOTH, VC_WARMSTART, VC_VFMT_NVFP4, VC_QK_NVFP4 = 1, 2, 8, 16, 32, 64
VC_FUSED_PROLOGUE = 128
FLAGS_DEFAULT = VC_VSMOOTH | VC_REPAIR | VC_KSMOOTH
D = 128

EXPORTED = [
    "vc_params_default", "vc_status_str", "vc_attn_workspace_bytes", "vc_attn_repair_count",
    "vc_attn_cluster", "vc_attn_quant_qk", "vc_attn_quant_v", "vc_attn_fwd", "vc_attn_fwd_ref_bf16",
    "vc_attn_expcast", "vc_attn_e4m3_encode", "vc_attn_device_status", "vc_attn_wait_selftest",
    "vc_attn_launch_count", "vc_attn_profile", "vc_attn_profile_read",
    "vc_attn_cluster_noalloc", "vc_attn_cluster_noalloc_max_bytes", "vc_attn_fwd_host",
]


class VcParams(ctypes.Structure):
    _fields_ = [("k", ctypes.c_int), ("iters", ctypes.c_int), ("rho", ctypes.c_float),
                ("softmax_scale", ctypes.c_float), ("expcast_bias", ctypes.c_int), ("flags", ctypes.c_uint)]


class VcError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_str(status)} (status {status})")
        self.status = status


_lock = threading.Lock()
_lib = None


def lib():
    """Load libvcattn.so (once). Raises if it is missing: no fallback exists."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                                   "`python -m bit_attention_diffusion_b200.build_lib`")
            L = ctypes.CDLL(LIB_PATH)
            P, I, Z, F, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_longlong
            PP = ctypes.POINTER(VcParams)
            L.vc_params_default.argtypes = [PP]
            L.vc_params_default.restype = None
            L.vc_status_str.argtypes = [I]
            L.vc_status_str.restype = ctypes.c_char_p
            L.vc_attn_workspace_bytes.argtypes = [I, I, I, I, PP]
            L.vc_attn_workspace_bytes.restype = Z
            L.vc_attn_repair_count.argtypes = [I, PP]
            L.vc_attn_repair_count.restype = I
            L.vc_attn_cluster.argtypes = [P, I, I, I, I, PP, P, P, P, Z, P]
            L.vc_attn_quant_qk.argtypes = [P, P, P, I, I, I, I, PP, P, P, P, P, P, Z, P]
            L.vc_attn_quant_v.argtypes = [P, P, I, I, I, I, PP, P, P, P, P, P, P, Z, P]
            L.vc_attn_fwd.argtypes = [P, P, P, I, I, I, I, P, PP, P, P, Z, P]
            L.vc_attn_fwd_host.argtypes = [P, P, P, I, I, I, I, PP, P, P, P, P, P, I, P, Z, P]
            L.vc_attn_fwd_ref_bf16.argtypes = [P, P, P, I, I, I, I, F, P, P]
            L.vc_attn_expcast.argtypes = [P, P, P, LL, P, P]
            L.vc_attn_e4m3_encode.argtypes = [P, LL, P, P]
            L.vc_attn_device_status.argtypes = [P, P]
            L.vc_attn_wait_selftest.argtypes = [P, LL, P]
            L.vc_attn_profile.argtypes = [I]
            L.vc_attn_profile_read.argtypes = [ctypes.POINTER(ctypes.c_float), I]
            L.vc_attn_profile_read.restype = I
            L.vc_attn_cluster_noalloc.argtypes = [P, I, I, I, I, PP, P, P, P]
            L.vc_attn_cluster_noalloc_max_bytes.argtypes = []
            L.vc_attn_cluster_noalloc_max_bytes.restype = Z
            L.vc_attn_launch_count.argtypes = []
            L.vc_attn_launch_count.restype = ctypes.c_ulonglong
            for n in EXPORTED:
                if n not in ("vc_params_default", "vc_status_str", "vc_attn_workspace_bytes",
                             "vc_attn_repair_count", "vc_attn_launch_count",
                             "vc_attn_cluster_noalloc_max_bytes"):
                    getattr(L, n).restype = I
            _lib = L
    return _lib


# ---------------------------------------------------------------- C-named wrappers
def params(k=8, iters=3, rho=0.005, softmax_scale=0.0, expcast_bias=120, flags=FLAGS_DEFAULT) -> VcParams:
    p = VcParams()
    lib().vc_params_default(ctypes.byref(p))
    p.k, p.iters, p.rho, p.softmax_scale, p.expcast_bias, p.flags = (
        int(k), int(iters), float(rho), float(softmax_scale), int(expcast_bias), int(flags))
    return p


def status_str(s: int) -> str:
    return lib().vc_status_str(int(s)).decode()


def vc_attn_workspace_bytes(B, H, N, d, p: VcParams) -> int:
    return int(lib().vc_attn_workspace_bytes(B, H, N, d, ctypes.byref(p)))


def vc_attn_repair_count(N, p: VcParams) -> int:
    return int(lib().vc_attn_repair_count(N, ctypes.byref(p)))


def vc_attn_cluster(V, B, H, N, d, p, perm, centroids, ws, ws_bytes, stream) -> int:
    return lib().vc_attn_cluster(V, B, H, N, d, ctypes.byref(p), perm, centroids, ws, ws_bytes, stream)


def vc_attn_cluster_noalloc(V, B, H, N, d, p, perm, centroids, stream) -> int:
    """vc_attn_cluster without a workspace (fixed 32 MiB library-owned scratch)."""
    return lib().vc_attn_cluster_noalloc(V, B, H, N, d, ctypes.byref(p), perm, centroids, stream)


def vc_attn_cluster_noalloc_max_bytes() -> int:
    return int(lib().vc_attn_cluster_noalloc_max_bytes())


def vc_attn_quant_qk(Q, K, perm, B, H, N, d, p, q8, sq, k8, sk, ws, ws_bytes, stream) -> int:
    return lib().vc_attn_quant_qk(Q, K, perm, B, H, N, d, ctypes.byref(p), q8, sq, k8, sk, ws, ws_bytes, stream)


def vc_attn_quant_v(V, perm, B, H, N, d, p, v8, v_scale, v_mean, rep_idx, rep_delta, ws, ws_bytes, stream) -> int:
    return lib().vc_attn_quant_v(V, perm, B, H, N, d, ctypes.byref(p), v8, v_scale, v_mean, rep_idx, rep_delta,
                                 ws, ws_bytes, stream)


def vc_attn_fwd(Q, K, V, B, H, N, d, perm, p, O, ws, ws_bytes, stream) -> int:
    return lib().vc_attn_fwd(Q, K, V, B, H, N, d, perm, ctypes.byref(p), O, ws, ws_bytes, stream)


def vc_attn_fwd_host(hQ, hK, hV, B, H, N, d, p, hO, dQ, dK, dV, dO, groups, ws, ws_bytes, stream) -> int:
    return lib().vc_attn_fwd_host(hQ, hK, hV, B, H, N, d, ctypes.byref(p), hO, dQ, dK, dV, dO, groups, ws, ws_bytes,
                                  stream)


def vc_attn_fwd_ref_bf16(Q, K, V, B, H, N, d, softmax_scale, O, stream) -> int:
    return lib().vc_attn_fwd_ref_bf16(Q, K, V, B, H, N, d, float(softmax_scale), O, stream)


def vc_attn_expcast(acc, alpha, c, n, out, stream) -> int:
    return lib().vc_attn_expcast(acc, alpha, c, n, out, stream)


def vc_attn_e4m3_encode(x, n, out, stream) -> int:
    return lib().vc_attn_e4m3_encode(x, n, out, stream)


def vc_attn_device_status(ws, stream) -> int:
    return lib().vc_attn_device_status(ws, stream)


def vc_attn_wait_selftest(ws, limit_cycles, stream) -> int:
    return lib().vc_attn_wait_selftest(ws, int(limit_cycles), stream)


def vc_attn_profile(on: bool) -> int:
    return lib().vc_attn_profile(1 if on else 0)


def vc_attn_profile_read() -> list:
    """Mean phase durations (ms) of the profiled vc_attn_fwd calls:
    [cluster, quant_v (Q/K quantization overlaps it on a side stream),
    further wait for quant_qk, attention]; [] if none was recorded."""
    buf = (ctypes.c_float * 4)()
    n = lib().vc_attn_profile_read(buf, 4)
    return [float(buf[i]) for i in range(n)]


def vc_attn_launch_count() -> int:
    return int(lib().vc_attn_launch_count())


# ---------------------------------------------------------------- torch conveniences
def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(st: int, where: str):
    if st != VC_OK:
        raise VcError(st, where)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _shape(x):
    assert x.dim() == 4 and x.shape[-1] == D and x.is_contiguous(), "expected contiguous [B,H,N,128]"
    B, H, N, d = x.shape
    return int(B), int(H), int(N), int(d)


def workspace(B, H, N, p: VcParams, device="cuda"):
    torch = _torch()
    nbytes = vc_attn_workspace_bytes(B, H, N, D, p)
    if nbytes == 0:
        raise VcError(VC_ERR_INVALID_ARG, "vc_attn_workspace_bytes")
    return torch.empty(nbytes, dtype=torch.uint8, device=device), nbytes


def fwd(q, k, v, perm=None, p: VcParams | None = None, out=None, ws=None, stream=None):
    """O = VC-Attention FP8 forward (bf16 [B,H,N,128] tensors on the GPU)."""
    torch = _torch()
    p = p or params()
    B, H, N, d = _shape(q)
    if ws is None:
        ws, nbytes = workspace(B, H, N, p, q.device)
    else:
        nbytes = ws.numel()
    if out is None:
        out = torch.empty_like(q)
    _check(vc_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, d, _ptr(perm), p, out.data_ptr(),
                       ws.data_ptr(), nbytes, _stream(stream)), "vc_attn_fwd")
    return out


def fwd_host(hq, hk, hv, groups: int, p: VcParams | None = None, hout=None, dev=None, ws=None, stream=None):
    """O = VC-Attention FP8 forward from host (CPU, ideally pinned) bf16 [B,H,N,128]
    tensors; the device staging tensors `dev` = (dQ, dK, dV, dO) and the
    workspace for one run of ceil(B*H/groups) heads are allocated if not given."""
    torch = _torch()
    p = p or params()
    B, H, N, d = _shape(hq)
    if hout is None:
        hout = torch.empty_like(hq, pin_memory=True)
    if dev is None:
        dev = tuple(torch.empty(hq.shape, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    gh = -(-(B * H) // min(groups, B * H))
    if ws is None:
        ws, nbytes = workspace(1, gh, N, p)
    else:
        nbytes = ws.numel()
    _check(vc_attn_fwd_host(hq.data_ptr(), hk.data_ptr(), hv.data_ptr(), B, H, N, d, p, hout.data_ptr(),
                            *(t.data_ptr() for t in dev), groups, ws.data_ptr(), nbytes, _stream(stream)),
           "vc_attn_fwd_host")
    return hout


def cluster(v, p: VcParams | None = None, ws=None, stream=None, init=None):
    """V-Smooth Group: returns (perm int32 [B,H,N], centroids fp32 [B,H,k,128]).
    `init` (fp32 [B,H,k,128] on the device): warm start from these centroids
    (VC_WARMSTART), e.g. the previous denoising step's."""
    torch = _torch()
    p = p or params()
    B, H, N, d = _shape(v)
    if ws is None:
        ws, nbytes = workspace(B, H, N, p, v.device)
    else:
        nbytes = ws.numel()
    perm = torch.empty((B, H, N), dtype=torch.int32, device=v.device)
    if init is None:
        cent = torch.empty((B, H, p.k, D), dtype=torch.float32, device=v.device)
    else:
        cent = init.to(dtype=torch.float32).contiguous().clone()
        p = VcParams(p.k, p.iters, p.rho, p.softmax_scale, p.expcast_bias, p.flags | VC_WARMSTART)
    _check(vc_attn_cluster(v.data_ptr(), B, H, N, d, p, perm.data_ptr(), cent.data_ptr(), ws.data_ptr(), nbytes,
                           _stream(stream)), "vc_attn_cluster")
    return perm, cent


class VSmoothSchedule:
    """Cross-step V-Smooth over a denoising run: the value grouping is
    recomputed (warm-started from the previous step's centroids) only in the
    first `cluster_fraction` of the steps; later steps reuse the last
    permutation. `perm(v, step)` returns the permutation to pass to fwd()."""

    def __init__(self, total_steps: int, cluster_fraction: float = 0.25, p: VcParams | None = None):
        self.total = int(total_steps)
        self.last_cluster_step = max(0, int(self.total * cluster_fraction + 0.5) - 1)
        self.p = p or params()
        self._perm = None
        self._cent = None

    def clusters_at(self, step: int) -> bool:
        return step <= self.last_cluster_step or self._perm is None

    def perm(self, v, step: int, ws=None, stream=None):
        if self.clusters_at(step):
            self._perm, self._cent = cluster(v, self.p, ws=ws, stream=stream, init=self._cent)
        return self._perm


def quant_qk(q, k, perm=None, p: VcParams | None = None, ws=None, stream=None):
    torch = _torch()
    p = p or params()
    B, H, N, d = _shape(q)
    Nb = (N + 127) // 128
    if ws is None:
        ws, nbytes = workspace(B, H, N, p, q.device)
    else:
        nbytes = ws.numel()
    q8 = torch.empty((B, H, Nb * 128, D), dtype=torch.uint8, device=q.device)
    k8 = torch.empty_like(q8)
    sq = torch.empty((B, H, Nb), dtype=torch.float32, device=q.device)
    sk = torch.empty_like(sq)
    _check(vc_attn_quant_qk(q.data_ptr(), k.data_ptr(), _ptr(perm), B, H, N, d, p, q8.data_ptr(), sq.data_ptr(),
                            k8.data_ptr(), sk.data_ptr(), ws.data_ptr(), nbytes, _stream(stream)),
           "vc_attn_quant_qk")
    return dict(q8=q8, sq=sq, k8=k8, sk=sk)


def quant_v(v, perm=None, p: VcParams | None = None, ws=None, stream=None):
    torch = _torch()
    p = p or params()
    B, H, N, d = _shape(v)
    Nb = (N + 127) // 128
    R = vc_attn_repair_count(N, p)
    if ws is None:
        ws, nbytes = workspace(B, H, N, p, v.device)
    else:
        nbytes = ws.numel()
    v8 = torch.empty((B, H, D, Nb * 128), dtype=torch.uint8, device=v.device)
    vscale = torch.empty((B, H, D), dtype=torch.float32, device=v.device)
    vmean = torch.empty((B, H, Nb, D), dtype=torch.bfloat16, device=v.device)
    rep_idx = torch.empty((B, H, max(R, 1)), dtype=torch.int32, device=v.device)
    rep_delta = torch.empty((B, H, max(R, 1), D), dtype=torch.bfloat16, device=v.device)
    _check(vc_attn_quant_v(v.data_ptr(), _ptr(perm), B, H, N, d, p, v8.data_ptr(), vscale.data_ptr(),
                           vmean.data_ptr(), rep_idx.data_ptr(), rep_delta.data_ptr(), ws.data_ptr(), nbytes,
                           _stream(stream)), "vc_attn_quant_v")
    return dict(v8=v8, vscale=vscale, vmean=vmean, rep_idx=rep_idx[..., :R], rep_delta=rep_delta[..., :R, :], R=R)


def fwd_ref_bf16(q, k, v, softmax_scale=0.0, out=None, stream=None):
    torch = _torch()
    B, H, N, d = _shape(q)
    if out is None:
        out = torch.empty_like(q)
    _check(vc_attn_fwd_ref_bf16(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, d, softmax_scale,
                                out.data_ptr(), _stream(stream)), "vc_attn_fwd_ref_bf16")
    return out


def expcast(acc, alpha, c, stream=None):
    torch = _torch()
    out = torch.empty(acc.numel(), dtype=torch.uint8, device=acc.device)
    _check(vc_attn_expcast(acc.data_ptr(), alpha.data_ptr(), c.data_ptr(), acc.numel(), out.data_ptr(),
                           _stream(stream)), "vc_attn_expcast")
    return out


def e4m3_encode(x, stream=None):
    torch = _torch()
    out = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    _check(vc_attn_e4m3_encode(x.data_ptr(), x.numel(), out.data_ptr(), _stream(stream)), "vc_attn_e4m3_encode")
    return out
