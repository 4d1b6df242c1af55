"""CPU oracle for VC-Attention (FP8 path and NVFP4-residual variant) - test infrastructure, not part of the product.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg may
import this package. The CUDA library never loads it and shares no code with
it. The bit-level steps are plain C in ``vc_oracle.c`` (built here with gcc);
exact attention is numpy float64 (a library matmul).

Page citations (by title and section):
  [VCA]  "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58×
         sem retreinamento": sections "Por que a atenção é o gargalo",
         "V-Smooth: corrigindo outliers de valor" (Group / Demean / Restore),
         "ExpCast-FP8: eliminando o gargalo do softmax".
  [IP73] "VC-Attention et FLUX 3 accélèrent la génération d'images sur
         Blackwell", section "Le compromis entre vitesse et fidélité" (rho).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vc_oracle.c")
_LIB = os.path.join(_HERE, "libvc_oracle.so")
_lock = threading.Lock()
_lib = None

TILE = 128
D = 128
DEFAULT_C = 120
DEFAULT_SCALE = float(np.float32(1.0 / np.sqrt(128.0)))

FLAG_VSMOOTH = 1
FLAG_REPAIR = 2
FLAG_KSMOOTH = 8
FLAG_VFMT_NVFP4 = 32
FLAG_QK_NVFP4 = 64  # full 4-bit path: Q and K in NVFP4 too (with FLAG_VFMT_NVFP4)
FLAGS_DEFAULT = FLAG_VSMOOTH | FLAG_REPAIR | FLAG_KSMOOTH


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no fused contraction, OpenMP over rows)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-fopenmp", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i32, f32, i64 = ctypes.c_int, ctypes.c_float, ctypes.c_longlong
            L.orc_bf16_value.restype = f32
            L.orc_bf16_value.argtypes = [ctypes.c_uint16]
            L.orc_bf16_round.restype = ctypes.c_uint16
            L.orc_bf16_round.argtypes = [f32]
            L.orc_e4m3_value.restype = ctypes.c_double
            L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
            L.orc_e4m3_encode.restype = ctypes.c_uint8
            L.orc_e4m3_encode.argtypes = [f32]
            L.orc_expcast_byte.restype = i32
            L.orc_expcast_byte.argtypes = [f32, f32, f32]
            L.orc_kappa.restype = f32
            L.orc_kappa.argtypes = [f32]
            L.orc_repair_count.restype = i32
            L.orc_repair_count.argtypes = [f32, i32]
            L.orc_kmeans_head.argtypes = [P, i32, i32, i32, i32, P, P, i32]
            L.orc_stable_sort_labels.argtypes = [P, i32, i32, P]
            L.orc_quant_qk_head.argtypes = [P, P, P, i32, i32, i32, P, P, P, P, P]
            L.orc_quant_v_head.argtypes = [P, P, i32, i32, i32, i32, P, P, P, P, P, P]
            L.orc_attn_vc_rows.argtypes = [P, P, P, P, P, P, P, P, P, i32, i32, i32, f32, i32,
                                           P, i32, P, P, P]
            L.orc_attn_exactv_rows.argtypes = [P, P, P, P, P, P, i32, i32, f32, i32, P, i32, P]
            L.orc_set_threads.argtypes = [i32]
            L.orc_get_threads.restype = i32
            L.orc_e4m3_encode_n.argtypes = [P, i64, P]
            L.orc_e4m3_value_n.argtypes = [P, i64, P]
            L.orc_bf16_round_n.argtypes = [P, i64, P]
            L.orc_expcast_n.argtypes = [P, P, P, i64, P]
            L.orc_expcast_bits_n.argtypes = [ctypes.c_uint32, i64, i32, f32, f32, P]
            L.orc_e2m1_value.restype = ctypes.c_double
            L.orc_e2m1_value.argtypes = [ctypes.c_uint8]
            L.orc_e2m1_encode.restype = ctypes.c_uint8
            L.orc_e2m1_encode.argtypes = [f32]
            L.orc_e2m1_encode_n.argtypes = [P, i64, P]
            L.orc_nvfp4_p_block.argtypes = [P, i32, P, P]
            L.orc_quant_v4_head.argtypes = [P, P, i32, i32, i32, i32, P, P, P, P, P, P, P]
            L.orc_attn_vc4_rows.argtypes = [P, P, P, P, P, P, P, P, P, P, i32, i32, i32, f32,
                                            P, i32, P, P, P]
            L.orc_quant_qk4_head.argtypes = [P, P, P, i32, i32, i32, P, P, P, P, P, P, P]
            L.orc_attn_vc44_rows.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, i32, i32, i32, f32,
                                             P, i32, P, P, P]
            _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- formats
def e4m3_value(codes) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().orc_e4m3_value_n(_p(c), c.size, _p(out))
    return out


def e4m3_encode(x) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, np.uint8)
    lib().orc_e4m3_encode_n(_p(a), a.size, _p(out))
    return out


def bf16_round(x) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, np.uint16)
    lib().orc_bf16_round_n(_p(a), a.size, _p(out))
    return out


def bf16_value(b) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def expcast(acc, alpha, c) -> np.ndarray:
    acc = np.ascontiguousarray(acc, dtype=np.float32)
    alpha = np.ascontiguousarray(np.broadcast_to(np.float32(alpha) if np.isscalar(alpha) else alpha,
                                                 acc.shape), dtype=np.float32)
    c = np.ascontiguousarray(np.broadcast_to(np.float32(c) if np.isscalar(c) else c, acc.shape),
                             dtype=np.float32)
    out = np.empty(acc.shape, np.uint8)
    lib().orc_expcast_n(_p(acc), _p(alpha), _p(c), acc.size, _p(out))
    return out


def expcast_bits(first: int, n: int, negative: bool, alpha: float, c: float) -> np.ndarray:
    """ExpCast bytes of the n consecutive binary32 bit patterns first, first+1, ...
    (sign bit set when `negative`), one alpha and c: the exhaustive sweeps."""
    out = np.empty(int(n), np.uint8)
    lib().orc_expcast_bits_n(int(first), int(n), int(bool(negative)), float(np.float32(alpha)),
                             float(np.float32(c)), _p(out))
    return out


def kappa(softmax_scale: float) -> np.float32:
    return np.float32(lib().orc_kappa(float(np.float32(softmax_scale))))


def repair_count(rho: float, N: int) -> int:
    return int(lib().orc_repair_count(float(np.float32(rho)), int(N)))


def set_threads(n: int) -> int:
    lib().orc_set_threads(int(n))
    return int(lib().orc_get_threads())


# ---------------------------------------------------------------- steps, one (b,h)
def kmeans_head(v_bits: np.ndarray, k: int = 8, iters: int = 3, init: np.ndarray | None = None):
    """V-Smooth Group: Lloyd k-means of one head's value tokens -> (centroids, labels).
    `init` (fp32 [k, d]): start from these centroids (warm start from the
    previous step) instead of the tokens floor(j N / k)."""
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    N, d = v.shape
    cent = np.empty((k, d), np.float32) if init is None else np.array(init, dtype=np.float32, copy=True, order="C")
    labels = np.empty(N, np.int32)
    lib().orc_kmeans_head(_p(v), N, d, k, iters, _p(cent), _p(labels), 0 if init is None else 1)
    return cent, labels


def stable_sort_labels(labels: np.ndarray, k: int) -> np.ndarray:
    lab = np.ascontiguousarray(labels, dtype=np.int32)
    perm = np.empty(lab.size, np.int32)
    lib().orc_stable_sort_labels(_p(lab), lab.size, k, _p(perm))
    return perm


def quant_qk_head(q_bits, k_bits, perm, ksmooth: bool = True):
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    kk = np.ascontiguousarray(k_bits, dtype=np.uint16)
    pm = np.ascontiguousarray(perm, dtype=np.int32)
    N, d = q.shape
    Nb = (N + TILE - 1) // TILE
    q8 = np.empty((Nb * TILE, d), np.uint8)
    k8 = np.empty((Nb * TILE, d), np.uint8)
    sq = np.empty(Nb, np.float32)
    sk = np.empty(Nb, np.float32)
    kbar = np.empty(d, np.float32)
    lib().orc_quant_qk_head(_p(q), _p(kk), _p(pm), N, d, int(bool(ksmooth)),
                            _p(q8), _p(sq), _p(k8), _p(sk), _p(kbar))
    return dict(q8=q8, sq=sq, k8=k8, sk=sk, kbar=kbar)


def quant_v_head(v_bits, perm, demean: bool = True, R: int = 0):
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    pm = np.ascontiguousarray(perm, dtype=np.int32)
    N, d = v.shape
    Nb = (N + TILE - 1) // TILE
    v8 = np.empty((Nb * TILE, d), np.uint8)
    vscale = np.empty(d, np.float32)
    vmean = np.empty((Nb, d), np.uint16)
    err = np.empty(N, np.float32)
    rep_idx = np.empty(max(R, 1), np.int32)
    rep_delta = np.empty((max(R, 1), d), np.uint16)
    lib().orc_quant_v_head(_p(v), _p(pm), N, d, int(bool(demean)), int(R), _p(v8), _p(vscale),
                           _p(vmean), _p(err), _p(rep_idx), _p(rep_delta))
    return dict(v8=v8, vscale=vscale, vmean=vmean, err=err,
                rep_idx=rep_idx[:R].copy(), rep_delta=rep_delta[:R].copy())


def attn_vc_rows(qk: dict, vq: dict, N: int, rows, softmax_scale: float = DEFAULT_SCALE,
                 C: int = DEFAULT_C):
    """Quantization-emulating attention for the given query rows of one head.

    Returns (out float64 [len(rows), d], row sums l, final frames F)."""
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    d = qk["q8"].shape[1]
    out = np.empty((rows.size, d), np.float64)
    out_l = np.empty(rows.size, np.float64)
    out_F = np.empty(rows.size, np.float32)
    R = int(vq["rep_idx"].size)
    ri = vq["rep_idx"] if R else np.zeros(1, np.int32)
    rd = vq["rep_delta"] if R else np.zeros((1, d), np.uint16)
    lib().orc_attn_vc_rows(_p(qk["q8"]), _p(qk["sq"]), _p(qk["k8"]), _p(qk["sk"]),
                           _p(vq["v8"]), _p(vq["vscale"]), _p(vq["vmean"]),
                           _p(np.ascontiguousarray(ri)), _p(np.ascontiguousarray(rd)), R,
                           int(N), d, float(kappa(softmax_scale)), int(C), _p(rows), rows.size,
                           _p(out), _p(out_l), _p(out_F))
    return out, out_l, out_F


def attn_exactv_rows(qk: dict, v_bits, perm, N: int, rows, softmax_scale: float = DEFAULT_SCALE,
                     C: int = DEFAULT_C):
    """Diagnostic: the same probability bytes as the method, exact values.

    ``out_method - out_exactv`` is the value-term error alone."""
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    pm = np.ascontiguousarray(perm, dtype=np.int32)
    d = qk["q8"].shape[1]
    out = np.empty((rows.size, d), np.float64)
    lib().orc_attn_exactv_rows(_p(qk["q8"]), _p(qk["sq"]), _p(qk["k8"]), _p(qk["sk"]), _p(v), _p(pm), int(N), d,
                               float(kappa(softmax_scale)), int(C), _p(rows), rows.size, _p(out))
    return out


# ---------------------------------------------------------------- NVFP4 variant
def e2m1_value(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    L = lib()
    table = np.array([L.orc_e2m1_value(i) for i in range(16)], np.float64)
    return table[c & 15]


def e2m1_encode(x) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, np.uint8)
    lib().orc_e2m1_encode_n(_p(a), a.size, _p(out))
    return out


def nvfp4_p_block(x):
    """NVFP4 codes of the probabilities 2^x of one block of <= 16 keys: (codes, scale code)."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    assert 0 < a.size <= 16
    codes = np.empty(a.size, np.uint8)
    sfc = np.empty(1, np.uint8)
    lib().orc_nvfp4_p_block(_p(a), a.size, _p(codes), _p(sfc))
    return codes, int(sfc[0])


def quant_v4_head(v_bits, perm, demean: bool = True, R: int = 0):
    """NVFP4 residual of one head: codes [N, d] (low nibble), block scale codes
    [ceil(N/16), d], per-channel global scales g [d], block means, token errors,
    the repair list and its deltas."""
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    pm = np.ascontiguousarray(perm, dtype=np.int32)
    N, d = v.shape
    Nb = (N + TILE - 1) // TILE
    codes = np.empty((N, d), np.uint8)
    sfc = np.empty(((N + 15) // 16, d), np.uint8)
    vscale = np.empty(d, np.float32)
    vmean = np.empty((Nb, d), np.uint16)
    err = np.empty(N, np.float32)
    rep_idx = np.empty(max(R, 1), np.int32)
    rep_delta = np.empty((max(R, 1), d), np.uint16)
    lib().orc_quant_v4_head(_p(v), _p(pm), N, d, int(bool(demean)), int(R), _p(codes), _p(sfc), _p(vscale),
                            _p(vmean), _p(err), _p(rep_idx), _p(rep_delta))
    return dict(codes=codes, sfc=sfc, vscale=vscale, vmean=vmean, err=err,
                rep_idx=rep_idx[:R].copy(), rep_delta=rep_delta[:R].copy())


def attn_vc4_rows(qk: dict, vq: dict, N: int, rows, softmax_scale: float = DEFAULT_SCALE):
    """The 4-bit variant's attention for the given query rows of one head.

    Returns (out float64 [len(rows), d], row sums l (2688 x the dequantized
    probabilities), final frames F)."""
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    d = qk["q8"].shape[1]
    out = np.empty((rows.size, d), np.float64)
    out_l = np.empty(rows.size, np.float64)
    out_F = np.empty(rows.size, np.float32)
    R = int(vq["rep_idx"].size)
    ri = vq["rep_idx"] if R else np.zeros(1, np.int32)
    rd = vq["rep_delta"] if R else np.zeros((1, d), np.uint16)
    lib().orc_attn_vc4_rows(_p(qk["q8"]), _p(qk["sq"]), _p(qk["k8"]), _p(qk["sk"]),
                            _p(vq["codes"]), _p(vq["sfc"]), _p(vq["vscale"]), _p(vq["vmean"]),
                            _p(np.ascontiguousarray(ri)), _p(np.ascontiguousarray(rd)), R,
                            int(N), d, float(kappa(softmax_scale)), _p(rows), rows.size,
                            _p(out), _p(out_l), _p(out_F))
    return out, out_l, out_F


def quant_qk4_head(q_bits, k_bits, perm, ksmooth: bool = True):
    """NVFP4 Q (original order) and K' (permuted, smoothed): codes [Nb*128, d]
    (low nibble), block scale codes [Nb*128, d/16], per-128-row-block global
    scales g [Nb] (powers of two), and the K channel means."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_bits, dtype=np.uint16)
    pm = np.ascontiguousarray(perm, dtype=np.int32)
    N, d = q.shape
    Nb = (N + TILE - 1) // TILE
    out = dict(qcodes=np.empty((Nb * TILE, d), np.uint8), qsfc=np.empty((Nb * TILE, d // 16), np.uint8),
               qg=np.empty(Nb, np.float32), kcodes=np.empty((Nb * TILE, d), np.uint8),
               ksfc=np.empty((Nb * TILE, d // 16), np.uint8), kg=np.empty(Nb, np.float32),
               kbar=np.empty(d, np.float32))
    lib().orc_quant_qk4_head(_p(q), _p(k), _p(pm), N, d, int(bool(ksmooth)), _p(out["qcodes"]), _p(out["qsfc"]),
                             _p(out["qg"]), _p(out["kcodes"]), _p(out["ksfc"]), _p(out["kg"]), _p(out["kbar"]))
    return out


def attn_vc44_rows(qk4: dict, vq: dict, N: int, rows, softmax_scale: float = DEFAULT_SCALE):
    """The full 4-bit path's attention for the given query rows of one head."""
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    d = qk4["qcodes"].shape[1]
    out = np.empty((rows.size, d), np.float64)
    out_l = np.empty(rows.size, np.float64)
    out_F = np.empty(rows.size, np.float32)
    R = int(vq["rep_idx"].size)
    ri = vq["rep_idx"] if R else np.zeros(1, np.int32)
    rd = vq["rep_delta"] if R else np.zeros((1, d), np.uint16)
    lib().orc_attn_vc44_rows(_p(qk4["qcodes"]), _p(qk4["qsfc"]), _p(qk4["qg"]), _p(qk4["kcodes"]),
                             _p(qk4["ksfc"]), _p(qk4["kg"]), _p(vq["codes"]), _p(vq["sfc"]), _p(vq["vscale"]),
                             _p(vq["vmean"]), _p(np.ascontiguousarray(ri)), _p(np.ascontiguousarray(rd)), R,
                             int(N), d, float(kappa(softmax_scale)), _p(rows), rows.size,
                             _p(out), _p(out_l), _p(out_F))
    return out, out_l, out_F


# ---------------------------------------------------------------- whole path
def head_prologue(q_bits, k_bits, v_bits, flags: int = FLAGS_DEFAULT, k: int = 8, iters: int = 3,
                  rho: float = 0.005, perm=None):
    """Cluster (unless perm is given), quantize Q/K and V, select the repair list."""
    N = q_bits.shape[0]
    cent = labels = None
    if perm is None:
        if flags & FLAG_VSMOOTH:
            cent, labels = kmeans_head(v_bits, k, iters)
            perm = stable_sort_labels(labels, k)
        else:
            perm = np.arange(N, dtype=np.int32)
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    R = repair_count(rho, N) if (flags & FLAG_REPAIR) else 0
    if flags & FLAG_QK_NVFP4:
        assert flags & FLAG_VFMT_NVFP4, "the full 4-bit path needs the NVFP4 residual too"
        qk = quant_qk4_head(q_bits, k_bits, perm, ksmooth=bool(flags & FLAG_KSMOOTH))
    else:
        qk = quant_qk_head(q_bits, k_bits, perm, ksmooth=bool(flags & FLAG_KSMOOTH))
    quant_v = quant_v4_head if (flags & FLAG_VFMT_NVFP4) else quant_v_head
    vq = quant_v(v_bits, perm, demean=bool(flags & FLAG_VSMOOTH), R=R)
    return dict(perm=perm, cent=cent, labels=labels, qk=qk, vq=vq, R=R)


def vc_attention_head(q_bits, k_bits, v_bits, rows=None, flags: int = FLAGS_DEFAULT, k: int = 8,
                      iters: int = 3, rho: float = 0.005, softmax_scale: float = DEFAULT_SCALE,
                      C: int = DEFAULT_C, perm=None):
    """O_vc for one head (rows default: all), plus the prologue's intermediates."""
    N = q_bits.shape[0]
    pro = head_prologue(q_bits, k_bits, v_bits, flags, k, iters, rho, perm)
    if rows is None:
        rows = np.arange(N, dtype=np.int32)
    if flags & FLAG_QK_NVFP4:
        out, l, F = attn_vc44_rows(pro["qk"], pro["vq"], N, rows, softmax_scale)
    elif flags & FLAG_VFMT_NVFP4:
        out, l, F = attn_vc4_rows(pro["qk"], pro["vq"], N, rows, softmax_scale)
    else:
        out, l, F = attn_vc_rows(pro["qk"], pro["vq"], N, rows, softmax_scale, C)
    pro.update(out=out, l=l, F=F, rows=np.asarray(rows, np.int32))
    return pro


def exact_attention_head(q_bits, k_bits, v_bits, rows=None, softmax_scale: float = DEFAULT_SCALE):
    """softmax(Q K^T * scale) V in float64 from the bf16 inputs (the plain definition)."""
    q = bf16_value(q_bits).astype(np.float64)
    kk = bf16_value(k_bits).astype(np.float64)
    v = bf16_value(v_bits).astype(np.float64)
    if rows is not None:
        q = q[np.asarray(rows)]
    s = (q @ kk.T) * float(np.float32(softmax_scale))
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ v) / p.sum(axis=1, keepdims=True)


def to_bf16_bits(x64: np.ndarray) -> np.ndarray:
    """Final output rounding: float64 -> binary32 -> bf16 (nearest-even)."""
    return bf16_round(np.asarray(x64, dtype=np.float64).astype(np.float32))
