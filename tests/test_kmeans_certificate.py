"""The error bound behind the k-means label certificate, checked numerically
on the CPU (test infrastructure; the GPU tests check the labels themselves
bit for bit against the oracle).

Page "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58× sem
retreinamento", section "V-Smooth: corrigindo outliers de valor", item Group.
The k <= 8 Lloyd pass decides a token's label from a tensor-core estimate
e_j = |v|^2 + |c_j|^2 - 2 v.(hi_j + lo_j) whenever every other cluster's
estimate exceeds the smallest by more than E_b + E_j, E_j = 2^-13 (|v|^2 +
|c_j|^2), and otherwise runs the pinned fp32 chains. `tests/kmeans_bound_pin.c`
(independent of the library and of the oracle) recomputes the pinned chains
and the estimates under four accumulation models of the tensor cores; the
bound |e_j - d~_j| <= E_j must hold everywhere, and no certified label may
differ from the chains' argmin. A planted smaller margin must let wrong labels
through on near-tie tokens, so the margin is what keeps them out.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
D = 128


@pytest.fixture(scope="module")
def pin(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("kmpin") / "libkmeans_pin.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           os.path.join(HERE, "kmeans_bound_pin.c"), "-o", out, "-lm"])
    L = ctypes.CDLL(out)
    P = ctypes.c_void_p
    L.pin_kmeans_bound.argtypes = [P, ctypes.c_int, P, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                   ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong),
                                   ctypes.POINTER(ctypes.c_longlong)]
    return L


def _bf16_bits(x):
    return oracle.to_bf16_bits(np.asarray(x, dtype=np.float32))


def _run(pin, vbits, cent, bscale=1.0):
    vbits = np.ascontiguousarray(vbits, dtype=np.uint16)
    cent = np.ascontiguousarray(cent, dtype=np.float32)
    n, k = vbits.shape[0], cent.shape[0]
    worst, wrong, acc = ctypes.c_double(), ctypes.c_longlong(), ctypes.c_longlong()
    rc = pin.pin_kmeans_bound(vbits.ctypes.data, n, cent.ctypes.data, k, D, ctypes.c_float(bscale),
                              ctypes.byref(worst), ctypes.byref(wrong), ctypes.byref(acc))
    assert rc == 0
    return worst.value, wrong.value, acc.value, 4 * n


def _workload_tokens(n, seed):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((n, D)).astype(np.float32)
    v[:, :8] += rng.normal(0.0, 2.0, 8).astype(np.float32)  # a shared channel bias
    out = rng.choice(n, n // 100, replace=False)
    v[out, rng.integers(0, D, out.size)] = rng.uniform(15, 30, out.size) * rng.choice([-1, 1], out.size)
    return _bf16_bits(v)


def _oracle_centroids(vbits, k, iters):
    """The centroids a Lloyd pass starts from after `iters` iterations."""
    cent, _ = oracle.kmeans_head(vbits, k=k, iters=iters)
    return cent


def test_bound_holds_on_workload_like_tokens(pin):
    vbits = _workload_tokens(1536, 11)
    for k, iters in ((8, 0), (8, 1), (8, 3), (4, 3), (2, 2)):
        cent = _oracle_centroids(vbits, k, iters)
        worst, wrong, acc, tot = _run(pin, vbits, cent)
        assert worst < 0.5, (k, iters, worst)
        assert wrong == 0, (k, iters)
        assert acc > 0.9 * tot, (k, iters, acc, tot)


def test_bound_holds_near_ties_and_extreme_scales(pin):
    rng = np.random.default_rng(12)
    cent = rng.standard_normal((8, D)).astype(np.float32)
    toks = []
    # near each centroid, and on the bisector of two centroids (plus tiny noise)
    for j in range(8):
        toks.append(cent[j] + 1e-3 * rng.standard_normal((24, D)).astype(np.float32))
        m = 0.5 * (cent[j] + cent[(j + 1) % 8])
        toks.append(m + 1e-4 * rng.standard_normal((24, D)).astype(np.float32))
    v = np.concatenate(toks)
    for scale in (1.0, 1e3, 1e-3, 2.0 ** 40, 2.0 ** -40):
        vb = _bf16_bits(v * scale)
        worst, wrong, acc, tot = _run(pin, vb, cent * np.float32(scale))
        assert worst < 0.5, (scale, worst)
        assert wrong == 0, scale
    # channels of very different magnitude within one token
    w = rng.standard_normal((256, D)).astype(np.float32) * np.float32(2.0) ** rng.integers(-20, 20, D)
    c2 = w[rng.choice(256, 8, replace=False)] * np.float32(1.001)
    worst, wrong, acc, tot = _run(pin, _bf16_bits(w), c2)
    assert worst < 0.5 and wrong == 0


def test_a_smaller_margin_lets_wrong_labels_through(pin):
    # two centroids 1e-6 apart (relative): the bf16 hi/lo split resolves a
    # centroid to about 2^-18, so the estimates cannot order the two and the
    # chains decide by rounding; with no margin the certificate would accept
    # the estimate's choice
    rng = np.random.default_rng(13)
    c0 = rng.standard_normal(D).astype(np.float32)
    c1 = (c0 * (1.0 + 1e-6 * rng.choice([-1.0, 1.0], D))).astype(np.float32)
    cent = np.stack([c0, c1])
    vb = _bf16_bits(rng.standard_normal((4000, D)))
    worst, wrong_kernel, acc_kernel, _ = _run(pin, vb, cent, 1.0)
    _, wrong_planted, _, _ = _run(pin, vb, cent, 0.0)
    assert worst < 0.5
    assert wrong_kernel == 0
    assert wrong_planted > 0
