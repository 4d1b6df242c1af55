"""GPU unit parity: ExpCast bytes and E4M3 codes bit-exact against the oracle,
through the C ABI; the bounded device wait reports a timeout instead of hanging."""
import numpy as np
import pytest

import oracle
from bit_attention_diffusion_b200 import vcattn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a B200"
    from bit_attention_diffusion_b200 import build_lib
    build_lib.build()
    return torch


def _pairs(rng, n):
    """acc random over many binades; each (2j, 2j+1) pair shares alpha and c."""
    mant = rng.integers(0, 1 << 23, n, dtype=np.uint32)
    ex = rng.integers(100, 152, n, dtype=np.uint32)
    sign = rng.integers(0, 2, n, dtype=np.uint32) << 31
    acc = (sign | (ex << 23) | mant).view(np.float32)
    alpha = np.repeat(rng.uniform(1e-4, 0.5, n // 2).astype(np.float32), 2)
    c = np.repeat(rng.integers(-600, 121, n // 2).astype(np.float32), 2)
    return acc, alpha, c


def test_expcast_bytes_bit_exact(torch):
    rng = np.random.default_rng(100)
    n = 1 << 22
    acc, alpha, c = _pairs(rng, n)
    acc[:8] = [np.inf, -np.inf, 0.0, -0.0, 1e-30, -1e-30, 3e38, -3e38]
    # the frame guarantees bytes <= C in the kernel; compare where the exact byte is <= 126
    want = oracle.expcast(acc, alpha, c)
    with np.errstate(invalid="ignore", over="ignore"):
        v = acc.astype(np.float64) * alpha + c
    keep = v < 126.0
    d = lambda a: torch.from_numpy(a).cuda()
    got = vcattn.expcast(d(acc), d(alpha), d(c)).cpu().numpy()
    assert np.array_equal(got[keep], want[keep]), np.nonzero(got[keep] != want[keep])[0][:10]
    assert keep.mean() > 0.5 and (want[keep] > 0).mean() > 0.05


def test_expcast_dense_sweep_over_byte_range(torch):
    """Every fp32 value of acc in [-(C+1), 2] (step 2^-12) with alpha = 1, c = 120."""
    acc = np.arange(-121 * 4096, 2 * 4096 + 1, dtype=np.float64) / 4096
    if acc.size % 2:
        acc = acc[:-1]
    acc = acc.astype(np.float32)
    alpha = np.ones_like(acc)
    c = np.full_like(acc, 120.0)
    want = oracle.expcast(acc, alpha, c)
    d = lambda a: torch.from_numpy(a).cuda()
    got = vcattn.expcast(d(acc), d(alpha), d(c)).cpu().numpy()
    assert np.array_equal(got, want)


@pytest.mark.parametrize("alpha,c", [(1.0, 120.0), (0.0553709, 112.0)])
def test_expcast_exhaustive_matches_oracle(torch, alpha, c):
    """Every binary32 score acc <= 0 with acc*alpha >= -(c+1) (about 1.1e9
    inputs per case, the range the oracle's exhaustive pin covers: every score
    that can reach a nonzero byte): the device bytes equal the oracle's, byte
    for byte. alpha = 1, c = 120 is the score in byte units against the row
    maximum's frame; the second case has a non-power-of-two alpha, so the
    fused product's rounding decides bytes."""
    alpha = float(np.float32(alpha))
    last = int(np.float32((c + 1.0) / alpha).view(np.uint32))
    while float(np.uint32(last).view(np.float32)) * alpha < c + 1.0:
        last += 1
    total = last + 1
    chunk = 1 << 27
    a_dev = torch.full((chunk,), alpha, dtype=torch.float32, device="cuda")
    c_dev = torch.full((chunk,), c, dtype=torch.float32, device="cuda")
    checked = 0
    for lo in range(0, total, chunk):
        n = min(chunk, total - lo)
        n += n & 1  # the entry point takes pairs; one extra input past the range is harmless
        acc = torch.arange(lo, lo + n, dtype=torch.int64, device="cuda").to(torch.int32).view(torch.float32).neg()
        got = vcattn.expcast(acc, a_dev[:n], c_dev[:n]).cpu().numpy()
        want = oracle.expcast_bits(lo, n, True, alpha, c)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, [(lo + int(i), int(got[i]), int(want[i])) for i in bad[:8]]
        checked += n
    assert checked >= total > 1_000_000_000


def test_e4m3_encoder_bit_exact(torch):
    rng = np.random.default_rng(101)
    n = 1 << 22
    mant = rng.integers(0, 1 << 23, n, dtype=np.uint32)
    ex = rng.integers(100, 140, n, dtype=np.uint32)
    sign = rng.integers(0, 2, n, dtype=np.uint32) << 31
    x = (sign | (ex << 23) | mant).view(np.float32)
    vals = oracle.e4m3_value(np.arange(0, 0x7F, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                        np.array([448, 464, 465, 1e9, -1e9, 0.0, -0.0, 2.0 ** -10], np.float32)])
    if x.size % 2:
        x = x[:-1]
    got = vcattn.e4m3_encode(torch.from_numpy(x).cuda()).cpu().numpy()
    assert np.array_equal(got, oracle.e4m3_encode(x))


def test_bounded_wait_reports_timeout(torch):
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    st = vcattn.vc_attn_wait_selftest(ws.data_ptr(), 20000, torch.cuda.current_stream().cuda_stream)
    assert st == vcattn.VC_OK
    assert vcattn.vc_attn_device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream) == \
        vcattn.VC_ERR_TIMEOUT
    # reading clears the word
    assert vcattn.vc_attn_device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream) == vcattn.VC_OK
    torch.cuda.synchronize()
