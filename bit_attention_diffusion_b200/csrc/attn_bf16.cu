// attn_bf16.cu - exact-softmax attention in BF16 on the tcgen05 tensor cores:
// the in-library comparator for the FP8 path (the pages compare against a
// BF16 FlashAttention-class kernel; this is our own, on the same tiling).
//
// One CTA per (128-query tile, b*h); warp 0 TMA producer, warp 1 TMEM owner and
// MMA issuer, warps 2-5 one thread per query row. S = Q K^T (bf16 x bf16 ->
// fp32 in TMEM, double-buffered); online softmax in log2 units with exp2 on
// the SFU; the running max used for P is only moved when the true max exceeds
// it by more than 8 (a factor 256, far inside fp32 and bf16 range), which keeps
// O rescales rare; P in bf16 to shared memory, two slots (tile t in slot t % 2),
// so the softmax of tile t+1 runs while PV(t) does: a tile waits for the PV of
// tile t-2 (its slot) and, only when it moves the max, for PV(t-1); O += P V
// with V consumed MN-major straight from its [token][channel] layout;
// O = acc / l.
#include "common.cuh"
#include "sm100.cuh"
#include "attn_bf16.cuh"

namespace vc {

namespace {

constexpr uint32_t SZ_T16 = 128 * 128 * 2;  // 128x128 bf16 tile = two 64-wide swizzle atoms
constexpr uint32_t ATOM = 16384;
constexpr int ST = 2;
constexpr uint32_t B_OFF_Q = 0;
constexpr uint32_t B_OFF_K = B_OFF_Q + SZ_T16;
constexpr uint32_t B_OFF_V = B_OFF_K + ST * SZ_T16;
constexpr uint32_t B_OFF_P = B_OFF_V + ST * SZ_T16;
constexpr uint32_t B_SMEM = B_OFF_P + 2 * SZ_T16 + 1024;
static_assert(B_SMEM <= 232448, "shared memory budget");

constexpr uint32_t IDESC_S = idesc_make(1, 1, 128, 128, false, false);  // Q K^T, both K-major
constexpr uint32_t IDESC_O = idesc_make(1, 1, 128, 128, false, true);   // P V, V MN-major

struct BarsB {
  uint64_t q, kfull[ST], kempty[ST], vfull[ST], vempty[ST], sfull[2], pfull[2], pvdone[2], main;
};

__device__ __forceinline__ uint64_t kdesc(const uint8_t *p) { return sdesc_sw128(smem_u32(p), 16, 1024); }
__device__ __forceinline__ uint64_t mndesc(const uint8_t *p) { return sdesc_sw128(smem_u32(p), ATOM, 1024); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

}  // namespace

__global__ void __launch_bounds__(192, 1)
    k_attn_ref_bf16(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnBf16Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = sm + B_OFF_Q, *sK = sm + B_OFF_K, *sV = sm + B_OFF_V, *sP = sm + B_OFF_P;
  __shared__ BarsB bars;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, bh = blockIdx.y, T = p.Nb;

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(&bars.q, 1);
    for (int i = 0; i < ST; ++i) {
      mbar_init(&bars.kfull[i], 1); mbar_init(&bars.kempty[i], 1);
      mbar_init(&bars.vfull[i], 1); mbar_init(&bars.vempty[i], 1);
    }
    mbar_init(&bars.sfull[0], 1); mbar_init(&bars.sfull[1], 1);
    mbar_init(&bars.pfull[0], 128); mbar_init(&bars.pfull[1], 128);
    mbar_init(&bars.pvdone[0], 1); mbar_init(&bars.pvdone[1], 1); mbar_init(&bars.main, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&s_tmem, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
    if (s_abort) return false;
    if (!mbar_wait(bar, parity)) {
      s_abort = 1;
      if (p.status) atomicOr(p.status, ST_TIMEOUT);
      return false;
    }
    return true;
  };

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmQ); prefetch_tmap(&tmK); prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(&bars.q, SZ_T16);
      tma_load_3d(sQ, &tmQ, &bars.q, 0, qt * 128, bh);
      tma_load_3d(sQ + ATOM, &tmQ, &bars.q, 64, qt * 128, bh);
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % ST;
        const uint32_t ph = (t / ST) & 1;
        ok = wait(&bars.kempty[s], ph ^ 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars.kfull[s], SZ_T16);
        tma_load_3d(sK + s * SZ_T16, &tmK, &bars.kfull[s], 0, t * 128, bh);
        tma_load_3d(sK + s * SZ_T16 + ATOM, &tmK, &bars.kfull[s], 64, t * 128, bh);
        ok = wait(&bars.vempty[s], ph ^ 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars.vfull[s], SZ_T16);
        tma_load_3d(sV + s * SZ_T16, &tmV, &bars.vfull[s], 0, t * 128, bh);
        tma_load_3d(sV + s * SZ_T16 + ATOM, &tmV, &bars.vfull[s], 64, t * 128, bh);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = wait(&bars.q, 0);
      tc_fence_after();
      auto issue_qk = [&](int t) -> bool {
        const int s = t % ST;
        if (!wait(&bars.kfull[s], (t / ST) & 1)) return false;
        tc_fence_after();
        const uint32_t d = tmem + (t & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ss(d, kdesc(sQ + (kk >> 2) * ATOM + 32 * (kk & 3)),
                     kdesc(sK + s * SZ_T16 + (kk >> 2) * ATOM + 32 * (kk & 3)), IDESC_S, kk > 0);
        mma_commit(&bars.kempty[s]);
        mma_commit(&bars.sfull[t & 1]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      if (ok && T > 1) ok = issue_qk(1);
      for (int t = 0; t < T && ok; ++t) {
        ok = wait(&bars.pfull[t & 1], (t >> 1) & 1);
        if (!ok) break;
        const int s = t % ST;
        ok = wait(&bars.vfull[s], (t / ST) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint8_t *sPt = sP + (t & 1) * SZ_T16;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ss(tmem + 256, kdesc(sPt + (kk >> 2) * ATOM + 32 * (kk & 3)), mndesc(sV + s * SZ_T16 + kk * 2048),
                     IDESC_O, (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars.vempty[s]);
        mma_commit(&bars.pvdone[t & 1]);
        if (t + 2 < T) ok = issue_qk(t + 2);
      }
      if (ok) mma_commit(&bars.main);
    }
  } else {
    const int q4 = warp & 3, r = q4 * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int tail = p.N - (T - 1) * 128;
    float m_use = -INFINITY, l = 0.0f;
    bool ok = true;
    auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
      const bool w = wait(bar, parity);
      return __all_sync(0xFFFFFFFFu, w);
    };
    for (int t = 0; t < T && ok; ++t) {
      const int b = t & 1;
      ok = wwait(&bars.sfull[b], (t >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t v[32];
        tmem_ld32(trow + b * 128 + 32 * i, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) s[32 * i + j] = __uint_as_float(v[j]);
      }
      if (t == T - 1 && tail < 128) {
#pragma unroll
        for (int j = 0; j < 128; ++j)
          if (j >= tail) s[j] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 126; j += 3) mx = fmax3(mx, fmax3(s[j], s[j + 1], s[j + 2]), mx);
      mx = fmax3(mx, s[126], s[127]);
      const float mt = mx * p.scale_log2;
      // slot t % 2 is free once PV(t-2) is complete
      if (t >= 2) {
        ok = wwait(&bars.pvdone[b], ((t >> 1) - 1) & 1);
        if (!ok) break;
      }
      if (t > 0) {
        const bool need = mt > m_use + 8.0f;
        if (__any_sync(0xFFFFFFFFu, need)) {
          // O must hold PV(0..t-1) before it is rescaled (PV(t-2) is complete,
          // so this barrier is at most one phase behind)
          ok = wwait(&bars.pvdone[b ^ 1], ((t - 1) >> 1) & 1);
          if (!ok) break;
          tc_fence_after();
          const float sc = need ? ex2(m_use - mt) : 1.0f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t v[32];
            tmem_ld32(trow + 256 + 32 * i, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * sc);
            tmem_st32(trow + 256 + 32 * i, v);
          }
          tmem_wait_st();
          l *= sc;
          if (need) m_use = mt;
        }
      } else {
        m_use = mt;
      }
      uint8_t *sPt = sP + b * SZ_T16;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 8 * ch + 2 * e;
          const float p0 = ex2(fmaf(s[j], p.scale_log2, -m_use));
          const float p1 = ex2(fmaf(s[j + 1], p.scale_log2, -m_use));
          l += p0 + p1;
          const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
          w[e] = *reinterpret_cast<const uint32_t *>(&pb);
        }
        *reinterpret_cast<uint4 *>(sPt + (ch >> 3) * ATOM + sw128_off(r, ch & 7)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars.pfull[b]);
    }
    if (ok) ok = wwait(&bars.main, 0);
    if (ok) {
      tc_fence_after();
      const int row = qt * 128 + r;
      uint16_t *orow = p.O + (static_cast<size_t>(bh) * p.N + row) * 128;
      const float inv = 1.0f / l;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t v[32];
        tmem_ld32(trow + 256 + 32 * i, v);
        tmem_wait_ld();
        if (row < p.N) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 ob = __floats2bfloat162_rn(__uint_as_float(v[8 * g + 2 * e]) * inv,
                                                              __uint_as_float(v[8 * g + 2 * e + 1]) * inv);
              w[e] = *reinterpret_cast<const uint32_t *>(&ob);
            }
            *reinterpret_cast<uint4 *>(orow + 32 * i + 8 * g) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

uint32_t attn_bf16_smem_bytes() { return B_SMEM; }

}  // namespace vc
