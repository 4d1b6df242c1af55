// attn_fp4.cu - the fused attention kernels of the 4-bit variants, sm_100a:
// the NVFP4-residual variant (QK^T in FP8) and the full 4-bit path (QK^T in
// NVFP4 as well); two query tiles per CTA sharing one TMEM score buffer.
//
// Page "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58× sem
// retreinamento": "V-Smooth: corrigindo outliers de valor", item Demean (the
// value residual quantized to NVFP4 for the 4-bit kernel) and item Restore
// (the block means come back through the online softmax's row sums);
// "ExpCast-FP8: eliminando o gargalo do softmax": ExpCast is 8-bit only, so
// here the probabilities come from an exp2 softmax and are quantized to NVFP4
// per 16 keys; "Por que a atenção é o gargalo": low-precision tensor cores for
// both products (the full 4-bit path). Page "VC-Attention et FLUX 3 accélèrent
// la génération d'images sur Blackwell", "Le compromis entre vitesse et
// fidélité": repair of the worst tokens.
//
// One CTA per (pair of 128-query tiles a, b; b*h); 11 warps:
//   warp 0     lane 0: Q_a, Q_b, the K tiles (ring), then the repair deltas;
//              lane 1: the NVFP4 V tile images (ring, one bulk copy each);
//              lane 2: the block-mean chunks (one per 32 KV tiles).
//   warp 1     allocates TMEM; copies the scale factors into TMEM and issues
//              PV (kind::mxf4nvf4, 16-element E4M3 scales) for both query
//              tiles, the block-mean restores and the repair products.
//   warp 2     issues QK^T for both query tiles (FP8, or kind::mxf4nvf4).
//   warps 3-6  softmax warpgroup of query tile a, warps 7-10 of tile b: one
//              thread per query row, all KV tiles of its own query tile, its
//              own running frame and row sums.
// QK^T alternates the score buffer S between the query tiles: S <- Q_a K(t),
// read out by warpgroup a; S <- Q_b K(t), read by b; S <- Q_a K(t+1) ...
// What is specific to the 4-bit products:
//   - The block-scaled FP4 MMA reads both operands from shared memory, so P_i
//     goes to a shared-memory slot [1 KB scales | 8 KB codes] per query tile;
//     the PV warp copies the slot's scales into TMEM (tcgen05.cp) right
//     before the product (two TMEM scale slots per query tile, by t % 2).
//   - Each softmax thread turns its row's 128 scores into 8 blocks of 16:
//     x = fma(acc, alpha/8, -F/8), p = 2^x, block scale sf = E4M3(448 * max p),
//     codes E2M1(p * fl(2688 / sf)), the multipliers from a 128-entry table.
//   - PV_i is one N = 144 product: B = the V tile's 128 channel rows plus 16
//     rows E, row 0 all E2M1 ones at scale 1.0, the others zero, so the row
//     sum l_t (sum of value(code) * sf over the tile, 2688 x the dequantized
//     probabilities) accumulates into the column after O_i; the warpgroup
//     reads it once PV_i(t) is complete and takes l_t as the difference of
//     two reads.
// TMEM (512 columns x 128 lanes): S [0,128); O_a [128,256) with its row-sum
// block [256,272); O_b [272,400) with [400,416); V scales of ring stage s at
// 416 + 16 s (+8 per K step; column +4 holds the constant scale of E); P
// scales of query tile i, slot j at TM_SFA + 16 i + 8 j (+4 per K step);
// full 4-bit path: Q scales of tile i at TM_QSF + 8 i, K' scales of slot j
// at TM_KSF + 8 j.
// O is kept in units of 2688 x p x v / g (g the channel's global scale, a power
// of two): O_acc = sum P * value(code) * vsf + sum_t l_t * mean_t / g +
// sum_R P' * delta / g, and the epilogue writes O = g_c * O_acc / l.
#include "common.cuh"
#include "sm100.cuh"
#include "attn_common.cuh"
#include "attn_fp4.cuh"

#include <type_traits>

namespace vc {

namespace {
using namespace attn;

constexpr uint32_t SZ_TILE8 = 128 * 128;                       // one 128x128 byte tile
constexpr uint32_t SZ_V4 = 128 * 64;                           // E2M1 codes of one V tile
constexpr uint32_t SZ_E4 = 16 * 64;                            // E rows
constexpr uint32_t SZ_VSTAGE = V4_SF_BYTES + SZ_V4 + SZ_E4;    // [scales | codes | E]
constexpr uint32_t SZ_PSLOT = V4_SF_BYTES + SZ_V4;             // [scales | codes]

// Shared memory and TMEM of the two QK^T formats. QK4: Q and K' as NVFP4 tile
// images ([scales | codes], 9 KB) instead of 16 KB E4M3 tiles; their scales
// take TMEM columns too, which one V ring stage fewer frees.
template <bool QK4>
struct Lay {
  static constexpr int KS = QK4 ? 4 : 3;  // K ring stages (the repair deltas take 32 KB of it)
  static constexpr int VS = QK4 ? 2 : 3;  // V ring stages
  static constexpr uint32_t SZ_QK = QK4 ? static_cast<uint32_t>(V4_TILE_BYTES) : SZ_TILE8;
  static constexpr uint32_t OFF_Q = 0;                      // Q_a, Q_b
  static constexpr uint32_t OFF_K = OFF_Q + 2 * SZ_QK;
  static constexpr uint32_t OFF_V = OFF_K + KS * SZ_QK;
  static constexpr uint32_t OFF_P = OFF_V + VS * SZ_VSTAGE;  // right after the V ring: a's repair P over both
  static constexpr uint32_t OFF_MU = OFF_P + 2 * SZ_PSLOT;   // one block-mean chunk; the repair's K rows later
  static constexpr uint32_t OFF_AR = OFF_MU + SZ_TILE8;      // restore A operands of a and b; b's repair P later
  static constexpr uint32_t OFF_LB = OFF_AR + 2 * SZ_TILE8;  // row-sum slots of a and b
  static constexpr uint32_t SMEM_USED = OFF_LB + 2 * 32 * 128 * 4;
  static constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // alignment slack
  static constexpr uint32_t TM_SFB = 416, TM_SFA = TM_SFB + 16 * VS, TM_QSF = TM_SFA + 32, TM_KSF = TM_QSF + 16;
  static_assert(SZ_QK % 1024 == 0 && SZ_VSTAGE % 1024 == 0 && SZ_PSLOT % 1024 == 0 && OFF_V % 1024 == 0 &&
                    OFF_P % 1024 == 0 && OFF_MU % 1024 == 0 && OFF_AR % 1024 == 0,
                "tile alignment");
  static_assert(VS * SZ_VSTAGE + 2 * SZ_PSLOT >= 2 * SZ_TILE8, "a's repair probabilities fit in the V ring and P slots");
  static_assert(KS * SZ_QK >= 2 * SZ_TILE8, "the repair deltas fit in the K ring");
  static_assert(SMEM_BYTES + 6144 <= 232448, "shared memory budget (dynamic + static)");
  static_assert(QK4 ? TM_KSF + 16 <= 512 : TM_SFA + 32 <= 512, "TMEM columns");
};

constexpr uint32_t TM_S = 0;
__device__ __forceinline__ constexpr uint32_t tm_o(int i) { return 128u + 144u * i; }  // O_i (+ row sums)
constexpr uint32_t IDESC_QK = idesc_make(0, 0, 128, 128, false, false);  // E4M3 x E4M3 -> f32, N = 128
constexpr uint32_t IDESC_QK4 = idesc_fp4_make(128, 128);                 // NVFP4 Q x NVFP4 K', N = 128
constexpr uint32_t IDESC_PV = idesc_fp4_make(128, 144);                  // NVFP4 P x NVFP4 [V | E], N = 144
constexpr uint32_t IDESC_BF = idesc_make(1, 1, 128, 128, false, false);  // bf16 x bf16 -> f32
constexpr float P_GLOBAL = 2688.0f;  // 6 * 448: block maximum -> E2M1 6 at scale 448

template <bool QK4>
struct Bars {
  static constexpr int KS = Lay<QK4>::KS, VS = Lay<QK4>::VS;
  uint64_t q, kfull[KS], kempty[KS], vfull[VS], vempty[VS], mufull, muempty;
  uint64_t sfull[2], sfree[2], pfull[2], pvdone[2], epi[2], rdone[2], repp[2];
  uint64_t main, repk, repdone, dt, fin;
};

__device__ __forceinline__ uint64_t desc128(const uint8_t *p) { return sdesc_sw128(smem_u32(p), 16, 1024); }

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two lanes of fma at once (one packed f32x2 instruction).
__device__ __forceinline__ float2 fma2(float a0, float a1, float b, float c) {
  float2 r;
  asm("{\n\t.reg .b64 a, b, c, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %4};\n\tmov.b64 c, {%5, %5};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
  return r;
}

// Two lanes of a product at once (one packed f32x2 instruction).
__device__ __forceinline__ float2 mul2(float a0, float a1, float b) {
  float2 r;
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %4};\n\t"
      "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a0), "f"(a1), "f"(b));
  return r;
}

// Eight values -> eight E2M1 codes (round to nearest even, saturating), value
// 2i in the low nibble of byte i. cvt...e2m1x2 puts its first source in the
// high nibble.
__device__ __forceinline__ uint32_t e2m1x8(const float *q) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
  return r;
}

// The E4M3 scale codes of the 8 key blocks of a row (bm: block maxima of the
// scores, -inf for a block without valid keys): sf = E4M3(fl(2^x_max * 448)).
__device__ __forceinline__ void p_scales(const float *bm, float al8, float nF8, uint32_t *sc) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a0 = ex2_approx(__fmaf_rn(bm[2 * i], al8, nF8));
    const float a1 = ex2_approx(__fmaf_rn(bm[2 * i + 1], al8, nF8));
    const uint32_t c2 = e4m3x2(__fmul_rn(a0, 448.0f), __fmul_rn(a1, 448.0f));
    sc[2 * i] = c2 & 0xFFu;
    sc[2 * i + 1] = (c2 >> 8) & 0xFFu;
  }
}

// 16 scores of one key block -> 8 bytes of E2M1 codes (w0: keys 0-7, w1: keys
// 8-15): code = E2M1(fl(2^x) * rcp), x = fma(acc, alpha/8, -F/8).
__device__ __forceinline__ void p_block(const float *s, float al8, float nF8, float rcp, uint32_t &w0,
                                        uint32_t &w1) {
  float q[16];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float2 x = fma2(s[2 * e], s[2 * e + 1], al8, nF8);
    const float2 pq = mul2(ex2_approx(x.x), ex2_approx(x.y), rcp);
    q[2 * e] = pq.x;
    q[2 * e + 1] = pq.y;
  }
  w0 = e2m1x8(q);
  w1 = e2m1x8(q + 8);
}

// The body of both kernels; QK4 selects the format of QK^T.
template <bool QK4>
__device__ __forceinline__ void attn4_body(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmMu,
                                           const CUtensorMap &tmDT, const AttnFp4Params &p) {
  using L = Lay<QK4>;
  constexpr int KS = L::KS, VS = L::VS;
  constexpr uint32_t SZ_QK = L::SZ_QK, TM_SFB = L::TM_SFB, TM_SFA = L::TM_SFA;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = sm + L::OFF_Q;
  uint8_t *sK = sm + L::OFF_K;
  uint8_t *sV = sm + L::OFF_V;
  uint8_t *sP = sm + L::OFF_P;
  uint8_t *sMu = sm + L::OFF_MU;
  uint8_t *sAr = sm + L::OFF_AR;
  float *sLb = reinterpret_cast<float *>(sm + L::OFF_LB);  // [2 query tiles][32 slots][128 rows]
  __shared__ Bars<QK4> bars;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ float s_vscale[128];
  __shared__ float s_skR[128];                    // sk of the repaired tokens' KV tiles
  __shared__ float s_rcp[128];                    // fl(2688 / value(code)) per E4M3 scale code
  __shared__ __align__(128) uint32_t s_esf[128];  // 512 bytes of E4M3 1.0: the scales of the E rows

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt0 = 2 * blockIdx.x, bh = blockIdx.y;
  const int T = p.Nb;
  const int nq = (qt0 + 1 < T) ? 2 : 1;  // query tiles of this CTA
  const int nrc = (p.R + 127) / 128;
  const int X_last = (T - 1) >> 5;       // the block-mean chunk restored after the loop

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(&bars.q, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(&bars.kfull[i], 1);
      mbar_init(&bars.kempty[i], 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(&bars.vfull[i], 1);
      mbar_init(&bars.vempty[i], 1);
    }
    mbar_init(&bars.mufull, 1);
    mbar_init(&bars.muempty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.sfull[i], 1);
      mbar_init(&bars.sfree[i], 4);
      mbar_init(&bars.pfull[i], 4);
      mbar_init(&bars.pvdone[i], 1);
      mbar_init(&bars.epi[i], 4);
      mbar_init(&bars.rdone[i], 1);
      mbar_init(&bars.repp[i], 4);
    }
    mbar_init(&bars.main, 2);  // one commit from each issuing warp
    mbar_init(&bars.repk, 4);
    mbar_init(&bars.repdone, 1);
    mbar_init(&bars.dt, 1);
    mbar_init(&bars.fin, 1);
    fence_mbar_init();
  }
  if (warp >= 3) {
    const int t = threadIdx.x - 96;  // 0..255
    // the E rows of every ring stage (16 rows x 64 bytes after the codes,
    // 64-byte swizzle): row 0 all E2M1 1.0 (0x22 = two ones), the others zero
    for (int i = t; i < VS * 64; i += 256) {
      const int s = i >> 6, rr = (i >> 2) & 15, ch = i & 3;
      const uint32_t v = rr == 0 ? 0x22222222u : 0u;
      *reinterpret_cast<uint4 *>(sV + s * SZ_VSTAGE + V4_SF_BYTES + SZ_V4 + sw64_off(rr, ch)) = make_uint4(v, v, v, v);
    }
    if (t < 128) {
      s_vscale[t] = p.vscale[static_cast<size_t>(bh) * 128 + t];
      s_esf[t] = 0x38383838u;  // E4M3 1.0
      // the P multiplier of scale code t; code 0 (and the NaN code 127, never
      // produced from a probability) give 0, so a block without a scale gets codes 0
      const float sfv = e4m3x2_value(static_cast<uint16_t>(t)).x;
      s_rcp[t] = (t == 0 || t == 127) ? 0.0f : __fdiv_rn(P_GLOBAL, sfv);
    }
    fence_proxy_async_smem();
  }
  if (warp == 1) tmem_alloc(&s_tmem, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  // One try_wait on the fast path; the abort flag (set by a warp whose wait
  // ran out) is read only when the phase is not complete yet.
  auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
    if (mbar_try_wait(smem_u32(bar), parity)) return true;
    if (s_abort) return false;
    if (!mbar_wait(bar, parity)) {
      s_abort = 1;
      atomicOr(p.status, ST_TIMEOUT);
      return false;
    }
    return true;
  };
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tmDT);
      mbar_arrive_expect_tx(&bars.q, nq * SZ_QK);
      if constexpr (QK4) {
        for (int i = 0; i < nq; ++i)
          bulk_load(sQ + i * SZ_QK, p.qimg + (static_cast<size_t>(bh) * T + qt0 + i) * SZ_QK, SZ_QK, &bars.q);
      } else {
        prefetch_tmap(&tmQ); prefetch_tmap(&tmK);
        for (int i = 0; i < nq; ++i)
          tma_load_2d(sQ + i * SZ_QK, &tmQ, &bars.q, 0, bh * p.Npad + (qt0 + i) * 128);
      }
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % KS;
        ok = wait(&bars.kempty[s], ((t / KS) & 1) ^ 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars.kfull[s], SZ_QK);
        if constexpr (QK4)
          bulk_load(sK + s * SZ_QK, p.kimg + (static_cast<size_t>(bh) * T + t) * SZ_QK, SZ_QK, &bars.kfull[s]);
        else
          tma_load_2d(sK + s * SZ_QK, &tmK, &bars.kfull[s], 0, bh * p.Npad + t * 128);
      }
      if (ok && nrc > 0) {
        ok = wait(&bars.main, 0);
        for (int rc = 0; rc < nrc && ok; ++rc) {
          if (rc > 0) ok = wait(&bars.repdone, (rc - 1) & 1);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars.dt, 2 * SZ_TILE8);
          tma_load_2d(sK, &tmDT, &bars.dt, rc * 128, bh * 128);
          tma_load_2d(sK + SZ_TILE8, &tmDT, &bars.dt, rc * 128 + 64, bh * 128);
        }
      }
    } else if (lane == 1) {
      const uint8_t *img = p.v4img + static_cast<size_t>(bh) * T * V4_TILE_BYTES;
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % VS;
        ok = wait(&bars.vempty[s], ((t / VS) & 1) ^ 1);
        if (!ok) break;
        // [scales | codes] of tile t in one copy; the E rows after them stay
        mbar_arrive_expect_tx(&bars.vfull[s], V4_TILE_BYTES);
        bulk_load(sV + s * SZ_VSTAGE, img + static_cast<size_t>(t) * V4_TILE_BYTES, V4_TILE_BYTES, &bars.vfull[s]);
      }
    } else if (lane == 2) {
      // block-mean chunk X is restored at KV tile 32X+32 (or after the loop);
      // the buffer is refilled once both query tiles' restores of X are done
      prefetch_tmap(&tmMu);
      bool ok = true;
      for (int X = 0; X <= X_last && ok; ++X) {
        if (X > 0) ok = wait(&bars.muempty, (X - 1) & 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars.mufull, SZ_TILE8);
        tma_load_2d(sMu, &tmMu, &bars.mufull, 0, (bh * p.nch32 + X) * 128);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    // Both warps run converged; descriptors are warp-uniform and each group of
    // tcgen05 instructions is issued by one elected lane.
    auto mwait = [&](uint64_t *bar, uint32_t parity) -> bool {
      const bool w = wait(bar, parity);
      return __all_sync(0xFFFFFFFFu, w);
    };
    const uint64_t dQ = desc128(sQ), dK = desc128(sK), dV = desc128(sV), dMu = desc128(sMu);
    const uint64_t dAr = desc128(sAr);
    constexpr uint64_t KSTEP = 32 >> 4, TSTEP = SZ_TILE8 >> 4;
    bool ok = true;
    if (warp == 2) {
      // S <- Q_i K^T in the order (a, t), (b, t), (a, t+1), ...: step k (k = t in
      // the loop, T + rc in the repair) of query tile i waits until the previous
      // product's warpgroup has read S out (sfree of that tile, its step)
      auto wait_s = [&](int i, int k) -> bool {
        if (i > 0) return mwait(&bars.sfree[i - 1], k & 1);
        return k == 0 || mwait(&bars.sfree[nq - 1], (k - 1) & 1);
      };
      // QK4: one product of step k for query tile i; the K' scales (from kimg
      // = the K' stage or the staged repair rows) go into slot k % 2 before
      // the first query tile's product of the step, Q_i's scales before its
      // first product (same thread: in issue order)
      auto qk4 = [&](int i, int k, const uint8_t *kimg) {
        const uint32_t ksf = tmem + L::TM_KSF + 8 * (k & 1), qsf = tmem + L::TM_QSF + 8 * i;
        if (k == 0) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) tmem_cp_sf(qsf + 4 * kk, sdesc_sf(smem_u32(sQ + i * SZ_QK + 512 * kk)));
        }
        if (i == 0) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) tmem_cp_sf(ksf + 4 * kk, sdesc_sf(smem_u32(kimg + 512 * kk)));
        }
        const uint64_t dq = sdesc_sw64(smem_u32(sQ + i * SZ_QK + V4_SF_BYTES)),
                       dk = sdesc_sw64(smem_u32(kimg + V4_SF_BYTES));
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_fp4_ss(tmem + TM_S, dq + 2 * kk, dk + 2 * kk, IDESC_QK4, qsf + 4 * kk, ksf + 4 * kk, kk > 0);
      };
      ok = mwait(&bars.q, 0);
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % KS;
        ok = mwait(&bars.kfull[s], (t / KS) & 1);
        for (int i = 0; i < nq && ok; ++i) {
          ok = wait_s(i, t);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            if constexpr (QK4) {
              qk4(i, t, sK + s * SZ_QK);
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_f8_ss(tmem + TM_S, dQ + TSTEP * i + KSTEP * kk, dK + TSTEP * s + KSTEP * kk, IDESC_QK, kk > 0);
            }
            mma_commit(&bars.sfull[i]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) mma_commit(&bars.kempty[s]);
        __syncwarp();
      }
      if (ok && elect_one()) mma_commit(&bars.main);
      __syncwarp();
      // repair scores S <- Q_i K_R^T, K_R staged by warpgroup a over the block-mean buffer
      for (int rc = 0; rc < nrc && ok; ++rc) {
        ok = mwait(&bars.repk, rc & 1);
        for (int i = 0; i < nq && ok; ++i) {
          ok = wait_s(i, T + rc);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            if constexpr (QK4) {
              qk4(i, T + rc, sMu);
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_f8_ss(tmem + TM_S, dQ + TSTEP * i + KSTEP * kk, dMu + KSTEP * kk, IDESC_QK, kk > 0);
            }
            mma_commit(&bars.sfull[i]);
          }
          __syncwarp();
        }
      }
    } else {
      // the scale column of the E rows (column +4 of every K step of every
      // stage) never changes: copied once, before the first product
      if (elect_one()) {
        const uint64_t de = sdesc_sf(smem_u32(s_esf));
#pragma unroll
        for (int s = 0; s < VS; ++s)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) tmem_cp_sf(tmem + TM_SFB + 16 * s + 8 * kk + 4, de);
      }
      __syncwarp();
      auto restore = [&](int i) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16_ss(tmem + tm_o(i), dAr + TSTEP * i + KSTEP * kk, dMu + KSTEP * kk, IDESC_BF, 1);
      };
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % VS;
        ok = mwait(&bars.vfull[s], (t / VS) & 1);
        // chunk X = t/32 - 1 is restored right before PV(t): its row sums were
        // written by the warpgroup in the frame of tile t, which O has after
        // the warpgroup's rescale for tile t (done before pfull(t))
        const bool rst = t >= 32 && (t & 31) == 0;
        if (ok && rst) ok = mwait(&bars.mufull, ((t >> 5) - 1) & 1);
        const uint8_t *vst = sV + s * SZ_VSTAGE;
        const uint32_t sfb = tmem + TM_SFB + 16 * s;
        for (int i = 0; i < nq && ok; ++i) {
          ok = mwait(&bars.pfull[i], t & 1);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            if (rst) {
              restore(i);
              if (i == nq - 1) mma_commit(&bars.muempty);
            }
            // the V stage's scales (once per tile) and P_i's, then the two
            // K = 64 products; a copy and the products after it run in issue order
            const uint8_t *pst = sP + i * SZ_PSLOT;
            const uint32_t sfa = tmem + TM_SFA + 16 * i + 8 * (t & 1);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              if (i == 0) tmem_cp_sf(sfb + 8 * kk, sdesc_sf(smem_u32(vst + 512 * kk)));
              tmem_cp_sf(sfa + 4 * kk, sdesc_sf(smem_u32(pst + 512 * kk)));
            }
            const uint64_t da = sdesc_sw64(smem_u32(pst + V4_SF_BYTES));
            const uint64_t db = sdesc_sw64(smem_u32(vst + V4_SF_BYTES));
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)  // a K step of 64 E2M1 values is 32 bytes: +2 in the address field
              mma_fp4_ss(tmem + tm_o(i), da + 2 * kk, db + 2 * kk, IDESC_PV, sfa + 4 * kk, sfb + 8 * kk,
                         (t > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&bars.pvdone[i]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) mma_commit(&bars.vempty[s]);
        __syncwarp();
      }
      if (ok && elect_one()) mma_commit(&bars.main);
      __syncwarp();
      // the last chunk, after the loop
      if (ok) ok = mwait(&bars.mufull, X_last & 1);
      for (int i = 0; i < nq && ok; ++i) {
        ok = mwait(&bars.epi[i], 0);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          restore(i);
          mma_commit(&bars.rdone[i]);
        }
        __syncwarp();
      }
      // repair: O_i += P_R,i (bf16) x (delta/g) (bf16); a's probabilities over
      // the V ring and P slots, b's over the restore operands
      for (int rc = 0; rc < nrc && ok; ++rc) {
        ok = mwait(&bars.dt, rc & 1);
        for (int i = 0; i < nq && ok; ++i) {
          ok = mwait(&bars.repp[i], rc & 1);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            const uint64_t dPr = i == 0 ? dV : dAr;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_f16_ss(tmem + tm_o(i), dPr + TSTEP * (kk >> 2) + KSTEP * (kk & 3),
                         dK + TSTEP * (kk >> 2) + KSTEP * (kk & 3), IDESC_BF, 1);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) mma_commit(&bars.repdone);
        __syncwarp();
      }
      if (ok && elect_one()) mma_commit(&bars.fin);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax rows
    // Warpgroup g (warps 3+4g .. 6+4g) owns query tile g of the pair; thread
    // row r = 32*(warp%4) + lane. Its row sums: lt (the tiles read so far) and
    // the slots of the current block-mean chunk, both in the frame F of its
    // latest tile; l_u is read at tile u+1, once PV(u) is complete.
    const int g = (warp - 3) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const bool active = g < nq;
    const uint32_t lrow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);  // this warp's lanes
    const int qt = qt0 + g;
    const float sqs = active ? p.sq[static_cast<size_t>(bh) * T + qt] : 0.0f;
    const float *skh = p.sk + static_cast<size_t>(bh) * T;
    float *lb = sLb + g * 32 * 128;       // [32 slots][128 rows]
    uint8_t *ar = sAr + g * SZ_TILE8;     // restore A operand
    uint8_t *pslot = sP + g * SZ_PSLOT;   // P_g
    const int tail = p.N - (T - 1) * 128;  // valid keys in the last tile
    bool ok = active;
    float F = -INFINITY;  // frame of the latest tile
    float lt = 0.0f;      // sum of the l_u read so far, frame F
    float lprev = 0.0f;   // last value read from the row-sum column
    auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
      const bool w = wait(bar, parity);
      return __all_sync(0xFFFFFFFFu, w);
    };
    // A operand of the restore MMA: row r = [hi(l_0..l_31) | lo(l_0..l_31)] in
    // bf16, the chunk's slots times sc (into the frame O will be in)
    auto flush = [&](int nvalid, float sc) {
      uint32_t hw[16], lw[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float l0 = (2 * i < nvalid) ? lb[(2 * i) * 128 + r] * sc : 0.0f;
        const float l1 = (2 * i + 1 < nvalid) ? lb[(2 * i + 1) * 128 + r] * sc : 0.0f;
        const __nv_bfloat16 h0 = __float2bfloat16_rn(l0), h1 = __float2bfloat16_rn(l1);
        const __nv_bfloat16 o0 = __float2bfloat16_rn(__fsub_rn(l0, __bfloat162float(h0)));
        const __nv_bfloat16 o1 = __float2bfloat16_rn(__fsub_rn(l1, __bfloat162float(h1)));
        hw[i] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
        lw[i] = static_cast<uint32_t>(__bfloat16_as_ushort(o0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(o1)) << 16);
      }
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        *reinterpret_cast<uint4 *>(ar + sw128_off(r, ch)) =
            make_uint4(hw[4 * ch], hw[4 * ch + 1], hw[4 * ch + 2], hw[4 * ch + 3]);
        *reinterpret_cast<uint4 *>(ar + sw128_off(r, ch + 4)) =
            make_uint4(lw[4 * ch], lw[4 * ch + 1], lw[4 * ch + 2], lw[4 * ch + 3]);
      }
    };
    // l_u = what PV(u) added to the row-sum column (PV(u) complete), into
    // chunk slot u % 32 and lt, both in frame F = F_u
    auto read_l = [&](int u) -> bool {
      if (!wwait(&bars.pvdone[g], u & 1)) return false;
      tc_fence_after();
      const float v = __uint_as_float(tmem_ld1(lrow + tm_o(g) + 128));
      tmem_wait_ld();
      const float l = __fsub_rn(v, lprev);
      lprev = v;
      lb[(u & 31) * 128 + r] = l;
      lt += l;
      return true;
    };

    // One KV tile t of this warpgroup's query tile. LAST: the ragged last tile.
    auto tile = [&](int t, auto last_tag) -> bool {
      constexpr bool LAST = decltype(last_tag)::value;
      const float skt = skh[t];
      if (!wwait(&bars.sfull[g], t & 1)) return false;
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int i = 0; i < 4; ++i) tmem_ld32(lrow + TM_S + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * i]));
      tmem_wait_ld();
      tc_fence_before();
      warp_arrive(&bars.sfree[g]);  // S may now take the other query tile's scores
      float s[128];
#pragma unroll
      for (int j = 0; j < 128; ++j) s[j] = __uint_as_float(sr[j]);
      if constexpr (LAST) {
#pragma unroll
        for (int j = 0; j < 128; ++j)
          if (j >= tail) s[j] = -INFINITY;
      }
      // the maxima of the 8 key blocks, then of the row
      float bm[8];
#pragma unroll
      for (int kb = 0; kb < 8; ++kb) {
        const float *x = &s[16 * kb];
        const float m0 = max3(x[0], x[1], x[2]), m1 = max3(x[3], x[4], x[5]), m2 = max3(x[6], x[7], x[8]);
        const float m3 = max3(x[9], x[10], x[11]), m4 = max3(x[12], x[13], x[14]);
        bm[kb] = max3(max3(m0, m1, m2), max3(m3, m4, x[15]), -INFINITY);
      }
      const float mx = max3(max3(bm[0], bm[1], bm[2]), max3(bm[3], bm[4], bm[5]), fmaxf(bm[6], bm[7]));
      const float alpha = __fmul_rn(__fmul_rn(sqs, skt), p.kappa);
      // F_t = max(F_{t-1}, 8 ceil(m_t / 8)): 8 ceil(running max / 8)
      const float Fn = fmaxf(F, 8.0f * ceilf(__fmul_rn(mx, alpha) * 0.125f));
      const bool need = t > 0 && Fn != F;
      const float sc = need ? frame_scale(F, Fn) : 1.0f;
      // NVFP4 probabilities against the frame Fn: the row's 64 bytes of codes
      // and its 8 scale bytes, in registers until P_g is free
      uint32_t cw[16], scw[2] = {0u, 0u};
      {
        const float al8 = __fmul_rn(alpha, 0.125f), nF8 = -Fn * 0.125f;
        uint32_t scb[8];
        p_scales(bm, al8, nF8, scb);
        if constexpr (LAST) {
#pragma unroll
          for (int kb = 0; kb < 8; ++kb)
            if (16 * kb >= tail) scb[kb] = 0u;  // no valid key: scale 0, codes 0
        }
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) scw[kb >> 2] |= scb[kb] << (8 * (kb & 3));
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) {
          p_block(&s[16 * kb], al8, nF8, s_rcp[scb[kb]], cw[2 * kb], cw[2 * kb + 1]);
          if constexpr (LAST) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              uint32_t keep = 0u;
#pragma unroll
              for (int e = 0; e < 8; ++e)
                if (16 * kb + 8 * q + e < tail) keep |= 0xFu << (4 * e);
              cw[2 * kb + q] &= keep;
            }
          }
        }
      }
      // PV(t-1) complete: P_g is free, O_g stable, and l_{t-1} can be read
      int nfill = 0;  // slots of the current chunk filled (frame F)
      if (t > 0) {
        if (!read_l(t - 1)) return false;
        nfill = ((t - 1) & 31) + 1;
        if (nfill == 32) {
          // chunk t/32 - 1 is complete: its row sums in frame Fn (O's frame
          // when the restore runs, right before PV(t))
          flush(32, sc);
          nfill = 0;
        }
      }
      // the codes (64-byte swizzle) and scale bytes into P_g
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
        *reinterpret_cast<uint4 *>(pslot + V4_SF_BYTES + sw64_off(r, ch)) =
            make_uint4(cw[4 * ch], cw[4 * ch + 1], cw[4 * ch + 2], cw[4 * ch + 3]);
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) *reinterpret_cast<uint32_t *>(pslot + v4_sf_off(r, 4 * kk)) = scw[kk];
      fence_proxy_async_smem();  // P_g and the restore operand are read by tcgen05.cp / the MMAs
      if (__any_sync(0xFFFFFFFFu, need)) {
        uint32_t o[128];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          tmem_ld32(lrow + tm_o(g) + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(&o[32 * i]));
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 128; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * sc);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          tmem_st32(lrow + tm_o(g) + 32 * i, *reinterpret_cast<const uint32_t(*)[32]>(&o[32 * i]));
        tmem_wait_st();
      }
      tc_fence_before();
      warp_arrive(&bars.pfull[g]);
      if (need) {
        lt *= sc;
        for (int i = 0; i < nfill; ++i) lb[i * 128 + r] *= sc;
      }
      F = Fn;
      return true;
    };

    const bool ragged = tail < 128;
    for (int t = 0; t < T - 1 && ok; ++t) ok = tile(t, std::false_type{});
    if (ok) ok = ragged ? tile(T - 1, std::true_type{}) : tile(T - 1, std::false_type{});
    if (ok) ok = read_l(T - 1);
    if (ok) {
      // the last chunk (tiles 32*X_last .. T-1), in frame F: restored after the loop
      flush(T - 32 * X_last, 1.0f);
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&bars.epi[g]);
      ok = wwait(&bars.rdone[g], 0);
    }

    // ---------------------------------------------------------- repair
    // Both final restores are complete once every softmax thread passes this
    // barrier: the block-mean buffer takes the repaired tokens' K rows (staged
    // by warpgroup a), a's bf16 probabilities go over the V ring and P slots,
    // b's over the restore operands. Every softmax thread takes the same
    // barriers on every path. P' = bf16(fl(2^x' * 2688)), x' = fma(acc,
    // alpha/8, -F/8): the unquantized probability of the repaired token in the
    // final frame, in the units of the NVFP4 products.
    softmax_bar256();
    const float nF8fin = -F * 0.125f;
    uint8_t *prep = g == 0 ? sV : sAr;
    for (int rc = 0; rc < nrc; ++rc) {
      if (ok && rc > 0) ok = wwait(&bars.repdone, (rc - 1) & 1);
      if (g == 0 && active) {
        const int i = rc * 128 + r;
        float skr = 0.0f;
        if constexpr (QK4) {
          // row pos % 128 of K' tile pos / 128: 64 bytes of codes and 8 scale
          // bytes, staged as row r of an image (rows past R: codes and scales 0)
          uint4 krow[4];
          uint32_t ksc[2] = {0u, 0u};
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) krow[ch] = make_uint4(0u, 0u, 0u, 0u);
          if (i < p.R) {
            const int pos = p.rep_idx[static_cast<size_t>(bh) * p.R + i];
            const uint8_t *img = p.kimg + (static_cast<size_t>(bh) * T + (pos >> 7)) * SZ_QK;
            const int rr = pos & 127;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
              krow[ch] = *reinterpret_cast<const uint4 *>(img + V4_SF_BYTES + sw64_off(rr, ch));
#pragma unroll
            for (int h = 0; h < 2; ++h) ksc[h] = *reinterpret_cast<const uint32_t *>(img + v4_sf_off(rr, 4 * h));
            skr = skh[pos >> 7];
          }
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) *reinterpret_cast<uint4 *>(sMu + V4_SF_BYTES + sw64_off(r, ch)) = krow[ch];
#pragma unroll
          for (int h = 0; h < 2; ++h) *reinterpret_cast<uint32_t *>(sMu + v4_sf_off(r, 4 * h)) = ksc[h];
        } else {
          uint4 krow[8];
          if (i < p.R) {
            const int pos = p.rep_idx[static_cast<size_t>(bh) * p.R + i];
            const uint4 *src = reinterpret_cast<const uint4 *>(p.k8 + (static_cast<size_t>(bh) * p.Npad + pos) * 128);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) krow[ch] = src[ch];
            skr = skh[pos >> 7];
          } else {
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) krow[ch] = make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4 *>(sMu + sw128_off(r, ch)) = krow[ch];
        }
        s_skR[r] = skr;
        fence_proxy_async_smem();
        tc_fence_before();
        warp_arrive(&bars.repk);
      }
      softmax_bar256();  // s_skR visible to both warpgroups
      if (!(ok && active)) continue;
      ok = wwait(&bars.sfull[g], (T + rc) & 1);
      if (!ok) continue;
      tc_fence_after();
      uint32_t sv[128];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(lrow + TM_S + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * q]));
      tmem_wait_ld();
      tc_fence_before();
      warp_arrive(&bars.sfree[g]);
      const int nval = min(128, p.R - rc * 128);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t *v = &sv[32 * q];
#pragma unroll
        for (int gg = 0; gg < 4; ++gg) {
          uint32_t outw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 32 * q + 8 * gg + 2 * e;
            const float a0 = __fmul_rn(__fmul_rn(__fmul_rn(sqs, s_skR[j]), p.kappa), 0.125f);
            const float a1 = __fmul_rn(__fmul_rn(__fmul_rn(sqs, s_skR[j + 1]), p.kappa), 0.125f);
            float p0 = __fmul_rn(ex2_approx(__fmaf_rn(__uint_as_float(v[8 * gg + 2 * e]), a0, nF8fin)), P_GLOBAL);
            float p1 = __fmul_rn(ex2_approx(__fmaf_rn(__uint_as_float(v[8 * gg + 2 * e + 1]), a1, nF8fin)), P_GLOBAL);
            if (j >= nval) p0 = 0.0f;
            if (j + 1 >= nval) p1 = 0.0f;
            const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
            outw[e] = *reinterpret_cast<const uint32_t *>(&pb);
          }
          const int jj = 32 * q + 8 * gg;  // first key of this 16-byte chunk
          *reinterpret_cast<uint4 *>(prep + (jj >> 6) * SZ_TILE8 + sw128_off(r, (jj & 63) >> 3)) =
              make_uint4(outw[0], outw[1], outw[2], outw[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&bars.repp[g]);
    }
    // ---------------------------------------------------------- epilogue
    if (ok) ok = wwait(&bars.fin, 0);
    if (ok) {
      tc_fence_after();
      // every product is complete: a stages over the K ring, b over the
      // restore operands
      const int row0 = qt * 128 + q4 * 32;
      uint8_t *stg = (g == 0 ? sK : sAr) + q4 * 32 * 256;
      store_o_rows(lrow + tm_o(g), s_vscale, lt, stg, p.O + (static_cast<size_t>(bh) * p.N + row0) * 128,
                   p.N - row0);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

__global__ void __launch_bounds__(352, 1)
    k_vc_attn_fwd4(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmMu, const __grid_constant__ CUtensorMap tmDT,
                   const AttnFp4Params p) {
  attn4_body<false>(tmQ, tmK, tmMu, tmDT, p);
}

__global__ void __launch_bounds__(352, 1)
    k_vc_attn_fwd44(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmMu, const __grid_constant__ CUtensorMap tmDT,
                    const AttnFp4Params p) {
  attn4_body<true>(tmQ, tmK, tmMu, tmDT, p);
}

uint32_t attn_fp4_smem_bytes(bool qk4) { return qk4 ? Lay<true>::SMEM_BYTES : Lay<false>::SMEM_BYTES; }

}  // namespace vc
