// attn_fp4.cu - the fused attention kernel of the NVFP4-residual variant, sm_100a.
//
// Page "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58× sem
// retreinamento": "V-Smooth: corrigindo outliers de valor", item Demean (the
// value residual quantized to NVFP4 for the 4-bit kernel) and item Restore
// (the block means come back through the online softmax's row sums);
// "ExpCast-FP8: eliminando o gargalo do softmax": ExpCast is 8-bit only, so
// here the probabilities come from an exp2 softmax and are quantized to NVFP4
// per 16 keys. QK^T stays FP8. Page "VC-Attention et FLUX 3 accélèrent la
// génération d'images sur Blackwell", "Le compromis entre vitesse et
// fidélité": repair of the worst tokens.
//
// One CTA per (128-query tile, b*h), 11 warps; the two softmax warpgroups
// take the KV tiles of that query tile in turn and hand the running frame from
// tile to tile:
//   warp 0     lane 0: Q, the K8 tiles (4-stage ring), then the repair deltas;
//              lane 1: the NVFP4 V tile images (scales + codes, one 9 KB bulk
//              copy per tile, 4-stage ring) and the block-mean chunks.
//   warp 1     allocates TMEM; copies the scale factors into TMEM and issues
//              PV (kind::mxf4nvf4, 16-element E4M3 scales), the block-mean
//              restores and the repair products.
//   warp 2     issues QK^T (FP8).
//   warps 3-10 two softmax warpgroups taking the KV tiles in turn, one thread
//              per query row.
// What is specific to the 4-bit products:
//   - P lives in shared memory: the block-scaled FP4 MMA reads both operands
//     from there. Three slots of [1 KB scales | 8 KB codes]; the PV warp copies
//     a slot's scales into TMEM (tcgen05.cp) right before the product.
//   - Each softmax thread turns its row's 128 scores into 8 blocks of 16:
//     x = fma(acc, alpha/8, -F/8), p = 2^x, block scale sf = E4M3(448 * max p),
//     codes E2M1(p * fl(2688 / sf)), the multipliers from a 128-entry table.
//   - PV is one N = 144 product: B = the V tile's 128 channel rows plus 16 rows
//     E holding one row of ones (E2M1 1.0, scale 1.0) at row s in ring stage s,
//     so the row sum l_t (sum of value(code) * sf over the tile, 2688 x the
//     dequantized probabilities) lands in accumulator column 128 + t % 4, and
//     every PV adds exact zeros to the other three.
//   - The full 4-bit path (QK4) takes Q and K' as NVFP4 tile images of the
//     same layout (rows = tokens, the K dimension = channels): QK^T is two
//     K = 64 steps of kind::mxf4nvf4, the Q tile's scales copied into TMEM
//     once, each K' tile's into one of two slots right before its product.
// TMEM (512 columns x 128 lanes): S double buffer [0,256); O [256,384); row
// sums [384,388) (the N = 144 accumulator spans [256,400)); V scales of ring
// stage s at 400 + 16 s (+8 per K step; column +4 holds the constant scale of
// E); P scales of slot i at 464 + 8 i (+4 per K step); QK4: Q scales at 488,
// K' scales of slot j at 496 + 8 j (+4 per K step).
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
constexpr int NPSLOT = 3;

// Shared memory and TMEM of the two QK^T formats. QK4: Q and K' as NVFP4 tile
// images ([scales | codes], 9 KB) instead of 16 KB E4M3 tiles; their scales
// take the last 24 TMEM columns.
template <bool QK4>
struct Lay {
  static constexpr int KS = 4;  // K ring stages
  static constexpr int VS = 4;  // V ring stages: stage t % 4 holds the ones row of row-sum column t % 4
  static constexpr uint32_t SZ_QK = QK4 ? static_cast<uint32_t>(V4_TILE_BYTES) : SZ_TILE8;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + SZ_QK;
  static constexpr uint32_t OFF_V = OFF_K + KS * SZ_QK;
  static constexpr uint32_t OFF_P = OFF_V + VS * SZ_VSTAGE;  // right after the V ring: the repair reuses both
  static constexpr uint32_t OFF_AR = OFF_P + NPSLOT * SZ_PSLOT;
  static constexpr uint32_t OFF_MU = OFF_AR + SZ_TILE8;
  static constexpr uint32_t OFF_LB = OFF_MU + 2 * SZ_TILE8;
  static constexpr uint32_t SMEM_USED = OFF_LB + 32 * 128 * 4;
  static constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // alignment slack
  // TMEM columns: S [0,256), O and row sums [256,400), V scales 16 per stage,
  // P scales 8 per slot, then (QK4) Q scales 8 and K scales 8 per slot (2)
  static constexpr uint32_t TM_SFB = 400, TM_SFA = TM_SFB + 16 * VS, TM_QSF = TM_SFA + 8 * NPSLOT,
                            TM_KSF = TM_QSF + 8;
  static_assert(SZ_QK % 1024 == 0 && SZ_VSTAGE % 1024 == 0 && SZ_PSLOT % 1024 == 0 && OFF_V % 1024 == 0 &&
                    OFF_P % 1024 == 0 && OFF_AR % 1024 == 0 && OFF_MU % 1024 == 0,
                "tile alignment");
  // repair staging: K rows (16 KB FP8 tile or 9 KB image) then 32 KB of bf16 P at +16 KB
  static_assert(VS * SZ_VSTAGE + NPSLOT * SZ_PSLOT >= 3 * SZ_TILE8, "repair staging fits in the V ring and P slots");
  static_assert(KS * SZ_QK >= 2 * SZ_TILE8, "the repair deltas fit in the K ring");
  static_assert(SMEM_BYTES + 8192 <= 232448, "shared memory budget (dynamic + static)");
  static_assert(!QK4 || TM_KSF + 16 <= 512, "TMEM columns");
  static_assert(QK4 || TM_SFA + 8 * NPSLOT <= 512, "TMEM columns");
};

constexpr uint32_t TM_S0 = 0, TM_O = 256, TM_L = 384;
constexpr int NPD = 8;  // PV completion barriers, indexed t % 8
__device__ __forceinline__ uint32_t lcol_of(int t) { return TM_L + (t & 3); }
constexpr uint32_t IDESC_QK = idesc_make(0, 0, 128, 128, false, false);  // E4M3 x E4M3 -> f32, N = 128
constexpr uint32_t IDESC_QK4 = idesc_fp4_make(128, 128);                 // NVFP4 Q x NVFP4 K', N = 128
constexpr uint32_t IDESC_PV = idesc_fp4_make(128, 144);                  // NVFP4 P x NVFP4 [V | E], N = 144
constexpr uint32_t IDESC_BF = idesc_make(1, 1, 128, 128, false, false);  // bf16 x bf16 -> f32
constexpr float P_GLOBAL = 2688.0f;  // 6 * 448: block maximum -> E2M1 6 at scale 448

template <bool QK4>
struct Bars {
  static constexpr int KS = Lay<QK4>::KS, VS = Lay<QK4>::VS;
  uint64_t q, kfull[KS], kempty[KS], vfull[VS], vempty[VS], mufull[2], muempty[2];
  uint64_t sfull[2], sfree[2], pfull[4], mxr[2], pvdone[NPD], bk, lflush, wgdone, main, epi, rdone, repk, reps,
      repp, repdone, dt, fin;
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
  constexpr uint32_t OFF_Q = L::OFF_Q, OFF_K = L::OFF_K, OFF_V = L::OFF_V, OFF_P = L::OFF_P, OFF_AR = L::OFF_AR,
                     OFF_MU = L::OFF_MU, OFF_LB = L::OFF_LB;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = sm + OFF_Q;
  uint8_t *sK = sm + OFF_K;
  uint8_t *sV = sm + OFF_V;
  uint8_t *sP = sm + OFF_P;
  uint8_t *sAr = sm + OFF_AR;
  uint8_t *sMu = sm + OFF_MU;
  float *sLb = reinterpret_cast<float *>(sm + OFF_LB);  // [32 slots][128 rows]
  __shared__ Bars<QK4> bars;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ float s_vscale[128];
  __shared__ float s_alphaR[128];
  __shared__ float s_F[128], s_ltot[128], s_lto[128], s_lprev[2][128];
  __shared__ float s_rcp[128];                            // fl(2688 / value(code)) per E4M3 scale code
  __shared__ __align__(128) uint32_t s_esf[128];          // 512 bytes of E4M3 1.0: the scales of the E rows

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, bh = blockIdx.y;
  const int T = p.Nb;
  const int nrc = (p.R + 127) / 128;
  const int X_epi0 = first_epilogue_chunk(T), X_epi1 = (T - 1) >> 5;

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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.mufull[i], 1); mbar_init(&bars.muempty[i], 1);
      mbar_init(&bars.sfull[i], 1); mbar_init(&bars.sfree[i], 4);
      mbar_init(&bars.mxr[i], 4);
    }
    for (int i = 0; i < NPD; ++i) mbar_init(&bars.pvdone[i], 1);
    // pfull is indexed t % 4: before a warpgroup arrives for tile t+4, its
    // bookkeeping of tile t+2 has waited for PV(t+1), so the issuer has already
    // consumed pfull(t); a barrier never runs two phases ahead of its waiter
    for (int i = 0; i < 4; ++i) mbar_init(&bars.pfull[i], 4);
    mbar_init(&bars.bk, 4); mbar_init(&bars.lflush, 4); mbar_init(&bars.wgdone, 4);
    mbar_init(&bars.main, 2);  // one commit from each issuing warp
    mbar_init(&bars.epi, 4); mbar_init(&bars.rdone, 1);
    mbar_init(&bars.repk, 4); mbar_init(&bars.reps, 1); mbar_init(&bars.repp, 4);
    mbar_init(&bars.repdone, 1); mbar_init(&bars.dt, 1); mbar_init(&bars.fin, 1);
    fence_mbar_init();
  }
  if (warp >= 3) {
    const int t = threadIdx.x - 96;  // 0..255
    // the E rows of the four ring stages (16 rows x 64 bytes after the codes,
    // 64-byte swizzle): zero except row s of stage s, all E2M1 1.0 (0x22 = two ones)
    for (int i = t; i < VS * 64; i += 256) {
      const int s = i >> 6, rr = (i >> 2) & 15, ch = i & 3;
      const uint32_t v = rr == s ? 0x22222222u : 0u;
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
      prefetch_tmap(&tmQ); prefetch_tmap(&tmK); prefetch_tmap(&tmDT);
      if constexpr (QK4) {
        mbar_arrive_expect_tx(&bars.q, SZ_QK);
        bulk_load(sQ, p.qimg + (static_cast<size_t>(bh) * T + qt) * SZ_QK, SZ_QK, &bars.q);
      } else {
        mbar_arrive_expect_tx(&bars.q, SZ_QK);
        tma_load_2d(sQ, &tmQ, &bars.q, 0, bh * p.Npad + qt * 128);
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
      prefetch_tmap(&tmMu);
      const uint8_t *img = p.v4img + static_cast<size_t>(bh) * T * V4_TILE_BYTES;
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        if ((t & 31) == 0) {
          const int X = t >> 5, s = X & 1;
          ok = wait(&bars.muempty[s], ((X >> 1) & 1) ^ 1);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars.mufull[s], SZ_TILE8);
          tma_load_2d(sMu + s * SZ_TILE8, &tmMu, &bars.mufull[s], 0, (bh * p.nch32 + X) * 128);
        }
        const int s = t % VS;
        ok = wait(&bars.vempty[s], ((t / VS) & 1) ^ 1);
        if (!ok) break;
        // [scales | codes] of tile t in one copy; the E rows after them stay
        mbar_arrive_expect_tx(&bars.vfull[s], V4_TILE_BYTES);
        bulk_load(sV + s * SZ_VSTAGE, img + static_cast<size_t>(t) * V4_TILE_BYTES, V4_TILE_BYTES, &bars.vfull[s]);
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
    const uint64_t dQ = desc128(sQ), dK = desc128(sK);
    const uint64_t dR = desc128(sV);  // the repair's staging (K rows, then bf16 P) over the V ring and P slots
    const uint64_t dAr = desc128(sAr), dMu = desc128(sMu);
    constexpr uint64_t KSTEP = 32 >> 4, TSTEP = SZ_TILE8 >> 4;
    bool ok = true;
    if (warp == 2) {
      // S(t) = Q8 K8(t)^T into S buffer t%2, once the warpgroup of tile t-2
      // has read S(t-2) out of it
      ok = mwait(&bars.q, 0);
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % KS;
        if (t >= 2) ok = mwait(&bars.sfree[t & 1], ((t - 2) >> 1) & 1);
        ok = ok && mwait(&bars.kfull[s], (t / KS) & 1);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t d = tmem + TM_S0 + (t & 1) * 128;
          if constexpr (QK4) {
            // K scales into slot t%2: its previous reader, QK(t-2), completed
            // before S(t-2) was read out (the sfree wait above)
            const uint8_t *kst = sK + s * SZ_QK;
            const uint32_t ksf = tmem + L::TM_KSF + 8 * (t & 1);
            if (t == 0) {  // the Q tile's scales, read by every QK^T of this CTA (same thread: in issue order)
#pragma unroll
              for (int kk = 0; kk < 2; ++kk) tmem_cp_sf(tmem + L::TM_QSF + 4 * kk, sdesc_sf(smem_u32(sQ + 512 * kk)));
            }
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) tmem_cp_sf(ksf + 4 * kk, sdesc_sf(smem_u32(kst + 512 * kk)));
            const uint64_t dq = sdesc_sw64(smem_u32(sQ + V4_SF_BYTES)), dk = sdesc_sw64(smem_u32(kst + V4_SF_BYTES));
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              mma_fp4_ss(d, dq + 2 * kk, dk + 2 * kk, IDESC_QK4, tmem + L::TM_QSF + 4 * kk, ksf + 4 * kk, kk > 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f8_ss(d, dQ + KSTEP * kk, dK + TSTEP * s + KSTEP * kk, IDESC_QK, kk > 0);
          }
          mma_commit(&bars.kempty[s]);
          mma_commit(&bars.sfull[t & 1]);
        }
        __syncwarp();
      }
      if (ok && elect_one()) mma_commit(&bars.main);
      __syncwarp();
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
      auto issue_restore = [&](int X) -> bool {
        const int s = X & 1;
        if (!mwait(&bars.mufull[s], (X >> 1) & 1)) return false;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ss(tmem + TM_O, dAr + KSTEP * kk, dMu + TSTEP * s + KSTEP * kk, IDESC_BF, 1);
          mma_commit(&bars.muempty[s]);
        }
        __syncwarp();
        return true;
      };
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % VS, slot = t % NPSLOT;
        ok = mwait(&bars.vfull[s], (t / VS) & 1);
        if (!ok) break;
        ok = mwait(&bars.pfull[t & 3], (t >> 2) & 1);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          // scales of V(t) and P(t) into TMEM, then the two K = 64 products;
          // a copy and the products after it run in issue order
          const uint8_t *vst = sV + s * SZ_VSTAGE, *pst = sP + slot * SZ_PSLOT;
          const uint32_t sfb = tmem + TM_SFB + 16 * s, sfa = tmem + TM_SFA + 8 * slot;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            tmem_cp_sf(sfb + 8 * kk, sdesc_sf(smem_u32(vst + 512 * kk)));
            tmem_cp_sf(sfa + 4 * kk, sdesc_sf(smem_u32(pst + 512 * kk)));
          }
          const uint64_t da = sdesc_sw64(smem_u32(pst + V4_SF_BYTES));
          const uint64_t db = sdesc_sw64(smem_u32(vst + V4_SF_BYTES));
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)  // a K step of 64 E2M1 values is 32 bytes: +2 in the address field
            mma_fp4_ss(tmem + TM_O, da + 2 * kk, db + 2 * kk, IDESC_PV, sfa + 4 * kk, sfb + 8 * kk,
                       (t > 0 || kk > 0) ? 1u : 0u);
        }
        __syncwarp();
        // block means of chunk X = (t-33)/32: their row sums were staged by the
        // tail of tile t in the frame of tile t, which O holds right after PV(t)
        if (t >= 33 && ((t - 33) & 31) == 0) {
          const int X = (t - 33) >> 5;
          ok = mwait(&bars.lflush, X & 1);
          if (ok) ok = issue_restore(X);
          if (!ok) break;
        }
        if (elect_one()) {
          mma_commit(&bars.vempty[s]);
          mma_commit(&bars.pvdone[t % NPD]);
        }
        __syncwarp();
      }
      if (ok && elect_one()) mma_commit(&bars.main);
      __syncwarp();
      // the restore chunks flushed after the loop, in order
      for (int X = X_epi0, e = 0; X <= X_epi1 && ok; ++X, ++e) {
        ok = mwait(&bars.epi, e & 1);
        if (!ok) break;
        tc_fence_after();
        ok = issue_restore(X);
        if (ok && elect_one()) mma_commit(&bars.rdone);
        __syncwarp();
      }
      // repair: the warpgroup's K rows and bf16 probabilities arrive after
      // `main`, so every QK^T and PV of the loop has completed
      for (int rc = 0; rc < nrc && ok; ++rc) {
        ok = mwait(&bars.repk, rc & 1);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          if constexpr (QK4) {
            // the staged K' rows: scales into K-scale slot 0 (every QK^T of
            // the loop completed before `main`), codes after them
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) tmem_cp_sf(tmem + L::TM_KSF + 4 * kk, sdesc_sf(smem_u32(sV + 512 * kk)));
            const uint64_t dq = sdesc_sw64(smem_u32(sQ + V4_SF_BYTES)), dk = sdesc_sw64(smem_u32(sV + V4_SF_BYTES));
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              mma_fp4_ss(tmem + TM_S0, dq + 2 * kk, dk + 2 * kk, IDESC_QK4, tmem + L::TM_QSF + 4 * kk,
                         tmem + L::TM_KSF + 4 * kk, kk > 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f8_ss(tmem + TM_S0, dQ + KSTEP * kk, dR + KSTEP * kk, IDESC_QK, kk > 0);
          }
          mma_commit(&bars.reps);
        }
        __syncwarp();
        ok = mwait(&bars.repp, rc & 1) && mwait(&bars.dt, rc & 1);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16_ss(tmem + TM_O, dR + TSTEP * (1 + (kk >> 2)) + KSTEP * (kk & 3),
                       dK + TSTEP * (kk >> 2) + KSTEP * (kk & 3), IDESC_BF, 1);
          mma_commit(&bars.repdone);
        }
        __syncwarp();
      }
      if (ok && elect_one()) mma_commit(&bars.fin);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax rows
    // Warpgroup g (warps 3+4g .. 6+4g) takes the tiles t with t % 2 == g;
    // thread row r = 32*(warp%4) + lane. The frame is handed from tile to
    // tile in order through s_F (mxr[t%2]). Row sums stay with the warpgroup
    // that owns the tile: lt_own (registers) and its own slots of sLb (slot
    // t%32 of every tile t of parity g), all in the frame of its latest tile;
    // l_t is the difference of two reads of column 384 + t % 4 (a warpgroup
    // owns columns g and g + 2). The two warpgroups meet only where a chunk of
    // 32 row sums is flushed for the block-mean restore, and at the end.
    const int g = (warp - 3) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float sqs = p.sq[static_cast<size_t>(bh) * T + qt];
    const float *skh = p.sk + static_cast<size_t>(bh) * T;
    const int tail = p.N - (T - 1) * 128;  // valid keys in the last tile
    bool ok = true;
    float F_own = 0.0f;   // frame of this warpgroup's latest tile
    float F_hand = 0.0f;  // frame handed over to this warpgroup's latest tile
    float lt_own = 0.0f;  // sum of l_u over this warpgroup's tiles read so far, in frame F_own
    float lprev0 = 0.0f, lprev1 = 0.0f;  // last values read from this warpgroup's two row-sum columns
    float sk_next = skh[g < T ? g : 0];
    auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
      const bool w = wait(bar, parity);
      return __all_sync(0xFFFFFFFFu, w);
    };
    // A operand of the restore MMA: row r = [hi(l_0..l_31) | lo(l_0..l_31)] in
    // bf16; the slots of the other warpgroup's parity are scaled by sc_other
    // into this warpgroup's frame
    auto flush = [&](int nvalid, float sc_other) {
      const float sc0 = g == 0 ? 1.0f : sc_other, sc1 = g == 1 ? 1.0f : sc_other;
      uint32_t hw[16], lw[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float l0 = (2 * i < nvalid) ? sLb[(2 * i) * 128 + r] * sc0 : 0.0f;
        float l1 = (2 * i + 1 < nvalid) ? sLb[(2 * i + 1) * 128 + r] * sc1 : 0.0f;
        const __nv_bfloat16 h0 = __float2bfloat16_rn(l0), h1 = __float2bfloat16_rn(l1);
        const __nv_bfloat16 o0 = __float2bfloat16_rn(__fsub_rn(l0, __bfloat162float(h0)));
        const __nv_bfloat16 o1 = __float2bfloat16_rn(__fsub_rn(l1, __bfloat162float(h1)));
        hw[i] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
        lw[i] = static_cast<uint32_t>(__bfloat16_as_ushort(o0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(o1)) << 16);
      }
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        *reinterpret_cast<uint4 *>(sAr + sw128_off(r, ch)) =
            make_uint4(hw[4 * ch], hw[4 * ch + 1], hw[4 * ch + 2], hw[4 * ch + 3]);
        *reinterpret_cast<uint4 *>(sAr + sw128_off(r, ch + 4)) =
            make_uint4(lw[4 * ch], lw[4 * ch + 1], lw[4 * ch + 2], lw[4 * ch + 3]);
      }
    };

    // One KV tile t (t % 2 == g). LAST: the ragged last tile (keys >= tail masked).
    auto tile = [&](int t, auto last_tag) -> bool {
      constexpr bool LAST = decltype(last_tag)::value;
      const int b = t & 1;
      const float skt = sk_next;
      if (t + 2 < T) sk_next = skh[t + 2];  // this warpgroup's next tile
      if (!wwait(&bars.sfull[b], (t >> 1) & 1)) return false;
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        tmem_ld32(trow + TM_S0 + b * 128 + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * i]));
      tmem_wait_ld();
      tc_fence_before();
      warp_arrive(&bars.sfree[b]);  // the issuer may now compute S(t+2) into this buffer
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
      // frame, taken over from tile t-1's warpgroup: F_t = max(F_{t-1}, 8 ceil(m_t / 8))
      float F_prev = -INFINITY;
      if (t > 0) {
        if (!wwait(&bars.mxr[(t - 1) & 1], ((t - 1) >> 1) & 1)) return false;
        F_prev = s_F[r];
      }
      const float Fn = fmaxf(F_prev, 8.0f * ceilf(__fmul_rn(mx, alpha) * 0.125f));
      if (t == 0) F_prev = Fn;
      s_F[r] = Fn;  // for tile t+1 (after the last tile it holds the final frame)
      if (t + 1 < T) warp_arrive(&bars.mxr[b]);
      const bool need = Fn != F_prev;
      const float sc = need ? frame_scale(F_prev, Fn) : 1.0f;
      const bool anyneed = __any_sync(0xFFFFFFFFu, need);
      // NVFP4 probabilities against the frame Fn into P slot t%3 (last read by
      // PV(t-3), complete since the bookkeeping of tile t-2 waited for it):
      // the row's 64 bytes of codes (64-byte swizzle) and its 8 scale bytes
      {
        const float al8 = __fmul_rn(alpha, 0.125f), nF8 = -Fn * 0.125f;
        uint8_t *slotp = sP + (t % NPSLOT) * SZ_PSLOT;
        uint32_t sc[8];
        p_scales(bm, al8, nF8, sc);
        if constexpr (LAST) {
#pragma unroll
          for (int kb = 0; kb < 8; ++kb)
            if (16 * kb >= tail) sc[kb] = 0u;  // no valid key: scale 0, codes 0
        }
        float rcp[8];
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) rcp[kb] = s_rcp[sc[kb]];
        uint32_t scw[2] = {0u, 0u};
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) scw[kb >> 2] |= sc[kb] << (8 * (kb & 3));
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {  // 32 keys = 2 blocks = one 16-byte chunk
          uint32_t w[4];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int kb = 2 * ch + h;
            p_block(&s[16 * kb], al8, nF8, rcp[kb], w[2 * h], w[2 * h + 1]);
            if constexpr (LAST) {
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                uint32_t keep = 0u;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  if (16 * kb + 8 * q + e < tail) keep |= 0xFu << (4 * e);
                w[2 * h + q] &= keep;
              }
            }
          }
          *reinterpret_cast<uint4 *>(slotp + V4_SF_BYTES + sw64_off(r, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) *reinterpret_cast<uint32_t *>(slotp + v4_sf_off(r, 4 * kk)) = scw[kk];
        fence_proxy_async_smem();  // the codes and scales are read by tcgen05.cp / the MMA
      }
      if (anyneed) {
        // O holds PV(0..t-1) in frame F_prev: rescale it before PV(t)
        if (!wwait(&bars.pvdone[(t - 1) % NPD], ((t - 1) / NPD) & 1)) return false;
        tc_fence_after();
        uint32_t o[128];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          tmem_ld32(trow + TM_O + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(&o[32 * i]));
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 128; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * sc);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          tmem_st32(trow + TM_O + 32 * i, *reinterpret_cast<const uint32_t(*)[32]>(&o[32 * i]));
        tmem_wait_st();
      }
      tc_fence_before();
      warp_arrive(&bars.pfull[t & 3]);

      // ---- row-sum bookkeeping of this warpgroup, off the PV path
      if (g == 0 && t >= 34 && ((t - 34) & 31) == 0) {
        if (!wwait(&bars.lflush, ((t - 34) >> 5) & 1)) return false;
      }
      if (t >= 1) {
        if (!wwait(&bars.pvdone[(t - 1) % NPD], ((t - 1) / NPD) & 1)) return false;
        tc_fence_after();
      }
      if (t >= 2) {
        // l_{t-2} (own previous tile, frame F_own): what PV(t-2) added to its column
        const float v = __uint_as_float(tmem_ld1(trow + lcol_of(t - 2)));
        tmem_wait_ld();
        float lraw;
        if ((t - 2) & 2) {
          lraw = __fsub_rn(v, lprev1);
          lprev1 = v;
        } else {
          lraw = __fsub_rn(v, lprev0);
          lprev0 = v;
        }
        const float scw = frame_scale(F_own, Fn);
        if (F_own != Fn) {
#pragma unroll
          for (int i = 0; i < 16; ++i) sLb[(2 * i + g) * 128 + r] *= scw;
        }
        const float lo = lraw * scw;
        lt_own = lt_own * scw + lo;
        const int slot = (t - 2) & 31;
        sLb[slot * 128 + r] = lo;
        if (slot == 31) {
          if (!wwait(&bars.bk, ((t - 33) >> 5) & 1)) return false;
          flush(32, sc);
          fence_proxy_async_smem();
          tc_fence_before();
          warp_arrive(&bars.lflush);  // the restore follows PV(t)
        }
      }
      if (g == 0 && t >= 32 && (t & 31) == 0) warp_arrive(&bars.bk);
      F_own = Fn;
      F_hand = F_prev;
      return true;
    };

    const bool ragged = tail < 128;
    for (int t = g; t < T - 1 && ok; t += 2) ok = tile(t, std::false_type{});
    if (ok && ((T - 1) & 1) == g)
      ok = ragged ? tile(T - 1, std::true_type{}) : tile(T - 1, std::false_type{});

    // ---------------------------------------------------------- end of the KV loop
    // The last tile's warpgroup takes the other's row-sum state, adds
    // l_{T-2} and l_{T-1}, flushes the remaining restore chunks and runs the
    // repair; both warpgroups write half of the output.
    const bool fin_wg = ((T - 1) & 1) == g;
    if (!fin_wg) {
      s_lto[r] = lt_own;  // frame F_{T-2}, the frame the last tile was handed
      s_lprev[0][r] = lprev0;
      s_lprev[1][r] = lprev1;
      warp_arrive(&bars.wgdone);
    }
    if (ok && fin_wg) ok = wwait(&bars.main, 0) && wwait(&bars.wgdone, 0);
    const float F_fin = F_own;  // frame of the last tile (meaningful in fin_wg)
    if (ok && fin_wg) {
      tc_fence_after();
      const float sc_o = frame_scale(F_hand, F_fin);  // other warpgroup's frame -> F_fin
      float lt = lt_own + s_lto[r] * sc_o;
      int e = 0;
      for (int u = (T >= 2 ? T - 2 : 0); u <= T - 1; ++u) {
        const float v = __uint_as_float(tmem_ld1(trow + lcol_of(u)));
        tmem_wait_ld();
        const int cix = (u >> 1) & 1;
        const float prev = u == T - 1 ? (cix ? lprev1 : lprev0) : s_lprev[cix][r];
        const float lu_raw = __fsub_rn(v, prev);
        const int slot = u & 31;
        sLb[slot * 128 + r] = lu_raw;
        lt += u == T - 1 ? lu_raw : lu_raw * sc_o;
        if (slot == 31 || u == T - 1) {
          if (e > 0) {  // the restore of the previous flush must have read sAr
            ok = wwait(&bars.rdone, (e - 1) & 1);
            if (!ok) break;
          }
          flush(slot + 1, sc_o);
          fence_proxy_async_smem();
          tc_fence_before();
          warp_arrive(&bars.epi);
          ++e;
        }
      }
      s_ltot[r] = lt;
    }
    // ---------------------------------------------------------- repair (the last tile's warpgroup)
    // P' = bf16(fl(2^x' * 2688)), x' = fma(acc, alpha/8, -F_fin/8): the
    // unquantized probability of the repaired token in the final frame, in the
    // units of the NVFP4 products.
    const float nF8fin = -F_fin * 0.125f;
    for (int rc = 0; rc < nrc && fin_wg; ++rc) {
      if (ok && rc > 0) ok = wwait(&bars.repdone, (rc - 1) & 1);
      if (!ok) {
        softmax_bar128(g);  // keep this warpgroup's barrier sequence on failure
        continue;
      }
      const int i = rc * 128 + r;
      const int nval = min(128, p.R - rc * 128);
      float al = 0.0f;
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
          for (int ch = 0; ch < 4; ++ch) krow[ch] = *reinterpret_cast<const uint4 *>(img + V4_SF_BYTES + sw64_off(rr, ch));
#pragma unroll
          for (int h = 0; h < 2; ++h) ksc[h] = *reinterpret_cast<const uint32_t *>(img + v4_sf_off(rr, 4 * h));
          al = __fmul_rn(__fmul_rn(sqs, skh[pos >> 7]), p.kappa);
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) *reinterpret_cast<uint4 *>(sV + V4_SF_BYTES + sw64_off(r, ch)) = krow[ch];
#pragma unroll
        for (int h = 0; h < 2; ++h) *reinterpret_cast<uint32_t *>(sV + v4_sf_off(r, 4 * h)) = ksc[h];
      } else {
        uint4 krow[8];
        if (i < p.R) {
          const int pos = p.rep_idx[static_cast<size_t>(bh) * p.R + i];
          const uint4 *src = reinterpret_cast<const uint4 *>(p.k8 + (static_cast<size_t>(bh) * p.Npad + pos) * 128);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) krow[ch] = src[ch];
          al = __fmul_rn(__fmul_rn(sqs, skh[pos >> 7]), p.kappa);
        } else {
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) krow[ch] = make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4 *>(sV + sw128_off(r, ch)) = krow[ch];
      }
      s_alphaR[r] = __fmul_rn(al, 0.125f);
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&bars.repk);
      softmax_bar128(g);  // s_alphaR visible to every row of this warpgroup
      ok = wwait(&bars.reps, rc & 1);
      if (!ok) continue;  // one barrier per iteration on every path
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t v[32];
        tmem_ld32(trow + TM_S0 + 32 * q, v);
        tmem_wait_ld();
#pragma unroll
        for (int gg = 0; gg < 4; ++gg) {
          uint32_t outw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 32 * q + 8 * gg + 2 * e;
            float p0 = __fmul_rn(ex2_approx(__fmaf_rn(__uint_as_float(v[8 * gg + 2 * e]), s_alphaR[j], nF8fin)),
                                 P_GLOBAL);
            float p1 = __fmul_rn(
                ex2_approx(__fmaf_rn(__uint_as_float(v[8 * gg + 2 * e + 1]), s_alphaR[j + 1], nF8fin)), P_GLOBAL);
            if (j >= nval) p0 = 0.0f;
            if (j + 1 >= nval) p1 = 0.0f;
            const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
            outw[e] = *reinterpret_cast<const uint32_t *>(&pb);
          }
          const int jj = 32 * q + 8 * gg;  // first key of this 16-byte chunk
          *reinterpret_cast<uint4 *>(sV + SZ_TILE8 + (jj >> 6) * SZ_TILE8 + sw128_off(r, (jj & 63) >> 3)) =
              make_uint4(outw[0], outw[1], outw[2], outw[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&bars.repp);
    }
    // ---------------------------------------------------------- epilogue (each warpgroup 64 columns)
    if (ok) ok = wwait(&bars.fin, 0);
    softmax_bar256();  // s_ltot final, from the last tile's warpgroup
    if (ok) {
      tc_fence_after();
      const int c0 = g * 64;
      const int row = qt * 128 + r;
      uint16_t *orow = p.O + (static_cast<size_t>(bh) * p.N + row) * 128;
      const float lrow = s_ltot[r];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        uint32_t v[32];
        tmem_ld32(trow + TM_O + c0 + 32 * i, v);
        tmem_wait_ld();
        if (row < p.N) {
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = c0 + 32 * i + 8 * gg + 2 * e;
              const float o0 = __fdiv_rn(__uint_as_float(v[8 * gg + 2 * e]) * s_vscale[c], lrow);
              const float o1 = __fdiv_rn(__uint_as_float(v[8 * gg + 2 * e + 1]) * s_vscale[c + 1], lrow);
              const __nv_bfloat162 ob = __floats2bfloat162_rn(o0, o1);
              w[e] = *reinterpret_cast<const uint32_t *>(&ob);
            }
            *reinterpret_cast<uint4 *>(orow + c0 + 32 * i + 8 * gg) = make_uint4(w[0], w[1], w[2], w[3]);
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
