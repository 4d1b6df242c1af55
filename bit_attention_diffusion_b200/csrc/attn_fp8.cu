// attn_fp8.cu - the fused VC-Attention FP8 forward kernel (sm_100a): two
// query tiles per CTA sharing one TMEM score buffer.
//
// Page "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58×
// sem retreinamento": low-bit tensor cores for QK^T and PV ("Por que a
// atenção é o gargalo"); the value block means restored through the online
// softmax's row sums ("V-Smooth: corrigindo outliers de valor", item
// Restore); the probability byte written from the log-domain score by one
// fused multiply-add ("ExpCast-FP8: eliminando o gargalo do softmax"). Page
// "VC-Attention et FLUX 3 accélèrent la génération d'images sur Blackwell",
// "Le compromis entre vitesse et fidélité": repair of the worst tokens.
//
// One CTA per (pair of 128-query tiles a, b; b*h). Each K8 / V8 tile is read
// once from shared memory per pair. Warp roles:
//   warp 0     lane 0: Q_a, Q_b, the K8 tiles (3-stage ring), then the repair
//              deltas; lane 1: the V8 tiles (3-stage ring); lane 2: the
//              block-mean chunks (one per 32 KV tiles).
//   warp 1     allocates TMEM; issues PV for both query tiles, the block-mean
//              restores and the repair products.
//   warp 2     issues QK^T for both query tiles.
//   warps 3-6  softmax warpgroup of query tile a, warps 7-10 of tile b: one
//              thread per query row, all KV tiles of its own query tile.
//              Each warpgroup keeps its own running max, frame and row sums,
//              so nothing is handed between warpgroups.
// TMEM (512 columns): one score buffer S [0,128) shared by the two query
// tiles; O_a [128,256) with its row-sum block [256,272); O_b [272,400) with
// [400,416); the probability bytes P_a [416,448) and P_b [448,480), the A
// operands of PV read from TMEM. QK^T alternates S between the query tiles:
// S <- Q_a K(t), read out by warpgroup a; S <- Q_b K(t), read by b; S <-
// Q_a K(t+1) ... A warpgroup holds S only for its register load, so the
// tensor pipe interleaves the four products of a KV tile (QK_a, QK_b, PV_a,
// PV_b) while the warpgroups compute bytes. PV_i is one N = 144 product: B = V
// tile followed by a 16-row block E (one row of E4M3 ones), D = [O_i | row
// sums], so l_t = sum_j p_tj of the decoded bytes accumulates into the
// column after O_i; the warpgroup reads it once PV_i(t) is complete (before
// it hands over the bytes of t+1) and takes l_t as the difference of two
// reads (the column is never rescaled: each l_t stays in its own frame).
// O is kept in "code units": O_acc = sum p * code + sum_t l_t * mean_t/s +
// sum_R p * delta/s, and the epilogue writes O = s_c * O_acc / l.
#include "common.cuh"
#include "sm100.cuh"
#include "attn_common.cuh"
#include "attn_fp8.cuh"
#include "expcast.cuh"

#include <type_traits>

namespace vc {

namespace {
using namespace attn;

constexpr int KS = 3;                        // K ring stages
constexpr int VS = 3;                        // V ring stages
constexpr uint32_t SZ_TILE8 = 128 * 128;     // one 128x128 byte tile
constexpr uint32_t SZ_EBLK = 2048;           // 16 rows x 128 bytes: row 0 ones, rows 1-15 zero
constexpr uint32_t SZ_VSTAGE = SZ_TILE8 + SZ_EBLK;  // [V | E]: the N = 144 B operand
constexpr uint32_t OFF_Q = 0;                       // Q_a, Q_b
constexpr uint32_t OFF_K = OFF_Q + 2 * SZ_TILE8;
constexpr uint32_t OFF_V = OFF_K + KS * SZ_TILE8;
constexpr uint32_t OFF_MU = OFF_V + VS * SZ_VSTAGE;  // one block-mean chunk; the repair's K rows later
constexpr uint32_t OFF_AR = OFF_MU + SZ_TILE8;       // restore A operands of a and b; b's repair P later
constexpr uint32_t OFF_LB = OFF_AR + 2 * SZ_TILE8;   // row-sum slots of a and b
constexpr uint32_t SMEM_USED = OFF_LB + 2 * 32 * 128 * 4;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // alignment slack
static_assert(SZ_VSTAGE % 1024 == 0 && OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && OFF_MU % 1024 == 0 &&
                  OFF_AR % 1024 == 0,
              "tile alignment");
static_assert(VS * SZ_VSTAGE >= 2 * SZ_TILE8, "a's repair probabilities fit in the V ring");
static_assert(SMEM_BYTES + 6144 <= 232448, "shared memory budget (dynamic + static)");

constexpr uint32_t TM_S = 0;                                                            // shared scores
__device__ __forceinline__ constexpr uint32_t tm_o(int i) { return 128u + 144u * i; }    // O_i (+ row sums)
__device__ __forceinline__ constexpr uint32_t tm_p(int i) { return 416u + 32u * i; }     // P_i
constexpr uint32_t IDESC_QK = idesc_make(0, 0, 128, 128, false, false);  // E4M3 x E4M3 -> f32, N = 128
constexpr uint32_t IDESC_PV = idesc_make(0, 0, 128, 144, false, false);  // [V | E], N = 144
constexpr uint32_t IDESC_BF = idesc_make(1, 1, 128, 128, false, false);  // bf16 x bf16 -> f32

struct Bars {
  uint64_t q, kfull[KS], kempty[KS], vfull[VS], vempty[VS], mufull, muempty;
  uint64_t sfull[2], sfree[2], pfull[2], pvdone[2], epi[2], rdone[2], repp[2];
  uint64_t main, repk, repdone, dt, fin;
};

__device__ __forceinline__ uint64_t desc128(const uint8_t *p) { return sdesc_sw128(smem_u32(p), 16, 1024); }

// tcgen05 MMA with the A operand read from TMEM (M = 128 lanes; K = 32 bytes
// per instruction = 8 columns of 4 packed E4M3 values) and B from shared memory.
__device__ __forceinline__ void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

}  // namespace

__global__ void __launch_bounds__(352, 1)
    k_vc_attn_fwd(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmMu,
                     const __grid_constant__ CUtensorMap tmDT, const AttnFp8Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = sm + OFF_Q;
  uint8_t *sK = sm + OFF_K;
  uint8_t *sV = sm + OFF_V;
  uint8_t *sMu = sm + OFF_MU;
  uint8_t *sAr = sm + OFF_AR;
  float *sLb = reinterpret_cast<float *>(sm + OFF_LB);  // [2 query tiles][32 slots][128 rows]
  __shared__ Bars bars;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ float s_vscale[128];
  __shared__ float s_skR[128];  // sk of the repaired tokens' KV tiles

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
    // the E block after the V tile of every stage: rows 128..143 of a K-major,
    // 128-byte-swizzled B operand, all zero except row 128, 1.0 (0x38) for every key
    for (int i = t; i < VS * 128; i += 256) {
      const int s = i >> 7, rr = (i >> 3) & 15, ch = i & 7;
      const uint32_t v = rr == 0 ? 0x38383838u : 0u;
      *reinterpret_cast<uint4 *>(sV + s * SZ_VSTAGE + SZ_TILE8 + sw128_off(rr, ch)) = make_uint4(v, v, v, v);
    }
    if (t < 128) s_vscale[t] = p.vscale[static_cast<size_t>(bh) * 128 + t];
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
      mbar_arrive_expect_tx(&bars.q, nq * SZ_TILE8);
      for (int i = 0; i < nq; ++i) tma_load_2d(sQ + i * SZ_TILE8, &tmQ, &bars.q, 0, bh * p.Npad + (qt0 + i) * 128);
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % KS;
        ok = wait(&bars.kempty[s], ((t / KS) & 1) ^ 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars.kfull[s], SZ_TILE8);
        tma_load_2d(sK + s * SZ_TILE8, &tmK, &bars.kfull[s], 0, bh * p.Npad + t * 128);
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
      prefetch_tmap(&tmV);
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % VS;
        ok = wait(&bars.vempty[s], ((t / VS) & 1) ^ 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars.vfull[s], SZ_TILE8);
        tma_load_2d(sV + s * SZ_VSTAGE, &tmV, &bars.vfull[s], t * 128, bh * 128);
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
    auto mwait = [&](uint64_t *bar, uint32_t parity) -> bool {
      const bool w = wait(bar, parity);
      return __all_sync(0xFFFFFFFFu, w);
    };
    const uint64_t dQ = desc128(sQ), dK = desc128(sK), dV = desc128(sV), dMu = desc128(sMu);
    const uint64_t dAr = desc128(sAr);
    constexpr uint64_t KSTEP = 32 >> 4, TSTEP = SZ_TILE8 >> 4, VSTEP = SZ_VSTAGE >> 4;
    bool ok = true;
    if (warp == 2) {
      // S <- Q_i K^T in the order (a, t), (b, t), (a, t+1), ...: step k (k = t in
      // the loop, T + rc in the repair) of query tile i waits until the previous
      // product's warpgroup has read S out (sfree of that tile, its step)
      auto wait_s = [&](int i, int k) -> bool {
        if (i > 0) return mwait(&bars.sfree[i - 1], k & 1);
        return k == 0 || mwait(&bars.sfree[nq - 1], (k - 1) & 1);
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
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f8_ss(tmem + TM_S, dQ + TSTEP * i + KSTEP * kk, dK + TSTEP * s + KSTEP * kk, IDESC_QK, kk > 0);
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
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f8_ss(tmem + TM_S, dQ + TSTEP * i + KSTEP * kk, dMu + KSTEP * kk, IDESC_QK, kk > 0);
            mma_commit(&bars.sfull[i]);
          }
          __syncwarp();
        }
      }
    } else {
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
        for (int i = 0; i < nq && ok; ++i) {
          ok = mwait(&bars.pfull[i], t & 1);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            if (rst) {
              restore(i);
              if (i == nq - 1) mma_commit(&bars.muempty);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f8_ts(tmem + tm_o(i), tmem + tm_p(i) + 8 * kk, dV + VSTEP * s + KSTEP * kk, IDESC_PV,
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
      // repair: O_i += P_R,i (bf16) x (delta/s) (bf16); a's probabilities over
      // the V ring, b's over the restore operands
      for (int rc = 0; rc < nrc && ok; ++rc) {
        ok = mwait(&bars.dt, rc & 1);
        for (int i = 0; i < nq && ok; ++i) {
          ok = mwait(&bars.repp[i], rc & 1);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            const uint64_t dP = i == 0 ? dV : dAr;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_f16_ss(tmem + tm_o(i), dP + TSTEP * (kk >> 2) + KSTEP * (kk & 3),
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
      float mx;
      {
        float mm[43];
#pragma unroll
        for (int j = 0; j < 42; ++j) mm[j] = max3(s[3 * j], s[3 * j + 1], s[3 * j + 2]);
        mm[42] = fmaxf(s[126], s[127]);
#pragma unroll
        for (int j = 0; j < 14; ++j) mm[j] = max3(mm[3 * j], mm[3 * j + 1], mm[3 * j + 2]);
        mm[14] = mm[42];
#pragma unroll
        for (int j = 0; j < 5; ++j) mm[j] = max3(mm[3 * j], mm[3 * j + 1], mm[3 * j + 2]);
        mx = max3(mm[0], mm[1], fmaxf(mm[2], fmaxf(mm[3], mm[4])));
      }
      const float alpha = __fmul_rn(__fmul_rn(sqs, skt), p.kappa);
      // F_t = max(F_{t-1}, 8 ceil(m_t / 8)): 8 ceil(running max / 8)
      const float Fn = fmaxf(F, 8.0f * ceilf(__fmul_rn(mx, alpha) * 0.125f));
      const bool need = t > 0 && Fn != F;
      const float sc = need ? frame_scale(F, Fn) : 1.0f;
      uint32_t w[32];
      {
        const float al24 = alpha * TWO_M24;
        const float c24 = (static_cast<float>(p.C) - Fn) * TWO_M24;
#pragma unroll
        for (int q = 0; q < 32; ++q) w[q] = expcast4(&s[4 * q], al24, c24);
        if constexpr (LAST) {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            uint32_t keep = 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (4 * q + e < tail) keep |= 0xFFu << (8 * e);
            w[q] &= keep;
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
          fence_proxy_async_smem();
          nfill = 0;
        }
      }
      tmem_st32(lrow + tm_p(g), w);
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
      }
      tmem_wait_st();  // the bytes and any O rescale are in TMEM
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
    // by warpgroup a), a's bf16 probabilities go over the V ring, b's over the
    // restore operands. Every softmax thread takes the same barriers on every
    // path.
    softmax_bar256();
    const float c24f = (static_cast<float>(p.C) - F) * TWO_M24;
    uint8_t *prep = g == 0 ? sV : sAr;
    for (int rc = 0; rc < nrc; ++rc) {
      if (ok && rc > 0) ok = wwait(&bars.repdone, (rc - 1) & 1);
      if (g == 0 && active) {
        const int i = rc * 128 + r;
        uint4 krow[8];
        float skr = 0.0f;
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
        // 32 scores -> 32 bf16 probabilities against the final frame
#pragma unroll
        for (int gg = 0; gg < 4; ++gg) {
          uint32_t outw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 32 * q + 8 * gg + 2 * e;
            const float a0 = __fmul_rn(__fmul_rn(sqs, s_skR[j]), p.kappa) * TWO_M24;
            const float a1 = __fmul_rn(__fmul_rn(sqs, s_skR[j + 1]), p.kappa) * TWO_M24;
            const uint32_t h = expcast2(__uint_as_float(v[8 * gg + 2 * e]), __uint_as_float(v[8 * gg + 2 * e + 1]),
                                        a0, a1, c24f);
            uint32_t b0 = h & 0xFFu, b1 = (h >> 16) & 0xFFu;
            if (j >= nval) b0 = 0u;
            if (j + 1 >= nval) b1 = 0u;
            const float2 pv = e4m3x2_value(static_cast<uint16_t>(b0 | (b1 << 8)));
            const __nv_bfloat162 pb = __floats2bfloat162_rn(pv.x, pv.y);
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

uint32_t attn_fp8_smem_bytes() { return SMEM_BYTES; }

}  // namespace vc
