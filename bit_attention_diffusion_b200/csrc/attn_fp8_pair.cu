// attn_fp8_pair.cu - the fused VC-Attention FP8 forward kernel on pairs of
// SMs (sm_100a, tcgen05 cta_group::2).
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
// One cluster of two CTAs (the two SMs of a pair) per (pair of 128-query tiles,
// b*h): CTA r owns query tile 2x + r. Every product is one M = 256 MMA over
// both SMs, issued by CTA 0: A rows 0-127 from CTA 0 (its query tile or its
// probabilities), 128-255 from CTA 1; B split along N, the first half in CTA
// 0's shared memory and the second in CTA 1's (each SM stages half of every K
// and V tile); D in each SM's own TMEM. Per SM the TMEM holds one query tile:
//   S0 [0,128), S1 [128,256)   two score buffers, S(t % 2) for KV tile t
//   O  [256,384), RS [384,400) PV is one N = 144 product, B = [V | E], E a
//                              16-row block whose row s (s = the V ring stage)
//                              is E4M3 ones: column RS+s accumulates the row
//                              sum of the decoded bytes of every tile staged
//                              in s; a tile's l_t is read two tiles later
//   P0 [400,432), P1 [432,464) the probability bytes of tiles t even / odd
// Warp roles (both CTAs):
//   warp 0     lane 0: Q, the K half tiles (ring), the repair deltas; lane 1:
//              the V half tiles (ring); lane 2: the block-mean half chunks.
//              Every copy of either CTA completes on CTA 0's barriers.
//   warp 1     allocates TMEM for the pair; in CTA 0 issues PV, the restores
//              and the repair products.
//   warp 2     in CTA 0 issues QK^T.
//   warps 3-10 softmax: warpgroup w takes the KV tiles t = w, w+2, ... (score
//              buffer S(w), probability slot P(w)), one thread per query row,
//              all 128 keys; while one warpgroup turns the scores of tile t
//              into bytes, the other reads tile t+1. The running frame goes
//              from tile to tile through shared memory (published as soon as
//              a warpgroup has its tile's maximum), each warpgroup keeps the
//              row sums of its own tiles with their frames.
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

constexpr int KS = 4;                        // K ring stages (half tiles)
constexpr int VS = 4;                        // V ring stages; at most 16 (one row-sum column each)
constexpr uint32_t SZ_Q = 128 * 128;         // one query tile, 128 rows x 128 bytes
constexpr uint32_t SZ_KH = 64 * 128;         // half a K tile: 64 keys
constexpr uint32_t V_ROWS0 = 72;             // V channels staged by CTA 0 (B rows 0-71)
constexpr uint32_t V_ROWS1 = 56;             // by CTA 1 (B rows 72-127), then the 16 E rows
constexpr uint32_t SZ_VH = 72 * 128;         // half of the N = 144 [V | E] operand
constexpr uint32_t SZ_MUH = 64 * 128;        // half a block-mean chunk: 64 channels x 64 bf16
constexpr uint32_t SZ_AR = 128 * 128;        // restore A operand: 128 rows x 64 bf16
constexpr int LSLOTS = 64;                   // row-sum slots: two restore chunks
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + SZ_Q;
constexpr uint32_t OFF_V = OFF_K + KS * SZ_KH;
constexpr uint32_t OFF_MU = OFF_V + VS * SZ_VH;   // block-mean chunk; the repair's K rows later
constexpr uint32_t OFF_AR = OFF_MU + SZ_MUH;
constexpr uint32_t OFF_LB = OFF_AR + SZ_AR;       // [LSLOTS][128] fp32 row sums
constexpr uint32_t OFF_PREV = OFF_LB + LSLOTS * 128 * 4;  // [VS][128] last value read per row-sum column
constexpr uint32_t OFF_FS = OFF_PREV + VS * 128 * 4;     // [LSLOTS][128] frame of each row-sum slot
constexpr uint32_t OFF_F = OFF_FS + LSLOTS * 128 * 4;     // [3][128] frame hand-over (two tiles, final)
constexpr uint32_t OFF_LT1 = OFF_F + 3 * 128 * 4;         // [2][128] warpgroup 1's row sum and its frame
constexpr uint32_t SMEM_USED = OFF_LT1 + 2 * 128 * 4;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // alignment slack
static_assert(VS <= 16, "one row-sum column per V stage");
static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && SZ_VH % 1024 == 0 && OFF_MU % 1024 == 0 &&
                  OFF_AR % 1024 == 0,
              "tile alignment");
static_assert(VS * SZ_VH >= 2 * 128 * 128, "the repair's bf16 probabilities fit in the V ring");
static_assert(KS * SZ_KH >= 2 * 64 * 128 && KS * SZ_KH >= 8 * 32 * 128, "repair deltas / epilogue staging");
static_assert(SMEM_BYTES + 4096 <= 232448, "shared memory budget (dynamic + static)");

__device__ __forceinline__ constexpr uint32_t tm_s(int b) { return 128u * b; }
constexpr uint32_t TM_O = 256;
constexpr uint32_t TM_RS = 384;
__device__ __forceinline__ constexpr uint32_t tm_p(int b) { return 400u + 32u * b; }
constexpr uint32_t IDESC_QK = idesc_make(0, 0, 256, 128, false, false);  // E4M3 x E4M3 -> f32
constexpr uint32_t IDESC_PV = idesc_make(0, 0, 256, 144, false, false);  // [V | E], N = 144
constexpr uint32_t IDESC_BF = idesc_make(1, 1, 256, 128, false, false);  // bf16 x bf16 -> f32
constexpr uint16_t PAIR = 3;                                              // both CTAs of the cluster

struct BarsPair {
  uint64_t q, kfull[KS], kempty[KS], vfull[VS], vempty[VS], mufull, muempty;
  uint64_t sfull[2], sfree[2], pfull[2], pvdone[2];
  uint64_t fbar[2][4];   // per warpgroup and 32-row group: the frame of its latest tile published
  uint64_t lslot[4];     // per 32-row group: warpgroup 0 wrote the row sum that completes a chunk
  uint64_t epi, rdone, repk, repp, repdone, dt, main, fin, drain;
};

__device__ __forceinline__ uint64_t desc128(const uint8_t *p) { return sdesc_sw128(smem_u32(p), 16, 1024); }

// One arrive per warp, on CTA 0's copy of a barrier (cluster address).
__device__ __forceinline__ void warp_arrive_cl(uint32_t bar_cl) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive_cl(bar_cl);
}

// Epilogue of one softmax warp: its 32 rows, channels [c0, c0+64) of O
// (TMEM columns taddr .. taddr+63) become O = s_c * O_acc / l in bf16. The
// rows are staged in `stg` (32 rows x 128 bytes; 16-byte chunk c of row r at
// chunk c XOR (r mod 8)) and written four half rows per warp store.
__device__ __forceinline__ void store_o_half(uint32_t taddr, const float *vscale, float l, uint8_t *stg,
                                             uint16_t *orow0, int nrows) {
  const int lane = threadIdx.x & 31;
  const float inv = __fdiv_rn(1.0f, l);
  uint8_t *mine = stg + lane * 128;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    uint32_t v[32];
    tmem_ld32(taddr + 32 * i, v);
    tmem_wait_ld();
#pragma unroll
    for (int gg = 0; gg < 4; ++gg) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 32 * i + 8 * gg + 2 * e;
        const float o0 = __uint_as_float(v[8 * gg + 2 * e]) * vscale[c] * inv;
        const float o1 = __uint_as_float(v[8 * gg + 2 * e + 1]) * vscale[c + 1] * inv;
        const __nv_bfloat162 ob = __floats2bfloat162_rn(o0, o1);
        w[e] = *reinterpret_cast<const uint32_t *>(&ob);
      }
      *reinterpret_cast<uint4 *>(mine + (((4 * i + gg) ^ (lane & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  __syncwarp();
  const int ch = lane & 7;
#pragma unroll 4
  for (int it = 0; it < 8; ++it) {
    const int rr = 4 * it + (lane >> 3);
    if (rr < nrows)
      *reinterpret_cast<uint4 *>(orow0 + static_cast<size_t>(rr) * 128 + 8 * ch) =
          *reinterpret_cast<const uint4 *>(stg + rr * 128 + ((ch ^ (rr & 7)) << 4));
  }
}

}  // namespace

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(352, 1)
    k_vc_attn_fwd_pair(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV0, const __grid_constant__ CUtensorMap tmV1,
                       const __grid_constant__ CUtensorMap tmMu, const __grid_constant__ CUtensorMap tmDT,
                       const AttnFp8Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = sm + OFF_Q;
  uint8_t *sK = sm + OFF_K;
  uint8_t *sV = sm + OFF_V;
  uint8_t *sMu = sm + OFF_MU;
  uint8_t *sAr = sm + OFF_AR;
  float *sLb = reinterpret_cast<float *>(sm + OFF_LB);      // [LSLOTS][128]
  float *sPrev = reinterpret_cast<float *>(sm + OFF_PREV);  // [VS][128]
  float *sFs = reinterpret_cast<float *>(sm + OFF_FS);      // [LSLOTS][128]
  float *sF = reinterpret_cast<float *>(sm + OFF_F);        // [3][128]
  float *sLt1 = reinterpret_cast<float *>(sm + OFF_LT1);    // [2][128]
  __shared__ BarsPair bars;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ float s_vscale[128];
  __shared__ float s_skR[128];  // sk of the repaired tokens' KV tiles
  __shared__ float s_lt[128];   // final row sums (warpgroup 0 -> 1)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool lead = rank == 0;
  const int bh = blockIdx.y;
  const int T = p.Nb;
  const int qt = 2 * (blockIdx.x >> 1) + static_cast<int>(rank);
  const bool active = qt < T;              // CTA 1 of the last pair may have no query tile
  const int qt_ld = active ? qt : T - 1;   // it still stages a valid tile (its scale is 0)
  const int nrc = (p.R + 127) / 128;
  const int X_last = (T - 1) >> 5;         // the last block-mean chunk
  const int X0 = first_epilogue_chunk(T);  // the first chunk restored after the loop

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
      mbar_init(&bars.sfree[i], 8);  // one warpgroup (4 warps) x 2 CTAs
      mbar_init(&bars.pfull[i], 8);
      mbar_init(&bars.pvdone[i], 1);
      for (int j = 0; j < 4; ++j) mbar_init(&bars.fbar[i][j], 1);  // the warp of those rows
    }
    for (int j = 0; j < 4; ++j) mbar_init(&bars.lslot[j], 1);
    mbar_init(&bars.epi, 8);   // warpgroup 0 of both CTAs
    mbar_init(&bars.rdone, 1);
    mbar_init(&bars.repk, 8);
    mbar_init(&bars.repp, 16);
    mbar_init(&bars.repdone, 1);
    mbar_init(&bars.dt, 1);
    mbar_init(&bars.main, 2);  // one commit from each issuing warp
    mbar_init(&bars.fin, 1);
    mbar_init(&bars.drain, 2);
    fence_mbar_init();
  }
  if (warp >= 3) {
    const int t = threadIdx.x - 96;  // 0..255
    if (rank == 1) {
      // the E rows after CTA 1's V channels in every stage: rows 56..71 of
      // the stage (B rows 128..143), row 56+j all E4M3 ones (0x38) iff j is
      // the stage's index, else zero
      for (int i = t; i < VS * 16 * 8; i += 256) {
        const int s = i >> 7, j = (i >> 3) & 15, ch = i & 7;
        const uint32_t v = j == s ? 0x38383838u : 0u;
        *reinterpret_cast<uint4 *>(sV + s * SZ_VH + sw128_off(V_ROWS1 + j, ch)) = make_uint4(v, v, v, v);
      }
    }
    if (t < 128) s_vscale[t] = p.vscale[static_cast<size_t>(bh) * 128 + t];
    for (int i = t; i < VS * 128; i += 256) sPrev[i] = 0.0f;
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc_pair(&s_tmem, 512);
    tc_fence_before();
  }
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialized before any remote arrive or copy
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  // Bounded wait; the abort flag (set by a warp whose wait ran out) is read
  // only when the phase is not complete yet.
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
  // CTA 0's copy of a barrier, in the cluster window
  auto at0 = [&](uint64_t *bar) -> uint32_t { return mapa_shared(smem_u32(bar), 0); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      prefetch_tmap(&tmQ); prefetch_tmap(&tmK); prefetch_tmap(&tmDT);
      if (lead) mbar_arrive_expect_tx(&bars.q, 2 * SZ_Q);
      tma_load_2d_pair(sQ, &tmQ, at0(&bars.q), 0, bh * p.Npad + qt_ld * 128);
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % KS;
        ok = wait(&bars.kempty[s], ((t / KS) & 1) ^ 1);
        if (!ok) break;
        if (lead) mbar_arrive_expect_tx(&bars.kfull[s], 2 * SZ_KH);
        tma_load_2d_pair(sK + s * SZ_KH, &tmK, at0(&bars.kfull[s]), 0, bh * p.Npad + t * 128 + 64 * rank);
      }
      if (ok && nrc > 0) {
        // the K ring takes this CTA's 64 channels of the repair deltas once
        // every product of the loop is complete
        ok = wait(&bars.main, 0);
        for (int rc = 0; rc < nrc && ok; ++rc) {
          if (rc > 0) ok = wait(&bars.repdone, (rc - 1) & 1);
          if (!ok) break;
          if (lead) mbar_arrive_expect_tx(&bars.dt, 4 * SZ_KH);
          tma_load_2d_pair(sK, &tmDT, at0(&bars.dt), rc * 128, bh * 128 + 64 * rank);
          tma_load_2d_pair(sK + SZ_KH, &tmDT, at0(&bars.dt), rc * 128 + 64, bh * 128 + 64 * rank);
        }
      }
    } else if (lane == 1) {
      prefetch_tmap(rank ? &tmV1 : &tmV0);
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % VS;
        ok = wait(&bars.vempty[s], ((t / VS) & 1) ^ 1);
        if (!ok) break;
        if (lead) mbar_arrive_expect_tx(&bars.vfull[s], (V_ROWS0 + V_ROWS1) * 128);
        tma_load_2d_pair(sV + s * SZ_VH, rank ? &tmV1 : &tmV0, at0(&bars.vfull[s]), t * 128,
                         bh * 128 + (rank ? V_ROWS0 : 0));
      }
    } else if (lane == 2) {
      // block-mean chunk X: restored before PV(32X+33), or after the loop;
      // the buffer is refilled once the restore of X is complete
      prefetch_tmap(&tmMu);
      bool ok = true;
      for (int X = 0; X <= X_last && ok; ++X) {
        if (X > 0) ok = wait(&bars.muempty, (X - 1) & 1);
        if (!ok) break;
        if (lead) mbar_arrive_expect_tx(&bars.mufull, 2 * SZ_MUH);
        tma_load_2d_pair(sMu, &tmMu, at0(&bars.mufull), 0, (bh * p.nch32 + X) * 128 + 64 * rank);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers (CTA 0)
    if (lead) {
      auto mwait = [&](uint64_t *bar, uint32_t parity) -> bool {
        const bool w = wait(bar, parity);
        return __all_sync(0xFFFFFFFFu, w);
      };
      const uint64_t dQ = desc128(sQ), dK = desc128(sK), dV = desc128(sV), dMu = desc128(sMu);
      const uint64_t dAr = desc128(sAr);
      constexpr uint64_t KSTEP = 32 >> 4, TSTEP = (128 * 128) >> 4, KHSTEP = SZ_KH >> 4, VSTEP = SZ_VH >> 4;
      bool ok = true;
      if (warp == 2) {
        // S(b) <- Q K(t)^T, b = t % 2, once the softmax of tile t-2 has read S(b)
        ok = mwait(&bars.q, 0);
        auto qk = [&](int u, uint64_t dB) -> bool {
          const int b = u & 1;
          if (u >= 2 && !mwait(&bars.sfree[b], ((u >> 1) - 1) & 1)) return false;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f8_ss_pair(tmem + tm_s(b), dQ + KSTEP * kk, dB + KSTEP * kk, IDESC_QK, kk > 0);
            mma_commit_pair(&bars.sfull[b], PAIR);
          }
          __syncwarp();
          return true;
        };
        for (int t = 0; t < T && ok; ++t) {
          const int s = t % KS;
          ok = mwait(&bars.kfull[s], (t / KS) & 1) && qk(t, dK + KHSTEP * s);
          if (!ok) break;
          if (elect_one()) mma_commit_pair(&bars.kempty[s], PAIR);
          __syncwarp();
        }
        if (ok && elect_one()) mma_commit_pair(&bars.main, PAIR);
        __syncwarp();
        // repair scores S <- Q K_R^T, K_R staged over the block-mean buffer
        for (int rc = 0; rc < nrc && ok; ++rc) ok = mwait(&bars.repk, rc & 1) && qk(T + rc, dMu);
      } else {
        auto restore = [&]() {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ss_pair(tmem + TM_O, dAr + KSTEP * kk, dMu + KSTEP * kk, IDESC_BF, 1);
        };
        for (int t = 0; t < T && ok; ++t) {
          const int s = t % VS, b = t & 1;
          ok = mwait(&bars.vfull[s], (t / VS) & 1) && mwait(&bars.pfull[b], (t >> 1) & 1);
          // chunk X is restored right before PV(32X+33): its row sums were
          // written in the frame of tile 32X+33, which O has after that
          // tile's rescale (done before pfull)
          const bool rst = t >= 33 && ((t - 33) & 31) == 0;
          if (ok && rst) ok = mwait(&bars.mufull, ((t - 33) >> 5) & 1);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            if (rst) {
              restore();
              mma_commit_pair(&bars.muempty, PAIR);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f8_ts_pair(tmem + TM_O, tmem + tm_p(b) + 8 * kk, dV + VSTEP * s + KSTEP * kk, IDESC_PV,
                             (t > 0 || kk > 0) ? 1u : 0u);
            mma_commit_pair(&bars.pvdone[b], PAIR);
            mma_commit_pair(&bars.vempty[s], PAIR);
          }
          __syncwarp();
        }
        if (ok && elect_one()) mma_commit_pair(&bars.main, PAIR);
        __syncwarp();
        // the chunks restored after the loop
        for (int X = X0; X <= X_last && ok; ++X) {
          ok = mwait(&bars.epi, (X - X0) & 1) && mwait(&bars.mufull, X & 1);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            restore();
            mma_commit_pair(&bars.rdone, PAIR);
            mma_commit_pair(&bars.muempty, PAIR);
          }
          __syncwarp();
        }
        // repair: O += P_R (bf16, over the V ring) x (delta/s) (bf16, over the K ring)
        for (int rc = 0; rc < nrc && ok; ++rc) {
          ok = mwait(&bars.dt, rc & 1) && mwait(&bars.repp, rc & 1);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_f16_ss_pair(tmem + TM_O, dV + TSTEP * (kk >> 2) + KSTEP * (kk & 3),
                              dK + KHSTEP * (kk >> 2) + KSTEP * (kk & 3), IDESC_BF, 1);
            mma_commit_pair(&bars.repdone, PAIR);
          }
          __syncwarp();
        }
        if (ok && elect_one()) mma_commit_pair(&bars.fin, PAIR);
        __syncwarp();
      }
      // whatever happened, every product this warp issued completes before
      // either CTA frees its TMEM
      if (elect_one()) mma_commit_pair(&bars.drain, 1);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax (both CTAs)
    // Warpgroup w takes the KV tiles t = w, w+2, w+4, ... (score buffer and
    // probability slot w), one thread per query row and all 128 keys. The
    // running frame is handed from tile to tile through shared memory: the
    // warpgroup of tile t publishes F_t as soon as it has the tile maximum.
    const int w = (warp - 3) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lrow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);  // this warp's lanes
    const float sqs = active ? p.sq[static_cast<size_t>(bh) * T + qt] : 0.0f;
    const float *skh = p.sk + static_cast<size_t>(bh) * T;
    const int tail = p.N - (T - 1) * 128;  // valid keys in the last tile
    const uint32_t sfree_cl = at0(&bars.sfree[w]), pfull_cl = at0(&bars.pfull[w]);
    bool ok = true;
    float Fown = -INFINITY;  // frame of this warpgroup's latest tile
    float lt = 0.0f;         // row sums of this warpgroup's tiles read so far, in frame Flt
    float Flt = -INFINITY;
    auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
      const bool v = wait(bar, parity);
      return __all_sync(0xFFFFFFFFu, v);
    };
    // l_u of this warpgroup's tile u (PV(u) complete, PV(u+VS) not issued):
    // what PV(u) added to row-sum column u % VS, into slot u % LSLOTS with
    // its frame Fu, and into lt
    auto read_l = [&](int u, float Fu) {
      const int col = u % VS;  // columns of even tiles are warpgroup 0's, of odd tiles warpgroup 1's
      const float v = __uint_as_float(tmem_ld1(lrow + TM_RS + col));
      tmem_wait_ld();
      const float l = __fsub_rn(v, sPrev[col * 128 + r]);
      sPrev[col * 128 + r] = v;
      sLb[(u % LSLOTS) * 128 + r] = l;
      sFs[(u % LSLOTS) * 128 + r] = Fu;
      if (Fu != Flt) {
        lt = Flt == -INFINITY ? 0.0f : lt * frame_scale(Flt, Fu);
        Flt = Fu;
      }
      lt += l;
    };
    // restore A operand, row r = [hi(l) | lo(l)] of the chunk's tiles in bf16,
    // every slot moved from its own frame into frame Fto (O's frame when the
    // restore runs)
    auto flush = [&](int X, int nvalid, float Fto) {
      uint32_t hw[16], lw[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float lv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int slot = (32 * X + 2 * i + e) % LSLOTS;
          lv[e] = (2 * i + e < nvalid) ? sLb[slot * 128 + r] * frame_scale(sFs[slot * 128 + r], Fto) : 0.0f;
        }
        const __nv_bfloat16 h0 = __float2bfloat16_rn(lv[0]), h1 = __float2bfloat16_rn(lv[1]);
        const __nv_bfloat16 o0 = __float2bfloat16_rn(__fsub_rn(lv[0], __bfloat162float(h0)));
        const __nv_bfloat16 o1 = __float2bfloat16_rn(__fsub_rn(lv[1], __bfloat162float(h1)));
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

    // One KV tile t (t % 2 == w). LAST: the ragged last tile.
    auto tile = [&](int t, auto last_tag) -> bool {
      constexpr bool LAST = decltype(last_tag)::value;
      const float skt = skh[t];
      if (!wwait(&bars.sfull[w], (t >> 1) & 1)) return false;
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int i = 0; i < 4; ++i) tmem_ld32(lrow + tm_s(w) + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * i]));
      tmem_wait_ld();
      tc_fence_before();
      warp_arrive_cl(sfree_cl);  // S(w) may take the scores of tile t+2
      const float Fprev_own = Fown;  // frame of this warpgroup's previous tile, t-2
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
      // F_t = max(F_{t-1}, 8 ceil(m_t / 8)): 8 ceil(running max / 8), with
      // F_{t-1} from the other warpgroup
      float Fp = -INFINITY;
      if (t > 0) {
        if (!wwait(&bars.fbar[w ^ 1][q4], ((t - 1) >> 1) & 1)) return false;
        Fp = sF[(w ^ 1) * 128 + r];
      }
      const float Fn = fmaxf(Fp, 8.0f * ceilf(__fmul_rn(mx, alpha) * 0.125f));
      sF[w * 128 + r] = Fn;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.fbar[w][q4]);
      uint32_t wb[32];
      {
        const float al24 = alpha * TWO_M24;
        const float c24 = (static_cast<float>(p.C) - Fn) * TWO_M24;
#pragma unroll
        for (int q = 0; q < 32; ++q) wb[q] = expcast4(&s[4 * q], al24, c24);
        if constexpr (LAST) {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            uint32_t keep = 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (4 * q + e < tail) keep |= 0xFFu << (8 * e);
            wb[q] &= keep;
          }
        }
      }
      // this warpgroup's previous tile: PV(t-2) complete, slot P(w) free, its
      // row sum readable (waited for only now, so that the PV has had the
      // whole tile to complete)
      if (t >= 2) {
        if (!wwait(&bars.pvdone[w], ((t >> 1) - 1) & 1)) return false;
        tc_fence_after();
        read_l(t - 2, Fprev_own);
        if (w == 0 && t >= 32 && ((t - 32) & 31) == 0) {
          // l_{t-2} completes chunk (t-32)/32 on this side; warpgroup 1
          // flushes it at tile t+1
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.lslot[q4]);
        }
      }
      const bool need = t > 0 && Fn != Fp;
      if (__any_sync(0xFFFFFFFFu, need)) {
        // the frame moves: O (PV(0..t-1), frame F_{t-1}) goes into frame Fn
        // before PV(t); PV(t-1) must be complete (PV(t-2) is, so that
        // barrier is at most one phase behind)
        if (!wwait(&bars.pvdone[w ^ 1], ((t - 1) >> 1) & 1)) return false;
        tc_fence_after();
        const float sc = need ? frame_scale(Fp, Fn) : 1.0f;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t o[64];
          tmem_ld32(lrow + TM_O + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
          tmem_ld32(lrow + TM_O + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 64; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * sc);
          tmem_st32(lrow + TM_O + 64 * hf, *reinterpret_cast<const uint32_t(*)[32]>(&o[0]));
          tmem_st32(lrow + TM_O + 64 * hf + 32, *reinterpret_cast<const uint32_t(*)[32]>(&o[32]));
        }
      }
      if (t >= 33 && ((t - 33) & 31) == 0) {
        // (t odd: warpgroup 1) chunk (t-33)/32 is complete: l_{t-2} was read
        // above, l_{t-3} by warpgroup 0 at tile t-1 (lslot); its row sums in
        // frame Fn for the restore issued right before PV(t)
        if (!wwait(&bars.lslot[q4], ((t - 33) >> 5) & 1)) return false;
        flush((t - 33) >> 5, 32, Fn);
        fence_proxy_async_smem();
      }
      tmem_st32(lrow + tm_p(w), wb);
      tmem_wait_st();  // the bytes and any O rescale are in TMEM
      tc_fence_before();
      warp_arrive_cl(pfull_cl);
      Fown = Fn;
      return true;
    };

    const bool ragged = tail < 128;
    for (int t = w; t < T - 1 && ok; t += 2) ok = tile(t, std::false_type{});
    if (ok && ((T - 1) & 1) == w) ok = ragged ? tile(T - 1, std::true_type{}) : tile(T - 1, std::false_type{});
    // every product of the loop is complete once PV(T-1) is. Parity waits
    // only tell the current phase from the one before, so each warpgroup
    // first waits for the PV of its own last tile (its barrier is then at most
    // that phase behind); after that PV(T-2) is complete, and with it every
    // earlier product, so PV(T-1)'s barrier cannot be two phases behind.
    const int tlast = ((T - 1 - w) & ~1) + w;  // this warpgroup's last tile (if w < T)
    if (ok && w < T) ok = wwait(&bars.pvdone[w], (tlast >> 1) & 1);
    if (ok) ok = wwait(&bars.pvdone[(T - 1) & 1], ((T - 1) >> 1) & 1);
    if (ok && w < T) {
      tc_fence_after();
      read_l(tlast, Fown);
    }
    if (w == 1) {
      sLt1[r] = lt;
      sLt1[128 + r] = Flt;
    }
    if (((T - 1) & 1) == w) sF[2 * 128 + r] = Fown;  // the final frame F_{T-1}
    softmax_bar256();
    const float F = sF[2 * 128 + r];
    if (ok && w == 0) {
      // the row sum over all tiles, in the final frame
      const float l0 = Flt == -INFINITY ? 0.0f : lt * frame_scale(Flt, F);
      const float F1 = sLt1[128 + r];
      const float l1 = F1 == -INFINITY ? 0.0f : sLt1[r] * frame_scale(F1, F);
      s_lt[r] = __fadd_rn(l0, l1);
      const uint32_t epi_cl = at0(&bars.epi);
      for (int X = X0; X <= X_last && ok; ++X) {
        flush(X, min(32, T - 32 * X), F);
        fence_proxy_async_smem();
        tc_fence_before();
        warp_arrive_cl(epi_cl);
        ok = wwait(&bars.rdone, (X - X0) & 1);  // the restore operand is read before the next flush
      }
    }

    // ---------------------------------------------------------- repair
    // The restores are complete once every softmax thread passes this
    // barrier: the block-mean buffer takes this CTA's half of the repaired
    // tokens' K rows (staged by warpgroup 0); warpgroup g writes its 64
    // columns of the bf16 probabilities over the V ring. Every softmax thread
    // takes the same barriers on every path.
    softmax_bar256();
    const int g = w;  // key half of the repair scores
    const float c24f = (static_cast<float>(p.C) - F) * TWO_M24;
    uint8_t *prep = sV + g * (128 * 128);
    const uint32_t repk_cl = at0(&bars.repk), repp_cl = at0(&bars.repp);
    for (int rc = 0; rc < nrc; ++rc) {
      if (ok && rc > 0) ok = wwait(&bars.repdone, (rc - 1) & 1);
      if (g == 0) {
        if (r < 64) {
          const int i = rc * 128 + 64 * static_cast<int>(rank) + r;
          uint4 krow[8];
          if (i < p.R) {
            const int pos = p.rep_idx[static_cast<size_t>(bh) * p.R + i];
            const uint4 *src = reinterpret_cast<const uint4 *>(p.k8 + (static_cast<size_t>(bh) * p.Npad + pos) * 128);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) krow[ch] = src[ch];
          } else {
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) krow[ch] = make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4 *>(sMu + sw128_off(r, ch)) = krow[ch];
        }
        fence_proxy_async_smem();
        tc_fence_before();
        warp_arrive_cl(repk_cl);
      } else {
        const int i = rc * 128 + r;
        s_skR[r] = i < p.R ? skh[p.rep_idx[static_cast<size_t>(bh) * p.R + i] >> 7] : 0.0f;
      }
      softmax_bar256();  // s_skR visible to both warpgroups
      const int u = T + rc, b = u & 1;
      uint32_t sv[64];
      bool got = false;
      if (ok) {
        ok = wwait(&bars.sfull[b], (u >> 1) & 1);
        if (ok) {
          tc_fence_after();
          tmem_ld32(lrow + tm_s(b) + 64 * g, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(lrow + tm_s(b) + 64 * g + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_wait_ld();
          tc_fence_before();
          got = true;
        }
      }
      // both halves of S(b) are read: warpgroup 0 releases it for both (the
      // barrier counts one warpgroup per CTA)
      softmax_bar256();
      if (g == 0) warp_arrive_cl(at0(&bars.sfree[b]));
      if (!got) continue;
      const int nval = min(128, p.R - rc * 128);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        // 32 scores -> 32 bf16 probabilities against the final frame
#pragma unroll
        for (int gg = 0; gg < 4; ++gg) {
          uint32_t outw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int jl = 32 * q + 8 * gg + 2 * e;  // key within this half
            const int j = 64 * g + jl;
            const float a0 = __fmul_rn(__fmul_rn(sqs, s_skR[j]), p.kappa) * TWO_M24;
            const float a1 = __fmul_rn(__fmul_rn(sqs, s_skR[j + 1]), p.kappa) * TWO_M24;
            const uint32_t h = expcast2(__uint_as_float(sv[jl]), __uint_as_float(sv[jl + 1]), a0, a1, c24f);
            uint32_t b0 = h & 0xFFu, b1 = (h >> 16) & 0xFFu;
            if (j >= nval) b0 = 0u;
            if (j + 1 >= nval) b1 = 0u;
            const float2 pv = e4m3x2_value(static_cast<uint16_t>(b0 | (b1 << 8)));
            const __nv_bfloat162 pb = __floats2bfloat162_rn(pv.x, pv.y);
            outw[e] = *reinterpret_cast<const uint32_t *>(&pb);
          }
          *reinterpret_cast<uint4 *>(prep + sw128_off(r, 4 * q + gg)) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive_cl(repp_cl);
    }
    // ---------------------------------------------------------- epilogue
    if (ok) ok = wwait(&bars.fin, 0);
    if (ok && active) {
      tc_fence_after();
      // every product is complete: the warps stage over the K ring
      const int row0 = qt * 128 + q4 * 32;
      uint8_t *stg = sK + (warp - 3) * 32 * 128;
      store_o_half(lrow + TM_O + 64 * g, s_vscale + 64 * g, s_lt[r], stg,
                   p.O + (static_cast<size_t>(bh) * p.N + row0) * 128 + 64 * g, p.N - row0);
    }
  }
  if (lead && (warp == 1 || warp == 2)) {
    // bounded: after a timeout there is nothing more to do for products that
    // never complete
    mbar_wait(&bars.drain, 0);
  }
  if (s_abort) {
    // a wait ran out: give copies still in flight a moment to land before the
    // shared memory is released
    const long long t0 = clock64();
    while (clock64() - t0 < 200000) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the other may still signal it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

uint32_t attn_fp8_pair_smem_bytes() { return SMEM_BYTES; }

}  // namespace vc
