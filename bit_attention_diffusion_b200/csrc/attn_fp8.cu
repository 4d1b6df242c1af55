// attn_fp8.cu - the fused VC-Attention FP8 forward kernel for sm_100a.
//
// Page "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58× sem
// retreinamento": low-bit tensor cores for both products QK^T and PV ("Por que
// a atenção é o gargalo"); the value block mean is restored through the row sum
// the online softmax keeps ("V-Smooth: corrigindo outliers de valor", item
// Restore); the probability byte is written from the log-domain score by one
// fused multiply-add ("ExpCast-FP8: eliminando o gargalo do softmax"). Page
// "VC-Attention et FLUX 3 accélèrent la génération d'images sur Blackwell",
// "Le compromis entre vitesse et fidélité": repair of the worst tokens.
//
// One CTA per (128-query tile, b*h). Warp roles:
//   warp 0     TMA producers: lane 0 Q once, the K8 tiles through a 4-stage
//              ring, then the repair deltas; lane 1 the V8 tiles through a
//              4-stage ring and the bf16 block-mean tiles (one per 32 KV tiles).
//   warp 1     allocates TMEM; issues PV (with the row sums), the block-mean
//              restores and the repair products.
//   warp 2     issues QK^T. Two issuing warps keep the tensor pipe fed: a wait
//              by one of them (~100 cycles even on a completed barrier while
//              MMAs run) overlaps the other's MMAs.
//   warps 3-10 two warpgroups that take the KV tiles in turn (tile t goes to
//              warpgroup t % 2), one thread per query row holding the whole
//              row of its tile: scores, running max, frame, ExpCast bytes,
//              O rescale when the frame moves, row-sum bookkeeping; at the end
//              the last tile's warpgroup does the final restore and the repair,
//              and both write the output.
// TMEM (512 columns x 128 lanes): S double buffer at [0,256); O at [272,400);
// row-sum columns at 256, 257 (odd tiles) and 400, 401 (even tiles); the
// probability bytes P in three slots of 32 columns (4 bytes per column) at
// [416,512), read by the PV MMA as its A operand straight from TMEM. The
// issuers run S(t) = Q8 K8(t)^T as soon as the warpgroup of tile t-2 has read
// S(t-2) out of the buffer, and PV(t) once the bytes are in. PV is one N = 144
// product: its B operand is the V tile plus a 16-row block E with one row of
// ones, placed after V for even tiles (D = [O | 400..415]) and before V for
// odd tiles (D = [256..271 | O]), so that l_t = sum_j p_tj of the decoded
// bytes accumulates into column 400 + (t/2)%2 or 256 + (t/2)%2. The warpgroup
// of tile t reads l_{t-2} there once PV(t-2) is complete (pvdone[(t-2)%8]),
// after it has handed the bytes of tile t to the issuer.
// O is kept in "code units": O_acc = sum p * code + sum_t l_t * mean_t/s + sum_R
// p * delta/s, and the epilogue writes O = s_c * O_acc / l.
#include "common.cuh"
#include "sm100.cuh"
#include "attn_common.cuh"
#include "attn_fp8.cuh"
#include "expcast.cuh"

#include <type_traits>

namespace vc {

namespace {
using namespace attn;

constexpr int KS = 4;  // K ring stages
constexpr int VS = 4;  // V ring stages
constexpr uint32_t SZ_TILE8 = 128 * 128;  // one 128x128 byte tile
constexpr uint32_t SZ_EBLK = 2048;         // 16 rows x 128 bytes: row 0 ones, rows 1-15 zero
// V ring: [V0][E][V1][V2][E][V3]. The PV MMA of an even stage reads N = 144
// rows V(128) + E(16) and writes [O | l_even]; an odd stage reads E(16) + V(128)
// and writes [l_odd | O]: one E block serves both neighbours.
__host__ __device__ constexpr uint32_t voff(int s) { return s * SZ_TILE8 + ((s + 1) >> 1) * SZ_EBLK; }
constexpr uint32_t SZ_VRING = VS * SZ_TILE8 + (VS / 2) * SZ_EBLK;
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + SZ_TILE8;
constexpr uint32_t OFF_V = OFF_K + KS * SZ_TILE8;
constexpr uint32_t OFF_AR = OFF_V + SZ_VRING;
constexpr uint32_t OFF_MU = OFF_AR + SZ_TILE8;
constexpr uint32_t OFF_LB = OFF_MU + 2 * SZ_TILE8;
constexpr uint32_t SMEM_USED = OFF_LB + 32 * 128 * 4;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // alignment slack
static_assert(VS == 4 && voff(1) % 1024 == 0 && voff(3) % 1024 == 0 && OFF_AR % 1024 == 0 && OFF_MU % 1024 == 0,
              "tile alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns: S double buffer [0,256); row sums of odd tiles at 256 + (t/2)%2
// (258..271 unused); O [272,400); row sums of even tiles at 400 + (t/2)%2
// (402..415 unused); P in three slots of 32 columns at [416,512). A row-sum
// column accumulates l_t over the tiles t that map to it (every fourth tile);
// the other PV products of its parity add exact zeros to it, so the value read
// between PV(t) and PV(t+4) is stable and l_t is the difference of two reads.
constexpr uint32_t TM_S0 = 0, TM_LO = 256, TM_O = 272, TM_LE = 400, TM_P = 416;
constexpr int NPD = 8;  // PV completion barriers, indexed t % 8
__device__ __forceinline__ uint32_t lcol_of(int t) { return ((t & 1) ? TM_LO : TM_LE) + ((t >> 1) & 1); }
constexpr uint32_t IDESC_QK = idesc_make(0, 0, 128, 128, false, false);  // E4M3 x E4M3 -> f32, N = 128
constexpr uint32_t IDESC_PV = idesc_make(0, 0, 128, 144, false, false);  // PV with the row-sum rows, N = 144
constexpr uint32_t IDESC_BF = idesc_make(1, 1, 128, 128, false, false);  // bf16 x bf16 -> f32

struct Bars {
  uint64_t q, kfull[KS], kempty[KS], vfull[VS], vempty[VS], mufull[2], muempty[2];
  uint64_t sfull[2], sfree[2], pfull[4], mxr[2], pvdone[NPD], bk, lflush, wgdone, main, epi, rdone, repk, reps,
      repp, repdone, dt, fin;
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
  uint8_t *sAr = sm + OFF_AR;
  uint8_t *sMu = sm + OFF_MU;
  float *sLb = reinterpret_cast<float *>(sm + OFF_LB);  // [32 slots][128 rows]
  __shared__ Bars bars;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ float s_vscale[128];
  __shared__ float s_alphaR[128];
  __shared__ float s_F[128], s_ltot[128], s_lto[128], s_lprev[2][128];

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
    // the two E blocks of the V ring: rows 0..15 of a K-major, 128-byte-swizzled
    // B operand, all zero except one row of 1.0 (0x38) for every key: row 0 in
    // the block of stages 0/1, row 1 in the block of stages 2/3, so that tiles
    // t and t+2 put their row sums into different columns
    {
      const int rr = (t >> 3) & 15, ch = t & 7, blk = t >> 7;
      uint8_t *eblk = sV + voff(2 * blk) + SZ_TILE8;
      const uint32_t v = rr == blk ? 0x38383838u : 0u;
      *reinterpret_cast<uint4 *>(eblk + sw128_off(rr, ch)) = make_uint4(v, v, v, v);
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
    // Lane 0 streams Q and the K tiles (then the repair deltas), lane 1 the V
    // tiles and the block-mean chunks: a K stage is freed by QK(t), long before
    // the V stage of the same tile is freed by PV(t).
    if (lane == 0) {
      prefetch_tmap(&tmQ); prefetch_tmap(&tmK); prefetch_tmap(&tmDT);
      mbar_arrive_expect_tx(&bars.q, SZ_TILE8);
      tma_load_2d(sQ, &tmQ, &bars.q, 0, bh * p.Npad + qt * 128);
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
      prefetch_tmap(&tmV); prefetch_tmap(&tmMu);
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
        mbar_arrive_expect_tx(&bars.vfull[s], SZ_TILE8);
        tma_load_2d(sV + voff(s), &tmV, &bars.vfull[s], t * 128, bh * 128);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    // Both warps run converged; descriptors are warp-uniform (a 32-byte step
    // along K adds 2 to the address field, a 16 KB tile step adds 1024), and
    // each group of tcgen05 instructions is issued by one elected lane.
    auto mwait = [&](uint64_t *bar, uint32_t parity) -> bool {
      const bool w = wait(bar, parity);
      return __all_sync(0xFFFFFFFFu, w);
    };
    const uint64_t dQ = desc128(sQ), dK = desc128(sK), dV = desc128(sV);
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
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_f8_ss(d, dQ + KSTEP * kk, dK + TSTEP * s + KSTEP * kk, IDESC_QK, kk > 0);
          mma_commit(&bars.kempty[s]);
          mma_commit(&bars.sfull[t & 1]);
        }
        __syncwarp();
      }
      if (ok && elect_one()) mma_commit(&bars.main);
      __syncwarp();
    } else {
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
        // V(t) lands long before the bytes: check it first, so that PV(t) goes
        // out as soon as pfull(t) completes
        const int s = t % VS;
        ok = mwait(&bars.vfull[s], (t / VS) & 1);
        if (!ok) break;
        ok = mwait(&bars.pfull[t & 3], (t >> 2) & 1);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          // even tile: B = V(t) + E, D = [O | l_even]; odd: B = E + V(t), D = [l_odd | O]
          const uint32_t pa = tmem + TM_P + 32 * (t % 3);
          const uint32_t d = tmem + ((t & 1) ? TM_LO : TM_O);
          const uint64_t bv = dV + ((voff(s) - (s & 1) * SZ_EBLK) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f8_ts(d, pa + 8 * kk, bv + KSTEP * kk, IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
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
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_f8_ss(tmem + TM_S0, dQ + KSTEP * kk, dV + KSTEP * kk, IDESC_QK, kk > 0);
          mma_commit(&bars.reps);
        }
        __syncwarp();
        ok = mwait(&bars.repp, rc & 1) && mwait(&bars.dt, rc & 1);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16_ss(tmem + TM_O, dV + TSTEP * (1 + (kk >> 2)) + KSTEP * (kk & 3),
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
    // thread row r = 32*(warp%4) + lane. The frame is handed from tile to tile
    // in order through s_F (mxr[t%2]). Row sums stay with the warpgroup that
    // owns the tile: lt_own (registers) and its own slots of sLb (slot t%32 of
    // every tile t of parity g), all in the frame of its latest tile; the two
    // warpgroups meet only where a chunk of 32 row sums is flushed for the
    // block-mean restore, and at the end.
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
    // every lane waits; the outcome is made warp-uniform so that the
    // .sync.aligned TMEM instructions below always see the whole warp
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
      // frame, taken over from tile t-1's warpgroup: F_t = max(F_{t-1}, 8 ceil(m_t / 8))
      // with m_t this tile's scaled row max, i.e. 8 ceil(running max / 8)
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
      // P slot t%3 was last read by PV(t-3), complete since the bookkeeping of
      // tile t-2 (which waited for PV(t-3) and, by commit order, all before it)
      // bytes against the frame Fn: one 32-column store of the row's 128
      // bytes, 4 per column
      {
        const float al24 = alpha * TWO_M24;
        const float c24 = (static_cast<float>(p.C) - Fn) * TWO_M24;
        uint32_t w[32];
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
        tmem_st32(trow + TM_P + 32 * (t % 3), w);
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
      }
      tmem_wait_st();  // the P bytes (and any O rescale) are in TMEM
      tc_fence_before();
      warp_arrive(&bars.pfull[t & 3]);

      // ---- row-sum bookkeeping of this warpgroup, off the PV path
      if (g == 0 && t >= 34 && ((t - 34) & 31) == 0) {
        // the other warpgroup flushed chunk (t-34)/32 at tile t-1: it has read
        // this warpgroup's slots once lflush completes
        if (!wwait(&bars.lflush, ((t - 34) >> 5) & 1)) return false;
      }
      // PV(t-1) complete, and with it every earlier PV: the P slot of tile t+2
      // (last read by PV(t-1)) is free, and l_{t-2} can be read
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
          // chunk (t-33)/32 is complete: the other warpgroup's slots are in the
          // frame of tile t-1 once its bookkeeping of that tile is done (bk)
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

    // this warpgroup's row-sum columns start at zero: odd tiles accumulate
    // onto theirs (the first even tile overwrites)
    tmem_st1(trow + lcol_of(g), 0u);
    tmem_st1(trow + lcol_of(g + 2), 0u);
    tmem_wait_st();
    const bool ragged = tail < 128;
    for (int t = g; t < T - 1 && ok; t += 2) ok = tile(t, std::false_type{});
    if (ok && ((T - 1) & 1) == g)
      ok = ragged ? tile(T - 1, std::true_type{}) : tile(T - 1, std::false_type{});

    // ---------------------------------------------------------- end of the KV loop
    // The warpgroup of the last tile (fin_wg) takes the other's row-sum state,
    // adds l_{T-2} and l_{T-1}, and flushes the remaining one or two restore
    // chunks; then it runs the repair; then both warpgroups write half of the
    // output columns each.
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
        // l_u: u = T-1 in frame F_fin, u = T-2 in frame F_hand (its slot keeps
        // the other warpgroup's frame convention)
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
    const float c24f = (static_cast<float>(p.C) - F_fin) * TWO_M24;
    for (int rc = 0; rc < nrc && fin_wg; ++rc) {
      if (ok && rc > 0) ok = wwait(&bars.repdone, (rc - 1) & 1);
      if (!ok) {
        softmax_bar128(g);  // keep this warpgroup's barrier sequence on failure
        continue;
      }
      const int i = rc * 128 + r;
      const int nval = min(128, p.R - rc * 128);
      uint4 krow[8];
      float al = 0.0f;
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
      s_alphaR[r] = al * TWO_M24;
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
        // 32 scores -> 32 bf16 probabilities (two 16-byte chunks per 8 values)
#pragma unroll
        for (int gg = 0; gg < 4; ++gg) {
          uint32_t outw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 32 * q + 8 * gg + 2 * e;
            const uint32_t h = expcast2(__uint_as_float(v[8 * gg + 2 * e]), __uint_as_float(v[8 * gg + 2 * e + 1]),
                                        s_alphaR[j], s_alphaR[j + 1], c24f);
            uint32_t b0 = h & 0xFFu, b1 = (h >> 16) & 0xFFu;
            if (j >= nval) b0 = 0u;
            if (j + 1 >= nval) b1 = 0u;
            const float2 pv = e4m3x2_value(static_cast<uint16_t>(b0 | (b1 << 8)));
            const __nv_bfloat162 pb = __floats2bfloat162_rn(pv.x, pv.y);
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

uint32_t attn_fp8_smem_bytes() { return SMEM_BYTES; }

}  // namespace vc
