// kmeans_tc.cu - one Lloyd pass of the V-Smooth grouping for k <= 8 with the
// labels decided on the tensor cores (sm_100a).
//
// Page "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58×
// sem retreinamento", section "V-Smooth: corrigindo outliers de valor", item
// Group: value tokens are grouped by online k-means so that each 128-token
// block holds similar tokens.
//
// The label of a token is the argmin over clusters of the pinned distance
// d~_j = fma chain over channels of fp32(v_c - c_jc)^2 (ties to the lowest
// cluster): the same arithmetic as k_kmeans_pass. Here a bf16 product on
// the tensor cores gives, for every token of a 128-token chunk, v . hi(c_j)
// and v . lo(c_j) (c_j = hi + lo + a remainder below 2^-18 |c_j|, hi and lo
// bf16), and each token's estimate e_j = |v|^2 - 2 (v.hi + v.lo) + |c_j|^2 is
// within E_j = 2^-13 (|v|^2 + |c_j|^2) of d~_j: the chain's rounding is
// below 130 * 2^-24 d, the estimate's (fp32 sums of 128 exact products,
// allowing 2^-15 of the absolute sum for the tensor cores' accumulation, the
// remainder, the fp32 combination) below 4.3e-5 (|v|^2 + |c_j|^2). When every
// other cluster's estimate exceeds the smallest one, e_b, by more than
// E_b + E_j, cluster b is the label (strictly smaller d~ than every other
// cluster, so no tie arises); otherwise the pinned chains of all clusters
// decide. Labels are therefore exactly k_kmeans_pass's.
//
// A block takes `cpb` consecutive 128-token chunks of one (b,h) and runs them
// through a ring of KS shared-memory stages, one warp role per step, each
// step handing the stage to the next through an mbarrier:
//   warp 0      TMA: the chunk, K-major with the 128-byte swizzle the MMA
//               reads (two 64-channel atoms), once the stage is empty;
//   warp 1      the product of the chunk with the centroid operand into the
//               stage's 16 TMEM columns, once the labels of the stage's
//               previous chunk have been read out of them;
//   warps 4-7   one token per thread (TMEM lane = token): |v|^2, the
//               estimates, the label or a place on the fallback list;
//   warps 2-3   the fallback list: the pinned chains, eight lanes per token
//               (lane j of the group is cluster j), four tokens per warp;
//   warps 8-15  update passes: warp j lists the chunk's tokens labelled j
//               and j ^ 4 and adds, in fp64, the first half of the first
//               list and the second half of the second, four rows per step
//               (lane l: channels 4l .. 4l+3), then frees the stage; in the
//               label pass warp j counts cluster j's tokens (the block's
//               counts go to pcnt for the permutation's scatter).
// No step waits for the whole block: a slow step (many fallback tokens, a
// large cluster) holds its stage, and the others go on until the ring is
// full. The last block of a (b,h) adds the blocks' partial sums in block order
// into the new centroids.
#include "common.cuh"
#include "prologue.cuh"
#include "sm100.cuh"

namespace vc {

namespace {

// The dynamic shared-memory base rounded up to a multiple of 1024 bytes by
// pointer arithmetic on the array itself, so that the compiler still knows the
// result points into shared memory and accesses through it compile to
// shared-memory instructions (an integer round trip would make them generic).
__device__ __forceinline__ uint8_t *smem_align1024(uint8_t *raw) {
  return raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
}

constexpr int KT_CHUNK_BYTES = TILE * D * 2;                     // 32 KB: two 16 KB atoms
constexpr int KS = KMEANS8TC_STAGES;                             // ring stages
constexpr uint32_t KT_IDESC = idesc_make(1, 1, 128, 16, false, false);  // bf16 x bf16 -> f32, N = 16

__device__ __forceinline__ uint32_t kt_off(int row, int ch16) {  // 16-byte chunk ch16 (0..15) of a token row
  return static_cast<uint32_t>((ch16 >> 3) * (TILE * 128)) + sw128_off(row, ch16 & 7);
}

// Chunk of rows [row0, row0+128) of the map over V (rows b*h*N + n): two
// 64-channel boxes into the two atoms, completing on `bar`.
__device__ __forceinline__ void kt_load_chunk(uint8_t *buf, const CUtensorMap *map, uint64_t *bar, int row0) {
  mbar_arrive_expect_tx(bar, KT_CHUNK_BYTES);
  tma_load_2d(buf, map, bar, 0, row0);
  tma_load_2d(buf + TILE * 128, map, bar, 64, row0);
}

__device__ __forceinline__ void kt_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Shared-memory loads at a 32-bit shared address. Volatile, so they stay
// after the barrier wait that precedes them; without a memory clobber, so the
// compiler may issue several before using the first.
__device__ __forceinline__ uint2 lds64_nc(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

}  // namespace

struct BarsKm {
  uint64_t full[KS], mma[KS], lab[KS], fbd[KS], empty[KS];
};

__global__ void __launch_bounds__(KM_THREADS, 2) k_kmeans_pass8tc(const __grid_constant__ CUtensorMap tmV, int N,
                                                                  int k, int cpb, int nblk, float *__restrict__ cent,
                                                                  int32_t *__restrict__ labels,
                                                                  double *__restrict__ psum, int *__restrict__ pcnt,
                                                                  unsigned *__restrict__ counter, int accumulate,
                                                                  uint32_t *__restrict__ status) {
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t *dsm = smem_align1024(dsm_raw);
  uint8_t *sB = dsm + KS * KT_CHUNK_BYTES;       // B operand: rows 0-7 hi(c_j), 8-15 lo(c_j); two 2 KB atoms
  __shared__ BarsKm bars;
  __shared__ float scc[8];                       // |c_j|^2
  __shared__ __align__(16) float scent[8][D + 4];  // fp32 centroids (rows padded: the 8 lanes of a chain group hit 8 banks)
  __shared__ int8_t slab[KS][TILE];              // label of each token of the stage's chunk (-1: not yet)
  __shared__ uint8_t sfb[KS][4][32];             // fallback tokens, per label warp
  __shared__ int snfb[KS][4];
  __shared__ __align__(16) uint8_t sidx[8][2][TILE];  // sum warp j: the chunk's tokens of clusters j, j^4
  __shared__ int s_fail;
  __shared__ int s_last;
  __shared__ uint32_t s_tmem;
  __shared__ int s_tma_issued, s_tma_seen, s_mma_issued, s_mma_seen;
  const int bh = blockIdx.y, blk = blockIdx.x, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  float *cent_h = cent + static_cast<size_t>(bh) * k * D;

  const int n_begin = blk * cpb * TILE;
  const int n_end = min(N, n_begin + cpb * TILE);
  const int nchunk = (n_end - n_begin + TILE - 1) / TILE;
  const int row_base = bh * N + n_begin;  // map row of the block's first token
  if (tid == 0) {
    for (int s = 0; s < KS; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.mma[s], 1);
      mbar_init(&bars.lab[s], 128);
      mbar_init(&bars.fbd[s], 64);
      mbar_init(&bars.empty[s], 256);
    }
    fence_mbar_init();
    prefetch_tmap(&tmV);
    s_fail = 0;
    s_tma_issued = min(KS, nchunk);
    s_tma_seen = 0;
    s_mma_issued = 0;
    s_mma_seen = 0;
    for (int i = 0; i < KS && i < nchunk; ++i)
      kt_load_chunk(dsm + i * KT_CHUNK_BYTES, &tmV, &bars.full[i], row_base + i * TILE);
  }

  // centroids: the bf16 hi/lo operand and |c_j|^2 (the pinned chains read
  // the fp32 centroids from global memory, through L1)
  if (tid < 16 * 16) {  // 16 rows x 16 chunks of 8 channels
    const int row = tid >> 4, ch16 = tid & 15, j = row & 7;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint16_t h2[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int c = 8 * ch16 + 2 * e + q;
        const float x = j < k ? cent_h[j * D + c] : 0.0f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(x);
        h2[q] = row < 8 ? __bfloat16_as_ushort(hi)
                        : __bfloat16_as_ushort(__float2bfloat16_rn(__fsub_rn(x, __bfloat162float(hi))));
      }
      w[e] = static_cast<uint32_t>(h2[0]) | (static_cast<uint32_t>(h2[1]) << 16);
    }
    *reinterpret_cast<uint4 *>(sB + (ch16 >> 3) * 2048 + sw128_off(row, ch16 & 7)) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if (warp < 16) {
    // |c_j|^2 in fp64, warp 8 + j
    const int j = warp - 8;
    double s2 = 0.0;
    if (j < k)
      for (int c = lane; c < D; c += 32) {
        const double x = cent_h[j * D + c];
        s2 += x * x;
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s2 += __shfl_xor_sync(0xFFFFFFFFu, s2, o);
    if (lane == 0) scc[j] = j < k ? static_cast<float>(s2) : 0.0f;
  }
  for (int i = tid; i < 8 * D; i += KM_THREADS) scent[i / D][i % D] = (i / D) < k ? cent_h[i] : 0.0f;
  if (warp == 1) tmem_alloc(&s_tmem, 64);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  double acc4[4] = {0.0, 0.0, 0.0, 0.0};  // sum warps: cluster warp - 8 (its first halves)
  double accB[4] = {0.0, 0.0, 0.0, 0.0};  // sum warps: cluster (warp - 8) ^ 4 (its second halves)
  int cnt_own = 0;  // tokens of cluster warp - 8 (sum warps)
  if (warp == 0) {
    // ---- TMA producer: chunk i into stage i % KS once chunk i - KS has left it
    if (lane == 0)
      for (int i = KS; i < nchunk; ++i) {
        const int s = i % KS;
        if (!mbar_wait(&bars.empty[s], ((i / KS) - 1) & 1)) {
          atomicOr(status, ST_TIMEOUT);
          s_fail = 1;
          break;
        }
        kt_load_chunk(dsm + s * KT_CHUNK_BYTES, &tmV, &bars.full[s], row_base + i * TILE);
        s_tma_issued = i + 1;
      }
  } else if (warp == 1) {
    // ---- MMA issuer: v . hi(c_j), v . lo(c_j) of chunk i into TMEM columns 16 s
    if (lane == 0) {
      const uint64_t dB = sdesc_sw128(smem_u32(sB), 16, 1024);
      for (int i = 0; i < nchunk; ++i) {
        const int s = i % KS;
        if (!mbar_wait(&bars.full[s], (i / KS) & 1)) {
          atomicOr(status, ST_TIMEOUT);
          s_fail = 1;
          break;
        }
        s_tma_seen = i + 1;
        if (i >= KS && !mbar_wait(&bars.lab[s], ((i / KS) - 1) & 1)) {  // the stage's columns were read
          atomicOr(status, ST_TIMEOUT);
          s_fail = 1;
          break;
        }
        tc_fence_after();
        const uint64_t dA = sdesc_sw128(smem_u32(dsm + s * KT_CHUNK_BYTES), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ss(tmem + 16u * s, dA + (kk >> 2) * ((TILE * 128) >> 4) + 2 * (kk & 3),
                     dB + (kk >> 2) * (2048 >> 4) + 2 * (kk & 3), KT_IDESC, kk > 0);
        mma_commit(&bars.mma[s]);
        s_mma_issued = i + 1;
      }
    }
  } else if (warp < 4) {
    // ---- fallback warps: the pinned chains of the undecided tokens, four
    // tokens per warp at a time (lane group g = lane / 8, cluster j = lane % 8)
    const int fw = warp - 2, g = lane >> 3, j = lane & 7;
    for (int i = 0; i < nchunk; ++i) {
      const int s = i % KS;
      const int n0 = n_begin + i * TILE;
      if (!mbar_wait(&bars.lab[s], (i / KS) & 1)) {
        if (lane == 0) atomicOr(status, ST_TIMEOUT);
        s_fail = 1;
        break;
      }
      const int c0 = snfb[s][0], c1 = snfb[s][1], c2 = snfb[s][2], c3 = snfb[s][3];
      const int nfb = c0 + c1 + c2 + c3;
      const uint32_t sbuf = smem_u32(dsm) + s * KT_CHUNK_BYTES;
      for (int f0 = 0; f0 < nfb; f0 += 8) {
        const int f = f0 + 2 * g + fw;
        int t2 = -1;
        if (f < nfb) {
          const int w = f < c0 ? 0 : f < c0 + c1 ? 1 : f < c0 + c1 + c2 ? 2 : 3;
          const int base = w == 0 ? 0 : w == 1 ? c0 : w == 2 ? c0 + c1 : c0 + c1 + c2;
          t2 = sfb[s][w][f - base];
        }
        float d = INFINITY;
        if (t2 >= 0 && j < k) {
          const float4 *cj = reinterpret_cast<const float4 *>(&scent[j][0]);
          float a = 0.0f;
          // channel order (the pinned chain); the next 8 channels' operands
          // are loaded while the current ones are accumulated
          uint4 w = lds128(sbuf + kt_off(t2, 0));
          float4 cA = cj[0], cB = cj[1];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            uint4 wn = w;
            float4 cAn = cA, cBn = cB;
            if (q < 15) {
              wn = lds128(sbuf + kt_off(t2, q + 1));
              cAn = cj[2 * q + 2];
              cBn = cj[2 * q + 3];
            }
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
            const float cc[8] = {cA.x, cA.y, cA.z, cA.w, cB.x, cB.y, cB.z, cB.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float v = (e & 1) ? __uint_as_float(ws[e >> 1] & 0xFFFF0000u) : __uint_as_float(ws[e >> 1] << 16);
              const float x = __fsub_rn(v, cc[e]);
              a = fmaf(x, x, a);
            }
            w = wn;
            cA = cAn;
            cB = cBn;
          }
          d = a;
        }
        int jmin = j < k ? j : 8;
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {  // within the lane group
          const float d2 = __shfl_xor_sync(0xFFFFFFFFu, d, o);
          const int j2 = __shfl_xor_sync(0xFFFFFFFFu, jmin, o);
          if (d2 < d || (d2 == d && j2 < jmin)) {
            d = d2;
            jmin = j2;
          }
        }
        if (j == 0 && t2 >= 0) {
          slab[s][t2] = static_cast<int8_t>(jmin);
          labels[static_cast<size_t>(bh) * N + n0 + t2] = jmin;
        }
      }
      __syncwarp();
      mbar_arrive(&bars.fbd[s]);
    }
  } else if (warp < 8) {
    // ---- label warps: one token per thread, TMEM lane = token
    const int tok = tid - 128, lw = warp - 4;
    for (int i = 0; i < nchunk; ++i) {
      const int s = i % KS;
      const int n0 = n_begin + i * TILE, cnt = min(TILE, n_end - n0);
      const uint32_t sbuf = smem_u32(dsm) + s * KT_CHUNK_BYTES;
      const bool w_ok = mbar_wait(&bars.mma[s], (i / KS) & 1);
      if (!__all_sync(0xFFFFFFFFu, w_ok)) {
        if (lane == 0) atomicOr(status, ST_TIMEOUT);
        s_fail = 1;
        break;
      }
      tc_fence_after();
      uint32_t dr[16];
      kt_ld16(tmem + (static_cast<uint32_t>(lw * 32) << 16) + 16u * s, dr);
      tmem_wait_ld();
      tc_fence_before();
      if (tid == 128) s_mma_seen = i + 1;
      int lab = 0;
      bool fallback = false;
      if (tok < cnt && k > 1) {
        // |v|^2: eight partial sums (16-byte chunk q into sum q % 8), then
        // added pairwise (any order keeps its rounding inside the bound)
        float vh[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) vh[q] = 0.0f;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const uint4 w = lds128(sbuf + kt_off(tok, q));
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = __uint_as_float(ws[e] << 16), x1 = __uint_as_float(ws[e] & 0xFFFF0000u);
            vh[q & 7] = fmaf(x0, x0, vh[q & 7]);
            vh[q & 7] = fmaf(x1, x1, vh[q & 7]);
          }
        }
        const float vv = __fadd_rn(__fadd_rn(__fadd_rn(vh[0], vh[1]), __fadd_rn(vh[2], vh[3])),
                                   __fadd_rn(__fadd_rn(vh[4], vh[5]), __fadd_rn(vh[6], vh[7])));
        float e[8];
        float best = INFINITY;
        int jb = 0;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const float dot = __fadd_rn(__uint_as_float(dr[jj]), __uint_as_float(dr[8 + jj]));
          e[jj] = __fsub_rn(__fadd_rn(vv, scc[jj]), 2.0f * dot);
          if (jj < k && e[jj] < best) {
            best = e[jj];
            jb = jj;
          }
        }
        lab = jb;
        const float bnd_b = 1.220703125e-4f * __fadd_rn(vv, scc[jb]);  // E_j = 2^-13 (|v|^2 + |c_j|^2)
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
          if (jj < k && jj != jb &&
              !(__fsub_rn(e[jj], best) > __fadd_rn(bnd_b, 1.220703125e-4f * __fadd_rn(vv, scc[jj]))))
            fallback = true;
      }
      slab[s][tok] = (tok < cnt && !fallback) ? static_cast<int8_t>(lab) : static_cast<int8_t>(-1);
      if (tok < cnt && !fallback) labels[static_cast<size_t>(bh) * N + n0 + tok] = lab;
      const unsigned fbm = __ballot_sync(0xFFFFFFFFu, fallback);
      if (fallback) sfb[s][lw][__popc(fbm & ((1u << lane) - 1u))] = static_cast<uint8_t>(tok);
      if (lane == 0) snfb[s][lw] = __popc(fbm);
      mbar_arrive(&bars.lab[s]);
    }
  } else {
    // ---- sum warps: warp 8 + j adds the first half of the chunk's tokens
    // labelled j and the second half of those labelled j ^ 4 (the halves split
    // at a multiple of four), so a large cluster is shared by two warps
    const int j = warp - 8, jb = j ^ 4;
    // fp64 sums of list positions [from, to) (from a multiple of 4), four rows
    // per step loaded together; the sums are exact, so the order does not
    // change them
    auto add_list = [&](const uint8_t *list, int from, int to, uint32_t sbuf, double (&acc)[4]) {
      double o[4] = {0.0, 0.0, 0.0, 0.0};
      for (int n = from; n < to; n += 4) {
        const uint32_t t4 = *reinterpret_cast<const uint32_t *>(list + n);  // four listed tokens
        uint2 w4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)  // (entries past the range are read, masked to a row of the chunk, dropped)
          w4[u] = lds64_nc(sbuf + kt_off((t4 >> (8 * u)) & 0x7Fu, lane >> 1) + 8 * (lane & 1));
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (n + u >= to) break;
          double *a = (u & 1) ? o : acc;
          a[0] += static_cast<double>(__uint_as_float(w4[u].x << 16));
          a[1] += static_cast<double>(__uint_as_float(w4[u].x & 0xFFFF0000u));
          a[2] += static_cast<double>(__uint_as_float(w4[u].y << 16));
          a[3] += static_cast<double>(__uint_as_float(w4[u].y & 0xFFFF0000u));
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[c] += o[c];
    };
    auto split = [](int c) { return min(c, (((c + 1) >> 1) + 3) & ~3); };  // first-half length
    for (int i = 0; i < nchunk; ++i) {
      const int s = i % KS;
      const int n0 = n_begin + i * TILE, cnt = min(TILE, n_end - n0);
      const uint32_t sbuf = smem_u32(dsm) + s * KT_CHUNK_BYTES;
      if (!mbar_wait(&bars.fbd[s], (i / KS) & 1)) {
        if (lane == 0) atomicOr(status, ST_TIMEOUT);
        s_fail = 1;
        break;
      }
      if (accumulate) {
        // the chunk's tokens of clusters j and jb, each listed in token order
        int ca = 0, cb = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int l = 32 * q + lane < cnt ? slab[s][32 * q + lane] : -1;
          const unsigned ba = __ballot_sync(0xFFFFFFFFu, l == j), bb = __ballot_sync(0xFFFFFFFFu, l == jb);
          const unsigned below = (1u << lane) - 1u;
          if (l == j) sidx[j][0][ca + __popc(ba & below)] = static_cast<uint8_t>(32 * q + lane);
          if (l == jb) sidx[j][1][cb + __popc(bb & below)] = static_cast<uint8_t>(32 * q + lane);
          ca += __popc(ba);
          cb += __popc(bb);
        }
        __syncwarp();
        if (j < k) {
          cnt_own += ca;
          add_list(sidx[j][0], 0, split(ca), sbuf, acc4);
        }
        if (jb < k) add_list(sidx[j][1], split(cb), cb, sbuf, accB);
        __syncwarp();  // the lists are rewritten for the next chunk
      } else if (j < k) {
        // the label pass: count the chunk's tokens of cluster j (the
        // permutation's scatter places each block's tokens from these counts)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          cnt_own += __popc(__ballot_sync(0xFFFFFFFFu, 32 * q + lane < cnt && slab[s][32 * q + lane] == j));
      }
      __syncwarp();
      mbar_arrive(&bars.empty[s]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (s_fail && tid == 0) {
    // a wait ran out: let the copies and products still in flight land before
    // the block leaves (bounded waits, again)
    for (int i = s_tma_seen; i < s_tma_issued; ++i)
      if (!mbar_wait(&bars.full[i % KS], (i / KS) & 1)) break;
    for (int i = s_mma_seen; i < s_mma_issued; ++i)
      if (!mbar_wait(&bars.mma[i % KS], (i / KS) & 1)) break;
  }
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 64);
  if (!accumulate) {
    if (warp >= 8 && warp - 8 < k && lane == 0) pcnt[(static_cast<size_t>(bh) * nblk + blk) * k + warp - 8] = cnt_own;
    return;
  }
  // each cluster's second halves go to its own sum warp over the chunk ring,
  // free now (every copy has landed and every read is done: barriers above)
  double *hand = reinterpret_cast<double *>(dsm);  // [cluster][channel]
  if (warp >= 8 && ((warp - 8) ^ 4) < k)
    *reinterpret_cast<double4 *>(hand + ((warp - 8) ^ 4) * D + 4 * lane) = make_double4(accB[0], accB[1], accB[2], accB[3]);
  __syncthreads();
  double *ps = psum + (static_cast<size_t>(bh) * nblk + blk) * k * D;
  int *pc = pcnt + (static_cast<size_t>(bh) * nblk + blk) * k;
  if (warp >= 8 && warp - 8 < k) {
    const double4 h = *reinterpret_cast<const double4 *>(hand + (warp - 8) * D + 4 * lane);
    *reinterpret_cast<double4 *>(ps + (warp - 8) * D + 4 * lane) =
        make_double4(acc4[0] + h.x, acc4[1] + h.y, acc4[2] + h.z, acc4[3] + h.w);
    if (lane == 0) pc[warp - 8] = cnt_own;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&counter[bh], 1u) == static_cast<unsigned>(nblk - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // every (cluster, channel) of the head: partial sums added in block order
  {
    const int c = tid & 127;
    for (int j = tid >> 7; j < k; j += KM_THREADS / 128) {
      double sum = 0.0;
      long long n = 0;
#pragma unroll 16
      for (int b = 0; b < nblk; ++b) {
        sum += __ldcg(psum + ((static_cast<size_t>(bh) * nblk + b) * k + j) * D + c);
        n += __ldcg(pcnt + (static_cast<size_t>(bh) * nblk + b) * k + j);
      }
      if (n > 0) cent_h[j * D + c] = static_cast<float>(sum / static_cast<double>(n));
    }
  }
  if (tid == 0) counter[bh] = 0u;
}

}  // namespace vc
