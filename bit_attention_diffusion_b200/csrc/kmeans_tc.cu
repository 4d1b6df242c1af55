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
// cluster, so no tie arises); otherwise the token goes on a list whose pinned
// chains (all clusters) the block's warps then run, one token per warp at a
// time. Labels are therefore exactly k_kmeans_pass's.
//
// Per block: `cpb` consecutive 128-token chunks of one (b,h), double-buffered
// in shared memory by TMA in the K-major 128-byte-swizzled layout the MMA
// reads (two 64-channel atoms per chunk). The product of chunk i+1 goes to the
// tensor cores, into the second of two 16-column accumulators, while chunk i
// is labelled: all 256 threads compute the tokens' |v|^2, then warps 0-3 take
// one token each (TMEM lane = token). In an update pass warp j then adds, in
// fp64, the channels of the chunk's tokens labelled j (lane l: channels 4l ..
// 4l+3; exact, so the order is free), and the last block of a (b,h) adds the
// blocks' partial sums in block order into the new centroids.
#include "common.cuh"
#include "prologue.cuh"
#include "sm100.cuh"

namespace vc {

namespace {

constexpr int KT_CHUNK_BYTES = TILE * D * 2;                     // 32 KB: two 16 KB atoms
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

}  // namespace

__global__ void __launch_bounds__(256, 3) k_kmeans_pass8tc(const __grid_constant__ CUtensorMap tmV, int N, int k,
                                                           int cpb, int nblk, float *__restrict__ cent,
                                                        int32_t *__restrict__ labels, double *__restrict__ psum,
                                                        int *__restrict__ pcnt, unsigned *__restrict__ counter,
                                                        int accumulate, uint32_t *__restrict__ status) {
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t *dsm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sB = dsm + 2 * KT_CHUNK_BYTES;        // B operand: rows 0-7 hi(c_j), 8-15 lo(c_j); two 2 KB atoms
  __shared__ float scc[8];                       // |c_j|^2
  __shared__ float svv[2][TILE];                 // |v|^2 over channels 0-63 / 64-127
  __shared__ int slab[TILE];
  __shared__ int sfb[TILE];                      // tokens the estimate cannot decide
  __shared__ int s_nfb;
  __shared__ int s_last;
  __shared__ uint32_t s_tmem;
  __shared__ uint64_t mbar[2], full[2];
  const int bh = blockIdx.y, blk = blockIdx.x, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  float *cent_h = cent + static_cast<size_t>(bh) * k * D;

  const int n_begin = blk * cpb * TILE;
  const int n_end = min(N, n_begin + cpb * TILE);
  const int nchunk = (n_end - n_begin + TILE - 1) / TILE;
  const int row_base = bh * N + n_begin;  // map row of the block's first token
  if (tid == 0) {
    mbar_init(&mbar[0], 1);
    mbar_init(&mbar[1], 1);
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_mbar_init();
    prefetch_tmap(&tmV);
    for (int i = 0; i < 2 && i < nchunk; ++i) kt_load_chunk(dsm + i * KT_CHUNK_BYTES, &tmV, &full[i], row_base + i * TILE);
  }

  // centroids: the bf16 hi/lo operand and |c_j|^2 (the pinned chains read
  // the fp32 centroids from global memory, through L1)
  for (int i = tid; i < 16 * 16; i += 256) {  // 16 rows x 16 chunks of 8 channels
    const int row = i >> 4, ch16 = i & 15, j = row & 7;
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
  }
  {
    // |c_j|^2 in fp64, warp j (8 warps)
    const int j = warp;
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
  if (warp == 0) tmem_alloc(&s_tmem, 32);
  if (tid == 0) s_nfb = 0;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint64_t dB = sdesc_sw128(smem_u32(sB), 16, 1024);
  // v . hi(c_j), v . lo(c_j) of chunk `ci` (landed) into D(ci % 2): columns 16 (ci % 2) ..
  auto issue_mma = [&](int ci) {
    const uint64_t dA = sdesc_sw128(smem_u32(dsm + (ci & 1) * KT_CHUNK_BYTES), 16, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_f16_ss(tmem + 16u * (ci & 1), dA + (kk >> 2) * ((TILE * 128) >> 4) + 2 * (kk & 3),
                 dB + (kk >> 2) * (2048 >> 4) + 2 * (kk & 3), KT_IDESC, kk > 0);
    mma_commit(&mbar[ci & 1]);
  };
  bool ok = true;
  if (tid == 0 && nchunk > 0) {
    ok = mbar_wait(&full[0], 0);
    if (ok) {
      tc_fence_after();
      issue_mma(0);
    } else {
      atomicOr(status, ST_TIMEOUT);
    }
  }

  // sums: warp j < k owns cluster j, lane l channels 4l .. 4l+3
  double acc4[4] = {0.0, 0.0, 0.0, 0.0};
  int cnt_own = 0;  // tokens of cluster `warp` (lane 0)
  for (int i = 0; i < nchunk; ++i) {
    const int n0 = n_begin + i * TILE, cnt = min(TILE, n_end - n0);
    uint8_t *buf = dsm + (i & 1) * KT_CHUNK_BYTES;
    // the chunk has landed (its product was issued when it did)
    const bool landed = ok && mbar_wait(&full[i & 1], (i >> 1) & 1);
    if (!__syncthreads_and(landed)) {
      if (tid == 0) atomicOr(status, ST_TIMEOUT);
      ok = false;
    }
    {
      // |v|^2 of token tid % 128 over channels [64 h, 64 h + 64), h = tid / 128
      const int t = tid & 127, h = tid >> 7;
      float a = 0.0f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 w = *reinterpret_cast<const uint4 *>(buf + kt_off(t, 8 * h + q));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = __uint_as_float(ws[e] << 16), x1 = __uint_as_float(ws[e] & 0xFFFF0000u);
          a = fmaf(x0, x0, a);
          a = fmaf(x1, x1, a);
        }
      }
      svv[h][t] = a;
    }
    __syncthreads();
    if (warp < 4) {
      const int tok = tid;  // TMEM lane tid
      const bool w_ok = ok && mbar_wait(&mbar[i & 1], (i >> 1) & 1);
      if (!__all_sync(0xFFFFFFFFu, w_ok)) {
        if (lane == 0) atomicOr(status, ST_TIMEOUT);
        ok = false;
      }
      tc_fence_after();
      uint32_t dr[16];
      kt_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + 16u * (i & 1), dr);
      tmem_wait_ld();
      tc_fence_before();
      int lab = 0;
      bool fallback = false;
      if (tok < cnt && k > 1) {
        const float vv = __fadd_rn(svv[0][tok], svv[1][tok]);
        float e[8], bnd[8];
        float best = INFINITY;
        int jb = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float dot = __fadd_rn(__uint_as_float(dr[j]), __uint_as_float(dr[8 + j]));
          e[j] = __fsub_rn(__fadd_rn(vv, scc[j]), 2.0f * dot);
          bnd[j] = 1.220703125e-4f * __fadd_rn(vv, scc[j]);  // E_j = 2^-13 (|v|^2 + |c_j|^2)
          if (j < k && e[j] < best) {
            best = e[j];
            jb = j;
          }
        }
        lab = jb;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < k && j != jb && !(__fsub_rn(e[j], best) > __fadd_rn(bnd[jb], bnd[j]))) fallback = true;
      }
      if (tok < cnt && !fallback) {
        slab[tok] = lab;
        labels[static_cast<size_t>(bh) * N + n0 + tok] = lab;
      }
      const unsigned fbm = __ballot_sync(0xFFFFFFFFu, fallback);
      int at = 0;
      if (lane == 0 && fbm) at = atomicAdd(&s_nfb, __popc(fbm));
      at = __shfl_sync(0xFFFFFFFFu, at, 0);
      if (fallback) sfb[at + __popc(fbm & ((1u << lane) - 1u))] = tok;
      if (warp == 0 && i + 1 < nchunk) {
        // the next chunk's product, into the other accumulator
        bool nxt = true;
        if (lane == 0) {
          nxt = ok && mbar_wait(&full[(i + 1) & 1], ((i + 1) >> 1) & 1);
          if (nxt) {
            tc_fence_after();
            issue_mma(i + 1);
          } else {
            atomicOr(status, ST_TIMEOUT);
          }
        }
        if (!__shfl_sync(0xFFFFFFFFu, nxt, 0)) ok = false;
      }
    }
    __syncthreads();
    {
      // ---- the pinned distances for the undecided tokens, one token per warp
      // at a time: lane j < k runs cluster j's chain over the channels in
      // order, then the warp takes the smallest (ties to the lowest cluster)
      const int nfb = s_nfb;
      for (int f = warp; f < nfb; f += 8) {
        const int t2 = sfb[f];
        float d = INFINITY;
        if (lane < k) {
          const float4 *cj = reinterpret_cast<const float4 *>(cent_h + lane * D);
          float a = 0.0f;
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const uint4 w = *reinterpret_cast<const uint4 *>(buf + kt_off(t2, q));
            const float4 c0 = cj[2 * q], c1 = cj[2 * q + 1];
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
            const float cc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float v = (e & 1) ? __uint_as_float(ws[e >> 1] & 0xFFFF0000u) : __uint_as_float(ws[e >> 1] << 16);
              const float x = __fsub_rn(v, cc[e]);
              a = fmaf(x, x, a);
            }
          }
          d = a;
        }
        int jmin = lane < k ? lane : 8;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float d2 = __shfl_xor_sync(0xFFFFFFFFu, d, o);
          const int j2 = __shfl_xor_sync(0xFFFFFFFFu, jmin, o);
          if (d2 < d || (d2 == d && j2 < jmin)) {
            d = d2;
            jmin = j2;
          }
        }
        if (lane == 0) {
          slab[t2] = jmin;
          labels[static_cast<size_t>(bh) * N + n0 + t2] = jmin;
        }
      }
    }
    if (accumulate) {
      __syncthreads();  // every label of the chunk is in slab
      // ---- fp64 sums: warp j adds the tokens labelled j, lane l its channels
      // 4l .. 4l+3 (exact, so the order is free)
      const int j = warp;
      if (j < k) {
        unsigned m[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) m[q] = __ballot_sync(0xFFFFFFFFu, 32 * q + lane < cnt && slab[32 * q + lane] == j);
        cnt_own += __popc(m[0]) + __popc(m[1]) + __popc(m[2]) + __popc(m[3]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          unsigned mm = m[q];
          while (mm) {
            const int t = 32 * q + __ffs(mm) - 1;
            mm &= mm - 1;
            const uint2 w = *reinterpret_cast<const uint2 *>(buf + kt_off(t, lane >> 1) + 8 * (lane & 1));
            acc4[0] += static_cast<double>(__uint_as_float(w.x << 16));
            acc4[1] += static_cast<double>(__uint_as_float(w.x & 0xFFFF0000u));
            acc4[2] += static_cast<double>(__uint_as_float(w.y << 16));
            acc4[3] += static_cast<double>(__uint_as_float(w.y & 0xFFFF0000u));
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // every read of this buffer and of D is done
    tc_fence_after();
    if (tid == 0) {
      s_nfb = 0;
      if (ok && i + 2 < nchunk) kt_load_chunk(buf, &tmV, &full[i & 1], row_base + (i + 2) * TILE);
    }
  }
  if (warp == 0) tmem_dealloc(tmem, 32);
  if (!accumulate) return;
  double *ps = psum + (static_cast<size_t>(bh) * nblk + blk) * k * D;
  int *pc = pcnt + (static_cast<size_t>(bh) * nblk + blk) * k;
  if (warp < k) {
    *reinterpret_cast<double4 *>(ps + warp * D + 4 * lane) = make_double4(acc4[0], acc4[1], acc4[2], acc4[3]);
    if (lane == 0) pc[warp] = cnt_own;
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
    for (int j = tid >> 7; j < k; j += 2) {
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
