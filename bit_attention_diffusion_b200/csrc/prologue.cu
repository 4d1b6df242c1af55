// prologue.cu - the HBM-bound steps before the attention kernel:
//   V-Smooth Group   k-means over value tokens + stable sort into the permutation
//   Q/K smoothing    per-(b,h) channel mean of K, 8-bit block quantization of Q, K'
//   V-Smooth Demean  block means, per-channel power-of-two residual scale,
//                    E4M3 residual codes (channel-major), token errors
//   rho-repair       top-R tokens by error, bf16 correction of their residual
// Sources: page "VC-Attention acelera atenção em modelos de vídeo de IA em até
// 3,58× sem retreinamento", sections "V-Smooth: corrigindo outliers de valor"
// (Group, Demean) and "Por que a atenção é o gargalo" (Q/K smoothing as prior
// art); page "VC-Attention et FLUX 3 accélèrent la génération d'images sur
// Blackwell", section "Le compromis entre vitesse et fidélité" (rho = 0.005).
#include "common.cuh"
#include "sm100.cuh"
#include "prologue.cuh"

namespace vc {

// ============================================================== k-means
// Init c_j = V[floor(j*N/k)].
__device__ __forceinline__ void kmeans_init_body(const uint16_t *__restrict__ V, int N, int k, float *__restrict__ cent, int bx, int by, int bz) {
  const int bh = bx;
  for (int j = 0; j < k; ++j) {
    const long long src = (static_cast<long long>(j) * N) / k;
    cent[(static_cast<size_t>(bh) * k + j) * D + threadIdx.x] =
        bf16_to_f32(V[(static_cast<size_t>(bh) * N + src) * D + threadIdx.x]);
  }
}
__global__ void k_kmeans_init(const uint16_t *__restrict__ V, int N, int k, float *__restrict__ cent) {
  kmeans_init_body(V, N, k, cent, blockIdx.x, blockIdx.y, blockIdx.z);
}

// One Lloyd pass over `cpb` consecutive 128-token chunks per block: assign
// labels (fp32 fma distances in channel order, ties to the lowest cluster) and,
// when `accumulate`, the block's fp64 per-cluster sums; the last block of a
// (b,h) reduces all blocks' sums in block order and writes the new centroids.
constexpr int KM_ROW_WORDS = 66;  // 128 bf16 = 64 words, padded to 66 (bank spread)

__global__ void __launch_bounds__(128) k_kmeans_pass(const uint16_t *__restrict__ V, int N, int k, int cpb,
                                                     int nblk, float *__restrict__ cent,
                                                     int32_t *__restrict__ labels, double *__restrict__ psum,
                                                     int *__restrict__ pcnt, unsigned *__restrict__ counter,
                                                     int accumulate) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t *sv = reinterpret_cast<uint32_t *>(smem);                       // 128 x 66 words
  float *scent = reinterpret_cast<float *>(smem + TILE * KM_ROW_WORDS * 4); // k x 128
  double *ssum = reinterpret_cast<double *>(scent + k * D);                // k x 128
  __shared__ int slab[TILE];
  __shared__ int scnt[64];
  __shared__ int s_last;

  const int bh = blockIdx.y, blk = blockIdx.x, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const uint16_t *Vh = V + static_cast<size_t>(bh) * N * D;
  float *cent_h = cent + static_cast<size_t>(bh) * k * D;

  for (int i = tid; i < k * D; i += TILE) scent[i] = cent_h[i];
  if (accumulate) {
    for (int i = tid; i < k * D; i += TILE) ssum[i] = 0.0;
    if (tid < 64) scnt[tid] = 0;
  }
  const int n_begin = blk * cpb * TILE;
  const int n_end = min(N, n_begin + cpb * TILE);
  for (int n0 = n_begin; n0 < n_end; n0 += TILE) {
    const int cnt = min(TILE, n_end - n0);
    __syncthreads();
    // coalesced load of the chunk: a warp reads one 256-byte row, 8 bytes per lane
    for (int r = warp; r < cnt; r += 4) {
      const uint2 w = *reinterpret_cast<const uint2 *>(Vh + static_cast<size_t>(n0 + r) * D + 4 * lane);
      sv[r * KM_ROW_WORDS + 2 * lane] = w.x;
      sv[r * KM_ROW_WORDS + 2 * lane + 1] = w.y;
    }
    __syncthreads();
    if (tid < cnt) {
      const uint32_t *row = sv + tid * KM_ROW_WORDS;
      int best = 0;
      float bestd = 0.0f;
      for (int j0 = 0; j0 < k; j0 += 8) {
        float acc[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) acc[jj] = 0.0f;
        for (int w = 0; w < 64; ++w) {
          const uint32_t pr = row[w];
          const float x0 = __uint_as_float(pr << 16), x1 = __uint_as_float(pr & 0xFFFF0000u);
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            if (j0 + jj < k) {
              const float d0 = __fsub_rn(x0, scent[(j0 + jj) * D + 2 * w]);
              acc[jj] = __fmaf_rn(d0, d0, acc[jj]);
              const float d1 = __fsub_rn(x1, scent[(j0 + jj) * D + 2 * w + 1]);
              acc[jj] = __fmaf_rn(d1, d1, acc[jj]);
            }
          }
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int j = j0 + jj;
          if (j < k && (j == 0 || acc[jj] < bestd)) {
            bestd = acc[jj];
            best = j;
          }
        }
      }
      slab[tid] = best;
      labels[static_cast<size_t>(bh) * N + n0 + tid] = best;
    }
    if (accumulate) {
      __syncthreads();
      // thread = channel: sums in token order, no write conflicts
      const int c = tid;
      const int wsel = c >> 1;
      const bool hi = c & 1;
      for (int r = 0; r < cnt; ++r) {
        const uint32_t pr = sv[r * KM_ROW_WORDS + wsel];
        const float x = hi ? __uint_as_float(pr & 0xFFFF0000u) : __uint_as_float(pr << 16);
        ssum[slab[r] * D + c] += static_cast<double>(x);
      }
      if (tid == 0)
        for (int r = 0; r < cnt; ++r) scnt[slab[r]] += 1;
    }
  }
  if (!accumulate) return;
  __syncthreads();
  double *ps = psum + (static_cast<size_t>(bh) * nblk + blk) * k * D;
  int *pc = pcnt + (static_cast<size_t>(bh) * nblk + blk) * k;
  for (int i = tid; i < k * D; i += TILE) ps[i] = ssum[i];
  if (tid < k) pc[tid] = scnt[tid];
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&counter[bh], 1u) == static_cast<unsigned>(nblk - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // last block of this (b,h): reduce in block order, new centroids
  for (int j = 0; j < k; ++j) {
    double s = 0.0;
    long long n = 0;
#pragma unroll 16
    for (int b = 0; b < nblk; ++b) {  // loads batched by the unroll, sums kept in block order
      s += __ldcg(psum + ((static_cast<size_t>(bh) * nblk + b) * k + j) * D + tid);
      n += __ldcg(pcnt + (static_cast<size_t>(bh) * nblk + b) * k + j);
    }
    if (n > 0) cent_h[j * D + tid] = static_cast<float>(s / static_cast<double>(n));
  }
  if (tid == 0) counter[bh] = 0u;
}

// The Lloyd pass for k <= 8 inside the one-launch prologue (the separate
// launch uses k_kmeans_pass8tc), same arithmetic per (token,
// cluster) as k_kmeans_pass: d = fp32(v - c) and acc = fma(d, d, acc) in
// channel order, two clusters per packed f32x2 instruction (each lane rounds
// exactly like the scalar instruction). 256 threads; the block's 128-token
// chunks are double-buffered in shared memory with cp.async (272-byte rows).
// Labels: two threads per token (clusters 0-3 and 4-7), centroids
// channel-major in shared memory ([c][8]); the halves combine with ties to the
// lower cluster. Sums: the chunk's tokens are sorted by label (stable, by
// ballots), then thread (channel pair, quarter) adds its two channels of the
// tokens of each label in fp64 registers; exact, so the order is free.
constexpr int KM8_ROW_BYTES = 272;
static_assert(KMEANS8_SMEM == 2 * TILE * KM8_ROW_BYTES, "chunk buffers");

__device__ __forceinline__ void sub_fma2(float x, float c0, float c1, float &a0, float &a1) {
  asm("{\n\t.reg .b64 xx, cc, dd, aa;\n\t"
      "mov.b64 xx, {%2, %2};\n\tmov.b64 cc, {%3, %4};\n\tmov.b64 aa, {%0, %1};\n\t"
      "sub.rn.f32x2 dd, xx, cc;\n\t"
      "fma.rn.f32x2 aa, dd, dd, aa;\n\t"
      "mov.b64 {%0, %1}, aa;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(x), "f"(c0), "f"(c1));
}

__device__ __forceinline__ void km8_load_chunk(uint8_t *buf, const uint16_t *Vh, int n0, int cnt) {
  const int g = threadIdx.x >> 4, c = threadIdx.x & 15;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = g + 16 * i;
    if (rr < cnt)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(
                       __cvta_generic_to_shared(buf + rr * KM8_ROW_BYTES + 16 * c))),
                   "l"(Vh + static_cast<size_t>(n0 + rr) * D + 8 * c)
                   : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void kmeans_pass8_body(const uint16_t *__restrict__ V, int N, int k, int cpb,
                                                      int nblk, float *__restrict__ cent,
                                                      int32_t *__restrict__ labels, double *__restrict__ psum,
                                                      int *__restrict__ pcnt, unsigned *__restrict__ counter,
                                                      int accumulate, int bx, int by, int bz) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ __align__(16) float scent[D * 8];  // [c][j]; j >= k unused
  __shared__ int slab[TILE];
  __shared__ int slist[TILE];
  __shared__ int sstart[9];
  __shared__ int s_last;
  const int bh = by, blk = bx, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const uint16_t *Vh = V + static_cast<size_t>(bh) * N * D;
  float *cent_h = cent + static_cast<size_t>(bh) * k * D;
  for (int i = tid; i < D * 8; i += 256) {
    const int c = i >> 3, j = i & 7;
    scent[i] = j < k ? cent_h[j * D + c] : 0.0f;
  }
  const int n_begin = blk * cpb * TILE;
  const int n_end = min(N, n_begin + cpb * TILE);
  const int nchunk = (n_end - n_begin + TILE - 1) / TILE;
  if (nchunk > 0) km8_load_chunk(dsm, Vh, n_begin, min(TILE, n_end - n_begin));
  double acc[8][2];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = 0.0;
  int cntj[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // tokens per label (thread 0)
  const int tok = warp * 16 + (lane & 15), half = lane >> 4;
  const int cp = tid & 63, qtr = tid >> 6;
  for (int i = 0; i < nchunk; ++i) {
    const int n0 = n_begin + i * TILE, cnt = min(TILE, n_end - n0);
    uint8_t *buf = dsm + (i & 1) * TILE * KM8_ROW_BYTES;
    if (i + 1 < nchunk) {
      km8_load_chunk(dsm + ((i + 1) & 1) * TILE * KM8_ROW_BYTES, Vh, n0 + TILE, min(TILE, n_end - n0 - TILE));
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    // ---- labels: this thread's four clusters 4*half .. 4*half+3 for token tok
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    if (tok < cnt) {
      const uint8_t *row = buf + tok * KM8_ROW_BYTES;
#pragma unroll 4
      for (int g8 = 0; g8 < 16; ++g8) {
        const uint4 w = *reinterpret_cast<const uint4 *>(row + 16 * g8);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = 8 * g8 + 2 * h + e;
            const float x = e ? __uint_as_float(ws[h] & 0xFFFF0000u) : __uint_as_float(ws[h] << 16);
            const float4 cc = *reinterpret_cast<const float4 *>(&scent[c * 8 + 4 * half]);
            sub_fma2(x, cc.x, cc.y, a0, a1);
            sub_fma2(x, cc.z, cc.w, a2, a3);
          }
        }
      }
    }
    const float av[4] = {a0, a1, a2, a3};
    int best = -1;
    float bestd = 0.0f;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j = 4 * half + jj;
      if (j < k && (best < 0 || av[jj] < bestd)) {
        bestd = av[jj];
        best = j;
      }
    }
    const float od = __shfl_xor_sync(0xFFFFFFFFu, bestd, 16);
    const int oj = __shfl_xor_sync(0xFFFFFFFFu, best, 16);
    // lower half first; the upper half wins only with a strictly smaller distance
    const float dlo = half ? od : bestd, dhi = half ? bestd : od;
    const int jlo = half ? oj : best, jhi = half ? best : oj;
    const int lab = (jhi >= 0 && dhi < dlo) ? jhi : jlo;
    if (half == 0 && tok < cnt) {
      slab[tok] = lab;
      labels[static_cast<size_t>(bh) * N + n0 + tok] = lab;
    }
    if (accumulate) {
      __syncthreads();
      // ---- stable sort of the chunk's tokens by label (warp 0)
      if (warp == 0) {
        int lm[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) lm[m] = (32 * m + lane < cnt) ? slab[32 * m + lane] : -1;
        const unsigned lt = (1u << lane) - 1u;
        int base = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j >= k) break;
          unsigned bm[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) bm[m] = __ballot_sync(0xFFFFFFFFu, lm[m] == j);
          if (lane == 0) sstart[j] = base;
          int pre = base;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            if (lm[m] == j) slist[pre + __popc(bm[m] & lt)] = 32 * m + lane;
            pre += __popc(bm[m]);
          }
          if (lane == 0) cntj[j] += pre - base;
          base = pre;
        }
        if (lane == 0) sstart[k] = base;
      }
      __syncthreads();
      // ---- fp64 sums: thread (channel pair cp, quarter qtr)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k) {
          const int e1 = sstart[j + 1];
          for (int ii = sstart[j] + qtr; ii < e1; ii += 4) {
            const uint32_t pr = *reinterpret_cast<const uint32_t *>(buf + slist[ii] * KM8_ROW_BYTES + 4 * cp);
            acc[j][0] += static_cast<double>(__uint_as_float(pr << 16));
            acc[j][1] += static_cast<double>(__uint_as_float(pr & 0xFFFF0000u));
          }
        }
      }
    }
    __syncthreads();  // the buffer is refilled by the load issued in the next iteration
  }
  if (!accumulate) return;
  // reduce the four quarters in shared memory (the chunk buffers are free now)
  double *red = reinterpret_cast<double *>(dsm);  // [4][8][128]
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    red[(qtr * 8 + j) * D + 2 * cp] = acc[j][0];
    red[(qtr * 8 + j) * D + 2 * cp + 1] = acc[j][1];
  }
  __syncthreads();
  double *ps = psum + (static_cast<size_t>(bh) * nblk + blk) * k * D;
  int *pc = pcnt + (static_cast<size_t>(bh) * nblk + blk) * k;
  for (int i = tid; i < k * D; i += 256) {
    const int j = i / D, c = i % D;
    ps[i] = red[(0 * 8 + j) * D + c] + red[(1 * 8 + j) * D + c] + red[(2 * 8 + j) * D + c] + red[(3 * 8 + j) * D + c];
  }
  if (tid == 0) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k) pc[j] = cntj[j];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&counter[bh], 1u) == static_cast<unsigned>(nblk - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // every (cluster, channel) of the head at once: thread (c = tid % 128,
  // cluster parity tid / 128) takes clusters j = parity, parity + 2, ...; the
  // partial sums are added in block order
  {
    const int c = tid & 127;
    for (int j = tid >> 7; j < k; j += 2) {
      double sum = 0.0;
      long long n = 0;
#pragma unroll 16
      for (int b = 0; b < nblk; ++b) {  // loads batched by the unroll
        sum += __ldcg(psum + ((static_cast<size_t>(bh) * nblk + b) * k + j) * D + c);
        n += __ldcg(pcnt + (static_cast<size_t>(bh) * nblk + b) * k + j);
      }
      if (n > 0) cent_h[j * D + c] = static_cast<float>(sum / static_cast<double>(n));
    }
  }
  if (tid == 0) counter[bh] = 0u;
}

// Stable counting sort of token indices by label, one block per (b,h): a
// histogram gives each label's start; then rounds of NT tokens scatter in
// order (rank among equal labels = earlier lanes of the warp + earlier warps).
template <int NT>
__device__ __forceinline__ void perm_sort_body(const int32_t *__restrict__ labels, int N, int k,
                                                    int32_t *__restrict__ perm, int bx, int by, int bz) {
  __shared__ int base[64];
  __shared__ int tot[64];
  __shared__ int wcnt[NT / 32][64];
  const int bh = bx, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t *lab = labels + static_cast<size_t>(bh) * N;
  int32_t *out = perm + static_cast<size_t>(bh) * N;
  if (tid < 64) base[tid] = 0;
  __syncthreads();
  for (int n = tid; n < N; n += NT) atomicAdd(&base[lab[n]], 1);
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int j = 0; j < k; ++j) {
      const int c = base[j];
      base[j] = run;
      run += c;
    }
  }
  for (int n0 = 0; n0 < N; n0 += NT) {
    for (int i = tid; i < (NT / 32) * 64; i += NT) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    const int n = n0 + tid;
    const int L = n < N ? lab[n] : -1;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, L);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (L >= 0 && rank == 0) wcnt[warp][L] = __popc(peers);
    __syncthreads();
    if (tid < k) {
      int run = 0;
      for (int w = 0; w < NT / 32; ++w) {
        const int c = wcnt[w][tid];
        wcnt[w][tid] = run;
        run += c;
      }
      tot[tid] = run;
    }
    __syncthreads();
    if (L >= 0) out[base[L] + wcnt[warp][L] + rank] = n;
    __syncthreads();
    if (tid < k) base[tid] += tot[tid];
  }
}
__global__ void __launch_bounds__(1024) k_perm_sort(const int32_t *__restrict__ labels, int N, int k,
                                                    int32_t *__restrict__ perm) {
  perm_sort_body<1024>(labels, N, k, perm, blockIdx.x, blockIdx.y, blockIdx.z);
}

// The same stable sort, spread over the k-means blocks of each (b,h) (k <= 8):
// block b of the Lloyd pass counted its tokens per label (pcnt[bh][b][j], the
// final label pass); label j's tokens of block b start at the tokens of the
// labels below j plus label j's tokens in the blocks before b, and the block
// scatters its own range [b cpb 128, (b+1) cpb 128) in rounds of 256 tokens.
__global__ void __launch_bounds__(256) k_perm_scatter(const int32_t *__restrict__ labels,
                                                      const int *__restrict__ pcnt, int N, int k, int cpb, int nblk,
                                                      int32_t *__restrict__ perm) {
  __shared__ int base[8], tot[8];
  __shared__ int wcnt[8][8];
  __shared__ int spc[PERM_SCATTER_MAX_BLOCKS * 8];  // the head's counts [block][label]
  const int blk = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_begin = blk * cpb * TILE, n_end = min(N, n_begin + cpb * TILE);
  const int32_t *lab = labels + static_cast<size_t>(bh) * N;
  int32_t *out = perm + static_cast<size_t>(bh) * N;
  const int *pc = pcnt + static_cast<size_t>(bh) * nblk * k;
  for (int i = tid; i < nblk * k; i += 256) spc[i] = pc[i];
  __syncthreads();
  if (warp < k) {
    // warp j: label j's tokens in all blocks (tot) and in the blocks before this one
    int all = 0, before = 0;
    for (int b = lane; b < nblk; b += 32) {
      const int c = spc[b * k + warp];
      all += c;
      if (b < blk) before += c;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      all += __shfl_xor_sync(0xFFFFFFFFu, all, o);
      before += __shfl_xor_sync(0xFFFFFFFFu, before, o);
    }
    if (lane == 0) {
      tot[warp] = all;
      base[warp] = before;
    }
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;  // tokens of the labels below j, all blocks
    for (int j = 0; j < k; ++j) {
      base[j] += run;
      run += tot[j];
    }
  }
  for (int n0 = n_begin; n0 < n_end; n0 += 256) {
    if (tid < 64) (&wcnt[0][0])[tid] = 0;
    __syncthreads();
    const int n = n0 + tid;
    const int L = n < n_end ? lab[n] : -1;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, L);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (L >= 0 && rank == 0) wcnt[warp][L] = __popc(peers);
    __syncthreads();
    if (tid < k) {
      int run = 0;
      for (int w = 0; w < 8; ++w) {
        const int c = wcnt[w][tid];
        wcnt[w][tid] = run;
        run += c;
      }
      tot[tid] = run;
    }
    __syncthreads();
    if (L >= 0) out[base[L] + wcnt[warp][L] + rank] = n;
    __syncthreads();
    if (tid < k) base[tid] += tot[tid];
  }
}

// ============================================================== streaming helpers
// The HBM-bound kernels below move a 128-row tile with 256 threads: thread
// (g, c) = (tid / 16, tid % 16) owns the 16-byte chunk c (channels 8c..8c+7)
// of rows g, g+16, ..., g+112, so every thread has eight independent 16-byte
// loads in flight and a warp covers two full rows per load.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void bf16x8(const uint4 &w, float *x) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(ws[i] << 16);
    x[2 * i + 1] = __uint_as_float(ws[i] & 0xFFFF0000u);
  }
}

// ============================================================== Q/K smoothing + quantization
// Channel sums of K in fp64 over a row range (one block per (chunk, b,h));
// the last block of a (b,h) adds the chunk sums in chunk order and writes the
// channel mean (0 without K smoothing).
__device__ __forceinline__ void kbar_body(const uint16_t *__restrict__ K, int N, int nchunk, int ksmooth,
                                              double *__restrict__ part, unsigned *__restrict__ counter,
                                              float *__restrict__ kbar, int bx, int by, int bz) {
  __shared__ double red[16][128];
  __shared__ int s_last;
  const int bh = by, ch = bx, tid = threadIdx.x;
  const int g = tid >> 4, c = tid & 15;
  const int rows = (N + nchunk - 1) / nchunk;
  const int r0 = ch * rows, r1 = min(N, r0 + rows);
  const uint16_t *Kh = K + static_cast<size_t>(bh) * N * D + 8 * c;
  double a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int r = r0 + g; r < r1; r += 64) {
    uint4 w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      w[u] = (r + 16 * u < r1) ? __ldg(reinterpret_cast<const uint4 *>(Kh + static_cast<size_t>(r + 16 * u) * D))
                               : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float x[8];
      bf16x8(w[u], x);
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] += static_cast<double>(x[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[g][8 * c + j] = a[j];
  __syncthreads();
  if (tid < 128) {
    double sum = 0.0;
#pragma unroll
    for (int i = 0; i < 16; ++i) sum += red[i][tid];
    part[(static_cast<size_t>(bh) * nchunk + ch) * D + tid] = sum;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&counter[bh], 1u) == static_cast<unsigned>(nchunk - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid < 128) {
    double sum = 0.0;
    for (int i = 0; i < nchunk; ++i) sum += __ldcg(part + (static_cast<size_t>(bh) * nchunk + i) * D + tid);
    kbar[static_cast<size_t>(bh) * D + tid] = ksmooth ? static_cast<float>(sum / static_cast<double>(N)) : 0.0f;
  }
  if (tid == 0) counter[bh] = 0u;
}
__global__ void __launch_bounds__(256) k_kbar(const uint16_t *__restrict__ K, int N, int nchunk, int ksmooth,
                                              double *__restrict__ part, unsigned *__restrict__ counter,
                                              float *__restrict__ kbar) {
  kbar_body(K, N, nchunk, ksmooth, part, counter, kbar, blockIdx.x, blockIdx.y, blockIdx.z);
}

// Block quantization: z = 0 -> Q rows [128t, 128t+128) in original order;
// z = 1 -> K rows perm[128t + r] minus the channel mean (z = blockIdx.z +
// zbase: one launch may take both, or Q and K separately). scale = amax/448,
// codes = E4M3(x * (448/amax)); rows past N get code 0.
__device__ __forceinline__ void qk_quant_body(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K,
                                                  const int32_t *__restrict__ perm, const float *__restrict__ kbar,
                                                  int N, int Npad, int zbase, uint8_t *__restrict__ q8,
                                                  float *__restrict__ sq, uint8_t *__restrict__ k8,
                                                  float *__restrict__ sk, int bx, int by, int bz) {
  __shared__ float wmax[8];
  const int t = bx, bh = by, z = bz + zbase;
  const int tid = threadIdx.x, g = tid >> 4, c = tid & 15;
  const int cnt = min(TILE, N - t * TILE);
  const uint16_t *src = (z == 0 ? Q : K) + static_cast<size_t>(bh) * N * D + 8 * c;
  int row[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = g + 16 * i, pos = t * TILE + rr;
    row[i] = rr < cnt ? ((z == 1 && perm != nullptr) ? __ldg(perm + static_cast<size_t>(bh) * N + pos) : pos) : -1;
  }
  uint4 w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = row[i] >= 0 ? __ldg(reinterpret_cast<const uint4 *>(src + static_cast<size_t>(row[i]) * D))
                       : make_uint4(0u, 0u, 0u, 0u);
  float kb[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (z == 1) {
    const float4 k0 = *reinterpret_cast<const float4 *>(kbar + static_cast<size_t>(bh) * D + 8 * c);
    const float4 k1 = *reinterpret_cast<const float4 *>(kbar + static_cast<size_t>(bh) * D + 8 * c + 4);
    kb[0] = k0.x; kb[1] = k0.y; kb[2] = k0.z; kb[3] = k0.w;
    kb[4] = k1.x; kb[5] = k1.y; kb[6] = k1.z; kb[7] = k1.w;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (row[i] < 0) continue;  // rows past N do not enter the block's amax
    float x[8];
    bf16x8(w[i], x);
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(z == 1 ? __fsub_rn(x[j], kb[j]) : x[j]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if ((tid & 31) == 0) wmax[tid >> 5] = amax;
  __syncthreads();
  amax = wmax[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, wmax[i]);
  const float scale = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 448.0f);
  const float mult = amax == 0.0f ? 0.0f : __fdiv_rn(448.0f, amax);
  uint8_t *dst = (z == 0 ? q8 : k8) + (static_cast<size_t>(bh) * Npad + static_cast<size_t>(t) * TILE) * D + 8 * c;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float x[8];
    bf16x8(w[i], x);
    uint32_t lo = 0, hi = 0;
    if (row[i] >= 0) {
      float y[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) y[j] = __fmul_rn(z == 1 ? __fsub_rn(x[j], kb[j]) : x[j], mult);
      lo = static_cast<uint32_t>(e4m3x2(y[0], y[1])) | (static_cast<uint32_t>(e4m3x2(y[2], y[3])) << 16);
      hi = static_cast<uint32_t>(e4m3x2(y[4], y[5])) | (static_cast<uint32_t>(e4m3x2(y[6], y[7])) << 16);
    }
    *reinterpret_cast<uint2 *>(dst + static_cast<size_t>(g + 16 * i) * D) = make_uint2(lo, hi);
  }
  if (tid == 0) (z == 0 ? sq : sk)[static_cast<size_t>(bh) * (Npad / TILE) + t] = scale;
}
__global__ void __launch_bounds__(256) k_qk_quant(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K,
                                                  const int32_t *__restrict__ perm, const float *__restrict__ kbar,
                                                  int N, int Npad, int zbase, uint8_t *__restrict__ q8,
                                                  float *__restrict__ sq, uint8_t *__restrict__ k8,
                                                  float *__restrict__ sk) {
  qk_quant_body(Q, K, perm, kbar, N, Npad, zbase, q8, sq, k8, sk, blockIdx.x, blockIdx.y, blockIdx.z);
}

// NVFP4 block quantization of the full 4-bit path, same grid and row mapping
// as k_qk_quant (z = 0: Q rows in original order; z = 1: K rows through perm
// minus the channel mean). Per block the power-of-two global scale g = 2^e,
// the least with amax <= 2688 * g (g = 1 for an all-zero block); per row and
// 16 channels sf = E4M3(fp32(b * 2^-e) / 6) of the block maximum b; codes
// E2M1(fp32(x * 2^-e) * fp32(1/sf)), 0 where sf is 0 and in rows past N. The
// tile image: scales, then rows of codes in the 64-byte swizzle (the layout
// of the V tile images, rows = tokens, the K dimension = channels).
__global__ void __launch_bounds__(256) k_qk_quant4(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K,
                                                   const int32_t *__restrict__ perm, const float *__restrict__ kbar,
                                                   int N, int Nb, int zbase, uint8_t *__restrict__ q4img,
                                                   float *__restrict__ gq, uint8_t *__restrict__ k4img,
                                                   float *__restrict__ gk) {
  __shared__ float wmax[8];
  const int t = blockIdx.x, bh = blockIdx.y, z = blockIdx.z + zbase;
  const int tid = threadIdx.x, g = tid >> 4, c = tid & 15;
  const int cnt = min(TILE, N - t * TILE);
  const uint16_t *src = (z == 0 ? Q : K) + static_cast<size_t>(bh) * N * D + 8 * c;
  int row[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = g + 16 * i, pos = t * TILE + rr;
    row[i] = rr < cnt ? ((z == 1 && perm != nullptr) ? __ldg(perm + static_cast<size_t>(bh) * N + pos) : pos) : -1;
  }
  uint4 w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = row[i] >= 0 ? __ldg(reinterpret_cast<const uint4 *>(src + static_cast<size_t>(row[i]) * D))
                       : make_uint4(0u, 0u, 0u, 0u);
  float kb[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (z == 1) {
    const float4 k0 = *reinterpret_cast<const float4 *>(kbar + static_cast<size_t>(bh) * D + 8 * c);
    const float4 k1 = *reinterpret_cast<const float4 *>(kbar + static_cast<size_t>(bh) * D + 8 * c + 4);
    kb[0] = k0.x; kb[1] = k0.y; kb[2] = k0.z; kb[3] = k0.w;
    kb[4] = k1.x; kb[5] = k1.y; kb[6] = k1.z; kb[7] = k1.w;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (row[i] < 0) continue;  // rows past N do not enter the block's amax
    float x[8];
    bf16x8(w[i], x);
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(z == 1 ? __fsub_rn(x[j], kb[j]) : x[j]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if ((tid & 31) == 0) wmax[tid >> 5] = amax;
  __syncthreads();
  amax = wmax[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, wmax[i]);
  int e = 0;
  if (amax > 0.0f) {
    int E;
    const float f = frexpf(amax, &E);  // amax = f * 2^E, f in [0.5, 1); 2688 = 0.65625 * 2^12
    e = (f > 0.65625f) ? E - 11 : E - 12;
  }
  // x * 2^-e in two exact steps when 2^-e is past the binary32 range (tiny blocks)
  const int eh = -e > 126 ? 64 : 0;
  const float m_hi = ldexpf(1.0f, eh), m_lo = ldexpf(1.0f, -e - eh);
  uint8_t *img = (z == 0 ? q4img : k4img) + (static_cast<size_t>(bh) * Nb + t) * V4_TILE_BYTES;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = g + 16 * i;
    float x[8], y[8];
    bf16x8(w[i], x);
    float b = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      y[j] = __fmul_rn(__fmul_rn(z == 1 ? __fsub_rn(x[j], kb[j]) : x[j], m_hi), m_lo);
      b = fmaxf(b, fabsf(y[j]));
    }
    b = fmaxf(b, __shfl_xor_sync(0xFFFFFFFFu, b, 1));  // the 16-channel block of threads c, c^1
    uint32_t sc = e4m3x2(__fdiv_rn(b, 6.0f), 0.0f) & 0xFFu;
    if (row[i] < 0) sc = 0u;
    const float sfv = e4m3x2_value(static_cast<uint16_t>(sc)).x;
    uint32_t codes = 0u;
    if (sfv != 0.0f) {
      const float rcp = __frcp_rn(sfv);
#pragma unroll
      for (int j = 0; j < 8; j += 2)
        codes |= e2m1x2(__fmul_rn(y[j], rcp), __fmul_rn(y[j + 1], rcp)) << (4 * j);
    }
    *reinterpret_cast<uint32_t *>(img + V4_SF_BYTES + sw64_off(r, c >> 2) + 4 * (c & 3)) = codes;
    if ((c & 1) == 0) img[v4_sf_off(r, c >> 1)] = static_cast<uint8_t>(sc);
  }
  if (tid == 0) (z == 0 ? gq : gk)[static_cast<size_t>(bh) * Nb + t] = ldexpf(1.0f, e);
}

// ============================================================== V demean + quantization
// The block's 128 rows (gathered through perm) are copied to shared memory
// with cp.async, row stride 272 bytes: 16-byte reads of one row per thread
// then hit 8 different bank groups per quarter warp.
constexpr int VQ_ROW_BYTES = 272;

__device__ __forceinline__ void gather_tile(uint8_t *sv, const uint16_t *Vh, const int32_t *permh, int p0, int cnt) {
  const int g = threadIdx.x >> 4, c = threadIdx.x & 15;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = g + 16 * i;
    uint8_t *d = sv + rr * VQ_ROW_BYTES + 16 * c;
    if (rr < cnt) {
      const int row = permh ? __ldg(permh + p0 + rr) : p0 + rr;
      cp_async16(d, Vh + static_cast<size_t>(row) * D + 8 * c);
    } else {
      *reinterpret_cast<uint4 *>(d) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  cp_async_wait_all();
}
__device__ __forceinline__ float sv_at(const uint8_t *sv, int r, int c) {
  const uint16_t b = *reinterpret_cast<const uint16_t *>(sv + r * VQ_ROW_BYTES + 2 * c);
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Pass 1: block means (fp64 sums over the block's tokens) and per-block
// residual amax; the last block of a (b,h) turns the channel amax into the
// power-of-two scale (the least with amax <= 448 * scale for E4M3 residuals,
// amax <= 2688 * scale, the NVFP4 global scale, for 4-bit ones). Thread (h, c): channel c over rows [64h, 64h+64).
__device__ __forceinline__ void quantv_pass1_body(const uint16_t *__restrict__ V, const int32_t *__restrict__ perm,
                                                      int N, int Nb, int demean, int fp4, uint16_t *__restrict__ vmean,
                                                      float *__restrict__ amax_part, float *__restrict__ vscale,
                                                      int *__restrict__ vexpo, unsigned *__restrict__ counter, int bx, int by, int bz) {
  extern __shared__ __align__(16) uint8_t dsm[];
  uint8_t *sv = dsm;  // 128 rows x 272 bytes
  __shared__ double ssum[2][128];
  __shared__ float smax[2][128];
  __shared__ int s_last;
  const int t = bx, bh = by, tid = threadIdx.x;
  const int p0 = t * TILE, cnt = min(TILE, N - p0);
  gather_tile(sv, V + static_cast<size_t>(bh) * N * D, perm ? perm + static_cast<size_t>(bh) * N : nullptr, p0, cnt);
  __syncthreads();
  const int c = tid & 127, h = tid >> 7;
  const int ra = 64 * h, rb = min(cnt, ra + 64);
  uint16_t mu = 0;
  if (demean) {
    double s = 0.0;
    for (int r = ra; r < rb; ++r) s += static_cast<double>(sv_at(sv, r, c));
    ssum[h][c] = s;
    __syncthreads();
    mu = f32_to_bf16_rn(static_cast<float>((ssum[0][c] + ssum[1][c]) / static_cast<double>(cnt)));
  }
  const float muf = bf16_to_f32(mu);
  float amax = 0.0f;
  for (int r = ra; r < rb; ++r) amax = fmaxf(amax, fabsf(__fsub_rn(sv_at(sv, r, c), muf)));
  smax[h][c] = amax;
  __syncthreads();
  if (h == 0) {
    vmean[(static_cast<size_t>(bh) * Nb + t) * D + c] = mu;
    amax_part[(static_cast<size_t>(bh) * Nb + t) * D + c] = fmaxf(smax[0][c], smax[1][c]);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&counter[bh], 1u) == static_cast<unsigned>(Nb - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid >= 128) return;
  float a = 0.0f;
#pragma unroll 32
  for (int b = 0; b < Nb; ++b) a = fmaxf(a, __ldcg(amax_part + (static_cast<size_t>(bh) * Nb + b) * D + c));
  int e = 0;
  float sc = 1.0f;
  if (a > 0.0f) {
    int E;
    const float f = frexpf(a, &E);  // a = f * 2^E, f in [0.5, 1)
    if (fp4)
      e = (f > 0.65625f) ? E - 11 : E - 12;  // NVFP4: a <= 2688 * 2^e, 2688 = 6 * 448 = 0.65625 * 2^12
    else
      e = (f > 0.875f) ? E - 8 : E - 9;      // E4M3: a <= 448 * 2^e, 448 = 0.875 * 2^9
    sc = ldexpf(1.0f, e);
  }
  vscale[static_cast<size_t>(bh) * D + c] = sc;
  vexpo[static_cast<size_t>(bh) * D + c] = e;
  if (c == 0) counter[bh] = 0u;
}
__global__ void __launch_bounds__(256) k_quantv_pass1(const uint16_t *__restrict__ V, const int32_t *__restrict__ perm,
                                                      int N, int Nb, int demean, int fp4, uint16_t *__restrict__ vmean,
                                                      float *__restrict__ amax_part, float *__restrict__ vscale,
                                                      int *__restrict__ vexpo, unsigned *__restrict__ counter) {
  quantv_pass1_body(V, perm, N, Nb, demean, fp4, vmean, amax_part, vscale, vexpo, counter, blockIdx.x, blockIdx.y, blockIdx.z);
}

// Pass 2: residual codes (written channel-major), per-token error, and the
// bf16 block means pre-divided by the channel scale for the in-kernel restore
// (mut2[bh][chunk][c][0..63]: slots 0..31 and 32..63 both hold tile
// chunk*32 + slot; unused slots of the last chunk are zero). Thread r < 128
// owns token r: its error is fmaf-accumulated in channel order; the residual,
// scaling and dequantization of a channel pair are packed f32x2 operations
// (each lane rounds as the scalar one; differences are sums with negated
// operands, exactly the same values). The codes of channels c0..c0+7 go over
// bytes c0..c0+7 of the token's own row, whose values there (channels below
// c0/2 + 4) have been read already; then every thread transposes 16 rows x 4
// channels in registers and writes four 16-byte pieces of channel rows. The
// tile therefore needs only its row buffer (six blocks per SM).
__device__ __forceinline__ void quantv_pass2_body(const uint16_t *__restrict__ V, const int32_t *__restrict__ perm,
                                                      int N, int Nb, int Npad, int nch32,
                                                      const uint16_t *__restrict__ vmean,
                                                      const float *__restrict__ vscale, const int *__restrict__ vexpo,
                                                      uint8_t *__restrict__ v8t, float *__restrict__ err,
                                                      uint16_t *__restrict__ mut2, int bx, int by, int bz) {
  extern __shared__ __align__(16) uint8_t dsm[];
  uint8_t *sv = dsm;                            // 128 rows x 272 bytes; then the codes, row-major
  __shared__ __align__(16) float snmu[D], smult[D], snscale[D];  // -mean, 2^-e, -scale
  const int t = bx, bh = by, tid = threadIdx.x;
  const int p0 = t * TILE, cnt = min(TILE, N - p0);
  gather_tile(sv, V + static_cast<size_t>(bh) * N * D, perm ? perm + static_cast<size_t>(bh) * N : nullptr, p0, cnt);
  if (tid < 128) {
    const int c = tid;
    const uint16_t mu = vmean[(static_cast<size_t>(bh) * Nb + t) * D + c];
    snmu[c] = -bf16_to_f32(mu);
    const int e = vexpo[static_cast<size_t>(bh) * D + c];
    smult[c] = ldexpf(1.0f, -e);
    snscale[c] = -vscale[static_cast<size_t>(bh) * D + c];
    // block mean / scale for the restore MMA (exact: bf16 divided by a power of two)
    const uint16_t ms = f32_to_bf16_rn(__fmul_rn(bf16_to_f32(mu), ldexpf(1.0f, -e)));
    const int ch = t / CHUNK32, slot = t % CHUNK32;
    uint16_t *m = mut2 + ((static_cast<size_t>(bh) * nch32 + ch) * D + c) * 64;
    m[slot] = ms;
    m[slot + 32] = ms;
    if (t == Nb - 1)
      for (int s2 = slot + 1; s2 < CHUNK32; ++s2) {
        m[s2] = 0;
        m[s2 + 32] = 0;
      }
  }
  __syncthreads();
  if (tid < 128) {
    const int r = tid;
    float acc = 0.0f;
    uint8_t *row = sv + r * VQ_ROW_BYTES;
#pragma unroll 2
    for (int c0 = 0; c0 < D; c0 += 8) {
      float x[8];
      bf16x8(*reinterpret_cast<const uint4 *>(row + 2 * c0), x);
      uint32_t cw[2] = {0u, 0u};  // the codes of channels c0 .. c0+7
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const int c = c0 + j;
        uint16_t codes = 0;
        if (r < cnt) {
          const float2 rr = __fadd2_rn(make_float2(x[j], x[j + 1]), *reinterpret_cast<const float2 *>(&snmu[c]));
          const float2 sr = __fmul2_rn(rr, *reinterpret_cast<const float2 *>(&smult[c]));
          codes = e4m3x2(sr.x, sr.y);
          const float2 nd = __fmul2_rn(e4m3x2_value(codes), *reinterpret_cast<const float2 *>(&snscale[c]));
          const float2 ee = __fadd2_rn(rr, nd);
          acc = __fmaf_rn(ee.x, ee.x, acc);
          acc = __fmaf_rn(ee.y, ee.y, acc);
        }
        cw[j >> 2] |= static_cast<uint32_t>(codes) << (8 * (j & 3));
      }
      *reinterpret_cast<uint2 *>(row + c0) = make_uint2(cw[0], cw[1]);  // over values already read
    }
    if (r < cnt) err[static_cast<size_t>(bh) * N + p0 + r] = acc;
  }
  __syncthreads();
  {
    // thread (rg, cg): rows 16 rg .. 16 rg + 15, channels 4 cg .. 4 cg + 3
    const int cg = tid & 31, rg = tid >> 5;
    uint32_t wv[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) wv[q] = *reinterpret_cast<const uint32_t *>(sv + (16 * rg + q) * VQ_ROW_BYTES + 4 * cg);
    uint32_t ch[4][4];  // [channel][4-row group]: the channel's bytes of those rows
#pragma unroll
    for (int g4 = 0; g4 < 4; ++g4) {
      const uint32_t t0 = __byte_perm(wv[4 * g4], wv[4 * g4 + 1], 0x5140);
      const uint32_t t1 = __byte_perm(wv[4 * g4], wv[4 * g4 + 1], 0x7362);
      const uint32_t t2 = __byte_perm(wv[4 * g4 + 2], wv[4 * g4 + 3], 0x5140);
      const uint32_t t3 = __byte_perm(wv[4 * g4 + 2], wv[4 * g4 + 3], 0x7362);
      ch[0][g4] = __byte_perm(t0, t2, 0x5410);
      ch[1][g4] = __byte_perm(t0, t2, 0x7632);
      ch[2][g4] = __byte_perm(t1, t3, 0x5410);
      ch[3][g4] = __byte_perm(t1, t3, 0x7632);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint4 *>(v8t + (static_cast<size_t>(bh) * D + 4 * cg + i) * Npad + p0 + 16 * rg) =
          make_uint4(ch[i][0], ch[i][1], ch[i][2], ch[i][3]);
  }
}
__global__ void __launch_bounds__(256) k_quantv_pass2(const uint16_t *__restrict__ V, const int32_t *__restrict__ perm,
                                                      int N, int Nb, int Npad, int nch32,
                                                      const uint16_t *__restrict__ vmean,
                                                      const float *__restrict__ vscale, const int *__restrict__ vexpo,
                                                      uint8_t *__restrict__ v8t, float *__restrict__ err,
                                                      uint16_t *__restrict__ mut2) {
  quantv_pass2_body(V, perm, N, Nb, Npad, nch32, vmean, vscale, vexpo, v8t, err, mut2, blockIdx.x, blockIdx.y, blockIdx.z);
}

// NVFP4 pass 2 (page "VC-Attention acelera atenção…", "V-Smooth: corrigindo
// outliers de valor", item Demean, the 4-bit residual): per 16-token block and
// channel the E4M3 scale sf = E4M3(fp32(b * 2^-e) / 6) of the block maximum
// b = max |r|; codes E2M1(fp32(r * 2^-e) * fp32(1/sf)); the per-token error
// of value(code) * sf * 2^e, fmaf-accumulated in channel order; the tile image
// (scales, then the swizzled channel rows of codes) and the block means / g
// for the restore, as in pass 2.
__global__ void __launch_bounds__(256) k_quantv4_pass2(const uint16_t *__restrict__ V, const int32_t *__restrict__ perm,
                                                       int N, int Nb, int nch32, const uint16_t *__restrict__ vmean,
                                                       const float *__restrict__ vscale, const int *__restrict__ vexpo,
                                                       uint8_t *__restrict__ v4img, float *__restrict__ err,
                                                       uint16_t *__restrict__ mut2) {
  extern __shared__ __align__(16) uint8_t dsm[];
  uint8_t *sv = dsm;                           // 128 rows x 272 bytes
  uint8_t *codeT = dsm + TILE * VQ_ROW_BYTES;  // 128 channels x 144 bytes, one code per byte
  __shared__ __align__(16) float smu[D], smult[D], sscale[D];
  __shared__ float srcp[8][D], ssfv[8][D];
  __shared__ __align__(16) uint8_t ssf[V4_SF_BYTES];
  const int t = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int p0 = t * TILE, cnt = min(TILE, N - p0);
  gather_tile(sv, V + static_cast<size_t>(bh) * N * D, perm ? perm + static_cast<size_t>(bh) * N : nullptr, p0, cnt);
  if (tid < 128) {
    const int c = tid;
    const uint16_t mu = vmean[(static_cast<size_t>(bh) * Nb + t) * D + c];
    smu[c] = bf16_to_f32(mu);
    const int e = vexpo[static_cast<size_t>(bh) * D + c];
    smult[c] = ldexpf(1.0f, -e);
    sscale[c] = vscale[static_cast<size_t>(bh) * D + c];
    const uint16_t ms = f32_to_bf16_rn(__fmul_rn(bf16_to_f32(mu), ldexpf(1.0f, -e)));
    const int ch = t / CHUNK32, slot = t % CHUNK32;
    uint16_t *m = mut2 + ((static_cast<size_t>(bh) * nch32 + ch) * D + c) * 64;
    m[slot] = ms;
    m[slot + 32] = ms;
    if (t == Nb - 1)
      for (int s2 = slot + 1; s2 < CHUNK32; ++s2) {
        m[s2] = 0;
        m[s2 + 32] = 0;
      }
  }
  __syncthreads();
  {
    // block scales: thread (c, jb = tid/128 + 2i)
    const int c = tid & 127;
    for (int jb = tid >> 7; jb < 8; jb += 2) {
      float b = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * jb + i;
        if (r < cnt) b = fmaxf(b, fabsf(__fsub_rn(sv_at(sv, r, c), smu[c])));
      }
      const uint32_t sc = e4m3x2(__fdiv_rn(__fmul_rn(b, smult[c]), 6.0f), 0.0f) & 0xFFu;
      const float sfv = e4m3x2_value(static_cast<uint16_t>(sc)).x;
      ssfv[jb][c] = sfv;
      srcp[jb][c] = sfv == 0.0f ? 0.0f : __frcp_rn(sfv);
      ssf[v4_sf_off(c, jb)] = static_cast<uint8_t>(sc);
    }
  }
  __syncthreads();
  if (tid < 128) {
    const int r = tid, jb = r >> 4;
    float acc = 0.0f;
    const uint8_t *row = sv + r * VQ_ROW_BYTES;
#pragma unroll 2
    for (int c0 = 0; c0 < D; c0 += 8) {
      float x[8];
      bf16x8(*reinterpret_cast<const uint4 *>(row + 2 * c0), x);
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const int c = c0 + j;
        uint32_t codes = 0;
        if (r < cnt) {
          const float r0 = __fsub_rn(x[j], smu[c]);
          const float r1 = __fsub_rn(x[j + 1], smu[c + 1]);
          codes = e2m1x2(__fmul_rn(__fmul_rn(r0, smult[c]), srcp[jb][c]),
                         __fmul_rn(__fmul_rn(r1, smult[c + 1]), srcp[jb][c + 1]));
          if (ssfv[jb][c] == 0.0f) codes &= 0xF0u;  // no scale: code 0 (not the -0 of a negative residual)
          if (ssfv[jb][c + 1] == 0.0f) codes &= 0x0Fu;
          const float2 dq = e2m1x2_value(codes);
          const float e0 = __fsub_rn(r0, __fmul_rn(__fmul_rn(dq.x, ssfv[jb][c]), sscale[c]));
          const float e1 = __fsub_rn(r1, __fmul_rn(__fmul_rn(dq.y, ssfv[jb][c + 1]), sscale[c + 1]));
          acc = __fmaf_rn(e0, e0, acc);
          acc = __fmaf_rn(e1, e1, acc);
        }
        codeT[c * 144 + r] = static_cast<uint8_t>(codes & 15u);
        codeT[(c + 1) * 144 + r] = static_cast<uint8_t>(codes >> 4);
      }
    }
    if (r < cnt) err[static_cast<size_t>(bh) * N + p0 + r] = acc;
  }
  __syncthreads();
  uint8_t *img = v4img + (static_cast<size_t>(bh) * Nb + t) * V4_TILE_BYTES;
  {
    // thread (c, h): the 16-byte chunks 2h and 2h+1 of channel row c (tokens 64h .. 64h+63)
    const int c = tid >> 1, h = tid & 1;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int ch = 2 * h + k;
      const uint8_t *src = codeT + c * 144 + 32 * ch;
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint2 b8 = *reinterpret_cast<const uint2 *>(src + 8 * q);
        uint32_t v = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v |= ((b8.x >> (8 * e)) & 15u) << (4 * e);
          v |= ((b8.y >> (8 * e)) & 15u) << (4 * e + 16);
        }
        w[q] = v;
      }
      *reinterpret_cast<uint4 *>(img + V4_SF_BYTES + sw64_off(c, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  if (tid < V4_SF_BYTES / 16)
    *reinterpret_cast<uint4 *>(img + 16 * tid) = *reinterpret_cast<const uint4 *>(ssf + 16 * tid);
}

// ============================================================== repair selection
// Top-R by error (float >= 0, so the bit pattern orders like the value), ties
// to the lowest permuted position; output ascending. One block per (b,h):
// radix select of the R-th largest key, then an ordered compaction.
template <int NT>
__device__ __forceinline__ void repair_select_body(const float *__restrict__ err, int N, int R,
                                                        int32_t *__restrict__ rep_idx, int bx, int by, int bz) {
  __shared__ unsigned hist[256];
  __shared__ unsigned s_prefix, s_need;
  __shared__ int wgt[NT / 32], weq[NT / 32];
  __shared__ int s_base_gt, s_base_eq;
  const int bh = bx, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const unsigned *key = reinterpret_cast<const unsigned *>(err + static_cast<size_t>(bh) * N);
  int32_t *out = rep_idx + static_cast<size_t>(bh) * R;
  if (tid == 0) {
    s_prefix = 0u;
    s_need = static_cast<unsigned>(R);
  }
  unsigned mask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
    const unsigned prefix = s_prefix;
    for (int n = tid; n < N; n += NT) {
      const unsigned kv = key[n];
      if ((kv & mask) == prefix) atomicAdd(&hist[(kv >> shift) & 0xFFu], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      unsigned need = s_need, run = 0u;
      int dsel = 0;
      for (int dgt = 255; dgt >= 0; --dgt) {
        if (run + hist[dgt] >= need) {
          dsel = dgt;
          break;
        }
        run += hist[dgt];
      }
      s_need = need - run;  // how many with exactly this digit prefix are still needed
      s_prefix = prefix | (static_cast<unsigned>(dsel) << shift);
    }
    mask |= 0xFFu << shift;
    __syncthreads();
  }
  const unsigned T = s_prefix;   // the R-th largest key
  const int need_eq = static_cast<int>(s_need);  // keys == T to take (lowest positions first)
  if (tid == 0) {
    s_base_gt = 0;
    s_base_eq = 0;
  }
  __syncthreads();
  for (int n0 = 0; n0 < N; n0 += NT) {
    const int n = n0 + tid;
    const unsigned kv = n < N ? key[n] : 0u;
    const bool gt = n < N && kv > T;
    const bool eq = n < N && kv == T;
    const unsigned bgt = __ballot_sync(0xFFFFFFFFu, gt), beq = __ballot_sync(0xFFFFFFFFu, eq);
    if (lane == 0) {
      wgt[warp] = __popc(bgt);
      weq[warp] = __popc(beq);
    }
    __syncthreads();
    int pre_gt = s_base_gt, pre_eq = s_base_eq;
    for (int w = 0; w < warp; ++w) {
      pre_gt += wgt[w];
      pre_eq += weq[w];
    }
    const unsigned lt = (1u << lane) - 1u;
    const int my_eq = pre_eq + __popc(beq & lt);
    const bool take = gt || (eq && my_eq < need_eq);
    // position in the ascending output = number of taken keys before n
    const int taken_eq_before = min(my_eq, need_eq);
    const int pos = pre_gt + __popc(bgt & lt) + taken_eq_before;
    if (take) out[pos] = n;
    __syncthreads();
    if (tid == 0) {
      int tg = 0, te = 0;
      for (int w = 0; w < NT / 32; ++w) {
        tg += wgt[w];
        te += weq[w];
      }
      s_base_gt += tg;
      s_base_eq += te;
    }
    __syncthreads();
  }
}
__global__ void __launch_bounds__(1024) k_repair_select(const float *__restrict__ err, int N, int R,
                                                        int32_t *__restrict__ rep_idx) {
  repair_select_body<1024>(err, N, R, rep_idx, blockIdx.x, blockIdx.y, blockIdx.z);
}

// Same selection for N <= 32768, with no serial step: the keys stay in
// registers (key i of thread t is position 512 i + t); each radix pass picks
// its digit with a block scan of the 256-bin histogram; the ordered compaction
// counts (chunk, warp) hits for all chunks at once, scans those counts once and
// writes every taken position in a second sweep.
constexpr int RS_T = 512, RS_KPT = 64, RS_W = RS_T / 32;

// Inclusive scan of one value per thread over the first `nthreads` threads
// (a multiple of 32, <= RS_T), through warp shuffles and one shared array.
__device__ __forceinline__ unsigned rs_block_scan(unsigned v, unsigned *wsum, int nthreads) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (tid < nthreads && lane == 31) wsum[warp] = x;
  __syncthreads();
  unsigned add = 0u;
  for (int w = 0; w < warp && tid < nthreads; ++w) add += wsum[w];
  __syncthreads();
  return x + add;
}

__global__ void __launch_bounds__(RS_T) k_repair_select_reg(const float *__restrict__ err, int N, int R,
                                                            int32_t *__restrict__ rep_idx) {
  __shared__ unsigned hist[256];
  __shared__ unsigned wsum[RS_W];
  __shared__ unsigned s_digit, s_run;
  __shared__ unsigned cgt[RS_KPT * RS_W], ceq[RS_KPT * RS_W];
  const int bh = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const unsigned *keyg = reinterpret_cast<const unsigned *>(err + static_cast<size_t>(bh) * N);
  int32_t *out = rep_idx + static_cast<size_t>(bh) * R;
  unsigned key[RS_KPT];
#pragma unroll
  for (int i = 0; i < RS_KPT; ++i) {
    const int n = RS_T * i + tid;
    key[i] = n < N ? __ldg(keyg + n) : 0u;
  }
  unsigned prefix = 0u, mask = 0u, need = static_cast<unsigned>(R);
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < RS_KPT; ++i)
      if (RS_T * i + tid < N && (key[i] & mask) == prefix) atomicAdd(&hist[(key[i] >> shift) & 0xFFu], 1u);
    __syncthreads();
    // thread j holds digit 255 - j: the inclusive scan over j counts the keys
    // whose digit is >= 255 - j; the digit where that count first reaches
    // `need` is the one of the R-th largest key (counts here sum to >= need)
    const unsigned c = tid < 256 ? hist[255 - tid] : 0u;
    const unsigned incl = rs_block_scan(c, wsum, 256);
    if (tid < 256 && incl >= need && incl - c < need) {
      s_digit = 255u - static_cast<unsigned>(tid);
      s_run = incl - c;
    }
    __syncthreads();
    need -= s_run;
    prefix |= s_digit << shift;
    mask |= 0xFFu << shift;
  }
  const unsigned T = prefix;  // the R-th largest key; `need` keys equal to T are taken
  // ---- ordered compaction (ascending position; ties to the lowest positions)
#pragma unroll
  for (int i = 0; i < RS_KPT; ++i) {
    const int n = RS_T * i + tid;
    const unsigned bg = __ballot_sync(0xFFFFFFFFu, n < N && key[i] > T);
    const unsigned be = __ballot_sync(0xFFFFFFFFu, n < N && key[i] == T);
    if (lane == 0) {
      cgt[i * RS_W + warp] = __popc(bg);
      ceq[i * RS_W + warp] = __popc(be);
    }
  }
  __syncthreads();
  {  // exclusive scan of the (chunk, warp) counts, two entries per thread
    const unsigned g0 = cgt[2 * tid], g1 = cgt[2 * tid + 1], e0 = ceq[2 * tid], e1 = ceq[2 * tid + 1];
    const unsigned ig = rs_block_scan(g0 + g1, wsum, RS_T);
    const unsigned ie = rs_block_scan(e0 + e1, wsum, RS_T);
    cgt[2 * tid] = ig - g0 - g1;
    cgt[2 * tid + 1] = ig - g1;
    ceq[2 * tid] = ie - e0 - e1;
    ceq[2 * tid + 1] = ie - e1;
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int i = 0; i < RS_KPT; ++i) {
    const int n = RS_T * i + tid;
    const bool gt = n < N && key[i] > T, eq = n < N && key[i] == T;
    const unsigned bg = __ballot_sync(0xFFFFFFFFu, gt), be = __ballot_sync(0xFFFFFFFFu, eq);
    const unsigned rank_eq = ceq[i * RS_W + warp] + __popc(be & lt);  // equal keys before this one
    const unsigned pos = cgt[i * RS_W + warp] + __popc(bg & lt) + min(rank_eq, need);
    if (gt || (eq && rank_eq < need)) out[pos] = n;
  }
}

// delta = bf16(r - value(code)*scale) for every repaired token; also the
// channel-major copy divided by the channel scale (deltat[bh][c][r], zero for
// r in [R, Rpad)) that the attention kernel's repair MMA reads.
__device__ __forceinline__ void repair_delta_body(const uint16_t *__restrict__ V, const int32_t *__restrict__ perm,
                                                      int N, int Nb, int R, int Rpad,
                                                      const int32_t *__restrict__ rep_idx,
                                                      const uint16_t *__restrict__ vmean,
                                                      const float *__restrict__ vscale, const int *__restrict__ vexpo,
                                                      uint16_t *__restrict__ rep_delta, uint16_t *__restrict__ deltat, int bx, int by, int bz) {
  const int bh = by, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = bx * 8 + warp;
  if (r >= Rpad) return;
  if (r >= R) {
    for (int i = 0; i < 4; ++i) deltat[(static_cast<size_t>(bh) * D + 4 * lane + i) * Rpad + r] = 0;
    return;
  }
  const int p = rep_idx[static_cast<size_t>(bh) * R + r];
  const int row = perm ? perm[static_cast<size_t>(bh) * N + p] : p;
  const int t = p / TILE;
  const uint2 w = *reinterpret_cast<const uint2 *>(V + (static_cast<size_t>(bh) * N + row) * D + 4 * lane);
  const float v[4] = {__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u), __uint_as_float(w.y << 16),
                      __uint_as_float(w.y & 0xFFFF0000u)};
  float res[4], mult[4], sc[4];
  for (int i = 0; i < 4; ++i) {
    const int c = 4 * lane + i;
    res[i] = __fsub_rn(v[i], bf16_to_f32(vmean[(static_cast<size_t>(bh) * Nb + t) * D + c]));
    mult[i] = ldexpf(1.0f, -vexpo[static_cast<size_t>(bh) * D + c]);
    sc[i] = vscale[static_cast<size_t>(bh) * D + c];
  }
  uint16_t dl[4];
  for (int i = 0; i < 4; i += 2) {
    const uint16_t codes = e4m3x2(__fmul_rn(res[i], mult[i]), __fmul_rn(res[i + 1], mult[i + 1]));
    const float2 dq = e4m3x2_value(codes);
    dl[i] = f32_to_bf16_rn(__fsub_rn(res[i], __fmul_rn(dq.x, sc[i])));
    dl[i + 1] = f32_to_bf16_rn(__fsub_rn(res[i + 1], __fmul_rn(dq.y, sc[i + 1])));
  }
  uint2 o;
  o.x = static_cast<uint32_t>(dl[0]) | (static_cast<uint32_t>(dl[1]) << 16);
  o.y = static_cast<uint32_t>(dl[2]) | (static_cast<uint32_t>(dl[3]) << 16);
  *reinterpret_cast<uint2 *>(rep_delta + (static_cast<size_t>(bh) * R + r) * D + 4 * lane) = o;
  for (int i = 0; i < 4; ++i) {
    const int c = 4 * lane + i;
    deltat[(static_cast<size_t>(bh) * D + c) * Rpad + r] = f32_to_bf16_rn(__fmul_rn(bf16_to_f32(dl[i]), mult[i]));
  }
}
__global__ void __launch_bounds__(256) k_repair_delta(const uint16_t *__restrict__ V, const int32_t *__restrict__ perm,
                                                      int N, int Nb, int R, int Rpad,
                                                      const int32_t *__restrict__ rep_idx,
                                                      const uint16_t *__restrict__ vmean,
                                                      const float *__restrict__ vscale, const int *__restrict__ vexpo,
                                                      uint16_t *__restrict__ rep_delta, uint16_t *__restrict__ deltat) {
  repair_delta_body(V, perm, N, Nb, R, Rpad, rep_idx, vmean, vscale, vexpo, rep_delta, deltat, blockIdx.x, blockIdx.y, blockIdx.z);
}

// The repair deltas of the NVFP4 residual: the token's codes are recomputed
// from its block's scale code in the tile image, exactly as pass 2 made them.
__global__ void __launch_bounds__(256) k_repair_delta4(const uint16_t *__restrict__ V,
                                                       const int32_t *__restrict__ perm, int N, int Nb, int R, int Rpad,
                                                       const int32_t *__restrict__ rep_idx,
                                                       const uint16_t *__restrict__ vmean,
                                                       const float *__restrict__ vscale, const int *__restrict__ vexpo,
                                                       const uint8_t *__restrict__ v4img,
                                                       uint16_t *__restrict__ rep_delta, uint16_t *__restrict__ deltat) {
  const int bh = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + warp;
  if (r >= Rpad) return;
  if (r >= R) {
    for (int i = 0; i < 4; ++i) deltat[(static_cast<size_t>(bh) * D + 4 * lane + i) * Rpad + r] = 0;
    return;
  }
  const int p = rep_idx[static_cast<size_t>(bh) * R + r];
  const int row = perm ? perm[static_cast<size_t>(bh) * N + p] : p;
  const int t = p / TILE, jb = (p % TILE) >> 4;
  const uint8_t *sfimg = v4img + (static_cast<size_t>(bh) * Nb + t) * V4_TILE_BYTES;
  const uint2 w = *reinterpret_cast<const uint2 *>(V + (static_cast<size_t>(bh) * N + row) * D + 4 * lane);
  const float v[4] = {__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u), __uint_as_float(w.y << 16),
                      __uint_as_float(w.y & 0xFFFF0000u)};
  float res[4], mult[4], sc[4], sfv[4], rcp[4];
  for (int i = 0; i < 4; ++i) {
    const int c = 4 * lane + i;
    res[i] = __fsub_rn(v[i], bf16_to_f32(vmean[(static_cast<size_t>(bh) * Nb + t) * D + c]));
    mult[i] = ldexpf(1.0f, -vexpo[static_cast<size_t>(bh) * D + c]);
    sc[i] = vscale[static_cast<size_t>(bh) * D + c];
    sfv[i] = e4m3x2_value(static_cast<uint16_t>(sfimg[v4_sf_off(c, jb)])).x;
    rcp[i] = sfv[i] == 0.0f ? 0.0f : __frcp_rn(sfv[i]);
  }
  uint16_t dl[4];
  for (int i = 0; i < 4; i += 2) {
    const uint32_t codes = e2m1x2(__fmul_rn(__fmul_rn(res[i], mult[i]), rcp[i]),
                                  __fmul_rn(__fmul_rn(res[i + 1], mult[i + 1]), rcp[i + 1]));
    const float2 dq = e2m1x2_value(codes);
    dl[i] = f32_to_bf16_rn(__fsub_rn(res[i], __fmul_rn(__fmul_rn(dq.x, sfv[i]), sc[i])));
    dl[i + 1] = f32_to_bf16_rn(__fsub_rn(res[i + 1], __fmul_rn(__fmul_rn(dq.y, sfv[i + 1]), sc[i + 1])));
  }
  uint2 o;
  o.x = static_cast<uint32_t>(dl[0]) | (static_cast<uint32_t>(dl[1]) << 16);
  o.y = static_cast<uint32_t>(dl[2]) | (static_cast<uint32_t>(dl[3]) << 16);
  *reinterpret_cast<uint2 *>(rep_delta + (static_cast<size_t>(bh) * R + r) * D + 4 * lane) = o;
  for (int i = 0; i < 4; ++i) {
    const int c = 4 * lane + i;
    deltat[(static_cast<size_t>(bh) * D + c) * Rpad + r] = f32_to_bf16_rn(__fmul_rn(bf16_to_f32(dl[i]), mult[i]));
  }
}

// ============================================================== misc
// ============================================================== one-launch prologue
// Grid-wide barrier of a cooperative launch: every block adds one to the
// counter (zeroed at the start of the call) and waits until it holds
// `target` = (barriers passed so far) x gridDim.x. Bounded: a wait that runs
// out sets the timeout bit in the status word and the block leaves the
// kernel; every waiting block reads that bit in its wait loop and leaves as
// soon as it is set, so a failed call ends about one limit after the first
// block gave up; nothing spins for ever.
__device__ bool grid_barrier(unsigned *count, unsigned target, uint32_t *status) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(count, 1u);
    const long long t0 = clock64();
    int ok = 1;
    while (true) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(count) : "memory");
      if (v >= target) break;
      if (clock64() - t0 > VC_WAIT_LIMIT_CYCLES) {
        atomicOr(status, ST_TIMEOUT);
        ok = 0;
        break;
      }
      unsigned st;
      asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(st) : "l"(status) : "memory");
      if (st & ST_TIMEOUT) {  // another block already gave up: this barrier cannot complete
        ok = 0;
        break;
      }
      __nanosleep(100);
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// The prologue of vc_attn_fwd (E4M3 path, k <= 8) as one persistent launch:
// the bodies of the separate kernels, each work item one of their blocks,
// with a grid barrier wherever a step reads what the previous one wrote.
//   1. k-means init (if clustering), the K channel means, Q quantization
//   2. each Lloyd pass (iters updates, then the final labels)
//   3. the stable permutation
//   4. K' quantization and V pass 1 (block means, channel scales)
//   5. V pass 2 (codes, token errors, restore operands)
//   6. repair selection, 7. repair deltas
// Every (b,h) step is the one the separate kernels compute, so every output
// is bit-identical to theirs.
__global__ void __launch_bounds__(256) k_prologue_fused(const FusedPrologueParams p) {
  unsigned passed = 0;
  auto sync = [&]() -> bool {
    ++passed;
    return grid_barrier(p.gsync, passed * gridDim.x, p.status);
  };
  const int BH = p.BH, Nb = p.Nb;
  {
    const int n_init = p.cluster ? BH : 0;
    const int n_kbar = p.ksmooth ? p.kb_nchunk * BH : BH;
    const int n_q = Nb * BH;
    for (int it = blockIdx.x; it < n_init + n_kbar + n_q; it += gridDim.x) {
      int i = it;
      if (i < n_init) {
        if (threadIdx.x < D) kmeans_init_body(p.V, p.N, p.k, p.cent, i, 0, 0);
      } else if ((i -= n_init) < n_kbar) {
        if (p.ksmooth)
          kbar_body(p.K, p.N, p.kb_nchunk, 1, p.kb_part, p.kb_counter, p.kbar, i % p.kb_nchunk, i / p.kb_nchunk, 0);
        else if (threadIdx.x < D)
          p.kbar[static_cast<size_t>(i) * D + threadIdx.x] = 0.0f;  // no K smoothing: mean 0
      } else {
        i -= n_kbar;
        qk_quant_body(p.Q, p.K, nullptr, p.kbar, p.N, p.Npad, 0, p.q8, p.sq, p.k8, p.sk, i % Nb, i / Nb, 0);
      }
      __syncthreads();
    }
  }
  if (!sync()) return;
  const int32_t *pm = p.perm_in;
  if (p.cluster) {
    for (int pass = 0; pass <= p.iters; ++pass) {
      for (int it = blockIdx.x; it < p.km_nblk * BH; it += gridDim.x) {
        kmeans_pass8_body(p.V, p.N, p.k, p.km_cpb, p.km_nblk, p.cent, p.labels, p.km_psum, p.km_pcnt,
                          p.km_counter, pass < p.iters ? 1 : 0, it % p.km_nblk, it / p.km_nblk, 0);
        __syncthreads();
      }
      if (!sync()) return;
    }
    for (int it = blockIdx.x; it < BH; it += gridDim.x) {
      perm_sort_body<256>(p.labels, p.N, p.k, p.perm, it, 0, 0);
      __syncthreads();
    }
    if (!sync()) return;
    pm = p.perm;
  }
  for (int it = blockIdx.x; it < 2 * Nb * BH; it += gridDim.x) {
    if (it < Nb * BH) {
      qk_quant_body(p.Q, p.K, pm, p.kbar, p.N, p.Npad, 1, p.q8, p.sq, p.k8, p.sk, it % Nb, it / Nb, 0);
    } else {
      const int i = it - Nb * BH;
      quantv_pass1_body(p.V, pm, p.N, Nb, p.demean, 0, p.vmean, p.amax_part, p.vscale, p.vexpo, p.vq_counter,
                        i % Nb, i / Nb, 0);
    }
    __syncthreads();
  }
  if (!sync()) return;
  for (int it = blockIdx.x; it < Nb * BH; it += gridDim.x) {
    quantv_pass2_body(p.V, pm, p.N, Nb, p.Npad, p.nch32, p.vmean, p.vscale, p.vexpo, p.v8t, p.err, p.mut2, it % Nb,
                      it / Nb, 0);
    __syncthreads();
  }
  if (p.R == 0) return;
  if (!sync()) return;
  for (int it = blockIdx.x; it < BH; it += gridDim.x) {
    repair_select_body<256>(p.err, p.N, p.R, p.rep_idx, it, 0, 0);
    __syncthreads();
  }
  if (!sync()) return;
  const int nrb = (p.Rpad + 7) / 8;
  for (int it = blockIdx.x; it < nrb * BH; it += gridDim.x) {
    repair_delta_body(p.V, pm, p.N, Nb, p.R, p.Rpad, p.rep_idx, p.vmean, p.vscale, p.vexpo, p.rep_delta, p.deltat,
                      it % nrb, it / nrb, 0);
    __syncthreads();
  }
}

__global__ void k_identity_perm(int32_t *perm, int N, long long total) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < total) perm[i] = static_cast<int32_t>(i % N);
}

}  // namespace vc
