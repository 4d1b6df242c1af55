// prologue.cuh - declarations of the prologue kernels (see prologue.cu).
#pragma once
#include <cstdint>
#include <cuda.h>

namespace vc {

__global__ void k_kmeans_init(const uint16_t *V, int N, int k, float *cent);
__global__ void k_kmeans_pass(const uint16_t *V, int N, int k, int cpb, int nblk, float *cent, int32_t *labels,
                              double *psum, int *pcnt, unsigned *counter, int accumulate);
// k <= 8 with the labels decided on the tensor cores (kmeans_tc.cu); status:
// the workspace status word (a bounded wait that runs out sets ST_TIMEOUT).
// tmV: 2-D map over V as [B*H*N rows][128] bf16, boxes of 64 channels x 128
// rows, 128-byte swizzle.
__global__ void k_kmeans_pass8tc(const __grid_constant__ CUtensorMap tmV, int N, int k, int cpb, int nblk, float *cent,
                                 int32_t *labels, double *psum, int *pcnt, unsigned *counter, int accumulate,
                                 uint32_t *status);
__global__ void k_perm_sort(const int32_t *labels, int N, int k, int32_t *perm);
// k <= 8: the stable sort spread over the k-means blocks, from the label
// pass's per-block counts pcnt[bh][block][label].
// At most PERM_SCATTER_MAX_BLOCKS k-means blocks per (b,h) (two per SM).
constexpr int PERM_SCATTER_MAX_BLOCKS = 2 * 148;
__global__ void k_perm_scatter(const int32_t *labels, const int *pcnt, int N, int k, int cpb, int nblk,
                               int32_t *perm);
__global__ void k_kbar(const uint16_t *K, int N, int nchunk, int ksmooth, double *part, unsigned *counter,
                       float *kbar);
__global__ void k_qk_quant(const uint16_t *Q, const uint16_t *K, const int32_t *perm, const float *kbar, int N,
                           int Npad, int zbase, uint8_t *q8, float *sq, uint8_t *k8, float *sk);
__global__ void k_qk_quant4(const uint16_t *Q, const uint16_t *K, const int32_t *perm, const float *kbar, int N,
                            int Nb, int zbase, uint8_t *q4img, float *gq, uint8_t *k4img, float *gk);
__global__ void k_quantv_pass1(const uint16_t *V, const int32_t *perm, int N, int Nb, int demean, int fp4, uint16_t *vmean,
                               float *amax_part, float *vscale, int *vexpo, unsigned *counter);
__global__ void k_quantv_pass2(const uint16_t *V, const int32_t *perm, int N, int Nb, int Npad, int nch32,
                               const uint16_t *vmean, const float *vscale, const int *vexpo, uint8_t *v8t, float *err,
                               uint16_t *mut2);
__global__ void k_quantv4_pass2(const uint16_t *V, const int32_t *perm, int N, int Nb, int nch32, const uint16_t *vmean,
                                const float *vscale, const int *vexpo, uint8_t *v4img, float *err, uint16_t *mut2);
__global__ void k_repair_select(const float *err, int N, int R, int32_t *rep_idx);
__global__ void k_repair_select_reg(const float *err, int N, int R, int32_t *rep_idx);
__global__ void k_repair_delta(const uint16_t *V, const int32_t *perm, int N, int Nb, int R, int Rpad,
                               const int32_t *rep_idx, const uint16_t *vmean, const float *vscale, const int *vexpo,
                               uint16_t *rep_delta, uint16_t *deltat);
__global__ void k_repair_delta4(const uint16_t *V, const int32_t *perm, int N, int Nb, int R, int Rpad,
                                const int32_t *rep_idx, const uint16_t *vmean, const float *vscale, const int *vexpo,
                                const uint8_t *v4img, uint16_t *rep_delta, uint16_t *deltat);
__global__ void k_identity_perm(int32_t *perm, int N, long long total);

// Arguments of the one-launch prologue (k_prologue_fused): the workspace
// arrays of the separate kernels and the sizes they are launched with.
struct FusedPrologueParams {
  const uint16_t *Q, *K, *V;
  int BH, N, Nb, Npad, nch32, k, iters, R, Rpad, km_cpb, km_nblk, kb_nchunk;
  int demean, ksmooth, cluster;  // cluster: k-means + permutation in this launch
  const int32_t *perm_in;        // the permutation when not clustering (null: identity)
  int32_t *perm, *labels;
  float *cent;
  double *km_psum;
  int *km_pcnt;
  unsigned *km_counter;
  double *kb_part;
  unsigned *kb_counter;
  float *kbar;
  uint8_t *q8, *k8, *v8t;
  float *sq, *sk, *amax_part, *vscale, *err;
  int *vexpo;
  uint16_t *vmean, *mut2, *rep_delta, *deltat;
  unsigned *vq_counter;
  int32_t *rep_idx;
  unsigned *gsync;   // grid-barrier counter, zero at launch
  uint32_t *status;  // device status word
};
// Cooperative launch only (every block resident): 256 threads, FUSED_SMEM of
// dynamic shared memory.
__global__ void k_prologue_fused(const FusedPrologueParams p);

constexpr int QUANTV1_SMEM = 128 * 272;              // gathered rows
constexpr int QUANTV2_SMEM = 128 * 272 + 128 * 144;  // NVFP4 pass 2: rows + transposed codes
constexpr int QUANTV2E_SMEM = 128 * 272;            // E4M3 pass 2: rows, then the codes in place
constexpr int KMEANS8_SMEM = 2 * 128 * 272;  // double-buffered chunk rows
constexpr int KMEANS8TC_STAGES = 3;   // chunk ring of k_kmeans_pass8tc
constexpr int KM_THREADS = 512;       // k_kmeans_pass8tc: 16 warps, two blocks per SM
constexpr int KMEANS8TC_SMEM = KMEANS8TC_STAGES * 128 * 256 + 4096 + 1024;  // swizzled chunks, centroid operand, alignment
constexpr int FUSED_SMEM = KMEANS8_SMEM > QUANTV2_SMEM ? KMEANS8_SMEM : QUANTV2_SMEM;  // the largest phase
constexpr int KMEANS_SMEM_FIXED = 128 * 66 * 4;  // chunk rows; + k*128*(4+8) for centroids and sums

}  // namespace vc
