// prologue.cuh - declarations of the prologue kernels (see prologue.cu).
#pragma once
#include <cstdint>

namespace vc {

__global__ void k_kmeans_init(const uint16_t *V, int N, int k, float *cent);
__global__ void k_kmeans_pass(const uint16_t *V, int N, int k, int cpb, int nblk, float *cent, int32_t *labels,
                              double *psum, int *pcnt, unsigned *counter, int accumulate);
__global__ void k_kmeans_pass8(const uint16_t *V, int N, int k, int cpb, int nblk, float *cent, int32_t *labels,
                               double *psum, int *pcnt, unsigned *counter, int accumulate);
__global__ void k_perm_sort(const int32_t *labels, int N, int k, int32_t *perm);
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

constexpr int QUANTV1_SMEM = 128 * 272;              // gathered rows
constexpr int QUANTV2_SMEM = 128 * 272 + 128 * 144;  // rows + transposed codes
constexpr int KMEANS8_SMEM = 2 * 128 * 272;  // double-buffered chunk rows
constexpr int KMEANS_SMEM_FIXED = 128 * 66 * 4;  // chunk rows; + k*128*(4+8) for centroids and sums

}  // namespace vc
