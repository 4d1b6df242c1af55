// api.cu - the C ABI of libvcattn (declared in include/vc_attn.h): argument
// validation, workspace layout, TMA tensor maps and kernel launches.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "attn_bf16.cuh"
#include "attn_fp4.cuh"
#include "attn_fp8.cuh"
#include "common.cuh"
#include "prologue.cuh"

namespace vc {

static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

Shape make_shape(int B, int H, int N, const vc_params &p, int R) {
  Shape s{};
  s.B = B;
  s.H = H;
  s.N = N;
  s.BH = B * H;
  s.Nb = (N + TILE - 1) / TILE;
  s.Npad = s.Nb * TILE;
  s.k = p.k;
  s.iters = p.iters;
  s.R = R;
  s.Rpad = R > 0 ? ((R + 127) / 128) * 128 : 0;
  s.nch32 = (s.Nb + CHUNK32 - 1) / CHUNK32;
  // k-means blocks per (b,h): two resident per SM for the k <= 8 pass (512
  // threads, a three-chunk ring), three for the generic pass
  const int target = std::max(1, ((p.k <= 8 ? 2 : 3) * 148) / s.BH);
  s.km_cpb = std::max(1, (s.Nb + target - 1) / target);
  s.km_nblk = (s.Nb + s.km_cpb - 1) / s.km_cpb;
  s.kb_nchunk = std::max(1, std::min(s.Nb, (4 * 148 + s.BH - 1) / s.BH));
  s.flags = p.flags;
  return s;
}

WsLayout make_layout(const Shape &s) {
  WsLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + std::max<size_t>(bytes, 1));
    return at;
  };
  const size_t BH = static_cast<size_t>(s.BH), N = static_cast<size_t>(s.N), Nb = static_cast<size_t>(s.Nb),
               Npad = static_cast<size_t>(s.Npad), k = static_cast<size_t>(s.k);
  L.status = take(256);
  L.gsync = take(256);  // grid-barrier counter of the one-launch prologue
  L.km_counter = take(BH * 4);
  L.vq_counter = take(BH * 4);
  L.kb_counter = take(BH * 4);
  L.cleared = o;
  L.perm = take(BH * N * 4);
  L.labels = take(BH * N * 4);
  L.cent = take(BH * k * D * 4);
  L.km_psum = take(BH * s.km_nblk * k * D * 8);
  L.km_pcnt = take(BH * s.km_nblk * k * 4);
  L.kbar_part = take(BH * s.kb_nchunk * D * 8);
  L.kbar = take(BH * D * 4);
  L.q8 = take(BH * Npad * D);
  L.sq = take(BH * Nb * 4);
  L.k8 = take(BH * Npad * D);
  L.sk = take(BH * Nb * 4);
  L.v8t = take(BH * D * Npad);
  L.vscale = take(BH * D * 4);
  L.vexpo = take(BH * D * 4);
  L.vmean = take(BH * Nb * D * 2);
  L.amax_part = take(BH * Nb * D * 4);
  L.mut2 = take(BH * s.nch32 * D * 64 * 2);
  L.err = take(BH * N * 4);
  L.rep_idx = take(BH * std::max(s.R, 1) * 4);
  L.rep_delta = take(BH * std::max(s.R, 1) * D * 2);
  L.deltat = take(BH * D * std::max(s.Rpad, 1) * 2);
  L.total = o;
  return L;
}

// The scratch of the clustering alone, when the permutation and the centroids
// are the caller's buffers: the status word and the k-means completion
// counters (zeroed per call), the labels and the k-means partial sums.
WsLayout make_cluster_layout(const Shape &s) {
  WsLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + std::max<size_t>(bytes, 1));
    return at;
  };
  const size_t BH = static_cast<size_t>(s.BH), N = static_cast<size_t>(s.N), k = static_cast<size_t>(s.k);
  L.status = take(256);
  L.km_counter = take(BH * 4);
  L.cleared = o;
  L.labels = take(BH * N * 4);
  L.km_psum = take(BH * s.km_nblk * k * D * 8);
  L.km_pcnt = take(BH * s.km_nblk * k * 4);
  L.total = o;
  return L;
}

}  // namespace vc

using namespace vc;

// ====================================================================== helpers
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D map over a row-major [outer][inner] array, 128-byte swizzle.
bool map2d(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, uint64_t inner, uint64_t outer,
           uint32_t box_in, uint32_t box_out) {
  EncodeTiledFn f = encoder();
  if (!f) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * static_cast<uint64_t>(esize)};
  cuuint32_t box[2] = {box_in, box_out};
  cuuint32_t es[2] = {1, 1};
  return f(m, dt, 2, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// 3-D map over bf16 [BH][N][128] with boxes of 64 channels x 128 rows x 1 head
// (rows past N read as zero).
bool map3d_bf16(CUtensorMap *m, const void *base, int N, int BH) {
  EncodeTiledFn f = encoder();
  if (!f) return false;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(N) * 256};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

vc_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VC_ERR_CUDA;
  static int ok_cache[64];  // 0 unknown, 1 ok, 2 unsupported
  if (dev < 0 || dev >= 64) return VC_ERR_UNSUPPORTED;
  if (ok_cache[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return VC_ERR_CUDA;
    ok_cache[dev] = (major == 10 && minor == 0) ? 1 : 2;
    if (ok_cache[dev] == 1) {
      if (cudaFuncSetAttribute(k_vc_attn_fwd, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(attn_fp8_smem_bytes())) != cudaSuccess ||
          cudaFuncSetAttribute(k_attn_ref_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(attn_bf16_smem_bytes())) != cudaSuccess ||
          cudaFuncSetAttribute(k_kmeans_pass, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               KMEANS_SMEM_FIXED + 64 * D * 12) != cudaSuccess ||
          cudaFuncSetAttribute(k_quantv_pass2, cudaFuncAttributeMaxDynamicSharedMemorySize, QUANTV2E_SMEM) !=
              cudaSuccess ||
          cudaFuncSetAttribute(k_quantv4_pass2, cudaFuncAttributeMaxDynamicSharedMemorySize, QUANTV2_SMEM) !=
              cudaSuccess ||
          cudaFuncSetAttribute(k_vc_attn_fwd4, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(attn_fp4_smem_bytes(false))) != cudaSuccess ||
          cudaFuncSetAttribute(k_vc_attn_fwd44, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(attn_fp4_smem_bytes(true))) != cudaSuccess ||
          cudaFuncSetAttribute(k_kmeans_pass8tc, cudaFuncAttributeMaxDynamicSharedMemorySize, KMEANS8TC_SMEM) !=
              cudaSuccess ||
          cudaFuncSetAttribute(k_kmeans_pass8tc, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared) != cudaSuccess ||
          cudaFuncSetAttribute(k_prologue_fused, cudaFuncAttributeMaxDynamicSharedMemorySize, FUSED_SMEM) !=
              cudaSuccess) {
        ok_cache[dev] = 0;
        return VC_ERR_CUDA;
      }
    }
  }
  return ok_cache[dev] == 1 ? VC_OK : VC_ERR_UNSUPPORTED;
}

vc_status check_params(const vc_params *p) {
  if (!p) return VC_ERR_INVALID_ARG;
  if (p->k < 1 || p->k > 64 || p->iters < 0 || p->iters > 64) return VC_ERR_INVALID_ARG;
  if (!(p->rho >= 0.0f && p->rho < 1.0f)) return VC_ERR_INVALID_ARG;
  if (!(p->softmax_scale >= 0.0f) || !std::isfinite(p->softmax_scale)) return VC_ERR_INVALID_ARG;
  if (p->expcast_bias < 8 || p->expcast_bias > 126) return VC_ERR_INVALID_ARG;
  if (p->flags & ~(VC_VSMOOTH | VC_REPAIR | VC_KSMOOTH | VC_WARMSTART | VC_VFMT_NVFP4 | VC_QK_NVFP4 |
                   VC_FUSED_PROLOGUE))
    return VC_ERR_INVALID_ARG;
  if ((p->flags & VC_QK_NVFP4) && !(p->flags & VC_VFMT_NVFP4)) return VC_ERR_INVALID_ARG;  // 4-bit QK needs 4-bit PV
  return VC_OK;
}

vc_status check_shape(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1) return VC_ERR_INVALID_ARG;
  if (d != 128) return VC_ERR_UNSUPPORTED;
  const long long Npad = ((static_cast<long long>(N) + 127) / 128) * 128;
  const long long elems = static_cast<long long>(B) * H * Npad * d;
  if (elems >= (1ll << 31)) return VC_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 65535) return VC_ERR_INVALID_ARG;  // grid.y
  return VC_OK;
}

struct Ws {
  uint8_t *base;
  WsLayout L;
  template <class T>
  T *at(size_t off) const { return reinterpret_cast<T *>(base + off); }
};

vc_status prep(int B, int H, int N, int d, const vc_params *p, void *ws, size_t ws_bytes, Shape *sh, Ws *w) {
  vc_status st = check_shape(B, H, N, d);
  if (st != VC_OK) return st;
  if ((st = check_params(p)) != VC_OK) return st;
  if (!ws || !aligned(ws, 256)) return VC_ERR_INVALID_ARG;
  *sh = make_shape(B, H, N, *p, vc_attn_repair_count(N, p));
  w->base = static_cast<uint8_t *>(ws);
  w->L = make_layout(*sh);
  if (ws_bytes < w->L.total) return VC_ERR_WORKSPACE;
  return VC_OK;
}

// Opt-in phase timing of vc_attn_fwd with CUDA events on the caller's stream:
// a ring of PROF_RING calls, read (and averaged) once after the timed loop.
constexpr int PROF_RING = 64;
struct Prof {
  bool on = false;
  int dev = -1;
  cudaEvent_t ev[PROF_RING][5] = {};
  int calls = 0;  // calls recorded since profiling was switched on
};
Prof g_prof;

void prof_mark(int i, cudaStream_t s) {
  if (g_prof.on) cudaEventRecord(g_prof.ev[g_prof.calls % PROF_RING][i], s);
}

vc_status last_error() { return cudaGetLastError() == cudaSuccess ? VC_OK : VC_ERR_CUDA; }

// Streams and events the library keeps per device for the life of the
// process, created on first use with that device current: the side stream of
// vc_attn_fwd (Q/K quantization beside the clustering and the V passes) with
// its fork, permutation-ready and join events, and the copy-in / copy-out
// streams of vc_attn_fwd_host with their events. Ordering with the caller's
// stream is by events only. Every call re-records the events, so a call holds
// the device's mutex while it enqueues work on them: concurrent calls from
// several host threads serialize on these streams.
struct DevCtx {
  std::mutex m_fwd, m_host;
  cudaStream_t side = nullptr;
  cudaEvent_t ev[3] = {};  // fork, permutation ready, join
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t hev[4] = {};  // start, copy-in done, compute done, last copy-out done
};
DevCtx g_devctx[64];

DevCtx *dev_ctx() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  return &g_devctx[dev];
}

// Create the missing streams / events (caller holds the matching mutex).
bool make_stream(cudaStream_t *s) {
  return *s || cudaStreamCreateWithFlags(s, cudaStreamNonBlocking) == cudaSuccess;
}
bool make_events(cudaEvent_t *ev, int n) {
  for (int i = 0; i < n; ++i)
    if (!ev[i] && cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) return false;
  return true;
}

// Clear the completion counters and the status word at the start of a call.
vc_status clear_small(const Ws &w, cudaStream_t s) {
  if (cudaMemsetAsync(w.base, 0, w.L.cleared, s) != cudaSuccess) return VC_ERR_CUDA;
  return VC_OK;
}

vc_status launch_cluster(const Shape &sh, const Ws &w, const uint16_t *V, int32_t *perm, float *cent,
                         cudaStream_t s) {
  int32_t *labels = w.at<int32_t>(w.L.labels);
  CUtensorMap tmv;
  if (sh.k <= 8 &&
      !map2d(&tmv, V, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, static_cast<uint64_t>(sh.BH) * sh.N, 64, TILE))
    return VC_ERR_CUDA;
  if (!(sh.flags & VC_WARMSTART)) {  // warm start: cent already holds the previous step's centroids
    k_kmeans_init<<<sh.BH, 128, 0, s>>>(V, sh.N, sh.k, cent);
    count_launch();
  }
  const size_t smem = KMEANS_SMEM_FIXED + static_cast<size_t>(sh.k) * D * 12;
  const dim3 grid(sh.km_nblk, sh.BH);
  for (int it = 0; it <= sh.iters; ++it) {
    if (sh.k <= 8)
      k_kmeans_pass8tc<<<grid, KM_THREADS, KMEANS8TC_SMEM, s>>>(tmv, sh.N, sh.k, sh.km_cpb, sh.km_nblk, cent, labels,
                                                         w.at<double>(w.L.km_psum), w.at<int>(w.L.km_pcnt),
                                                         w.at<unsigned>(w.L.km_counter), it < sh.iters ? 1 : 0,
                                                         w.at<uint32_t>(w.L.status));
    else
      k_kmeans_pass<<<grid, 128, smem, s>>>(V, sh.N, sh.k, sh.km_cpb, sh.km_nblk, cent, labels,
                                            w.at<double>(w.L.km_psum), w.at<int>(w.L.km_pcnt),
                                            w.at<unsigned>(w.L.km_counter), it < sh.iters ? 1 : 0);
    count_launch();
  }
  if (sh.k <= 8 && sh.km_nblk <= PERM_SCATTER_MAX_BLOCKS)
    k_perm_scatter<<<grid, 256, 0, s>>>(labels, w.at<int>(w.L.km_pcnt), sh.N, sh.k, sh.km_cpb, sh.km_nblk, perm);
  else
    k_perm_sort<<<sh.BH, 1024, 0, s>>>(labels, sh.N, sh.k, perm);
  count_launch();
  return VC_OK;
}

// parts: QK_Q = the K channel means and Q (no permutation needed), QK_K = K'
// through perm (after QK_Q on the same stream); both in one launch for QK_QK.
enum { QK_Q = 1, QK_K = 2, QK_QK = 3 };
void launch_quant_qk(const Shape &sh, const Ws &w, const uint16_t *Q, const uint16_t *K, const int32_t *perm,
                     uint8_t *q8, float *sq, uint8_t *k8, float *sk, cudaStream_t s, int parts = QK_QK) {
  const int ks = (sh.flags & VC_KSMOOTH) ? 1 : 0;
  double *part = w.at<double>(w.L.kbar_part);
  float *kbar = w.at<float>(w.L.kbar);
  if (!(parts & QK_Q)) {
    // K' alone: the means were computed by an earlier QK_Q launch on this stream
  } else if (ks) {
    k_kbar<<<dim3(sh.kb_nchunk, sh.BH), 256, 0, s>>>(K, sh.N, sh.kb_nchunk, 1, part, w.at<unsigned>(w.L.kb_counter),
                                                     kbar);
    count_launch();
  } else {
    cudaMemsetAsync(kbar, 0, static_cast<size_t>(sh.BH) * D * sizeof(float), s);  // no K smoothing: mean 0
  }
  const int zbase = (parts & QK_Q) ? 0 : 1, nz = parts == QK_QK ? 2 : 1;
  if (sh.flags & VC_QK_NVFP4)
    k_qk_quant4<<<dim3(sh.Nb, sh.BH, nz), 256, 0, s>>>(Q, K, perm, kbar, sh.N, sh.Nb, zbase, q8, sq, k8, sk);
  else
    k_qk_quant<<<dim3(sh.Nb, sh.BH, nz), 256, 0, s>>>(Q, K, perm, kbar, sh.N, sh.Npad, zbase, q8, sq, k8, sk);
  count_launch();
}

void launch_quant_v(const Shape &sh, const Ws &w, const uint16_t *V, const int32_t *perm, uint8_t *v8t,
                    float *vscale, uint16_t *vmean, int32_t *rep_idx, uint16_t *rep_delta, cudaStream_t s) {
  const int demean = (sh.flags & VC_VSMOOTH) ? 1 : 0;
  const int fp4 = (sh.flags & VC_VFMT_NVFP4) ? 1 : 0;
  int *vexpo = w.at<int>(w.L.vexpo);
  k_quantv_pass1<<<dim3(sh.Nb, sh.BH), 256, QUANTV1_SMEM, s>>>(V, perm, sh.N, sh.Nb, demean, fp4, vmean,
                                                     w.at<float>(w.L.amax_part), vscale, vexpo,
                                                     w.at<unsigned>(w.L.vq_counter));
  count_launch();
  if (fp4)
    k_quantv4_pass2<<<dim3(sh.Nb, sh.BH), 256, QUANTV2_SMEM, s>>>(V, perm, sh.N, sh.Nb, sh.nch32, vmean, vscale,
                                                                  vexpo, v8t, w.at<float>(w.L.err),
                                                                  w.at<uint16_t>(w.L.mut2));
  else
    k_quantv_pass2<<<dim3(sh.Nb, sh.BH), 256, QUANTV2E_SMEM, s>>>(V, perm, sh.N, sh.Nb, sh.Npad, sh.nch32, vmean,
                                                                 vscale, vexpo, v8t, w.at<float>(w.L.err),
                                                                 w.at<uint16_t>(w.L.mut2));
  count_launch();
  if (sh.R > 0) {
    if (sh.N <= 512 * 64)
      k_repair_select_reg<<<sh.BH, 512, 0, s>>>(w.at<float>(w.L.err), sh.N, sh.R, rep_idx);
    else
      k_repair_select<<<sh.BH, 1024, 0, s>>>(w.at<float>(w.L.err), sh.N, sh.R, rep_idx);
    count_launch();
    if (fp4)
      k_repair_delta4<<<dim3((sh.Rpad + 7) / 8, sh.BH), 256, 0, s>>>(V, perm, sh.N, sh.Nb, sh.R, sh.Rpad, rep_idx,
                                                                     vmean, vscale, vexpo, v8t, rep_delta,
                                                                     w.at<uint16_t>(w.L.deltat));
    else
      k_repair_delta<<<dim3((sh.Rpad + 7) / 8, sh.BH), 256, 0, s>>>(V, perm, sh.N, sh.Nb, sh.R, sh.Rpad, rep_idx,
                                                                    vmean, vscale, vexpo, rep_delta,
                                                                    w.at<uint16_t>(w.L.deltat));
    count_launch();
  }
}

// Blocks of the one-launch prologue: every block must be resident at once
// (cooperative launch), so the grid is the occupancy limit times the SMs.
int fused_grid() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (!cache[dev]) {
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_prologue_fused, 256, FUSED_SMEM) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return 0;
    cache[dev] = per_sm * sms;
  }
  return cache[dev];
}

// The whole prologue of vc_attn_fwd (E4M3 path, k <= 8) as one launch.
vc_status launch_prologue_fused(const Shape &sh, const Ws &w, const uint16_t *Q, const uint16_t *K,
                                const uint16_t *V, const int32_t *perm, bool cluster, cudaStream_t s) {
  FusedPrologueParams fp{};
  fp.Q = Q; fp.K = K; fp.V = V;
  fp.BH = sh.BH; fp.N = sh.N; fp.Nb = sh.Nb; fp.Npad = sh.Npad; fp.nch32 = sh.nch32; fp.k = sh.k;
  fp.iters = sh.iters; fp.R = sh.R; fp.Rpad = sh.Rpad; fp.km_cpb = sh.km_cpb; fp.km_nblk = sh.km_nblk;
  fp.kb_nchunk = sh.kb_nchunk;
  fp.demean = (sh.flags & VC_VSMOOTH) ? 1 : 0;
  fp.ksmooth = (sh.flags & VC_KSMOOTH) ? 1 : 0;
  fp.cluster = cluster ? 1 : 0;
  fp.perm_in = perm;
  fp.perm = w.at<int32_t>(w.L.perm); fp.labels = w.at<int32_t>(w.L.labels); fp.cent = w.at<float>(w.L.cent);
  fp.km_psum = w.at<double>(w.L.km_psum); fp.km_pcnt = w.at<int>(w.L.km_pcnt);
  fp.km_counter = w.at<unsigned>(w.L.km_counter);
  fp.kb_part = w.at<double>(w.L.kbar_part); fp.kb_counter = w.at<unsigned>(w.L.kb_counter);
  fp.kbar = w.at<float>(w.L.kbar);
  fp.q8 = w.at<uint8_t>(w.L.q8); fp.k8 = w.at<uint8_t>(w.L.k8); fp.v8t = w.at<uint8_t>(w.L.v8t);
  fp.sq = w.at<float>(w.L.sq); fp.sk = w.at<float>(w.L.sk); fp.amax_part = w.at<float>(w.L.amax_part);
  fp.vscale = w.at<float>(w.L.vscale); fp.err = w.at<float>(w.L.err); fp.vexpo = w.at<int>(w.L.vexpo);
  fp.vmean = w.at<uint16_t>(w.L.vmean); fp.mut2 = w.at<uint16_t>(w.L.mut2);
  fp.rep_delta = w.at<uint16_t>(w.L.rep_delta); fp.deltat = w.at<uint16_t>(w.L.deltat);
  fp.vq_counter = w.at<unsigned>(w.L.vq_counter); fp.rep_idx = w.at<int32_t>(w.L.rep_idx);
  fp.gsync = w.at<unsigned>(w.L.gsync); fp.status = w.at<uint32_t>(w.L.status);
  const int grid = fused_grid();
  if (grid <= 0) return VC_ERR_CUDA;
  void *args[] = {&fp};
  if (cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(k_prologue_fused), dim3(grid), dim3(256), args,
                                  FUSED_SMEM, s) != cudaSuccess)
    return VC_ERR_CUDA;
  count_launch();
  return VC_OK;
}

float kappa_of(float softmax_scale) {
  return static_cast<float>(8.0 * 1.4426950408889634074 * static_cast<double>(softmax_scale));
}
float scale_or_default(float s) { return s > 0.0f ? s : static_cast<float>(1.0 / std::sqrt(128.0)); }

}  // namespace

// ====================================================================== C ABI
extern "C" {

void vc_params_default(vc_params *p) {
  if (!p) return;
  p->k = 8;
  p->iters = 3;
  p->rho = 0.005f;
  p->softmax_scale = 0.0f;
  p->expcast_bias = 120;
  p->flags = VC_VSMOOTH | VC_REPAIR | VC_KSMOOTH;
}

const char *vc_status_str(vc_status s) {
  switch (s) {
    case VC_OK: return "ok";
    case VC_ERR_INVALID_ARG: return "invalid argument";
    case VC_ERR_UNSUPPORTED: return "unsupported (d must be 128; device must be compute capability 10.0)";
    case VC_ERR_WORKSPACE: return "workspace too small";
    case VC_ERR_CUDA: return "CUDA runtime error";
    case VC_ERR_TIMEOUT: return "a bounded device wait ran out";
  }
  return "unknown status";
}

int vc_attn_repair_count(int N, const vc_params *p) {
  if (!p || !(p->flags & VC_REPAIR) || N < 1) return 0;
  double r = std::ceil(static_cast<double>(p->rho) * static_cast<double>(N));
  if (r < 0) r = 0;
  if (r > N) r = N;
  return static_cast<int>(r);
}

size_t vc_attn_workspace_bytes(int B, int H, int N, int d, const vc_params *p) {
  if (check_shape(B, H, N, d) != VC_OK || check_params(p) != VC_OK) return 0;
  return make_layout(make_shape(B, H, N, *p, vc_attn_repair_count(N, p))).total;
}

vc_status vc_attn_cluster(const void *V, int B, int H, int N, int d, const vc_params *p, int32_t *perm,
                          float *centroids, void *ws, size_t ws_bytes, void *stream) {
  Shape sh;
  Ws w;
  vc_status st = prep(B, H, N, d, p, ws, ws_bytes, &sh, &w);
  if (st != VC_OK) return st;
  if (!V || !perm || !aligned(V, 16) || !aligned(perm, 16) || (centroids && !aligned(centroids, 16)) ||
      ((sh.flags & VC_WARMSTART) && !centroids))
    return VC_ERR_INVALID_ARG;
  if ((st = check_device()) != VC_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = clear_small(w, s)) != VC_OK) return st;
  if ((st = launch_cluster(sh, w, static_cast<const uint16_t *>(V), perm, centroids ? centroids : w.at<float>(w.L.cent),
                           s)) != VC_OK)
    return st;
  return last_error();
}

vc_status vc_attn_quant_qk(const void *Q, const void *K, const int32_t *perm, int B, int H, int N, int d,
                           const vc_params *p, uint8_t *q8, float *sq, uint8_t *k8, float *sk, void *ws,
                           size_t ws_bytes, void *stream) {
  Shape sh;
  Ws w;
  vc_status st = prep(B, H, N, d, p, ws, ws_bytes, &sh, &w);
  if (st != VC_OK) return st;
  if (!Q || !K || !q8 || !sq || !k8 || !sk || !aligned(Q, 16) || !aligned(K, 16) || !aligned(q8, 16) ||
      !aligned(k8, 16) || !aligned(sq, 4) || !aligned(sk, 4) || (perm && !aligned(perm, 4)))
    return VC_ERR_INVALID_ARG;
  if ((st = check_device()) != VC_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = clear_small(w, s)) != VC_OK) return st;
  launch_quant_qk(sh, w, static_cast<const uint16_t *>(Q), static_cast<const uint16_t *>(K), perm, q8, sq, k8, sk, s);
  return last_error();
}

vc_status vc_attn_quant_v(const void *V, const int32_t *perm, int B, int H, int N, int d, const vc_params *p,
                          uint8_t *v8, float *v_scale, void *v_mean, int32_t *rep_idx, void *rep_delta, void *ws,
                          size_t ws_bytes, void *stream) {
  Shape sh;
  Ws w;
  vc_status st = prep(B, H, N, d, p, ws, ws_bytes, &sh, &w);
  if (st != VC_OK) return st;
  if (!V || !v8 || !v_scale || !v_mean || !aligned(V, 16) || !aligned(v8, 16) || !aligned(v_scale, 4) ||
      !aligned(v_mean, 4) || (perm && !aligned(perm, 4)))
    return VC_ERR_INVALID_ARG;
  if (sh.R > 0 && (!rep_idx || !rep_delta || !aligned(rep_idx, 4) || !aligned(rep_delta, 8)))
    return VC_ERR_INVALID_ARG;
  if ((st = check_device()) != VC_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = clear_small(w, s)) != VC_OK) return st;
  launch_quant_v(sh, w, static_cast<const uint16_t *>(V), perm, v8, v_scale, static_cast<uint16_t *>(v_mean),
                 rep_idx, static_cast<uint16_t *>(rep_delta), s);
  return last_error();
}

vc_status vc_attn_fwd(const void *Q, const void *K, const void *V, int B, int H, int N, int d, const int32_t *perm,
                      const vc_params *p, void *O, void *ws, size_t ws_bytes, void *stream) {
  Shape sh;
  Ws w;
  vc_status st = prep(B, H, N, d, p, ws, ws_bytes, &sh, &w);
  if (st != VC_OK) return st;
  if (!Q || !K || !V || !O || !aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) ||
      (perm && !aligned(perm, 4)))
    return VC_ERR_INVALID_ARG;
  if ((st = check_device()) != VC_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint16_t *Qh = static_cast<const uint16_t *>(Q), *Kh = static_cast<const uint16_t *>(K),
                 *Vh = static_cast<const uint16_t *>(V);
  if ((st = clear_small(w, s)) != VC_OK) return st;
  prof_mark(0, s);
  uint8_t *q8 = w.at<uint8_t>(w.L.q8), *k8 = w.at<uint8_t>(w.L.k8), *v8t = w.at<uint8_t>(w.L.v8t);
  float *sq = w.at<float>(w.L.sq), *sk = w.at<float>(w.L.sk), *vscale = w.at<float>(w.L.vscale);
  int32_t *rep_idx = w.at<int32_t>(w.L.rep_idx);
  const bool clusters = !perm && (sh.flags & VC_VSMOOTH);
  const bool fused = (sh.flags & VC_FUSED_PROLOGUE) && sh.k <= 8 &&
                     !(sh.flags & (VC_VFMT_NVFP4 | VC_QK_NVFP4));
  if (fused) {
    // the whole prologue in one launch; its time is reported as the first phase
    if ((st = launch_prologue_fused(sh, w, Qh, Kh, Vh, perm, clusters, s)) != VC_OK) return st;
    prof_mark(1, s);
    prof_mark(2, s);
    prof_mark(3, s);
  } else {
    // Q/K quantization on a side stream (disjoint workspace regions). When this
    // call clusters, the K channel means and Q (which do not depend on the
    // permutation) start with the call, concurrent with the clustering, and K'
    // follows once the permutation is known; otherwise Q and K' are one launch.
    // Either way they run concurrently with the V passes, and the attention
    // kernel waits for both streams. Per-call events, released once the work
    // completes.
    DevCtx *dc = dev_ctx();
    if (!dc) return VC_ERR_CUDA;
    std::lock_guard<std::mutex> lock(dc->m_fwd);
    if (!make_stream(&dc->side) || !make_events(dc->ev, 3)) return VC_ERR_CUDA;
    cudaStream_t side = dc->side;
    const cudaEvent_t *ev = dc->ev;
    if (cudaEventRecord(ev[0], s) != cudaSuccess || cudaStreamWaitEvent(side, ev[0], 0) != cudaSuccess)
      return VC_ERR_CUDA;
    if (clusters) launch_quant_qk(sh, w, Qh, Kh, nullptr, q8, sq, k8, sk, side, QK_Q);
    const int32_t *pm = perm;
    if (clusters) {
      Shape cold = sh;  // vc_attn_fwd has no centroid input: always the default start
      cold.flags &= ~VC_WARMSTART;
      if ((st = launch_cluster(cold, w, Vh, w.at<int32_t>(w.L.perm), w.at<float>(w.L.cent), s)) != VC_OK) return st;
      pm = w.at<int32_t>(w.L.perm);
    }
    prof_mark(1, s);
    // from here on a failed record or wait returns after joining what was
    // already forked, so that no work of this call stays unordered
    bool evok = cudaEventRecord(ev[1], s) == cudaSuccess && cudaStreamWaitEvent(side, ev[1], 0) == cudaSuccess;
    if (evok) launch_quant_qk(sh, w, Qh, Kh, pm, q8, sq, k8, sk, side, clusters ? QK_K : QK_QK);
    const bool joined = cudaEventRecord(ev[2], side) == cudaSuccess;
    if (evok && joined)
      launch_quant_v(sh, w, Vh, pm, v8t, vscale, w.at<uint16_t>(w.L.vmean), rep_idx, w.at<uint16_t>(w.L.rep_delta),
                     s);
    prof_mark(2, s);
    if (!joined || cudaStreamWaitEvent(s, ev[2], 0) != cudaSuccess || !evok) return VC_ERR_CUDA;
    prof_mark(3, s);
  }

  const bool fp4 = (sh.flags & VC_VFMT_NVFP4) != 0;
  const bool qk4 = (sh.flags & VC_QK_NVFP4) != 0;
  CUtensorMap tq, tk, tv, tmu, tdt;
  const uint64_t rows = static_cast<uint64_t>(sh.BH) * sh.Npad;
  bool ok = map2d(&tq, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 128, rows, 128, 128) &&
            map2d(&tk, k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 128, rows, 128, 128) &&
            (fp4 || map2d(&tv, v8t, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, sh.Npad, static_cast<uint64_t>(sh.BH) * 128,
                          128, 128)) &&
            map2d(&tmu, w.at<uint16_t>(w.L.mut2), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64,
                  static_cast<uint64_t>(sh.BH) * sh.nch32 * 128, 64, 128);
  if (ok) {
    if (sh.R > 0)
      ok = map2d(&tdt, w.at<uint16_t>(w.L.deltat), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sh.Rpad,
                 static_cast<uint64_t>(sh.BH) * 128, 64, 128);
    else
      tdt = tmu;  // unused when R == 0
  }
  if (!ok) return VC_ERR_CUDA;
  if (fp4) {
    AttnFp4Params ap{};
    ap.N = sh.N;
    ap.Nb = sh.Nb;
    ap.Npad = sh.Npad;
    ap.nch32 = sh.nch32;
    ap.R = sh.R;
    ap.Rpad = sh.Rpad;
    ap.kappa = kappa_of(scale_or_default(p->softmax_scale));
    ap.sq = sq;
    ap.sk = sk;
    ap.vscale = vscale;
    ap.v4img = v8t;
    ap.qimg = qk4 ? q8 : nullptr;
    ap.kimg = qk4 ? k8 : nullptr;
    ap.rep_idx = rep_idx;
    ap.k8 = k8;
    ap.O = static_cast<uint16_t *>(O);
    ap.status = w.at<uint32_t>(w.L.status);
    if (qk4)
      k_vc_attn_fwd44<<<dim3((sh.Nb + 1) / 2, sh.BH), 352, attn_fp4_smem_bytes(true), s>>>(tq, tk, tmu, tdt, ap);
    else
      k_vc_attn_fwd4<<<dim3((sh.Nb + 1) / 2, sh.BH), 352, attn_fp4_smem_bytes(false), s>>>(tq, tk, tmu, tdt, ap);
    count_launch();
    prof_mark(4, s);
    if (g_prof.on) ++g_prof.calls;
    return last_error();
  }
  AttnFp8Params ap{};
  ap.N = sh.N;
  ap.Nb = sh.Nb;
  ap.Npad = sh.Npad;
  ap.nch32 = sh.nch32;
  ap.R = sh.R;
  ap.Rpad = sh.Rpad;
  ap.C = p->expcast_bias;
  ap.kappa = kappa_of(scale_or_default(p->softmax_scale));
  ap.sq = sq;
  ap.sk = sk;
  ap.vscale = vscale;
  ap.rep_idx = rep_idx;
  ap.k8 = k8;
  ap.O = static_cast<uint16_t *>(O);
  ap.status = w.at<uint32_t>(w.L.status);
  k_vc_attn_fwd<<<dim3((sh.Nb + 1) / 2, sh.BH), 352, attn_fp8_smem_bytes(), s>>>(tq, tk, tv, tmu, tdt, ap);
  count_launch();
  prof_mark(4, s);
  if (g_prof.on) ++g_prof.calls;
  return last_error();
}

vc_status vc_attn_profile(int on) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VC_ERR_CUDA;
  if (on) {
    if (g_prof.dev != dev) {
      for (int c = 0; c < PROF_RING; ++c)
        for (int i = 0; i < 5; ++i)
          if (cudaEventCreate(&g_prof.ev[c][i]) != cudaSuccess) return VC_ERR_CUDA;
      g_prof.dev = dev;
    }
    g_prof.on = true;
  } else {
    g_prof.on = false;
  }
  g_prof.calls = 0;
  return VC_OK;
}

int vc_attn_profile_read(float *ms, int max_n) {
  const int n = std::min(g_prof.calls, PROF_RING);
  if (!ms || max_n < 4 || n == 0) return 0;
  double acc[4] = {0, 0, 0, 0};
  for (int c = 0; c < n; ++c) {
    const int slot = (g_prof.calls - n + c) % PROF_RING;
    if (cudaEventSynchronize(g_prof.ev[slot][4]) != cudaSuccess) return 0;
    for (int i = 0; i < 4; ++i) {
      float t = 0.0f;
      if (cudaEventElapsedTime(&t, g_prof.ev[slot][i], g_prof.ev[slot][i + 1]) != cudaSuccess) return 0;
      acc[i] += t;
    }
  }
  for (int i = 0; i < 4; ++i) ms[i] = static_cast<float>(acc[i] / n);
  return 4;
}

// End-to-end forward from host buffers: runs of consecutive heads, copy-in on
// one stream, compute on the caller's stream, copy-out on another; each stream
// waits for the event of the previous stage of the same run. An event can be
// re-recorded after a wait has been issued on it (the wait binds to the record
// current at the time of the wait), so one event per direction suffices.
vc_status vc_attn_fwd_host(const void *hQ, const void *hK, const void *hV, int B, int H, int N, int d,
                           const vc_params *p, void *hO, void *dQ, void *dK, void *dV, void *dO, int groups,
                           void *ws, size_t ws_bytes, void *stream) {
  vc_status st = check_shape(B, H, N, d);
  if (st != VC_OK) return st;
  if ((st = check_params(p)) != VC_OK) return st;
  if (!hQ || !hK || !hV || !hO || !dQ || !dK || !dV || !dO || groups < 1 || !aligned(dQ, 16) || !aligned(dK, 16) ||
      !aligned(dV, 16) || !aligned(dO, 16) || !ws || !aligned(ws, 256))
    return VC_ERR_INVALID_ARG;
  const long long BH = static_cast<long long>(B) * H;
  const int G = static_cast<int>(std::min<long long>(groups, BH));
  const int gh = static_cast<int>((BH + G - 1) / G);
  // the workspace must hold one run of gh heads; vc_attn_fwd checks the rest
  if (vc_attn_workspace_bytes(1, gh, N, d, p) > ws_bytes) return VC_ERR_WORKSPACE;
  st = check_device();
  if (st != VC_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DevCtx *dc = dev_ctx();
  if (!dc) return VC_ERR_CUDA;
  std::lock_guard<std::mutex> lock(dc->m_host);
  if (!make_stream(&dc->s_in) || !make_stream(&dc->s_out) || !make_events(dc->hev, 4)) return VC_ERR_CUDA;
  cudaStream_t s_in = dc->s_in, s_out = dc->s_out;
  cudaEvent_t ev_start = dc->hev[0], ev_in = dc->hev[1], ev_out = dc->hev[2], ev_done = dc->hev[3];
  bool ok = cudaEventRecord(ev_start, s) == cudaSuccess && cudaStreamWaitEvent(s_in, ev_start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(s_out, ev_start, 0) == cudaSuccess;
  const size_t head_bytes = static_cast<size_t>(N) * d * sizeof(uint16_t);
  for (int g = 0; g < G && ok && st == VC_OK; ++g) {
    const long long h0 = static_cast<long long>(g) * gh;
    if (h0 >= BH) break;
    const int hn = static_cast<int>(std::min<long long>(gh, BH - h0));
    const size_t off = static_cast<size_t>(h0) * head_bytes, bytes = static_cast<size_t>(hn) * head_bytes;
    auto at = [&](const void *base) { return static_cast<const char *>(base) + off; };
    auto atw = [&](void *base) { return static_cast<char *>(base) + off; };
    ok = cudaMemcpyAsync(atw(dQ), at(hQ), bytes, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
         cudaMemcpyAsync(atw(dK), at(hK), bytes, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
         cudaMemcpyAsync(atw(dV), at(hV), bytes, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
         cudaEventRecord(ev_in, s_in) == cudaSuccess && cudaStreamWaitEvent(s, ev_in, 0) == cudaSuccess;
    if (!ok) break;
    st = vc_attn_fwd(at(dQ), at(dK), at(dV), 1, hn, N, d, nullptr, p, atw(dO), ws, ws_bytes, stream);
    if (st != VC_OK) break;
    ok = cudaEventRecord(ev_out, s) == cudaSuccess && cudaStreamWaitEvent(s_out, ev_out, 0) == cudaSuccess &&
         cudaMemcpyAsync(atw(hO), at(dO), bytes, cudaMemcpyDeviceToHost, s_out) == cudaSuccess;
  }
  // the caller's stream resumes after the last copy-out (also on an error path,
  // so that nothing of this call is left running unordered)
  const bool tail_ok = cudaEventRecord(ev_done, s_out) == cudaSuccess && cudaStreamWaitEvent(s, ev_done, 0) == cudaSuccess;
  if (st != VC_OK) return st;
  return (ok && tail_ok) ? VC_OK : VC_ERR_CUDA;
}

vc_status vc_attn_fwd_ref_bf16(const void *Q, const void *K, const void *V, int B, int H, int N, int d,
                               float softmax_scale, void *O, void *stream) {
  vc_status st = check_shape(B, H, N, d);
  if (st != VC_OK) return st;
  if (!(softmax_scale >= 0.0f) || !std::isfinite(softmax_scale)) return VC_ERR_INVALID_ARG;
  if (!Q || !K || !V || !O || !aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16))
    return VC_ERR_INVALID_ARG;
  if ((st = check_device()) != VC_OK) return st;
  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  if (!map3d_bf16(&tq, Q, N, BH) || !map3d_bf16(&tk, K, N, BH) || !map3d_bf16(&tv, V, N, BH)) return VC_ERR_CUDA;
  AttnBf16Params ap{};
  ap.N = N;
  ap.Nb = (N + 127) / 128;
  ap.scale_log2 = static_cast<float>(static_cast<double>(scale_or_default(softmax_scale)) * 1.4426950408889634074);
  ap.O = static_cast<uint16_t *>(O);
  ap.status = nullptr;  // no workspace here: a timeout shows as a wrong result only
  k_attn_ref_bf16<<<dim3(ap.Nb, BH), 192, attn_bf16_smem_bytes(), static_cast<cudaStream_t>(stream)>>>(tq, tk, tv, ap);
  count_launch();
  return last_error();
}

vc_status vc_attn_device_status(void *ws, void *stream) {
  if (!ws || !aligned(ws, 256)) return VC_ERR_INVALID_ARG;
  uint32_t v = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return VC_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return VC_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) return VC_ERR_CUDA;
  return (v & ST_TIMEOUT) ? VC_ERR_TIMEOUT : VC_OK;
}

unsigned long long vc_attn_launch_count(void) { return g_launches.load(); }

}  // extern "C"

// ====================================================================== allocation-free clustering
// For callers that cannot allocate device memory at the point where they
// cluster (see vc_attn_cluster_noalloc in vc_attn.h): the clustering scratch
// lives in a fixed device array that the library owns for the life of the
// process on every device that loads it.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch for each device, looked up once per
// device (with that device current) by cudaGetSymbolAddress. In host code the
// symbol itself is only a host-side stand-in and must never be passed to a
// kernel.
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64] = {};

vc_status noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VC_ERR_CUDA;
  if (dev < 0 || dev >= 64) return VC_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return VC_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return VC_OK;
}

}  // namespace

extern "C" vc_status vc_attn_cluster_noalloc(const void *V, int B, int H, int N, int d, const vc_params *p,
                                             int32_t *perm, float *centroids, void *stream) {
  vc_status st = check_shape(B, H, N, d);
  if (st != VC_OK) return st;
  if ((st = check_params(p)) != VC_OK) return st;
  if (!V || !perm || !centroids || !aligned(V, 16) || !aligned(perm, 16) || !aligned(centroids, 16))
    return VC_ERR_INVALID_ARG;
  Shape sh = make_shape(B, H, N, *p, vc_attn_repair_count(N, p));
  // the clustering's own scratch only: perm and centroids are the caller's
  WsLayout L = make_cluster_layout(sh);
  if (L.total > kNoAllocScratchBytes) return VC_ERR_WORKSPACE;
  if ((st = check_device()) != VC_OK) return st;
  void *scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != VC_OK) return st;
  Ws w;
  w.base = static_cast<uint8_t *>(scratch);
  w.L = L;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the completion counters must start at zero; the array keeps the previous call's contents
  if ((st = clear_small(w, s)) != VC_OK) return st;
  if ((st = launch_cluster(sh, w, static_cast<const uint16_t *>(V), perm, centroids, s)) != VC_OK) return st;
  const cudaError_t e = cudaGetLastError();
  if (e == cudaErrorContextIsDestroyed || e == cudaErrorDeviceUninitialized || e == cudaErrorInvalidResourceHandle) {
    // the context that held the array is gone: look its address up again next time
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
      std::lock_guard<std::mutex> lock(g_noalloc_mu);
      g_noalloc_ptr[dev] = nullptr;
    }
  }
  return e == cudaSuccess ? VC_OK : VC_ERR_CUDA;
}

extern "C" size_t vc_attn_cluster_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }
