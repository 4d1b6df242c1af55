// misc.cu - element-wise device entry points that expose, for testing, the
// exact device code the attention and quantization kernels use: ExpCast and
// the hardware E4M3 encoder.
#include "common.cuh"
#include "expcast.cuh"

namespace vc {

__global__ void k_expcast(const float *__restrict__ acc, const float *__restrict__ alpha,
                          const float *__restrict__ c, long long npairs, uint8_t *__restrict__ out) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= npairs) return;
  const long long j = 2 * i;
  const uint32_t h = expcast2(acc[j], acc[j + 1], alpha[j] * TWO_M24, alpha[j] * TWO_M24, c[j] * TWO_M24);
  out[j] = static_cast<uint8_t>(h & 0xFFu);
  out[j + 1] = static_cast<uint8_t>((h >> 16) & 0xFFu);
}

__global__ void k_e4m3_encode(const float *__restrict__ x, long long npairs, uint8_t *__restrict__ out) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= npairs) return;
  const uint16_t c = e4m3x2(x[2 * i], x[2 * i + 1]);
  out[2 * i] = static_cast<uint8_t>(c & 0xFFu);
  out[2 * i + 1] = static_cast<uint8_t>(c >> 8);
}

}  // namespace vc

using namespace vc;

extern "C" vc_status vc_attn_expcast(const float *acc, const float *alpha, const float *c, long long n, uint8_t *out,
                                     void *stream) {
  if (n < 0 || (n & 1) || (n > 0 && (!acc || !alpha || !c || !out))) return VC_ERR_INVALID_ARG;
  if (n == 0) return VC_OK;
  const long long np = n / 2;
  k_expcast<<<static_cast<unsigned>((np + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(acc, alpha, c,
                                                                                                     np, out);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? VC_OK : VC_ERR_CUDA;
}

extern "C" vc_status vc_attn_e4m3_encode(const float *x, long long n, uint8_t *out, void *stream) {
  if (n < 0 || (n & 1) || (n > 0 && (!x || !out))) return VC_ERR_INVALID_ARG;
  if (n == 0) return VC_OK;
  const long long np = n / 2;
  k_e4m3_encode<<<static_cast<unsigned>((np + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, np, out);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? VC_OK : VC_ERR_CUDA;
}

// ---------------------------------------------------------------- bounded-wait self test
// One thread waits on an mbarrier that nothing ever arrives at, with a limit
// of `limit_cycles`; when the wait gives up it records ST_TIMEOUT in the
// status word, exactly as the attention kernels do, and returns.
#include "sm100.cuh"
namespace vc {
__global__ void k_wait_selftest(uint32_t *status, long long limit_cycles) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (!mbar_wait(&bar, 0, limit_cycles)) atomicOr(status, ST_TIMEOUT);
}
}  // namespace vc

extern "C" vc_status vc_attn_wait_selftest(void *ws, long long limit_cycles, void *stream) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) || limit_cycles < 1 || limit_cycles > (1ll << 32))
    return VC_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) return VC_ERR_CUDA;
  k_wait_selftest<<<1, 1, 0, s>>>(static_cast<uint32_t *>(ws), limit_cycles);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? VC_OK : VC_ERR_CUDA;
}
