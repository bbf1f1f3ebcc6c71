// vc_testing.cu -- test hooks declared in include/vc_attn_testing.h: the
// production device functions run element by element, and the bounded wait run
// against a barrier that is never completed.
#include <cuda_runtime.h>

#include <algorithm>
#include <stdint.h>

#include "../../include/vc_attn_testing.h"
#include "vc_common.cuh"
#include "vc_sm100.cuh"

namespace vc {
namespace {

__global__ void e4m3_round_kernel(const float* __restrict__ x, uint8_t* __restrict__ out, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = cvt_e4m3(x[i]);
}

__global__ void e2m1_round_kernel(const float* __restrict__ x, uint8_t* __restrict__ out, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = cvt_e2m1x2(x[i], 0.0f) & 0xF;
}

__global__ void expcast_kernel(const float* __restrict__ t, const float* __restrict__ c,
                               const float* __restrict__ M, int32_t bias_b, uint8_t* __restrict__ out, int64_t n,
                               int32_t hot) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float bias = expcast_bias(bias_b, M[i]);
    const float c8 = 8.0f * c[i];
    out[i] = hot ? (uint8_t)(__float_as_uint(expcast_z(t[i], c8, bias)) & 0xFFu)
                 : (uint8_t)expcast_code(t[i], c8, bias);
  }
}

__global__ void bounded_wait_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit_ns, nullptr)) report_status(status, VC_ERR_TIMEOUT);
  __syncthreads();
}

int grid_for(int64_t n) { return (int)std::min<int64_t>(4096, std::max<int64_t>(1, (n + 255) / 256)); }

}  // namespace
}  // namespace vc

static vc_status_t launched(cudaError_t e) { return e == cudaSuccess ? VC_OK : VC_ERR_CUDA; }

extern "C" {

vc_status_t vc_attn_test_e4m3_round(const float* x, uint8_t* codes, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !codes))) return VC_ERR_INVALID_ARG;
  if (n == 0) return VC_OK;
  vc::e4m3_round_kernel<<<vc::grid_for(n), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, codes, n);
  return launched(cudaGetLastError());
}

vc_status_t vc_attn_test_e2m1_round(const float* x, uint8_t* codes, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !codes))) return VC_ERR_INVALID_ARG;
  if (n == 0) return VC_OK;
  vc::e2m1_round_kernel<<<vc::grid_for(n), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, codes, n);
  return launched(cudaGetLastError());
}

vc_status_t vc_attn_test_expcast(const float* t, const float* c, const float* M, int32_t bias_b, uint8_t* codes,
                                 int64_t n, int32_t hot, void* stream) {
  if (n < 0 || (n > 0 && (!t || !c || !M || !codes))) return VC_ERR_INVALID_ARG;
  if (n == 0) return VC_OK;
  vc::expcast_kernel<<<vc::grid_for(n), 256, 0, static_cast<cudaStream_t>(stream)>>>(t, c, M, bias_b, codes, n,
                                                                                       hot);
  return launched(cudaGetLastError());
}

vc_status_t vc_attn_test_bounded_wait(int32_t* dev_status, uint64_t limit_ns, void* stream) {
  if (!dev_status || limit_ns > 10000000000ull) return VC_ERR_INVALID_ARG;
  vc::bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_status, limit_ns);
  return launched(cudaGetLastError());
}

}  // extern "C"
