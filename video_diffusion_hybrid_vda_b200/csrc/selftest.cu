// Diagnostic entry point: the Softmax's two exponential paths on given
// inputs, so tests can bound the FMA-pipe exponential against the MUFU one
// and against an exact reference.
#include "common.cuh"
#include "exp2_fma.cuh"

namespace vdn {
namespace {

__global__ void exp2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y_fma,
                                     float* __restrict__ y_mufu, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i];
  const float x1 = i + 1 < n ? x[i + 1] : 0.f;
  const uint64_t r = exp2_fma_x2(f32x2_pack(x0, x1));
  y_fma[i] = f32x2_lo(r);
  y_mufu[i] = exp2_mufu(x0);
  if (i + 1 < n) {
    y_fma[i + 1] = f32x2_hi(r);
    y_mufu[i + 1] = exp2_mufu(x1);
  }
}

}  // namespace
}  // namespace vdn

extern "C" vdn_status vdn_selftest_exp2(const float* x, float* y_fma, float* y_mufu, int n,
                                        void* stream) {
  if (n < 0 || (n > 0 && (!x || !y_fma || !y_mufu))) return VDN_ERR_INVALID_ARG;
  if (n == 0) return VDN_OK;
  const int threads = 256;
  const int blocks = ((n + 1) / 2 + threads - 1) / threads;
  vdn::exp2_selftest_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      x, y_fma, y_mufu, n);
  return cudaGetLastError() == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}
