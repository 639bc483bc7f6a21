// MXFP8 quantization of a bf16 operand (see mxfp8.cuh for the format and
// the scale layout): one thread per (row, 32-element block); reads 64 bytes,
// writes 32 bytes of codes and one scale byte.  HBM-bound.  Rows between R
// and the next multiple of 128 get the unit scale byte 127, so the last
// tile's scale block is fully defined.
#include <cuda_bf16.h>

#include "common.cuh"
#include "mxfp8.cuh"
#include "ptx.cuh"

namespace vdn {
namespace {

__global__ void mx_quantize_kernel(const __nv_bfloat16* __restrict__ x, int64_t ld, int R, int K,
                                   uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  const int kblocks = K / 32;
  const int rpad = (R + 127) / 128 * 128;
  const int64_t total = static_cast<int64_t>(rpad) * kblocks;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / kblocks;
    const int kb = static_cast<int>(i % kblocks);
    uint8_t byte = 127;
    if (r < R) {
      const uint4* src = reinterpret_cast<const uint4*>(x + r * ld + 32 * kb);
      float v[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 u = __ldg(src + c);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack_bf16x2(w[e]);
          v[8 * c + 2 * e] = f.x;
          v[8 * c + 2 * e + 1] = f.y;
        }
      }
      uint4 codes[2];
      byte = mx_quantize_block(v, codes);
      uint4* dst = reinterpret_cast<uint4*>(q + r * K + 32 * kb);
      dst[0] = codes[0];
      dst[1] = codes[1];
    }
    sf[mx_sf_offset(r, kb, K / 128)] = byte;
  }
}

}  // namespace

cudaError_t launch_mx_quantize(cudaStream_t st, const void* x, int64_t ld, int R, int K,
                               uint8_t* q, uint8_t* sf) {
  const int64_t total = static_cast<int64_t>((R + 127) / 128 * 128) * (K / 32);
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 148 * 16 ? want : 148 * 16);
  mx_quantize_kernel<<<blocks, threads, 0, st>>>(static_cast<const __nv_bfloat16*>(x), ld, R, K,
                                                 q, sf);
  return cudaGetLastError();
}

}  // namespace vdn

using namespace vdn;

extern "C" {

size_t vdn_mxfp8_scale_bytes(int64_t rows, int64_t cols) {
  if (rows < 1 || cols < 128 || cols % 128 != 0) return 0;
  return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>(cols / 128) * 512;
}

vdn_status vdn_mxfp8_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld, void* q,
                              void* sf, void* stream) {
  NvtxRange nvtx("vdn_mxfp8_quantize");
  if (x == nullptr || q == nullptr || sf == nullptr) return VDN_ERR_INVALID_ARG;
  if (rows < 1 || rows >= (int64_t(1) << 31) || cols < 128 || cols % 128 != 0 ||
      cols >= (int64_t(1) << 30) || ld < cols || ld % 8 != 0)
    return VDN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(q) & 15))
    return VDN_ERR_INVALID_ARG;
  if (launch_mx_quantize(static_cast<cudaStream_t>(stream), x, ld, static_cast<int>(rows),
                         static_cast<int>(cols), static_cast<uint8_t*>(q),
                         static_cast<uint8_t*>(sf)) != cudaSuccess)
    return VDN_ERR_CUDA;
  return VDN_OK;
}

}  // extern "C"
