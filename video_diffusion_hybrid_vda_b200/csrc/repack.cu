// Head-block repacking between layouts with different per-head widths.
//
// The tensor-core kernels take head dims of 64 or 128 (and the fuse GEMMs a
// hidden size that 256-wide tiles divide).  Smaller heads (d = 16 or 32) are
// run by copying each head's columns into a wider zero-padded block of a
// workspace, running the wide kernels, and copying the real columns back.
// Zero padding is exact for every step of the layer: padded key/value dims
// add zero blocks to A and B (P gets an identity block, C and the states
// zero blocks), padded q/k dims add nothing to a score, padded v dims give
// zero outputs, and the RMSNorm divides by the true head dim.
#include <cuda_bf16.h>

#include "common.cuh"
#include "repack.cuh"

namespace vdn {
namespace {

// dst[rb*dr_dst + jr][cb*dc_dst + jc] =
//     (jr < dr_src && jc < dc_src) ? src[rb*dr_src + jr][cb*dc_src + jc] : 0
template <typename T>
__global__ void repack_kernel(T* __restrict__ dst, int64_t ld_dst, const T* __restrict__ src,
                              int64_t ld_src, int rblocks, int dr_dst, int dr_src, int cblocks,
                              int dc_dst, int dc_src) {
  const int64_t rows = static_cast<int64_t>(rblocks) * dr_dst;
  const int64_t cols = static_cast<int64_t>(cblocks) * dc_dst;
  const int64_t total = rows * cols;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = idx / cols, c = idx % cols;
    const int64_t rb = r / dr_dst, jr = r % dr_dst;
    const int64_t cb = c / dc_dst, jc = c % dc_dst;
    T v = static_cast<T>(0.0f);
    if (jr < dr_src && jc < dc_src) v = src[(rb * dr_src + jr) * ld_src + cb * dc_src + jc];
    dst[r * ld_dst + c] = v;
  }
}

template <typename T>
cudaError_t launch_repack_t(cudaStream_t st, T* dst, int64_t ld_dst, const T* src,
                            int64_t ld_src, int rblocks, int dr_dst, int dr_src, int cblocks,
                            int dc_dst, int dc_src) {
  const int64_t total = static_cast<int64_t>(rblocks) * dr_dst * cblocks * dc_dst;
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 4096 ? want : 4096);
  repack_kernel<T><<<blocks, threads, 0, st>>>(dst, ld_dst, src, ld_src, rblocks, dr_dst, dr_src,
                                               cblocks, dc_dst, dc_src);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_repack_bf16(cudaStream_t st, void* dst, int64_t ld_dst, const void* src,
                               int64_t ld_src, int rblocks, int dr_dst, int dr_src, int cblocks,
                               int dc_dst, int dc_src) {
  return launch_repack_t(st, static_cast<__nv_bfloat16*>(dst), ld_dst,
                         static_cast<const __nv_bfloat16*>(src), ld_src, rblocks, dr_dst, dr_src,
                         cblocks, dc_dst, dc_src);
}

cudaError_t launch_repack_f32(cudaStream_t st, float* dst, int64_t ld_dst, const float* src,
                              int64_t ld_src, int rblocks, int dr_dst, int dr_src, int cblocks,
                              int dc_dst, int dc_src) {
  return launch_repack_t(st, dst, ld_dst, src, ld_src, rblocks, dr_dst, dr_src, cblocks, dc_dst,
                         dc_src);
}

}  // namespace vdn
