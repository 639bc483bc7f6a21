// Head-block repacking (see repack.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace vdn {

// dst[rb*dr_dst + jr][cb*dc_dst + jc] =
//     (jr < dr_src && jc < dc_src) ? src[rb*dr_src + jr][cb*dc_src + jc] : 0
// for rb < rblocks, jr < dr_dst, cb < cblocks, jc < dc_dst.
cudaError_t launch_repack_bf16(cudaStream_t st, void* dst, int64_t ld_dst, const void* src,
                               int64_t ld_src, int rblocks, int dr_dst, int dr_src, int cblocks,
                               int dc_dst, int dc_src);
cudaError_t launch_repack_f32(cudaStream_t st, float* dst, int64_t ld_dst, const float* src,
                              int64_t ld_src, int rblocks, int dr_dst, int dr_src, int cblocks,
                              int dc_dst, int dc_src);

// Padded head width used for head dims the tensor-core kernels do not take.
inline int padded_head_dim(int d) { return d <= 64 ? 64 : d; }

}  // namespace vdn
