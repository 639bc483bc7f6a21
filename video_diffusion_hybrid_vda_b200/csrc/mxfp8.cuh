// MXFP8 block quantization (OCP Microscaling: E4M3 elements, one UE8M0
// power-of-two scale per 32 consecutive elements along K), shared by the
// quantizer kernel and the GEMM epilogue that writes its output in MXFP8.
//
//   e = floor(log2(max |v|)) - 8, clamped to [-127, 127] (-127 for a zero
//   block); codes = E4M3(v * 2^-e), rounded to nearest even and saturated
//   at +-448; scale byte = e + 127.
// The scales of an [R, K] operand are stored in the tile layout the
// block-scaled MMA reads through tcgen05.cp: per 128-row x 128-column tile
// one 512-byte block holding the scale of (row r, K-block kb) at byte
// (r % 32) * 16 + ((r % 128) / 32) * 4 + kb % 4, tiles ordered
// [row tile][column tile].
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace vdn {

__host__ __device__ __forceinline__ int64_t mx_sf_offset(int64_t r, int kb, int ktiles) {
  return ((r >> 7) * ktiles + (kb >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (kb & 3);
}

// One MX block: 32 E4M3 codes (memory order) and the returned scale byte.
__device__ __forceinline__ uint8_t mx_quantize_block(const float (&v)[32], uint4 (&codes)[2]) {
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(v[e]));
  // floor(log2(amax)) is the unbiased exponent of a normal float; a zero or
  // subnormal maximum clamps to the smallest scale
  const int ef = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
  const int e = ef == 0 ? -127 : max(-127, min(127, ef - 127 - 8));
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e, exact
  uint32_t w[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(v[4 * q] * inv, v[4 * q + 1] * inv), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(v[4 * q + 2] * inv, v[4 * q + 3] * inv), __NV_SATFINITE, __NV_E4M3);
    w[q] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
  }
  codes[0] = make_uint4(w[0], w[1], w[2], w[3]);
  codes[1] = make_uint4(w[4], w[5], w[6], w[7]);
  return static_cast<uint8_t>(e + 127);
}

}  // namespace vdn
