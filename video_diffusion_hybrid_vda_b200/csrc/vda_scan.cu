// Bidirectional frame scan of Video DeltaNet's linear branch ("Video
// DeltaNet", 10100.com article, 方法概述 item 2 and the figure caption under
// 效率阶梯: a forward and a backward scan over the latent frames):
//
//   S_fwd_t = alpha_t S_fwd_{t-1} P_t + C_t      t = 0 .. T-1, S_fwd_{-1} = 0
//   S_bwd_t = alpha_t S_bwd_{t+1} P_t + C_t      t = T-1 .. 0, S_bwd_T   = 0
//
// which is (alpha_t S_prev + B_t)(I + A_t)^-1 with P_t = (I + A_t)^-1 and
// C_t = B_t P_t precomputed by the solve.  Rows of S evolve independently
// (row r of S_t only needs row r of S_{t-1}), so the state is split into
// blocks of R rows: one CTA per (row block, head, direction), all resident
// at once, each running all T steps with its rows of S in shared memory
// (transposed) and P_t, C_t streamed from L2.  Arithmetic is fp32 FMA; each
// thread owns a 4 x 4 tile of the new state.
#include "common.cuh"

namespace vdn {
namespace {

constexpr int kScanRows = 16;  // rows of S per CTA
constexpr int kTile = 4;       // 4 x 4 outputs per thread

template <int DH>
__global__ void __launch_bounds__((kScanRows / kTile) * (DH / kTile))
    vda_scan_kernel(const float* __restrict__ P, const float* __restrict__ C,
                    const float* __restrict__ alpha, float* __restrict__ states, int T, int H) {
  constexpr int CG = DH / kTile;  // column groups
  __shared__ __align__(16) float St[DH][kScanRows];  // S^T of this CTA's rows

  const int rb = blockIdx.x;  // row block
  const int h = blockIdx.y;
  const int dir = blockIdx.z;  // 0 forward, 1 backward
  const int cg = threadIdx.x % CG;
  const int rg = threadIdx.x / CG;
  const int row0 = rb * kScanRows + rg * kTile;  // first row of this thread's tile
  const int col0 = cg * kTile;

  for (int i = threadIdx.x; i < DH * kScanRows; i += blockDim.x) (&St[0][0])[i] = 0.f;
  __syncthreads();

  const int64_t mat_stride = static_cast<int64_t>(DH) * DH;
  float* out_dir = states + static_cast<int64_t>(dir) * T * H * mat_stride;

#pragma unroll 1
  for (int step = 0; step < T; ++step) {
    const int t = dir == 0 ? step : T - 1 - step;
    const float a = __ldg(alpha + t * H + h);
    const float* Pt = P + (static_cast<int64_t>(t) * H + h) * mat_stride;
    const float* Ct = C + (static_cast<int64_t>(t) * H + h) * mat_stride;

    float acc[kTile][kTile];
#pragma unroll
    for (int r = 0; r < kTile; ++r)
#pragma unroll
      for (int e = 0; e < kTile; ++e) acc[r][e] = 0.f;

    if (step > 0) {
#pragma unroll 8
      for (int k = 0; k < DH; ++k) {
        const float4 p = __ldg(reinterpret_cast<const float4*>(Pt + k * DH + col0));
        const float4 s = *reinterpret_cast<const float4*>(&St[k][rg * kTile]);
        const float sv[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
        for (int r = 0; r < kTile; ++r) {
          acc[r][0] = fmaf(sv[r], p.x, acc[r][0]);
          acc[r][1] = fmaf(sv[r], p.y, acc[r][1]);
          acc[r][2] = fmaf(sv[r], p.z, acc[r][2]);
          acc[r][3] = fmaf(sv[r], p.w, acc[r][3]);
        }
      }
    }
    float snew[kTile][kTile];
#pragma unroll
    for (int r = 0; r < kTile; ++r) {
      const float4 c = __ldg(reinterpret_cast<const float4*>(Ct + (row0 + r) * DH + col0));
      snew[r][0] = fmaf(a, acc[r][0], c.x);
      snew[r][1] = fmaf(a, acc[r][1], c.y);
      snew[r][2] = fmaf(a, acc[r][2], c.z);
      snew[r][3] = fmaf(a, acc[r][3], c.w);
      float* dst = out_dir + (static_cast<int64_t>(t) * H + h) * mat_stride +
                   static_cast<int64_t>(row0 + r) * DH + col0;
      *reinterpret_cast<float4*>(dst) = make_float4(snew[r][0], snew[r][1], snew[r][2], snew[r][3]);
    }
    __syncthreads();  // every thread has finished reading St
#pragma unroll
    for (int e = 0; e < kTile; ++e)
      *reinterpret_cast<float4*>(&St[col0 + e][rg * kTile]) =
          make_float4(snew[0][e], snew[1][e], snew[2][e], snew[3][e]);
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_vda_scan(const Launch& ctx, const vdn_shape& s, const float* P,
                            const float* C, const float* alpha, float* states) {
  if (s.d == 128) {
    dim3 grid(128 / kScanRows, s.H, 2);
    vda_scan_kernel<128><<<grid, (kScanRows / kTile) * (128 / kTile), 0, ctx.stream>>>(
        P, C, alpha, states, s.T, s.H);
  } else if (s.d == 64) {
    dim3 grid(64 / kScanRows, s.H, 2);
    vda_scan_kernel<64><<<grid, (kScanRows / kTile) * (64 / kTile), 0, ctx.stream>>>(
        P, C, alpha, states, s.T, s.H);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace vdn
