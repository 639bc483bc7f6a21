// Batched SPD solve for the VDA closed form ("Video DeltaNet", 10100.com
// article, 方法概述 item 2: S_t = (S_bar_t + B_t)(I + A_t)^-1).
//
// Per (frame t, head h), one CTA of 512 threads:
//   1. Cholesky  L L^T = I + A   (right-looking, the matrix held in registers
//      as 4x8 (d=128) tiles per thread; the scaled pivot column is published
//      through shared memory each step and L is kept in shared memory);
//   2. forward substitution  L Y = [I | B^T];
//   3. back substitution     L^T X = Y   ->  X = [P | C^T],
//      P = (I + A)^-1 and C = B P (because (I + A) C^T = B^T).
// The solve factors the symmetric part of the prep's A (the tensor-core
// product rounds beta*k on one side only, so A is symmetric up to that).
// I + A is symmetric positive definite with eigenvalues >= 1 (beta >= 0),
// so no pivoting is needed; a non-positive or NaN pivot is reported as
// VDN_ERR_NUMERIC in the status word.
// This step is FP32-ALU and latency bound (d^3-order work per problem).
#include "common.cuh"
#include "ptx.cuh"

namespace vdn {
namespace {

constexpr int kSolveThreads = 512;  // 32 row groups x 16 column groups

template <int DH>
struct SolveCfg {
  static constexpr int RA = DH / 32;        // rows per thread
  static constexpr int CB = DH / 16;        // matrix columns per thread (phase 1)
  static constexpr int RG = (2 * DH) / 64;  // 4-wide column groups of the RHS per thread
  static constexpr int LD = DH + 1;         // padded smem row stride of L
  static constexpr int SMEM = DH * LD * 4 + 2 * (2 * DH) * 4;
};

// Scale row group `ka` of the register tile by `dinv`, write it back and
// publish it (4 floats per 64-column group) to shared memory.  Written with
// predicated selects so the tile stays in registers.
template <int RA, int RG>
__device__ __forceinline__ void publish_row(float (&r)[RA][RG][4], int ka, float dinv,
                                            float* dst) {
#pragma unroll
  for (int g = 0; g < RG; ++g) {
    float y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float v = r[0][g][e];
#pragma unroll
      for (int a = 1; a < RA; ++a) v = (a == ka) ? r[a][g][e] : v;
      y[e] = v * dinv;
#pragma unroll
      for (int a = 0; a < RA; ++a) r[a][g][e] = (a == ka) ? y[e] : r[a][g][e];
    }
    *reinterpret_cast<float4*>(dst + 64 * g) = make_float4(y[0], y[1], y[2], y[3]);
  }
}

template <int DH>
__global__ void __launch_bounds__(kSolveThreads, 1)
    vda_solve_kernel(const float* __restrict__ A, const float* __restrict__ B,
                     float* __restrict__ P, float* __restrict__ Cout, uint32_t* status) {
  using Cfg = SolveCfg<DH>;
  extern __shared__ float sm[];
  float* Ls = sm;                    // [DH][LD], lower triangle of L
  float* buf0 = sm + DH * Cfg::LD;   // two 2*DH broadcast buffers
  float* buf1 = buf0 + 2 * DH;

  const int tx = threadIdx.x & 15;
  const int ty = threadIdx.x >> 4;
  const int64_t mat = static_cast<int64_t>(blockIdx.x) * DH * DH;
  const float* Am = A + mat;
  const float* Bm = B + mat;
  bool bad = false;

  // ---------------------------------------------------------------- phase 1
  float m[Cfg::RA][Cfg::CB];
#pragma unroll
  for (int a = 0; a < Cfg::RA; ++a)
#pragma unroll
    for (int b = 0; b < Cfg::CB; ++b) {
      const int i = ty + 32 * a, k = tx + 16 * b;
      // A from the prep is symmetric up to the bf16 rounding of beta*k on
      // one operand; the solve uses its symmetric part (A + A^T) / 2.
      m[a][b] = 0.5f * (__ldg(Am + i * DH + k) + __ldg(Am + k * DH + i)) + (i == k ? 1.f : 0.f);
    }

#pragma unroll 1
  for (int j = 0; j < DH; ++j) {
    float* col = (j & 1) ? buf1 : buf0;
    // owners of column j publish it
    if (tx == (j & 15)) {
      // select column j >> 4 of the tile with predicated moves (no dynamic
      // register indexing)
      const int jb = j >> 4;
#pragma unroll
      for (int a = 0; a < Cfg::RA; ++a) {
        float vsel = m[a][0];
#pragma unroll
        for (int b = 1; b < Cfg::CB; ++b) vsel = (b == jb) ? m[a][b] : vsel;
        col[ty + 32 * a] = vsel;
      }
    }
    __syncthreads();
    float piv = col[j];
    if (!(piv > 0.f)) {  // also catches NaN
      bad = true;
      piv = 1.f;
    }
    const float s = sqrtf(piv);
    const float inv = 1.f / s;
    if (threadIdx.x < DH) {
      const int i = threadIdx.x;
      Ls[i * Cfg::LD + j] = i > j ? col[i] * inv : (i == j ? s : 0.f);
    }
    float li[Cfg::RA], lk[Cfg::CB];
#pragma unroll
    for (int a = 0; a < Cfg::RA; ++a) li[a] = col[ty + 32 * a] * inv;
#pragma unroll
    for (int b = 0; b < Cfg::CB; ++b) lk[b] = col[tx + 16 * b] * inv;
#pragma unroll
    for (int a = 0; a < Cfg::RA; ++a) {
      if (32 * a + 31 <= j) continue;  // whole row group already factored
#pragma unroll
      for (int b = 0; b < Cfg::CB; ++b) {
        if (16 * b + 15 <= j) continue;
        const int i = ty + 32 * a, k = tx + 16 * b;
        if (i > j && k > j) m[a][b] = fmaf(-li[a], lk[b], m[a][b]);
      }
    }
    // the next step writes the other buffer; the one after that rewrites
    // this one only after the next step's barrier, so one barrier suffices
  }
  __syncthreads();  // L complete in shared memory

  // ---------------------------------------------------------------- phase 2
  // RHS columns c = 64 g + 4 tx + e; c < DH: identity, c >= DH: B^T.
  float r[Cfg::RA][Cfg::RG][4];
#pragma unroll
  for (int a = 0; a < Cfg::RA; ++a)
#pragma unroll
    for (int g = 0; g < Cfg::RG; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = ty + 32 * a, c = 64 * g + 4 * tx + e;
        r[a][g][e] = c < DH ? (i == c ? 1.f : 0.f) : __ldg(Bm + (c - DH) * DH + i);
      }

#pragma unroll 1
  for (int k = 0; k < DH; ++k) {
    float* row = (k & 1) ? buf1 : buf0;
    const float dinv = 1.f / Ls[k * Cfg::LD + k];
    if (ty == (k & 31)) {
      publish_row<Cfg::RA, Cfg::RG>(r, k >> 5, dinv, row + 4 * tx);
    }
    __syncthreads();
#pragma unroll
    for (int a = 0; a < Cfg::RA; ++a) {
      if (32 * a + 31 <= k) continue;
      const int i = ty + 32 * a;
      const float lik = i > k ? Ls[i * Cfg::LD + k] : 0.f;
#pragma unroll
      for (int g = 0; g < Cfg::RG; ++g) {
        const float4 y = *reinterpret_cast<const float4*>(row + 64 * g + 4 * tx);
        r[a][g][0] = fmaf(-lik, y.x, r[a][g][0]);
        r[a][g][1] = fmaf(-lik, y.y, r[a][g][1]);
        r[a][g][2] = fmaf(-lik, y.z, r[a][g][2]);
        r[a][g][3] = fmaf(-lik, y.w, r[a][g][3]);
      }
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- phase 3
#pragma unroll 1
  for (int k = DH - 1; k >= 0; --k) {
    float* row = (k & 1) ? buf1 : buf0;
    const float dinv = 1.f / Ls[k * Cfg::LD + k];
    if (ty == (k & 31)) {
      publish_row<Cfg::RA, Cfg::RG>(r, k >> 5, dinv, row + 4 * tx);
    }
    __syncthreads();
#pragma unroll
    for (int a = 0; a < Cfg::RA; ++a) {
      if (32 * a >= k) continue;  // rows i >= k are final
      const int i = ty + 32 * a;
      const float lki = i < k ? Ls[k * Cfg::LD + i] : 0.f;
#pragma unroll
      for (int g = 0; g < Cfg::RG; ++g) {
        const float4 x = *reinterpret_cast<const float4*>(row + 64 * g + 4 * tx);
        r[a][g][0] = fmaf(-lki, x.x, r[a][g][0]);
        r[a][g][1] = fmaf(-lki, x.y, r[a][g][1]);
        r[a][g][2] = fmaf(-lki, x.z, r[a][g][2]);
        r[a][g][3] = fmaf(-lki, x.w, r[a][g][3]);
      }
    }
  }

  // ---------------------------------------------------------------- store
  float* Pm = P + mat;
  float* Cm = Cout + mat;
#pragma unroll
  for (int a = 0; a < Cfg::RA; ++a) {
    const int i = ty + 32 * a;
#pragma unroll
    for (int g = 0; g < Cfg::RG; ++g) {
      const int c0 = 64 * g + 4 * tx;
      if (c0 < DH) {
        *reinterpret_cast<float4*>(Pm + i * DH + c0) =
            make_float4(r[a][g][0], r[a][g][1], r[a][g][2], r[a][g][3]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) Cm[(c0 - DH + e) * DH + i] = r[a][g][e];
      }
    }
  }
  if (bad) record_status(status, kStatusNumeric);
}

template <int DH>
cudaError_t launch_solve_dh(const Launch& ctx, const vdn_shape& s, const float* A,
                            const float* B, float* P, float* C) {
  using Cfg = SolveCfg<DH>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(vda_solve_kernel<DH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  vda_solve_kernel<DH><<<s.T * s.H, kSolveThreads, Cfg::SMEM, ctx.stream>>>(A, B, P, C,
                                                                             ctx.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_vda_solve(const Launch& ctx, const vdn_shape& s, const float* A,
                             const float* B, float* P, float* C) {
  if (s.d == 128) return launch_solve_dh<128>(ctx, s, A, B, P, C);
  if (s.d == 64) return launch_solve_dh<64>(ctx, s, A, B, P, C);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
