// Batched SPD solve for the VDA closed form ("Video DeltaNet", 10100.com
// article, 方法概述 item 2: S_t = (S_bar_t + B_t)(I + A_t)^-1).
//
// Per (frame t, head h) one CTA of 256 threads (two CTAs per SM, so two
// problems hide each other's barrier latency) produces
//   P_t = (I + A_sym)^-1,   A_sym = (A + A^T) / 2
// (the tensor-core product in the prep rounds beta*k on one operand only, so
// A is symmetric up to that rounding).  Two solvers:
//
//  Cholesky (default):
//   1. L L^T = I + A_sym, right-looking; the matrix lives in registers
//      (8x8 per thread at d = 128), the scaled pivot column is published
//      through shared memory each step and L is kept in shared memory;
//   2. W = L^-1 by forward substitution against I (row k of W is published
//      each step; column blocks that are still zero are skipped);
//   3. P = W^T W as a shared-memory product (no barriers inside the loop);
//      W is lower triangular, so entry (i, c) sums rows k >= max(i, c) only.
//  Gauss-Jordan (the inverse the pages' own kernels use):
//   one in-register sweep over the pivots, publishing the pivot row and
//   column each step, leaves (I + A_sym)^-1.
// The scan multiplies (alpha S + B_t) by P_t itself, so no B P is formed here.
//
// I + A_sym is symmetric positive definite with eigenvalues >= 1 (beta >= 0),
// so neither solver pivots; a non-positive or NaN pivot is reported as
// VDN_ERR_NUMERIC.  This step is FP32-ALU and latency bound.
#include "common.cuh"
#include "ptx.cuh"

namespace vdn {
namespace {

constexpr int kThreads = 256;  // 16 row groups x 16 column groups

template <int DH>
struct SolveCfg {
  static constexpr int RA = DH / 16;   // rows per thread (rows ty + 16 a)
  static constexpr int CB = DH / 16;   // columns per thread (cols tx + 16 b)
  static constexpr int RG = DH / 64;   // 4-wide column groups of W per thread
  static constexpr int LD = DH + 1;    // row stride of L (column accesses)
  static constexpr int LD2 = DH + 4;   // row stride of W / P (float4 rows)
  static constexpr int MAT = DH * LD2; // floats of the matrix buffer (>= DH * LD)
  static constexpr int TR = DH / 16;   // products: TR x TR tile per thread
  static constexpr int SMEM = MAT * 4 + 4 * DH * 4;
};

// Scale row group `ka` of the register tile by `dinv`, write it back and
// publish it (4 floats per 64-column group) to shared memory.  Predicated
// selects keep the tile in registers.
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

// Load (I + A_sym) into the register tile m (rows ty + 16 a, cols tx + 16 b).
template <int DH>
__device__ __forceinline__ void load_spd(const float* __restrict__ Am,
                                         float (&m)[SolveCfg<DH>::RA][SolveCfg<DH>::CB],
                                         int ty, int tx) {
#pragma unroll
  for (int a = 0; a < SolveCfg<DH>::RA; ++a)
#pragma unroll
    for (int b = 0; b < SolveCfg<DH>::CB; ++b) {
      const int i = ty + 16 * a, k = tx + 16 * b;
      m[a][b] = 0.5f * (__ldg(Am + i * DH + k) + __ldg(Am + k * DH + i)) + (i == k ? 1.f : 0.f);
    }
}

// ---------------------------------------------------------------- Cholesky

template <int DH>
__global__ void __launch_bounds__(kThreads, 2)
    vda_solve_kernel(const float* __restrict__ A, float* __restrict__ P, uint32_t* status) {
  using Cfg = SolveCfg<DH>;
  extern __shared__ float sm[];
  float* Ls = sm;                    // [DH][LD]: L, later W and P ([DH][LD2])
  float* buf0 = sm + Cfg::MAT;       // two 2*DH broadcast buffers
  float* buf1 = buf0 + 2 * DH;
  const int tx = threadIdx.x & 15;
  const int ty = threadIdx.x >> 4;
  const int64_t mat = static_cast<int64_t>(blockIdx.x) * DH * DH;
  bool bad = false;

  // ---------------------------------------------------------------- 1. Cholesky
  {
    float m[Cfg::RA][Cfg::CB];
    load_spd<DH>(A + mat, m, ty, tx);
#pragma unroll 1
    for (int j = 0; j < DH; ++j) {
      float* col = (j & 1) ? buf1 : buf0;
      if (tx == (j & 15)) {  // owners of column j publish it
        const int jb = j >> 4;
#pragma unroll
        for (int a = 0; a < Cfg::RA; ++a) {
          float v = m[a][0];
#pragma unroll
          for (int b = 1; b < Cfg::CB; ++b) v = (b == jb) ? m[a][b] : v;
          col[ty + 16 * a] = v;
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
      for (int a = 0; a < Cfg::RA; ++a) li[a] = col[ty + 16 * a] * inv;
#pragma unroll
      for (int b = 0; b < Cfg::CB; ++b) lk[b] = col[tx + 16 * b] * inv;
#pragma unroll
      for (int a = 0; a < Cfg::RA; ++a) {
        if (16 * a + 15 <= j) continue;  // whole row group already factored
#pragma unroll
        for (int b = 0; b < Cfg::CB; ++b) {
          if (16 * b + 15 <= j) continue;
          const int i = ty + 16 * a, k = tx + 16 * b;
          if (i > j && k > j) m[a][b] = fmaf(-li[a], lk[b], m[a][b]);
        }
      }
      // one barrier per step: the next step writes the other buffer
    }
  }
  __syncthreads();  // L complete in shared memory

  // ---------------------------------------------------------------- 2. W = L^-1
  // forward substitution against I; columns c = 64 g + 4 tx + e, rows ty + 16 a
  {
    float r[Cfg::RA][Cfg::RG][4];
#pragma unroll
    for (int a = 0; a < Cfg::RA; ++a)
#pragma unroll
      for (int g = 0; g < Cfg::RG; ++g)
#pragma unroll
        for (int e = 0; e < 4; ++e) r[a][g][e] = (ty + 16 * a == 64 * g + 4 * tx + e) ? 1.f : 0.f;
#pragma unroll 1
    for (int k = 0; k < DH; ++k) {
      float* row = (k & 1) ? buf1 : buf0;
      const float dinv = 1.f / Ls[k * Cfg::LD + k];
      if (ty == (k & 15)) publish_row<Cfg::RA, Cfg::RG>(r, k >> 4, dinv, row + 4 * tx);
      __syncthreads();
#pragma unroll
      for (int a = 0; a < Cfg::RA; ++a) {
        if (16 * a + 15 <= k) continue;
        const int i = ty + 16 * a;
        const float lik = i > k ? Ls[i * Cfg::LD + k] : 0.f;
#pragma unroll
        for (int g = 0; g < Cfg::RG; ++g) {
          if (64 * g > k) continue;  // W[k][c] = 0 for c > k
          const float4 y = *reinterpret_cast<const float4*>(row + 64 * g + 4 * tx);
          r[a][g][0] = fmaf(-lik, y.x, r[a][g][0]);
          r[a][g][1] = fmaf(-lik, y.y, r[a][g][1]);
          r[a][g][2] = fmaf(-lik, y.z, r[a][g][2]);
          r[a][g][3] = fmaf(-lik, y.w, r[a][g][3]);
        }
      }
    }
    __syncthreads();  // all reads of L done: the buffer now takes W
#pragma unroll
    for (int a = 0; a < Cfg::RA; ++a)
#pragma unroll
      for (int g = 0; g < Cfg::RG; ++g)
        *reinterpret_cast<float4*>(sm + (ty + 16 * a) * Cfg::LD2 + 64 * g + 4 * tx) =
            make_float4(r[a][g][0], r[a][g][1], r[a][g][2], r[a][g][3]);
  }
  __syncthreads();

  // ---------------------------------------------------------------- 3. P = W^T W
  {
    constexpr int TR = Cfg::TR;
    const int i0 = (threadIdx.x >> 4) * TR, c0 = (threadIdx.x & 15) * TR;
    float acc[TR][TR];
#pragma unroll
    for (int a = 0; a < TR; ++a)
#pragma unroll
      for (int b = 0; b < TR; ++b) acc[a][b] = 0.f;
    // W[k][i] = 0 for k < i: rows below max(i0, c0) add nothing to the tile
#pragma unroll 2
    for (int k = max(i0, c0); k < DH; ++k) {
      const float* wk = sm + k * Cfg::LD2;
      float wi[TR], wc[TR];
#pragma unroll
      for (int a = 0; a < TR; a += 4) {
        const float4 v = *reinterpret_cast<const float4*>(wk + i0 + a);
        wi[a] = v.x; wi[a + 1] = v.y; wi[a + 2] = v.z; wi[a + 3] = v.w;
      }
#pragma unroll
      for (int b = 0; b < TR; b += 4) {
        const float4 v = *reinterpret_cast<const float4*>(wk + c0 + b);
        wc[b] = v.x; wc[b + 1] = v.y; wc[b + 2] = v.z; wc[b + 3] = v.w;
      }
#pragma unroll
      for (int a = 0; a < TR; ++a)
#pragma unroll
        for (int b = 0; b < TR; ++b) acc[a][b] = fmaf(wi[a], wc[b], acc[a][b]);
    }
    float* Pm = P + mat;
#pragma unroll
    for (int a = 0; a < TR; ++a)
#pragma unroll
      for (int b = 0; b < TR; b += 4)
        *reinterpret_cast<float4*>(Pm + (i0 + a) * DH + c0 + b) =
            make_float4(acc[a][b], acc[a][b + 1], acc[a][b + 2], acc[a][b + 3]);
  }
  if (bad) record_status(status, kStatusNumeric);
}

// ---------------------------------------------------------------- Gauss-Jordan
//   M[p][p] <- 1/piv,  M[p][k] <- M[p][k]/piv,  M[i][p] <- -M[i][p]/piv,
//   M[i][k] <- M[i][k] - M[i][p] M[p][k] / piv          (i, k != p)
// over p = 0..d-1 leaves (I + A_sym)^-1; the pivots are Schur-complement
// diagonals of an SPD matrix with eigenvalues >= 1.
template <int DH>
__global__ void __launch_bounds__(kThreads, 2)
    vda_solve_gj_kernel(const float* __restrict__ A, float* __restrict__ P, uint32_t* status) {
  using Cfg = SolveCfg<DH>;
  extern __shared__ float sm[];
  float* rowb = sm + Cfg::MAT;   // 2 x [DH] pivot rows
  float* colb = rowb + 2 * DH;   // 2 x [DH] pivot columns
  const int tx = threadIdx.x & 15;
  const int ty = threadIdx.x >> 4;
  const int64_t mat = static_cast<int64_t>(blockIdx.x) * DH * DH;
  bool bad = false;

  float m[Cfg::RA][Cfg::CB];
  load_spd<DH>(A + mat, m, ty, tx);
#pragma unroll 1
  for (int p = 0; p < DH; ++p) {
    float* rb = rowb + (p & 1) * DH;
    float* cb = colb + (p & 1) * DH;
    if (ty == (p & 15)) {  // owners of row p
      const int pa = p >> 4;
#pragma unroll
      for (int b = 0; b < Cfg::CB; ++b) {
        float v = m[0][b];
#pragma unroll
        for (int a = 1; a < Cfg::RA; ++a) v = (a == pa) ? m[a][b] : v;
        rb[tx + 16 * b] = v;
      }
    }
    if (tx == (p & 15)) {  // owners of column p
      const int pb = p >> 4;
#pragma unroll
      for (int a = 0; a < Cfg::RA; ++a) {
        float v = m[a][0];
#pragma unroll
        for (int b = 1; b < Cfg::CB; ++b) v = (b == pb) ? m[a][b] : v;
        cb[ty + 16 * a] = v;
      }
    }
    __syncthreads();
    float piv = rb[p];
    if (!(piv > 0.f)) {  // also catches NaN
      bad = true;
      piv = 1.f;
    }
    const float inv = 1.f / piv;
    float fi[Cfg::RA], rk[Cfg::CB];
#pragma unroll
    for (int a = 0; a < Cfg::RA; ++a) fi[a] = cb[ty + 16 * a] * inv;
#pragma unroll
    for (int b = 0; b < Cfg::CB; ++b) rk[b] = rb[tx + 16 * b];
#pragma unroll
    for (int a = 0; a < Cfg::RA; ++a) {
      const int i = ty + 16 * a;
#pragma unroll
      for (int b = 0; b < Cfg::CB; ++b) {
        const int k = tx + 16 * b;
        const float upd = fmaf(-fi[a], rk[b], m[a][b]);
        const float rowp = (k == p) ? inv : rk[b] * inv;
        m[a][b] = (i == p) ? rowp : ((k == p) ? -fi[a] : upd);
      }
    }
    // one barrier per step: the next step writes the other buffer pair
  }
  float* Pm = P + mat;
#pragma unroll
  for (int a = 0; a < Cfg::RA; ++a)
#pragma unroll
    for (int b = 0; b < Cfg::CB; ++b) Pm[(ty + 16 * a) * DH + tx + 16 * b] = m[a][b];
  if (bad) record_status(status, kStatusNumeric);
}

template <int DH>
cudaError_t launch_solve_dh(const Launch& ctx, const vdn_shape& s, const float* A, float* P,
                            int solver) {
  using Cfg = SolveCfg<DH>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(vda_solve_kernel<DH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(vda_solve_gj_kernel<DH>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (solver == VDN_SOLVER_GAUSS_JORDAN)
    vda_solve_gj_kernel<DH><<<s.T * s.H, kThreads, Cfg::SMEM, ctx.stream>>>(A, P, ctx.status);
  else
    vda_solve_kernel<DH><<<s.T * s.H, kThreads, Cfg::SMEM, ctx.stream>>>(A, P, ctx.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_vda_solve(const Launch& ctx, const vdn_shape& s, const float* A, float* P) {
  const int solver = current_vda_solver();
  if (s.d == 128) return launch_solve_dh<128>(ctx, s, A, P, solver);
  if (s.d == 64) return launch_solve_dh<64>(ctx, s, A, P, solver);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
