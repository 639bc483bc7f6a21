// Batched SPD solve for the VDA closed form ("Video DeltaNet", 10100.com
// article, 方法概述 item 2: S_t = (S_bar_t + B_t)(I + A_t)^-1).
//
// Per (frame t, head h), one CTA of 512 threads:
//   1. Cholesky  L L^T = I + A_sym  (right-looking; the matrix lives in
//      registers as 4x8 (d=128) tiles per thread, the scaled pivot column is
//      published through shared memory each step, L is kept in shared
//      memory);
//   2. W = L^-1 by forward substitution against I (row k of W is published
//      each step; column blocks that are still zero are skipped);
//   3. P = (I + A)^-1 = W^T W and 4. C = B P, both as shared-memory GEMMs
//      without barriers inside their loops.
// A_sym = (A + A^T) / 2: the tensor-core product in the prep rounds
// beta*k on one operand only, so A is symmetric up to that rounding.
// I + A is symmetric positive definite with eigenvalues >= 1 (beta >= 0),
// so no pivoting is needed; a non-positive or NaN pivot is reported as
// VDN_ERR_NUMERIC in the status word.  This step is FP32-ALU bound.
#include "common.cuh"
#include "ptx.cuh"

namespace vdn {
namespace {

constexpr int kSolveThreads = 512;  // 32 row groups x 16 column groups

template <int DH>
struct SolveCfg {
  static constexpr int RA = DH / 32;        // rows per thread (strided by 32)
  static constexpr int CB = DH / 16;        // matrix columns per thread (phase 1)
  static constexpr int RG = DH / 64;        // 4-wide column groups of W per thread
  static constexpr int LD = DH + 1;         // padded row stride of L (column access)
  static constexpr int LD2 = DH + 4;        // row stride of W, P, B (float4 rows)
  static constexpr int MAT = DH * LD2;      // floats per matrix buffer (>= DH * LD)
  static constexpr int SMEM = 2 * MAT * 4 + 2 * (2 * DH) * 4;
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

// C = B P for one (frame, head): B staged through shared memory `Bs`, P
// already in shared memory `Ps` (both [DH][LD2]); each of the 512 threads
// computes a (DH/32) x (DH/16) tile.  Caller synchronises before the call.
template <int DH>
__device__ __forceinline__ void c_equals_b_times_p(const float* __restrict__ Bm, const float* Ps,
                                                   float* Bs, float* __restrict__ Cm) {
  using Cfg = SolveCfg<DH>;
  constexpr int PR = DH / 32, PC = DH / 16;
  const int i0 = (threadIdx.x >> 4) * PR, c0 = (threadIdx.x & 15) * PC;
  for (int idx = threadIdx.x; idx < DH * DH / 4; idx += kSolveThreads) {
    const int rr = idx / (DH / 4), cc = idx % (DH / 4);
    *reinterpret_cast<float4*>(Bs + rr * Cfg::LD2 + 4 * cc) =
        __ldg(reinterpret_cast<const float4*>(Bm) + idx);
  }
  __syncthreads();
  float acc[PR][PC];
#pragma unroll
  for (int a = 0; a < PR; ++a)
#pragma unroll
    for (int b = 0; b < PC; ++b) acc[a][b] = 0.f;
#pragma unroll 2
  for (int k = 0; k < DH; k += 4) {
    float bv[PR][4];
#pragma unroll
    for (int a = 0; a < PR; ++a) {
      const float4 v = *reinterpret_cast<const float4*>(Bs + (i0 + a) * Cfg::LD2 + k);
      bv[a][0] = v.x; bv[a][1] = v.y; bv[a][2] = v.z; bv[a][3] = v.w;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      float pc[PC];
#pragma unroll
      for (int b = 0; b < PC; b += 4) {
        const float4 v = *reinterpret_cast<const float4*>(Ps + (k + kk) * Cfg::LD2 + c0 + b);
        pc[b] = v.x; pc[b + 1] = v.y; pc[b + 2] = v.z; pc[b + 3] = v.w;
      }
#pragma unroll
      for (int a = 0; a < PR; ++a)
#pragma unroll
        for (int b = 0; b < PC; ++b) acc[a][b] = fmaf(bv[a][kk], pc[b], acc[a][b]);
    }
  }
#pragma unroll
  for (int a = 0; a < PR; ++a)
#pragma unroll
    for (int b = 0; b < PC; b += 4)
      *reinterpret_cast<float4*>(Cm + (i0 + a) * DH + c0 + b) =
          make_float4(acc[a][b], acc[a][b + 1], acc[a][b + 2], acc[a][b + 3]);
}

// Gauss-Jordan variant (the inverse the pages' own kernels use): one sweep
// over the pivots p = 0..d-1 of the symmetric positive definite I + A_sym,
// with the whole matrix in registers (4x8 per thread, d = 128).  Each step
// publishes pivot row p and pivot column p through shared memory and applies
//   M[p][p] <- 1/piv,  M[p][k] <- M[p][k]/piv,  M[i][p] <- -M[i][p]/piv,
//   M[i][k] <- M[i][k] - M[i][p] M[p][k] / piv          (i, k != p),
// which leaves (I + A)^-1 after the last pivot.  No pivoting is needed: the
// pivots are Schur-complement diagonals of an SPD matrix with eigenvalues
// >= 1.  Then C = B P as in the Cholesky kernel.
template <int DH>
__global__ void __launch_bounds__(kSolveThreads, 1)
    vda_solve_gj_kernel(const float* __restrict__ A, const float* __restrict__ B,
                        float* __restrict__ P, float* __restrict__ Cout, uint32_t* status) {
  using Cfg = SolveCfg<DH>;
  extern __shared__ float sm[];
  float* Ws = sm;                    // [DH][LD2]: B for the C product
  float* Xs = sm + Cfg::MAT;         // [DH][LD2]: P
  float* rowb = sm + 2 * Cfg::MAT;   // 2 x [DH] pivot rows
  float* colb = rowb + 2 * DH;       // 2 x [DH] pivot columns
  const int tx = threadIdx.x & 15;
  const int ty = threadIdx.x >> 4;
  const int64_t mat = static_cast<int64_t>(blockIdx.x) * DH * DH;
  const float* Am = A + mat;
  bool bad = false;

  float m[Cfg::RA][Cfg::CB];
#pragma unroll
  for (int a = 0; a < Cfg::RA; ++a)
#pragma unroll
    for (int b = 0; b < Cfg::CB; ++b) {
      const int i = ty + 32 * a, k = tx + 16 * b;
      m[a][b] = 0.5f * (__ldg(Am + i * DH + k) + __ldg(Am + k * DH + i)) + (i == k ? 1.f : 0.f);
    }
#pragma unroll 1
  for (int p = 0; p < DH; ++p) {
    float* rb = rowb + (p & 1) * DH;
    float* cb = colb + (p & 1) * DH;
    if (ty == (p & 31)) {  // owners of row p
      const int pa = p >> 5;
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
        cb[ty + 32 * a] = v;
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
    for (int a = 0; a < Cfg::RA; ++a) fi[a] = cb[ty + 32 * a] * inv;
#pragma unroll
    for (int b = 0; b < Cfg::CB; ++b) rk[b] = rb[tx + 16 * b];
#pragma unroll
    for (int a = 0; a < Cfg::RA; ++a) {
      const int i = ty + 32 * a;
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
#pragma unroll
  for (int a = 0; a < Cfg::RA; ++a)
#pragma unroll
    for (int b = 0; b < Cfg::CB; ++b) {
      const int i = ty + 32 * a, k = tx + 16 * b;
      Xs[i * Cfg::LD2 + k] = m[a][b];
      P[mat + i * DH + k] = m[a][b];
    }
  __syncthreads();
  c_equals_b_times_p<DH>(B + mat, Xs, Ws, Cout + mat);
  if (bad) record_status(status, kStatusNumeric);
}

template <int DH>
__global__ void __launch_bounds__(kSolveThreads, 1)
    vda_solve_kernel(const float* __restrict__ A, const float* __restrict__ B,
                     float* __restrict__ P, float* __restrict__ Cout, uint32_t* status) {
  using Cfg = SolveCfg<DH>;
  extern __shared__ float sm[];
  float* Ls = sm;                    // [DH][LD], lower triangle of L
  float* buf0 = sm + 2 * Cfg::MAT;   // two 2*DH broadcast buffers
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
  // W = L^-1: forward substitution against I.  Columns c = 64 g + 4 tx + e.
  // Row k of W is zero beyond column k, so column group g only takes part
  // once k >= 64 g.
  float r[Cfg::RA][Cfg::RG][4];
#pragma unroll
  for (int a = 0; a < Cfg::RA; ++a)
#pragma unroll
    for (int g = 0; g < Cfg::RG; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) r[a][g][e] = (ty + 32 * a == 64 * g + 4 * tx + e) ? 1.f : 0.f;

#pragma unroll 1
  for (int k = 0; k < DH; ++k) {
    float* row = (k & 1) ? buf1 : buf0;
    const float dinv = 1.f / Ls[k * Cfg::LD + k];
    if (ty == (k & 31)) publish_row<Cfg::RA, Cfg::RG>(r, k >> 5, dinv, row + 4 * tx);
    __syncthreads();
#pragma unroll
    for (int a = 0; a < Cfg::RA; ++a) {
      if (32 * a + 31 <= k) continue;
      const int i = ty + 32 * a;
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
  __syncthreads();  // all reads of L done: its buffer now takes W

  float* Ws = sm;             // [DH][LD2]
  float* Xs = sm + Cfg::MAT;  // [DH][LD2]: P, then read by phase 4
#pragma unroll
  for (int a = 0; a < Cfg::RA; ++a)
#pragma unroll
    for (int g = 0; g < Cfg::RG; ++g)
      *reinterpret_cast<float4*>(Ws + (ty + 32 * a) * Cfg::LD2 + 64 * g + 4 * tx) =
          make_float4(r[a][g][0], r[a][g][1], r[a][g][2], r[a][g][3]);
  __syncthreads();

  // ---------------------------------------------------------------- phase 3
  // P = W^T W: each thread a (DH/32) x (DH/16) tile, rows 4 rg.., cols CW cg..
  constexpr int PR = DH / 32;   // rows per thread
  constexpr int PC = DH / 16;   // cols per thread
  const int rg = threadIdx.x >> 4;   // 0..31
  const int cg = threadIdx.x & 15;   // 0..15
  const int i0 = rg * PR, c0 = cg * PC;
  float acc[PR][PC];
#pragma unroll
  for (int a = 0; a < PR; ++a)
#pragma unroll
    for (int b = 0; b < PC; ++b) acc[a][b] = 0.f;
#pragma unroll 4
  for (int k = 0; k < DH; ++k) {
    const float* wk = Ws + k * Cfg::LD2;
    float wi[PR], wc[PC];
#pragma unroll
    for (int a = 0; a < PR; a += 2) {
      const float2 v = *reinterpret_cast<const float2*>(wk + i0 + a);
      wi[a] = v.x;
      wi[a + 1] = v.y;
    }
#pragma unroll
    for (int b = 0; b < PC; b += 4) {
      const float4 v = *reinterpret_cast<const float4*>(wk + c0 + b);
      wc[b] = v.x; wc[b + 1] = v.y; wc[b + 2] = v.z; wc[b + 3] = v.w;
    }
#pragma unroll
    for (int a = 0; a < PR; ++a)
#pragma unroll
      for (int b = 0; b < PC; ++b) acc[a][b] = fmaf(wi[a], wc[b], acc[a][b]);
  }
  float* Pm = P + mat;
#pragma unroll
  for (int a = 0; a < PR; ++a)
#pragma unroll
    for (int b = 0; b < PC; b += 4) {
      const float4 v = make_float4(acc[a][b], acc[a][b + 1], acc[a][b + 2], acc[a][b + 3]);
      *reinterpret_cast<float4*>(Xs + (i0 + a) * Cfg::LD2 + c0 + b) = v;
      *reinterpret_cast<float4*>(Pm + (i0 + a) * DH + c0 + b) = v;
    }
  __syncthreads();  // P complete in Xs; W no longer needed: its buffer takes B

  // ---------------------------------------------------------------- phase 4
  c_equals_b_times_p<DH>(Bm, Xs, Ws, Cout + mat);
  if (bad) record_status(status, kStatusNumeric);
}

template <int DH>
cudaError_t launch_solve_dh(const Launch& ctx, const vdn_shape& s, const float* A,
                            const float* B, float* P, float* C, int solver) {
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
    vda_solve_gj_kernel<DH><<<s.T * s.H, kSolveThreads, Cfg::SMEM, ctx.stream>>>(A, B, P, C,
                                                                                ctx.status);
  else
    vda_solve_kernel<DH><<<s.T * s.H, kSolveThreads, Cfg::SMEM, ctx.stream>>>(A, B, P, C,
                                                                             ctx.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_vda_solve(const Launch& ctx, const vdn_shape& s, const float* A,
                             const float* B, float* P, float* C) {
  const int solver = current_vda_solver();
  if (s.d == 128) return launch_solve_dh<128>(ctx, s, A, B, P, C, solver);
  if (s.d == 64) return launch_solve_dh<64>(ctx, s, A, B, P, C, solver);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
