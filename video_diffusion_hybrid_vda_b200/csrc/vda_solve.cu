// Batched SPD solve for the VDA closed form ("Video DeltaNet", 10100.com
// article, 方法概述 item 2: S_t = (S_bar_t + B_t)(I + A_t)^-1).
//
// Per (frame t, head h) one CTA of 256 threads (two CTAs per SM, so two
// problems hide each other's barrier latency) produces
//   P_t = (I + A_sym)^-1,   A_sym = (A + A^T) / 2
// (the tensor-core product in the prep rounds beta*k on one operand only, so
// A is symmetric up to that rounding).  Two solvers:
//
//  Cholesky (default): blocked in 16 x 16 blocks; one warp factors and
//   inverts each diagonal block with shuffles, every thread takes part in
//   the panel and trailing block products; then W = L^-1 by blocked forward
//   substitution and P = W^T W (see the kernel's own comment).
//  Gauss-Jordan (the inverse the pages' own kernels use):
//   one in-register sweep over the pivots, publishing the pivot row and
//   column each step, leaves (I + A_sym)^-1.
// The scan multiplies (alpha S + B_t) by P_t itself, so no B P is formed here.
//
// I + A_sym is symmetric positive definite with eigenvalues >= 1 (beta >= 0),
// so neither solver pivots; a non-positive or NaN pivot is reported as
// VDN_ERR_NUMERIC.  This step is FP32-ALU and latency bound.
#include "common.cuh"
#include "exp2_fma.cuh"
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
//
// Blocked in 16 x 16 blocks (NB = DH / 16 block rows).  Thread (ty, tx)
// holds element (ty, tx) of every block, so block products need no
// reshuffling: a block (a, b) of the register tile is m[a][b].
//
//  1. factor, for p = 0 .. NB-1:
//     a. every thread stages block column p (rows >= 16p) in Apan;
//     b. warp 0 factors the diagonal block with shuffles (lane j holds
//        column j; the pivot column is broadcast row by row) into L_pp and
//        inverts it, W_pp = L_pp^-1 (one column per lane); both to smem;
//     c. L_ip = A_ip W_pp^T for the blocks below (16-term dot products);
//     d. trailing update A_ab -= L_ap L_bp^T for p < b <= a (packed f32x2);
//  2. W = L^-1 in place, block row by block row:
//     W_ij = -W_ii sum_{k=j}^{i-1} L_ik W_kj   (j < i);
//  3. P = W^T W over the rows where W can be nonzero (k >= max(i, c)).
// About 54 barriers in all (the unblocked form needs two per column).
template <int DH>
struct CholCfg {
  static constexpr int NB = DH / 16;
  static constexpr int LDL = DH + 4;   // row stride of L / W (float4 rows)
  static constexpr int LDP = 20;       // row stride of the 16-wide staging blocks
  static constexpr int SMEM = (DH * LDL + DH * LDP + NB * 16 * LDP) * 4;
};

template <int DH>
__global__ void __launch_bounds__(kThreads, 2)
    vda_solve_kernel(const float* __restrict__ A, float* __restrict__ P, uint32_t* status) {
  using Cfg = CholCfg<DH>;
  constexpr int NB = Cfg::NB;
  constexpr int LDL = Cfg::LDL;
  constexpr int LDP = Cfg::LDP;
  extern __shared__ __align__(16) float sm[];
  float* Ls = sm;                       // [DH][LDL]: L (lower blocks), then W
  float* Apan = Ls + DH * LDL;          // [DH][LDP]: block column p before scaling
  float* Wd = Apan + DH * LDP;          // [NB][16][LDP]: W_pp = L_pp^-1
  const int tx = threadIdx.x & 15;
  const int ty = threadIdx.x >> 4;
  const int64_t mat = static_cast<int64_t>(blockIdx.x) * DH * DH;
  const float* Am = A + mat;
  bool bad = false;

  // strictly upper blocks of L / W stay zero (the product in 3 reads them)
  for (int e = threadIdx.x; e < DH * DH; e += kThreads) {
    const int r = e / DH, c = e % DH;
    if ((c >> 4) > (r >> 4)) Ls[r * LDL + c] = 0.f;
  }

  // lower blocks of I + (A + A^T) / 2 into registers
  float m[NB][NB];
#pragma unroll
  for (int a = 0; a < NB; ++a)
#pragma unroll
    for (int b = 0; b <= a; ++b) {
      const int i = 16 * a + ty, k = 16 * b + tx;
      m[a][b] = 0.5f * (__ldg(Am + i * DH + k) + __ldg(Am + k * DH + i)) + (i == k ? 1.f : 0.f);
    }

  // ---------------------------------------------------------------- 1. factor
#pragma unroll
  for (int p = 0; p < NB; ++p) {
#pragma unroll
    for (int a = p; a < NB; ++a) Apan[(16 * a + ty) * LDP + tx] = m[a][p];
    __syncthreads();

    if (threadIdx.x < 32) {
      // lane j (mod 16) holds column j of the diagonal block
      const int j = threadIdx.x & 15;
      float dc[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) dc[r] = Apan[(16 * p + r) * LDP + j];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float piv = __shfl_sync(0xffffffffu, dc[c], c);
        if (!(piv > 0.f)) {  // also catches NaN
          bad = true;
          piv = 1.f;
        }
        const float f = dc[c] / piv;  // D[c][j] / D[c][c]
#pragma unroll
        for (int r = c + 1; r < 16; ++r) {
          const float v = __shfl_sync(0xffffffffu, dc[r], c);  // D[r][c]
          if (j > c) dc[r] = fmaf(-v, f, dc[r]);
        }
        if (j == c) {
          const float sq = sqrtf(piv);
          const float is = 1.f / sq;
#pragma unroll
          for (int r = c + 1; r < 16; ++r) dc[r] *= is;
          dc[c] = sq;
        }
      }
#pragma unroll
      for (int r = 0; r < 16; ++r)
        if (r < j) dc[r] = 0.f;
      if (threadIdx.x < 16)
#pragma unroll
        for (int r = 0; r < 16; ++r) Ls[(16 * p + r) * LDL + 16 * p + j] = dc[r];
      __syncwarp();
      // column j of W_pp by forward substitution (rows above j come out 0)
      float w[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float* lr = Ls + (16 * p + r) * LDL + 16 * p;
        float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int k = 0; k < r; ++k) acc = fmaf(-lr[k], w[k], acc);
        w[r] = acc / lr[r];
      }
      if (threadIdx.x < 16)
#pragma unroll
        for (int r = 0; r < 16; ++r) Wd[(p * 16 + r) * LDP + j] = w[r];
    }
    __syncthreads();

    if (p + 1 < NB) {
      // L_ip = A_ip W_pp^T: row ty of A_ip against row tx of W_pp
      uint64_t wr[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(Wd + (p * 16 + tx) * LDP + 4 * q);
        wr[2 * q] = v.x;
        wr[2 * q + 1] = v.y;
      }
#pragma unroll
      for (int i = p + 1; i < NB; ++i) {
        uint64_t acc = 0ull;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(Apan + (16 * i + ty) * LDP + 4 * q);
          acc = f32x2_fma(v.x, wr[2 * q], acc);
          acc = f32x2_fma(v.y, wr[2 * q + 1], acc);
        }
        Ls[(16 * i + ty) * LDL + 16 * p + tx] = f32x2_lo(acc) + f32x2_hi(acc);
      }
      __syncthreads();
      // trailing update of the lower blocks right of panel p
#pragma unroll
      for (int a = p + 1; a < NB; ++a) {
        uint64_t la[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const ulonglong2 v =
              *reinterpret_cast<const ulonglong2*>(Ls + (16 * a + ty) * LDL + 16 * p + 4 * q);
          la[2 * q] = v.x;
          la[2 * q + 1] = v.y;
        }
#pragma unroll
        for (int b = p + 1; b <= a; ++b) {
          uint64_t acc = 0ull;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const ulonglong2 v =
                *reinterpret_cast<const ulonglong2*>(Ls + (16 * b + tx) * LDL + 16 * p + 4 * q);
            acc = f32x2_fma(la[2 * q], v.x, acc);
            acc = f32x2_fma(la[2 * q + 1], v.y, acc);
          }
          m[a][b] -= f32x2_lo(acc) + f32x2_hi(acc);
        }
      }
    }
  }

  // ---------------------------------------------------------------- 2. W = L^-1
  // (the barrier closing the last factor step made L complete)
  Ls[ty * LDL + tx] = Wd[ty * LDP + tx];  // W_00
  __syncthreads();
#pragma unroll
  for (int i = 1; i < NB; ++i) {
    float t[NB];
#pragma unroll
    for (int j = 0; j < i; ++j) t[j] = 0.f;
#pragma unroll
    for (int k = 0; k < i; ++k) {
      float lr[16];  // row ty of L_ik
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(Ls + (16 * i + ty) * LDL + 16 * k + 4 * q);
        lr[4 * q] = v.x; lr[4 * q + 1] = v.y; lr[4 * q + 2] = v.z; lr[4 * q + 3] = v.w;
      }
#pragma unroll
      for (int j = 0; j <= k; ++j)
#pragma unroll
        for (int n = 0; n < 16; ++n) t[j] = fmaf(lr[n], Ls[(16 * k + n) * LDL + 16 * j + tx], t[j]);
    }
    __syncthreads();  // every read of L_i* is done
#pragma unroll
    for (int j = 0; j < i; ++j) Ls[(16 * i + ty) * LDL + 16 * j + tx] = t[j];
    __syncthreads();
    float wi[16];  // row ty of W_ii
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = *reinterpret_cast<const float4*>(Wd + (i * 16 + ty) * LDP + 4 * q);
      wi[4 * q] = v.x; wi[4 * q + 1] = v.y; wi[4 * q + 2] = v.z; wi[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int j = 0; j < i; ++j) {
      float acc = 0.f;
#pragma unroll
      for (int n = 0; n < 16; ++n) acc = fmaf(wi[n], Ls[(16 * i + n) * LDL + 16 * j + tx], acc);
      t[j] = -acc;
    }
    __syncthreads();  // every read of T_i* is done
#pragma unroll
    for (int j = 0; j < i; ++j) Ls[(16 * i + ty) * LDL + 16 * j + tx] = t[j];
    Ls[(16 * i + ty) * LDL + 16 * i + tx] = Wd[(i * 16 + ty) * LDP + tx];
    __syncthreads();
  }

  // ---------------------------------------------------------------- 3. P = W^T W
  {
    constexpr int TR = DH / 16;
    const int i0 = (threadIdx.x >> 4) * TR, c0 = (threadIdx.x & 15) * TR;
    uint64_t acc[TR][TR / 2];
#pragma unroll
    for (int a = 0; a < TR; ++a)
#pragma unroll
      for (int b = 0; b < TR / 2; ++b) acc[a][b] = 0ull;
    // W[k][i] = 0 for k < i: rows below max(i0, c0) add nothing to the tile
#pragma unroll 2
    for (int k = max(i0, c0); k < DH; ++k) {
      const float* wk = Ls + k * LDL;
      float wi[TR];
      uint64_t wc[TR / 2];
#pragma unroll
      for (int a = 0; a < TR; a += 4) {
        const float4 v = *reinterpret_cast<const float4*>(wk + i0 + a);
        wi[a] = v.x; wi[a + 1] = v.y; wi[a + 2] = v.z; wi[a + 3] = v.w;
      }
#pragma unroll
      for (int b = 0; b < TR / 2; b += 2) {
        const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(wk + c0 + 2 * b);
        wc[b] = v.x;
        wc[b + 1] = v.y;
      }
#pragma unroll
      for (int a = 0; a < TR; ++a) {
        const uint64_t aa = f32x2_pack(wi[a], wi[a]);
#pragma unroll
        for (int b = 0; b < TR / 2; ++b) acc[a][b] = f32x2_fma(aa, wc[b], acc[a][b]);
      }
    }
    float* Pm = P + mat;
#pragma unroll
    for (int a = 0; a < TR; ++a)
#pragma unroll
      for (int b = 0; b < TR / 2; b += 2)
        *reinterpret_cast<float4*>(Pm + (i0 + a) * DH + c0 + 2 * b) =
            make_float4(f32x2_lo(acc[a][b]), f32x2_hi(acc[a][b]), f32x2_lo(acc[a][b + 1]),
                        f32x2_hi(acc[a][b + 1]));
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
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         CholCfg<DH>::SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(vda_solve_gj_kernel<DH>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (solver == VDN_SOLVER_GAUSS_JORDAN)
    vda_solve_gj_kernel<DH><<<s.T * s.H, kThreads, Cfg::SMEM, ctx.stream>>>(A, P, ctx.status);
  else
    vda_solve_kernel<DH><<<s.T * s.H, kThreads, CholCfg<DH>::SMEM, ctx.stream>>>(A, P,
                                                                                 ctx.status);
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
