// Batched SPD solve for the VDA closed form ("Video DeltaNet", 10100.com
// article, 方法概述 item 2: S_t = (S_bar_t + B_t)(I + A_t)^-1).
//
// Per (frame t, head h) one CTA of 256 threads (two CTAs per SM, so two
// problems hide each other's barrier latency) produces
//   P_t = (I + A_sym)^-1,   A_sym = (A + A^T) / 2
// (the tensor-core product in the prep rounds beta*k on one operand only, so
// A is symmetric up to that rounding).  Two solvers:
//
//  Cholesky: blocked in 16 x 16 blocks; one warp factors and
//   inverts each diagonal block with shuffles, every thread takes part in
//   the panel and trailing block products; then W = L^-1 by blocked forward
//   substitution and P = W^T W (see the kernel's own comment).
//  Gauss-Jordan (default; the inverse the pages' own kernels use): one
//   in-register sweep over the pivots, each thread holding a contiguous
//   block of the matrix, the pivot row and column published each step,
//   leaves (I + A_sym)^-1.
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

// ---------------------------------------------------------------- Cholesky
//
// Blocked in 16 x 16 blocks (NB = DH / 16 block rows), the matrix in shared
// memory (lower blocks; strictly upper blocks held at zero), thread (ty, tx)
// working on element (ty, tx) of every block it touches:
//  1. factor, for p = 0 .. NB-1:
//     a. warp 0 factors the diagonal block with shuffles (lane j holds
//        column j; the pivot column is broadcast row by row) and inverts it,
//        W_pp = L_pp^-1 (one column per lane), which replaces the block;
//     b. L_ip = A_ip W_pp^T for the blocks below, into a panel buffer;
//     c. trailing update A_ab -= L_ap L_bp^T (p < b <= a, packed f32x2),
//        and L_ip copied into block column p;
//  2. W = L^-1 in place, block row by block row:
//     W_ij = -W_ii sum_{k=j}^{i-1} L_ik W_kj   (j < i);
//  3. P = W^T W over the rows where W can be nonzero (k >= max(i, c)).
// The block loops are runtime loops, so the program stays small (each
// step's code is fetched once and reused); only the 16-step factorization
// of a diagonal block is unrolled.  About 40 barriers in all.
template <int DH>
struct CholCfg {
  static constexpr int NB = DH / 16;
  static constexpr int LDL = DH + 4;   // row stride of the matrix (float4 rows)
  static constexpr int LDP = 20;       // row stride of the 16-wide panel buffer, of the
                                       // transposed T blocks (aliasing it) and of WTd
  static constexpr int PANEL = DH * LDP;
  static constexpr int WTD = NB * 16 * LDP;  // transposed diagonal blocks W_pp^T
  static constexpr int SMEM = (DH * LDL + PANEL + 16 + WTD) * 4;
};

// A 16-float row of shared memory (16-byte aligned) into registers, and
// its dot product with another such row (packed f32x2, pairs summed last).
__device__ __forceinline__ void load_row16(const float* x, ulonglong2 (&r)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) r[q] = *reinterpret_cast<const ulonglong2*>(x + 4 * q);
}

__device__ __forceinline__ float dot16_reg(const ulonglong2 (&a)[4], const float* y) {
  uint64_t acc = 0ull;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const ulonglong2 b = *reinterpret_cast<const ulonglong2*>(y + 4 * q);
    acc = f32x2_fma(a[q].x, b.x, acc);
    acc = f32x2_fma(a[q].y, b.y, acc);
  }
  return f32x2_lo(acc) + f32x2_hi(acc);
}

template <int DH>
__global__ void __launch_bounds__(kThreads, 2)
    vda_solve_kernel(const float* __restrict__ A, float* __restrict__ P, uint32_t* status) {
  using Cfg = CholCfg<DH>;
  constexpr int NB = Cfg::NB;
  constexpr int LDL = Cfg::LDL;
  constexpr int LDP = Cfg::LDP;
  extern __shared__ __align__(16) float sm[];
  float* Ls = sm;                   // [DH][LDL]: the matrix, then L / W blocks
  float* Pan = Ls + DH * LDL;       // [DH][LDP] panel L_ip; in step 2 the T_ij^T rows
  float* idg = Pan + Cfg::PANEL;    // [16] 1 / L_pp[r][r]
  float* WTd = idg + 16;            // [NB][16][LDP] W_pp^T
  const int tx = threadIdx.x & 15;
  const int ty = threadIdx.x >> 4;
  const int64_t mat = static_cast<int64_t>(blockIdx.x) * DH * DH;
  const float* Am = A + mat;
  bool bad = false;

  // ---------------------------------------------------------------- load
  // A row-major into shared memory (coalesced), then I + (A + A^T) / 2 on
  // the lower blocks and zero on the strictly upper ones
  for (int e = threadIdx.x; e < DH * DH / 4; e += kThreads) {
    const int r = e / (DH / 4), c4 = e % (DH / 4);
    *reinterpret_cast<float4*>(Ls + r * LDL + 4 * c4) =
        __ldg(reinterpret_cast<const float4*>(Am + r * DH + 4 * c4));
  }
  __syncthreads();
  {
    constexpr int PER = DH * DH / kThreads;
    float v[PER];
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int e = threadIdx.x + kThreads * q;
      const int r = e / DH, c = e % DH;
      v[q] = (c >> 4) > (r >> 4) ? 0.f
                                 : 0.5f * (Ls[r * LDL + c] + Ls[c * LDL + r]) + (r == c ? 1.f : 0.f);
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int e = threadIdx.x + kThreads * q;
      Ls[(e / DH) * LDL + e % DH] = v[q];
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- 1. factor
#pragma unroll 1
  for (int p = 0; p < NB; ++p) {
    float* Dg = Ls + (16 * p) * LDL + 16 * p;  // diagonal block (p, p)
    if (threadIdx.x < 32) {
      // lane j (mod 16) holds column j of the diagonal block
      const int j = threadIdx.x & 15;
      float dc[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) dc[r] = Dg[r * LDL + j];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float piv = __shfl_sync(0xffffffffu, dc[c], c);
        if (!(piv > 0.f)) {  // also catches NaN
          bad = true;
          piv = 1.f;
        }
        // rsqrt and products (not the correctly rounded sqrt and reciprocal,
        // whose longer sequences sit on this serial chain); the pivot column
        // goes to the other lanes through shared memory in one burst
        const float is = rsqrtf(piv);                         // 1 / L[c][c]
        const float f = (j > c) ? dc[c] * (is * is) : 0.f;  // D[c][j] / D[c][c]
        const float sq = piv * is;                            // L[c][c]
        float* colc = Pan + (16 * p) * LDP;  // 16 floats; panel rows 16p.. are free
        if (threadIdx.x == c)
#pragma unroll
          for (int r = 0; r < 16; ++r) colc[r] = dc[r];
        __syncwarp();
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          if (r > c) {
            const float v = colc[r];  // D[r][c]
            dc[r] = (j == c) ? dc[r] * is : fmaf(-v, f, dc[r]);
          }
        }
        __syncwarp();  // every lane has read the column before the next pivot's
        if (j == c) dc[c] = sq;
        if (threadIdx.x == c) idg[c] = is;
      }
      // L_pp (zero above the diagonal) into the panel rows 16p.. (free now)
      float* Lp = Pan + (16 * p) * LDP;
      if (threadIdx.x < 16)
#pragma unroll
        for (int r = 0; r < 16; ++r) Lp[r * LDP + j] = r < j ? 0.f : dc[r];
      __syncwarp();
      // column j of W_pp by forward substitution (rows above j come out 0)
      float w[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float* lr = Lp + r * LDP;
        float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int k = 0; k < r; ++k) acc = fmaf(-lr[k], w[k], acc);
        w[r] = acc * idg[r];
      }
      if (threadIdx.x < 16) {
#pragma unroll
        for (int r = 0; r < 16; ++r) Dg[r * LDL + j] = w[r];
        // row j of W_pp^T, for the products of step 2
        float* wt = WTd + (16 * p + j) * LDP;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<float4*>(wt + 4 * q) =
              make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      }
    }
    __syncthreads();
    if (p + 1 == NB) break;

    // L_ip = A_ip W_pp^T: row ty of A_ip against row tx of W_pp (that row
    // held in registers across the block rows i: half the shared loads)
    {
      ulonglong2 wr[4];
      load_row16(Dg + tx * LDL, wr);
#pragma unroll 1
      for (int i = p + 1; i < NB; ++i)
        Pan[(16 * i + ty) * LDP + tx] = dot16_reg(wr, Ls + (16 * i + ty) * LDL + 16 * p);
    }
    __syncthreads();

    // trailing update of the lower blocks right of panel p (row ty of L_ap
    // in registers across the block columns b); L_ip into place
#pragma unroll 1
    for (int a = p + 1; a < NB; ++a) {
      ulonglong2 la[4];
      load_row16(Pan + (16 * a + ty) * LDP, la);
#pragma unroll 1
      for (int b = p + 1; b <= a; ++b)
        Ls[(16 * a + ty) * LDL + 16 * b + tx] -= dot16_reg(la, Pan + (16 * b + tx) * LDP);
      Ls[(16 * a + ty) * LDL + 16 * p + tx] = Pan[(16 * a + ty) * LDP + tx];
    }
    __syncthreads();
  }

  // ---------------------------------------------------------------- 2. W = L^-1
  // Block row by block row: T_ij = sum_{k=j}^{i-1} L_ik W_kj (j < i), then
  // W_ij = -W_ii T_ij.  Every product pairs two contiguous 16-float rows:
  // W_kj is read through its transpose, kept in the strictly upper block
  // (j, k) of the matrix buffer for k > j (nothing else reads those blocks)
  // and in WTd for k = j, and T through its transpose in the panel buffer.
  // Block row 0 holds W_00 already; the diagonal blocks hold W_ii.
  {
    constexpr int NT = NB - 1;  // T blocks of the last block row
#pragma unroll 1
    for (int i = 1; i < NB; ++i) {
      const float* li = Ls + (16 * i + ty) * LDL;  // row ty of block row i
      float t[NT];
#pragma unroll
      for (int j = 0; j < NT; ++j) t[j] = 0.f;
#pragma unroll 1
      for (int k = 0; k < i; ++k) {
        ulonglong2 lr[4];
        load_row16(li + 16 * k, lr);  // row ty of L_ik, for every j <= k
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          if (j <= k) {
            const float* wt = j == k ? WTd + (16 * j + tx) * LDP
                                     : Ls + (16 * j + tx) * LDL + 16 * k;  // row tx of W_kj^T
            t[j] += dot16_reg(lr, wt);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < NT; ++j)
        if (j < i) Pan[(16 * j + tx) * LDP + ty] = t[j];  // T_ij^T
      __syncthreads();  // T complete; every read of L_i* is done
      ulonglong2 wi[4];
      load_row16(li + 16 * i, wi);  // row ty of W_ii
#pragma unroll 1
      for (int j = 0; j < i; ++j) {
        const float w = -dot16_reg(wi, Pan + (16 * j + tx) * LDP);  // W_ij[ty][tx]
        Ls[(16 * i + ty) * LDL + 16 * j + tx] = w;
        Ls[(16 * j + tx) * LDL + 16 * i + ty] = w;  // W_ij^T into block (j, i)
      }
      __syncthreads();  // W_i* complete; T free again
    }
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
//
// Thread (ty, tx) of the 16 x 16 grid holds the R x R block of rows
// R ty .. R ty + R-1 and columns R tx .. R tx + R-1 (R = DH / 16) in
// registers as packed pairs.  The pivots are walked in groups of R, the R
// pivots of a group unrolled, so the pivot's row or column inside an
// owner's block is a compile-time index.  Each step: the lanes holding
// row p and the half-warp holding column p publish them (double-buffered in
// shared memory, one barrier per step), every thread applies the rank-1
// update to its block with packed f32x2 FMAs, and the owners overwrite
// row p, column p and the pivot.
//
// The row group ty is the lane within a half-warp and the column group tx
// the half-warp.  The column owners' work (extracting and rewriting one
// element of each of R packed rows) is the longer of the two divergent
// paths; this way it runs in one half-warp, while the row owners' few
// multiplies fall on two lanes of every warp.  The other way round, every
// warp waited on the column work each step (0.57 against 0.46 ms for 2448
// matrices of 128 x 128 on a B200).
template <int DH>
__global__ void __launch_bounds__(kThreads, 2)
    vda_solve_gj_kernel(const float* __restrict__ A, float* __restrict__ P, uint32_t* status) {
  constexpr int R = DH / 16;  // rows (and columns) per thread
  constexpr int H2 = R / 2;   // packed pairs per row
  __shared__ __align__(16) float rowb[2][DH];
  __shared__ __align__(16) float colb[2][DH];
  const int tx = threadIdx.x >> 4;
  const int ty = threadIdx.x & 15;
  const int64_t mat = static_cast<int64_t>(blockIdx.x) * DH * DH;
  const float* Am = A + mat;
  bool bad = false;

  // I + (A + A^T) / 2 on this thread's block: its rows, then the rows of
  // its columns (whole 32-byte sectors per lane either way)
  uint64_t m[R][H2];
#pragma unroll
  for (int a = 0; a < R; ++a) {
    const float* src = Am + (R * ty + a) * DH + R * tx;
#pragma unroll
    for (int q = 0; q < R / 4; ++q) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(src + 4 * q));
      m[a][2 * q] = f32x2_pack(v.x, v.y);
      m[a][2 * q + 1] = f32x2_pack(v.z, v.w);
    }
  }
#pragma unroll
  for (int b = 0; b < R; ++b) {
    const float* src = Am + (R * tx + b) * DH + R * ty;
    float t[R];
#pragma unroll
    for (int q = 0; q < R / 4; ++q) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(src + 4 * q));
      t[4 * q] = v.x;
      t[4 * q + 1] = v.y;
      t[4 * q + 2] = v.z;
      t[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int a = 0; a < R; ++a) {
      float lo = f32x2_lo(m[a][b / 2]), hi = f32x2_hi(m[a][b / 2]);
      const float dg = (R * ty + a == R * tx + b) ? 1.f : 0.f;
      if (b & 1)
        hi = 0.5f * (hi + t[a]) + dg;
      else
        lo = 0.5f * (lo + t[a]) + dg;
      m[a][b / 2] = f32x2_pack(lo, hi);
    }
  }

  // row and column r of the blocks of row / column group g into buffer buf
  auto publish = [&](int buf, int g, int r) {
    if (ty == g) {
#pragma unroll
      for (int q = 0; q < R / 4; ++q)
        *reinterpret_cast<float4*>(&rowb[buf][R * tx + 4 * q]) =
            make_float4(f32x2_lo(m[r][2 * q]), f32x2_hi(m[r][2 * q]),
                        f32x2_lo(m[r][2 * q + 1]), f32x2_hi(m[r][2 * q + 1]));
    }
    if (tx == g) {
      float c[R];
#pragma unroll
      for (int a = 0; a < R; ++a) c[a] = (r & 1) ? f32x2_hi(m[a][r / 2]) : f32x2_lo(m[a][r / 2]);
#pragma unroll
      for (int q = 0; q < R / 4; ++q)
        *reinterpret_cast<float4*>(&colb[buf][R * ty + 4 * q]) =
            make_float4(c[4 * q], c[4 * q + 1], c[4 * q + 2], c[4 * q + 3]);
    }
  };
  publish(0, 0, 0);
  __syncthreads();
#pragma unroll 1
  for (int g = 0; g < 16; ++g) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int p = R * g + r;
      const int buf = r & 1;  // R is even: the parity of p
      float piv = rowb[buf][p];
      if (!(piv > 0.f)) {  // also catches NaN
        bad = true;
        piv = 1.f;
      }
      const float inv = __frcp_rn(piv);
      const uint64_t ninv2 = f32x2_pack(-inv, -inv);
      uint64_t nrk[H2];  // -M[p][k] / piv at this thread's columns
#pragma unroll
      for (int q = 0; q < R / 4; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(&rowb[buf][R * tx + 4 * q]);
        nrk[2 * q] = f32x2_mul(f32x2_pack(v.x, v.y), ninv2);
        nrk[2 * q + 1] = f32x2_mul(f32x2_pack(v.z, v.w), ninv2);
      }
      float col[R];  // M[i][p] at this thread's rows
#pragma unroll
      for (int q = 0; q < R / 4; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(&colb[buf][R * ty + 4 * q]);
        col[4 * q] = v.x;
        col[4 * q + 1] = v.y;
        col[4 * q + 2] = v.z;
        col[4 * q + 3] = v.w;
      }
#pragma unroll
      for (int a = 0; a < R; ++a) {
        const uint64_t c2 = f32x2_pack(col[a], col[a]);
#pragma unroll
        for (int b = 0; b < H2; ++b) m[a][b] = f32x2_fma(c2, nrk[b], m[a][b]);
      }
      if (ty == g) {  // row p: M[p][k] / piv
#pragma unroll
        for (int b = 0; b < H2; ++b) m[r][b] = f32x2_mul(nrk[b], f32x2_pack(-1.f, -1.f));
      }
      if (tx == g) {  // column p: -M[i][p] / piv, and the pivot 1 / piv
#pragma unroll
        for (int a = 0; a < R; ++a) {
          const float v = (a == r && ty == g) ? inv : -col[a] * inv;
          float lo = f32x2_lo(m[a][r / 2]), hi = f32x2_hi(m[a][r / 2]);
          if (r & 1)
            hi = v;
          else
            lo = v;
          m[a][r / 2] = f32x2_pack(lo, hi);
        }
      }
      // the next step's row and column into the other buffer (its readers
      // all passed the barrier that ended the step before this one)
      if (p + 1 < DH) {
        if (r + 1 < R)
          publish((r + 1) & 1, g, r + 1);
        else
          publish(0, g + 1, 0);
      }
      __syncthreads();
    }
  }
  float* Pm = P + mat;
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int q = 0; q < R / 4; ++q)
      *reinterpret_cast<float4*>(Pm + (R * ty + a) * DH + R * tx + 4 * q) =
          make_float4(f32x2_lo(m[a][2 * q]), f32x2_hi(m[a][2 * q]), f32x2_lo(m[a][2 * q + 1]),
                      f32x2_hi(m[a][2 * q + 1]));
  if (bad) record_status(status, kStatusNumeric);
}

template <int DH>
cudaError_t launch_solve_dh(const Launch& ctx, const vdn_shape& s, const float* A, float* P,
                            int solver) {
  static std::atomic<uint64_t> chol_set{0};
  if (cudaError_t e = set_smem_once(vda_solve_kernel<DH>, CholCfg<DH>::SMEM, chol_set)) return e;
  if (solver == VDN_SOLVER_GAUSS_JORDAN)
    vda_solve_gj_kernel<DH><<<s.T * s.H, kThreads, 0, ctx.stream>>>(A, P, ctx.status);
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
