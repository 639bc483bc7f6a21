// Bidirectional frame scan of Video DeltaNet's linear branch ("Video
// DeltaNet", 10100.com article, 方法概述 item 2 and the figure caption under
// 效率阶梯: a forward and a backward scan over the latent frames):
//
//   S_fwd_t = (alpha_t S_fwd_{t-1} + B_t) P_t    t = 0 .. T-1, S_fwd_{-1} = 0
//   S_bwd_t = (alpha_t S_bwd_{t+1} + B_t) P_t    t = T-1 .. 0, S_bwd_T   = 0
//
// with P_t = (I + A_t)^-1 from the solve.  Rows of S evolve independently
// (row r of S_t needs only row r of S_{t-1}), so each CTA owns a block of
// rows of one head's state in one direction and runs all T steps; every CTA
// of the grid is resident at once.  The block is 8 x TR rows: TR = 8 (two
// blocks per state at d = 128), or, when three blocks per state still fit
// the SMs once, TR = 6 (48-row blocks, the last one 32 rows with the rest
// masked), which shortens each step by a quarter.  Per step the CTA stages P_t (d x d fp32) and
// its rows of B_t (one contiguous block) into shared memory with bulk
// copies, double-buffered so that step t+1's operands land while step t
// computes (nothing on a step's critical path waits on global memory).
// Each thread first writes its tile of the bracket alpha S_prev + B_t into
// the shared rows (row stride d + 4, so four consecutive k of a row are one
// float4 and the rows of a warp fall in different banks), then computes TR
// rows x 8 columns of the new state with packed f32x2 FMA: per k it loads TR
// state and 8 P values for 8 TR FMA, a ratio at which shared-memory
// bandwidth (32 floats per clock per SM) keeps up with the FMA pipes.  The
// CTA's two halves split the k range of the product (two warps per SM
// sub-partition keep the packed FMAs issuing); the upper half hands its
// partial sums over through the step's B buffer, already consumed.  A
// thread's columns are two interleaved groups of 4 (4c.., d/2 + 4c..), so
// each quarter warp reads 128 contiguous bytes of P.
// Multiplying the bracket (rather than adding a precomputed B_t P_t) keeps
// the d^3 product C = B P out of the solve, at the price of one product at
// the first step.  The scan is serial over T and FP32-ALU bound.
//
// Adjoint mode (kAdjoint) runs the two scans of the gradient pass.  With
// G_t = sum_i dO_i q_i^T, the sensitivity of the loss to the bracket of
// each direction obeys
//   D_t = (alpha_u D_u + G_t) P_t,   u = the frame the same scan visited
// one step earlier (t - 1 going forward in time, t + 1 going backward):
// the same step with G in place of B and the decay of the previous frame.
// Output direction 0 (forward in time) is the adjoint of the backward scan,
// direction 1 the adjoint of the forward scan.
#include "common.cuh"
#include "exp2_fma.cuh"
#include "ptx.cuh"

namespace vdn {
namespace {

constexpr int kGroups = 8;  // row groups per CTA (TR rows each)
constexpr int kTC = 8;      // columns per thread

template <int DH, int TR>
struct ScanCfg {
  static constexpr int ROWS = kGroups * TR;           // rows of S per CTA
  static constexpr int BLOCKS = (DH + ROWS - 1) / ROWS;  // row blocks per state
  static constexpr int HALF = kGroups * (DH / kTC);  // threads per k half
  static constexpr int THREADS = 2 * HALF;           // 256 (d=128), 128 (d=64)
  static constexpr int P_BYTES = DH * DH * 4;
  static constexpr int X_BYTES = ROWS * DH * 4;  // the CTA's rows of B_t (or G_t)
  static constexpr int LDS = DH + 4;  // row stride of the state rows in shared memory
  static constexpr int SMEM = 2 * P_BYTES + 2 * X_BYTES + ROWS * LDS * 4 + 64;
};

template <int DH, int TR, bool kAdjoint>
__global__ void __launch_bounds__(ScanCfg<DH, TR>::THREADS, 1)
    vda_scan_kernel(const float* __restrict__ P, const float* __restrict__ X,
                    const float* __restrict__ alpha, float* __restrict__ states, int T, int H,
                    uint32_t* status, uint64_t budget_ns) {
  using Cfg = ScanCfg<DH, TR>;
  constexpr int CG = DH / kTC;  // column groups
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* Pbuf = reinterpret_cast<float*>(smem_raw);                  // 2 x [DH][DH]
  float* Xbuf = reinterpret_cast<float*>(smem_raw + 2 * Cfg::P_BYTES);  // 2 x [ROWS][DH]
  float* Ss = reinterpret_cast<float*>(smem_raw + 2 * Cfg::P_BYTES + 2 * Cfg::X_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + 2 * Cfg::P_BYTES +
                                               2 * Cfg::X_BYTES + Cfg::ROWS * Cfg::LDS * 4);

  const int rb = blockIdx.x;  // row block
  const int h = blockIdx.y;
  const int dir = blockIdx.z;  // 0 forward, 1 backward
  const int half = threadIdx.x / Cfg::HALF;  // which half of the k range
  const int lt = threadIdx.x % Cfg::HALF;
  const int cg = lt % CG;
  const int rg = lt / CG;
  const int lrow0 = rg * TR;                   // first local row of the thread's tile
  const int row0 = rb * Cfg::ROWS + lrow0;     // first row of S
  // rows of this block inside the state (the last block may be partial)
  const int nrows = min(Cfg::ROWS, DH - rb * Cfg::ROWS);
  const int x_bytes = nrows * DH * 4;
  // the thread's columns: [colA, colA + 4) and [colB, colB + 4)
  const int colA = 4 * cg, colB = DH / 2 + 4 * cg;
  const int64_t mat = static_cast<int64_t>(DH) * DH;
  float* out_dir = states + static_cast<int64_t>(dir) * T * H * mat;
  auto frame = [&](int step) { return dir == 0 ? step : T - 1 - step; };
  // both operands of the step that visits frame(step), into buffer `buf`
  auto stage = [&](int step, int buf) {
    const int64_t th = static_cast<int64_t>(frame(step)) * H + h;
    mbar_arrive_expect_tx(&full[buf], Cfg::P_BYTES + x_bytes);
    bulk_load(Pbuf + buf * DH * DH, P + th * mat, Cfg::P_BYTES, &full[buf]);
    bulk_load(Xbuf + buf * Cfg::ROWS * DH,
              X + th * mat + static_cast<int64_t>(rb) * Cfg::ROWS * DH, x_bytes, &full[buf]);
  };

  for (int i = threadIdx.x; i < Cfg::ROWS * Cfg::LDS; i += blockDim.x) Ss[i] = 0.f;
  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_mbar_init();
    stage(0, 0);
  }
  __syncthreads();

  float sprev[TR][kTC];  // the thread's tile of the previous step's state
#pragma unroll
  for (int r = 0; r < TR; ++r)
#pragma unroll
    for (int c = 0; c < kTC; ++c) sprev[r][c] = 0.f;

  // forward: the decay of the frame being absorbed; adjoint: of the frame
  // visited one step earlier (unused at step 0, where the carried term is 0).
  // Read one step ahead, so no step waits on it.
  auto decay = [&](int step) {
    return !kAdjoint ? __ldg(alpha + frame(step) * H + h)
                     : (step > 0 ? __ldg(alpha + frame(step - 1) * H + h) : 0.f);
  };
  float a_next = decay(0);

  int issued = 1;
#pragma unroll 1
  for (int step = 0; step < T; ++step) {
    const int t = frame(step);
    const int b = step & 1;
    if (threadIdx.x == 0 && step + 1 < T) {
      // buffer b^1 was last read in step-1, which every thread has left
      stage(step + 1, b ^ 1);
      ++issued;
    }
    const float a = a_next;
    if (step + 1 < T) a_next = decay(step + 1);
    // U = a S_prev + X_t into the shared rows; every thread left the previous
    // step's reads behind the barrier that closed it, and the barrier below
    // publishes U before the multiply
    const bool ok = mbar_wait(&full[b], (step >> 1) & 1, budget_ns);
    float* Xt = Xbuf + b * Cfg::ROWS * DH;
    // rows past the state (masked block tail) carry junk that stays in
    // their own rows and is never stored
#pragma unroll
    for (int r = 0; r < TR; ++r) {
      if (half != 0) break;  // the lower half holds the state
      const float4 xa = *reinterpret_cast<const float4*>(Xt + (lrow0 + r) * DH + colA);
      const float4 xb = *reinterpret_cast<const float4*>(Xt + (lrow0 + r) * DH + colB);
      float* srow = Ss + (lrow0 + r) * Cfg::LDS;
      *reinterpret_cast<float4*>(srow + colA) =
          make_float4(fmaf(a, sprev[r][0], xa.x), fmaf(a, sprev[r][1], xa.y),
                      fmaf(a, sprev[r][2], xa.z), fmaf(a, sprev[r][3], xa.w));
      *reinterpret_cast<float4*>(srow + colB) =
          make_float4(fmaf(a, sprev[r][4], xb.x), fmaf(a, sprev[r][5], xb.y),
                      fmaf(a, sprev[r][6], xb.z), fmaf(a, sprev[r][7], xb.w));
    }
    if (!__syncthreads_and(ok)) {
      if (threadIdx.x == 0) record_status(status, kStatusTimeout);
      break;
    }
    const float* Pt = Pbuf + b * DH * DH;
    // acc2[r][q]: columns (colA + 2q, +1) for q < 2, (colB + 2(q-2), +1) for q >= 2
    uint64_t acc2[TR][kTC / 2];
#pragma unroll
    for (int r = 0; r < TR; ++r)
#pragma unroll
      for (int q = 0; q < kTC / 2; ++q) acc2[r][q] = 0ull;
    {
#pragma unroll 1
      for (int k = half * (DH / 2); k < (half + 1) * (DH / 2); k += 4) {
        float sr[TR][4];
#pragma unroll
        for (int r = 0; r < TR; ++r) {
          const float4 v = *reinterpret_cast<const float4*>(Ss + (lrow0 + r) * Cfg::LDS + k);
          sr[r][0] = v.x; sr[r][1] = v.y; sr[r][2] = v.z; sr[r][3] = v.w;
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const ulonglong2 pa = *reinterpret_cast<const ulonglong2*>(Pt + (k + kk) * DH + colA);
          const ulonglong2 pb = *reinterpret_cast<const ulonglong2*>(Pt + (k + kk) * DH + colB);
#pragma unroll
          for (int r = 0; r < TR; ++r) {
            const uint64_t ss = f32x2_pack(sr[r][kk], sr[r][kk]);
            acc2[r][0] = f32x2_fma(ss, pa.x, acc2[r][0]);
            acc2[r][1] = f32x2_fma(ss, pa.y, acc2[r][1]);
            acc2[r][2] = f32x2_fma(ss, pb.x, acc2[r][2]);
            acc2[r][3] = f32x2_fma(ss, pb.y, acc2[r][3]);
          }
        }
      }
    }
    // the upper half's partial sums, through the consumed B buffer
    if (half != 0) {
#pragma unroll
      for (int r = 0; r < TR; ++r) {
        *reinterpret_cast<ulonglong2*>(Xt + (lrow0 + r) * DH + colA) =
            make_ulonglong2(acc2[r][0], acc2[r][1]);
        *reinterpret_cast<ulonglong2*>(Xt + (lrow0 + r) * DH + colB) =
            make_ulonglong2(acc2[r][2], acc2[r][3]);
      }
    }
    __syncthreads();  // partials visible; every read of Ss and Pbuf b is done
    if (half == 0) {
#pragma unroll
      for (int r = 0; r < TR; ++r) {
        const ulonglong2 ua = *reinterpret_cast<const ulonglong2*>(Xt + (lrow0 + r) * DH + colA);
        const ulonglong2 ub = *reinterpret_cast<const ulonglong2*>(Xt + (lrow0 + r) * DH + colB);
        const uint64_t v[4] = {f32x2_add(acc2[r][0], ua.x), f32x2_add(acc2[r][1], ua.y),
                               f32x2_add(acc2[r][2], ub.x), f32x2_add(acc2[r][3], ub.y)};
#pragma unroll
        for (int q = 0; q < kTC / 2; ++q) {
          sprev[r][2 * q] = f32x2_lo(v[q]);
          sprev[r][2 * q + 1] = f32x2_hi(v[q]);
        }
        if (lrow0 + r < nrows) {
          float* dst = out_dir + (static_cast<int64_t>(t) * H + h) * mat +
                       static_cast<int64_t>(row0 + r) * DH;
          *reinterpret_cast<float4*>(dst + colA) =
              make_float4(sprev[r][0], sprev[r][1], sprev[r][2], sprev[r][3]);
          *reinterpret_cast<float4*>(dst + colB) =
              make_float4(sprev[r][4], sprev[r][5], sprev[r][6], sprev[r][7]);
        }
      }
    }
    __syncthreads();  // the partials are read: buffer b may be refilled
  }
  // the bulk copies this CTA started must land before it exits
  if (threadIdx.x == 0) {
    for (int s = (issued > 2 ? issued - 2 : 0); s < issued; ++s)
      mbar_wait(&full[s & 1], (s >> 1) & 1, 200000000ull);
  }
}

template <int DH, int TR, bool kAdjoint>
cudaError_t launch_scan_tr(const Launch& ctx, const vdn_shape& s, const float* P, const float* X,
                           const float* alpha, float* states) {
  using Cfg = ScanCfg<DH, TR>;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_once(vda_scan_kernel<DH, TR, kAdjoint>, Cfg::SMEM, smem_set))
    return e;
  dim3 grid(Cfg::BLOCKS, s.H, 2);
  vda_scan_kernel<DH, TR, kAdjoint><<<grid, Cfg::THREADS, Cfg::SMEM, ctx.stream>>>(
      P, X, alpha, states, s.T, s.H, ctx.status, ctx.budget_ns);
  return cudaGetLastError();
}

// The finer row blocks (TR = 6 at d = 128, 4 at d = 64) when their grid is
// resident at once (one CTA per SM: each holds two P_t buffers), else the
// 64-row blocks.
template <int DH, bool kAdjoint>
cudaError_t launch_scan_dh(const Launch& ctx, const vdn_shape& s, const float* P, const float* X,
                           const float* alpha, float* states) {
  constexpr int TR_FINE = DH == 128 ? 6 : 4;
  const int64_t fine_ctas = static_cast<int64_t>(ScanCfg<DH, TR_FINE>::BLOCKS) * s.H * 2;
  if (fine_ctas <= sm_count_of_current_device())
    return launch_scan_tr<DH, TR_FINE, kAdjoint>(ctx, s, P, X, alpha, states);
  return launch_scan_tr<DH, 8, kAdjoint>(ctx, s, P, X, alpha, states);
}

}  // namespace

cudaError_t launch_vda_scan(const Launch& ctx, const vdn_shape& s, const float* P,
                            const float* B, const float* alpha, float* states) {
  if (s.d == 128) return launch_scan_dh<128, false>(ctx, s, P, B, alpha, states);
  if (s.d == 64) return launch_scan_dh<64, false>(ctx, s, P, B, alpha, states);
  return cudaErrorInvalidValue;
}

cudaError_t launch_vda_adjoint_scan(const Launch& ctx, const vdn_shape& s, const float* P,
                                    const float* G, const float* alpha, float* adj) {
  if (s.d == 128) return launch_scan_dh<128, true>(ctx, s, P, G, alpha, adj);
  if (s.d == 64) return launch_scan_dh<64, true>(ctx, s, P, G, alpha, adj);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
