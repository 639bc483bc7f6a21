// Gradient pass of Video DeltaNet's linear branch ("Video DeltaNet",
// 10100.com article, 方法概述 items 2 and 3: the closed-form frame update and
// the staged alignment that trains the branch).  Two kernels of that pass
// live here; the others are modes of the forward kernels (the transposed
// mode of the read-out for dq, which at head dim 128 also forms G, and the
// gram mode of the prep kernel for G at head dims 64 and below; the
// adjoint mode of the scan for D).
//
// With S_t = U_t P_t, U_t = alpha S_prev + B_t, P_t = (I + A_t)^-1 and the
// adjoint states D_t = dL/dU_t of both scans:
//
//   combine, per (t, h):
//     dA_t     = -(S_fwd_t^T D_fwd_t + S_bwd_t^T D_bwd_t)
//     E_t      = dA_t + dA_t^T                  (A_t is symmetric)
//     dalpha_t = <D_fwd_t, S_fwd_{t-1}> + <D_bwd_t, S_bwd_{t+1}>
//   per token i of frame t (dB_t = D_fwd_t + D_bwd_t):
//     a_i = E_t k_i + dB_t^T v_i,  w_i = dB_t k_i
//     dk_i = beta_i a_i,  dv_i = beta_i w_i,
//     dbeta_i = k_i . (E_t k_i / 2 + dB_t^T v_i) = (k_i . a_i + v_i . w_i) / 2
//   (v_i . w_i = k_i . dB_t^T v_i), so one pass over k and v gives all three.
#include "common.cuh"
#include "ptx.cuh"

namespace vdn {
namespace {

// ---------------------------------------------------------------- combine
//
// One CTA per (t, h); thread (ra, cb) owns the 8 x 8 block of dA at rows
// 8 ra.., columns 8 cb...  dA is a sum of outer products of matching rows
// (row k of S and row k of D), so 16-row chunks of the four matrices are
// staged in shared memory and every thread accumulates its block from them.
// FP32 throughout; 4 d^3 flops and 6 d^2 floats read per (t, h).
template <int DH>
struct CombineCfg {
  static constexpr int THREADS = (DH / 8) * (DH / 8);  // 256 (d=128), 64 (d=64)
  static constexpr int KC = 16;                        // rows per chunk
  static constexpr int LDA = DH + 1;                   // dA row stride (transposed reads)
  static constexpr int SMEM = 4 * KC * DH * 4 + DH * LDA * 4 + 32 * 4;
};

template <int DH>
__global__ void __launch_bounds__(CombineCfg<DH>::THREADS)
    vda_grad_combine_kernel(const float* __restrict__ states, const float* __restrict__ adj,
                            float* __restrict__ E, float* __restrict__ dalpha, int T, int H) {
  using Cfg = CombineCfg<DH>;
  constexpr int CB = DH / 8;
  extern __shared__ __align__(16) float sm[];
  float* cf = sm;                          // [KC][DH] rows of S_fwd
  float* cdf = cf + Cfg::KC * DH;          // D_fwd
  float* cb_ = cdf + Cfg::KC * DH;         // S_bwd
  float* cdb = cb_ + Cfg::KC * DH;         // D_bwd
  float* dA = cdb + Cfg::KC * DH;          // [DH][LDA]
  float* red = dA + DH * Cfg::LDA;         // [32]

  const int t = blockIdx.x / H;
  const int h = blockIdx.x % H;
  const int64_t mm = static_cast<int64_t>(DH) * DH;
  const int64_t tot = static_cast<int64_t>(T) * H * mm;
  const int64_t mat = (static_cast<int64_t>(t) * H + h) * mm;
  const float* Sf = states + mat;
  const float* Sb = states + tot + mat;
  const float* Db = adj + mat;        // direction 0: adjoint of the backward scan
  const float* Df = adj + tot + mat;  // direction 1: adjoint of the forward scan
  const float* Sf_prev = t > 0 ? states + mat - static_cast<int64_t>(H) * mm : nullptr;
  const float* Sb_next = t + 1 < T ? states + tot + mat + static_cast<int64_t>(H) * mm : nullptr;

  const int tid = threadIdx.x;
  const int a0 = (tid / CB) * 8, b0 = (tid % CB) * 8;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  float dal = 0.f;

#pragma unroll 1
  for (int k0 = 0; k0 < DH; k0 += Cfg::KC) {
    constexpr int V4 = Cfg::KC * DH / 4;
    for (int idx = tid; idx < V4; idx += Cfg::THREADS) {
      const int64_t g = static_cast<int64_t>(k0) * DH + 4 * idx;
      const float4 df = __ldg(reinterpret_cast<const float4*>(Df + g));
      const float4 db = __ldg(reinterpret_cast<const float4*>(Db + g));
      reinterpret_cast<float4*>(cf)[idx] = __ldg(reinterpret_cast<const float4*>(Sf + g));
      reinterpret_cast<float4*>(cb_)[idx] = __ldg(reinterpret_cast<const float4*>(Sb + g));
      reinterpret_cast<float4*>(cdf)[idx] = df;
      reinterpret_cast<float4*>(cdb)[idx] = db;
      if (Sf_prev != nullptr) {
        const float4 p = __ldg(reinterpret_cast<const float4*>(Sf_prev + g));
        dal += df.x * p.x + df.y * p.y + df.z * p.z + df.w * p.w;
      }
      if (Sb_next != nullptr) {
        const float4 n = __ldg(reinterpret_cast<const float4*>(Sb_next + g));
        dal += db.x * n.x + db.y * n.y + db.z * n.z + db.w * n.w;
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < Cfg::KC; ++r) {
      const float4 fa0 = *reinterpret_cast<const float4*>(cf + r * DH + a0);
      const float4 fa1 = *reinterpret_cast<const float4*>(cf + r * DH + a0 + 4);
      const float4 ba0 = *reinterpret_cast<const float4*>(cb_ + r * DH + a0);
      const float4 ba1 = *reinterpret_cast<const float4*>(cb_ + r * DH + a0 + 4);
      const float4 fb0 = *reinterpret_cast<const float4*>(cdf + r * DH + b0);
      const float4 fb1 = *reinterpret_cast<const float4*>(cdf + r * DH + b0 + 4);
      const float4 bb0 = *reinterpret_cast<const float4*>(cdb + r * DH + b0);
      const float4 bb1 = *reinterpret_cast<const float4*>(cdb + r * DH + b0 + 4);
      const float sa[8] = {fa0.x, fa0.y, fa0.z, fa0.w, fa1.x, fa1.y, fa1.z, fa1.w};
      const float ta[8] = {ba0.x, ba0.y, ba0.z, ba0.w, ba1.x, ba1.y, ba1.z, ba1.w};
      const float sd[8] = {fb0.x, fb0.y, fb0.z, fb0.w, fb1.x, fb1.y, fb1.z, fb1.w};
      const float td[8] = {bb0.x, bb0.y, bb0.z, bb0.w, bb1.x, bb1.y, bb1.z, bb1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(ta[i], td[j], fmaf(sa[i], sd[j], acc[i][j]));
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) dA[(a0 + i) * Cfg::LDA + b0 + j] = -acc[i][j];
  // dalpha: warp sums, then one thread adds the warp partials
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dal += __shfl_xor_sync(0xffffffffu, dal, o);
  if ((tid & 31) == 0) red[tid >> 5] = dal;
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
    for (int w = 0; w < Cfg::THREADS / 32; ++w) s += red[w];
    dalpha[t * H + h] = s;
  }
  float* Et = E + mat;
  for (int idx = tid; idx < DH * DH; idx += Cfg::THREADS) {
    const int a = idx / DH, b = idx % DH;
    Et[idx] = dA[a * Cfg::LDA + b] + dA[b * Cfg::LDA + a];
  }
}

// ---------------------------------------------------------------- dk, dbeta
//
// One CTA per (t, h), laid out like the read-out: the two d x d operands
// (E_t and dB_t) are rounded to bf16 once into 128B-swizzled tiles, TMA
// streams the frame's k and v tiles [128 tokens x d], one thread issues
//   Y = K E     (B operand K-major; E is symmetric)
//   Z = V dB    (B operand MN-major: the dB tile holds rows of dB)
// into a double-buffered TMEM pair, and four epilogue warps (one row each)
// combine Y, Z, the k row (read back from the swizzled stage) and beta into
// dk (bf16, TMA store through the frame view) and dbeta (fp32).  A stage is
// released by the epilogue once it has read k; HBM-bound: k and v are read
// once, dk written once.
template <int DH>
struct GradKCfg {
  static constexpr int SLABS = DH / 64;
  static constexpr int TILE = SLABS * 128 * 128;  // 128 tokens x DH bf16
  static constexpr int STAGES = DH == 128 ? 2 : 3;
  static constexpr int OPS = SLABS * DH * 128;     // DH x DH bf16
  static constexpr int OUT_BUFS = DH == 128 ? 1 : 2;
  static constexpr int TMEM_COLS = 4 * DH;         // (Y, Z) x 2 buffers
  static constexpr int THREADS = 192;
  static constexpr int SMEM = 1024 + STAGES * 2 * TILE + 2 * OPS + OUT_BUFS * TILE + 256;
};

// fp32 [DH][DH] (sum of one or two matrices) -> bf16 swizzled tile, rows = first index
template <int DH, int NT>
__device__ __forceinline__ void to_bf16_tile(uint8_t* tile, const float* m0, const float* m1) {
  constexpr int CHUNKS = DH * DH / 8;
  for (int ci = threadIdx.x; ci < CHUNKS; ci += NT) {
    const int r = ci / (DH / 8);
    const int cc = ci % (DH / 8);
    const float4* p0 = reinterpret_cast<const float4*>(m0 + r * DH + cc * 8);
    float4 f0 = __ldg(p0), f1 = __ldg(p0 + 1);
    if (m1 != nullptr) {
      const float4* p1 = reinterpret_cast<const float4*>(m1 + r * DH + cc * 8);
      const float4 g0 = __ldg(p1), g1 = __ldg(p1 + 1);
      f0 = make_float4(f0.x + g0.x, f0.y + g0.y, f0.z + g0.z, f0.w + g0.w);
      f1 = make_float4(f1.x + g1.x, f1.y + g1.y, f1.z + g1.z, f1.w + g1.w);
    }
    uint4 u;
    u.x = pack_bf16x2(f0.x, f0.y);
    u.y = pack_bf16x2(f0.z, f0.w);
    u.z = pack_bf16x2(f1.x, f1.y);
    u.w = pack_bf16x2(f1.z, f1.w);
    *reinterpret_cast<uint4*>(tile + (cc / 8) * (DH * 128) + sw128_offset(r, cc % 8)) = u;
  }
}

template <int DH>
__global__ void __launch_bounds__(GradKCfg<DH>::THREADS, 1)
    vda_grad_k_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap,
                      const __grid_constant__ CUtensorMap dkmap, const float* __restrict__ E,
                      const float* __restrict__ adj, const float* __restrict__ beta,
                      float* __restrict__ dbeta, __nv_bfloat16* __restrict__ dv, int64_t ld_dv,
                      int T, int N, int H, uint32_t* status, uint64_t budget_ns) {
  using Cfg = GradKCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem;                                  // [STAGES][K tile | V tile]
  uint8_t* ebuf = stages + Cfg::STAGES * 2 * Cfg::TILE;    // E_t
  uint8_t* dbbuf = ebuf + Cfg::OPS;                        // dB_t
  uint8_t* obuf = dbbuf + Cfg::OPS;                        // dk staging
  uint64_t* full = reinterpret_cast<uint64_t*>(obuf + Cfg::OUT_BUFS * Cfg::TILE);
  uint64_t* empty = full + Cfg::STAGES;
  uint64_t* tfull = empty + Cfg::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int t = blockIdx.x / H;
  const int h = blockIdx.x % H;
  const int ntiles = (N + 127) / 128;
  const uint32_t warp = warp_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 128);  // the epilogue threads, after reading k
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
    tma_prefetch_desc(&dkmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  {
    const int64_t mm = static_cast<int64_t>(DH) * DH;
    const int64_t mat = (static_cast<int64_t>(t) * H + h) * mm;
    to_bf16_tile<DH, Cfg::THREADS>(ebuf, E + mat, nullptr);
    to_bf16_tile<DH, Cfg::THREADS>(dbbuf, adj + mat, adj + static_cast<int64_t>(T) * H * mm + mat);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto kstage = [&](int s) { return stages + s * 2 * Cfg::TILE; };
  auto vstage = [&](int s) { return stages + s * 2 * Cfg::TILE + Cfg::TILE; };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      int issued = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % Cfg::STAGES;
        if (j >= Cfg::STAGES &&
            !mbar_wait(&empty[s], ((j / Cfg::STAGES) & 1) ^ 1, budget_ns)) {
          record_status(status, kStatusTimeout);
          break;
        }
        mbar_arrive_expect_tx(&full[s], 2 * Cfg::TILE);
        for (int sl = 0; sl < Cfg::SLABS; ++sl) {
          tma_load_3d(kstage(s) + sl * 16384, &kmap, &full[s], h * DH + 64 * sl, j * 128, t);
          tma_load_3d(vstage(s) + sl * 16384, &vmap, &full[s], h * DH + 64 * sl, j * 128, t);
        }
        ++issued;
      }
      for (int j = (issued > Cfg::STAGES ? issued - Cfg::STAGES : 0); j < issued; ++j)
        if (!mbar_wait(&full[j % Cfg::STAGES], (j / Cfg::STAGES) & 1, 200000000ull))
          record_status(status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      // a = K E + V dB (one accumulator), w = K dB^T: dB's tile is the
      // MN-major B operand of the first and the K-major one of the second
      constexpr uint32_t idesc_k = idesc_bf16(128, DH, false, false);
      constexpr uint32_t idesc_mn = idesc_bf16(128, DH, false, true);
      const uint32_t eb = smem_u32(ebuf);
      const uint32_t db = smem_u32(dbbuf);
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % Cfg::STAGES;
        const int b = j & 1;
        if (j >= 2 && !mbar_wait(&tempty[b], ((j >> 1) & 1) ^ 1, budget_ns)) {
          record_status(status, kStatusTimeout);
          break;
        }
        if (!mbar_wait(&full[s], (j / Cfg::STAGES) & 1, budget_ns)) {
          record_status(status, kStatusTimeout);
          break;
        }
        tc_fence_after();
        const uint32_t kb = smem_u32(kstage(s));
        const uint32_t vb = smem_u32(vstage(s));
        const uint32_t ty = tmem + b * 2 * DH;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t eoff = (kk >> 2) * (DH * 128) + (kk & 3) * 32;
          umma_ss(ty, sdesc_sw128(kb + aoff, 16, 1024), sdesc_sw128(eb + eoff, 16, 1024), idesc_k,
                  kk > 0);
          umma_ss(ty, sdesc_sw128(vb + aoff, 16, 1024),
                  sdesc_sw128(db + kk * 2048, DH * 128, 1024), idesc_mn, 1);
          umma_ss(ty + DH, sdesc_sw128(kb + aoff, 16, 1024), sdesc_sw128(db + eoff, 16, 1024),
                  idesc_k, kk > 0);
        }
        umma_commit(&tfull[b]);
      }
      umma_commit(mma_done);  // every MMA of this CTA, also after an early exit
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t quarter = warp & 3;
    const int row = quarter * 32 + lane_id();
    const bool leader = threadIdx.x == 64;
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % Cfg::STAGES;
      const int b = j & 1;
      const int tok = j * 128 + row;
      // this token's rows of dk, dv and dbeta are stored only inside the
      // frame (and inside the tensors: checked in debug builds)
      const bool store = tok < N && in_bounds(status, static_cast<int64_t>(t) * N + tok,
                                              static_cast<int64_t>(T) * N,
                                              static_cast<int64_t>(h) * DH, DH,
                                              static_cast<int64_t>(H) * DH);
      const float bt =
          tok < N ? __ldg(beta + (static_cast<int64_t>(t) * N + tok) * H + h) : 0.f;
      if (leader) bulk_wait_read<Cfg::OUT_BUFS - 1>();  // staging buffer free again
      // tfull: Y and Z are ready; full[s] (already complete, and it cannot
      // move on before this warp releases stage s): the k tile is visible
      // to this thread's plain loads
      const bool ok = mbar_wait(&tfull[b], (j >> 1) & 1, budget_ns) &&
                      mbar_wait(&full[s], (j / Cfg::STAGES) & 1, budget_ns);
      if (!named_bar_and(1, 128, ok)) {
        if (!ok) record_status(status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      uint8_t* ob = obuf + (j % Cfg::OUT_BUFS) * Cfg::TILE;
      const uint8_t* ks = kstage(s);
      const uint8_t* vs = vstage(s);
      const uint32_t taddr = tmem + b * 2 * DH + ((quarter * 32) << 16);
      // this token's row of dv, written from registers (16 bytes at a time)
      __nv_bfloat16* dvrow = dv + (static_cast<int64_t>(t) * N + tok) * ld_dv + h * DH;
      float dbt = 0.f;
#pragma unroll 1
      for (int c = 0; c < DH; c += 32) {
        uint32_t ra[32], rw[32];
        tmem_ld32(taddr + c, ra);
        tmem_ld32(taddr + DH + c, rw);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = ((c & 63) >> 3) + q;  // 16-byte chunk within the 128-byte row
          const uint32_t off = (c >> 6) * 16384 + sw128_offset(row, chunk);
          const uint4 kw = *reinterpret_cast<const uint4*>(ks + off);
          const uint4 vw = *reinterpret_cast<const uint4*>(vs + off);
          const uint32_t kwa[4] = {kw.x, kw.y, kw.z, kw.w};
          const uint32_t vwa[4] = {vw.x, vw.y, vw.z, vw.w};
          uint32_t o[4], ov[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 kf = unpack_bf16x2(kwa[e]);
            const float2 vf = unpack_bf16x2(vwa[e]);
            const float a0 = __uint_as_float(ra[8 * q + 2 * e]);
            const float a1 = __uint_as_float(ra[8 * q + 2 * e + 1]);
            const float w0 = __uint_as_float(rw[8 * q + 2 * e]);
            const float w1 = __uint_as_float(rw[8 * q + 2 * e + 1]);
            dbt = fmaf(kf.x, a0, dbt);
            dbt = fmaf(kf.y, a1, dbt);
            dbt = fmaf(vf.x, w0, dbt);
            dbt = fmaf(vf.y, w1, dbt);
            o[e] = pack_bf16x2(bt * a0, bt * a1);
            ov[e] = pack_bf16x2(bt * w0, bt * w1);
          }
          *reinterpret_cast<uint4*>(ob + off) = make_uint4(o[0], o[1], o[2], o[3]);
          if (store)
            *reinterpret_cast<uint4*>(dvrow + c + 8 * q) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[b]);
      mbar_arrive(&empty[s]);  // k and v of this stage are no longer needed
      if (store) dbeta[(static_cast<int64_t>(t) * N + tok) * H + h] = 0.5f * dbt;
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (leader) {
        for (int sl = 0; sl < Cfg::SLABS; ++sl)
          tma_store_3d(&dkmap, ob + sl * 16384, h * DH + 64 * sl, j * 128, t);
        bulk_commit();
      }
    }
    if (leader) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    mbar_wait(mma_done, 0, 200000000ull);
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

template <int DH>
cudaError_t launch_combine_dh(const Launch& ctx, const vdn_shape& s, const float* states,
                              const float* adj, float* E, float* dalpha) {
  using Cfg = CombineCfg<DH>;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_once(vda_grad_combine_kernel<DH>, Cfg::SMEM, smem_set)) return e;
  vda_grad_combine_kernel<DH><<<s.T * s.H, Cfg::THREADS, Cfg::SMEM, ctx.stream>>>(
      states, adj, E, dalpha, s.T, s.H);
  return cudaGetLastError();
}

template <int DH>
cudaError_t launch_grad_k_dh(const Launch& ctx, const vdn_shape& s, const CUtensorMap& kmap,
                             const CUtensorMap& vmap, const CUtensorMap& dkmap, const float* E,
                             const float* adj, const float* beta, float* dbeta, void* dv,
                             int64_t ld_dv) {
  using Cfg = GradKCfg<DH>;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_once(vda_grad_k_kernel<DH>, Cfg::SMEM, smem_set)) return e;
  vda_grad_k_kernel<DH><<<s.T * s.H, Cfg::THREADS, Cfg::SMEM, ctx.stream>>>(
      kmap, vmap, dkmap, E, adj, beta, dbeta, static_cast<__nv_bfloat16*>(dv), ld_dv, s.T, s.N,
      s.H, ctx.status, ctx.budget_ns);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_vda_grad_combine(const Launch& ctx, const vdn_shape& s, const float* states,
                                    const float* adj, float* E, float* dalpha) {
  if (s.d == 128) return launch_combine_dh<128>(ctx, s, states, adj, E, dalpha);
  if (s.d == 64) return launch_combine_dh<64>(ctx, s, states, adj, E, dalpha);
  return cudaErrorInvalidValue;
}

cudaError_t launch_vda_grad_k(const Launch& ctx, const vdn_shape& s, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, const CUtensorMap& dkmap, const float* E,
                              const float* adj, const float* beta, float* dbeta, void* dv,
                              int64_t ld_dv) {
  if (s.d == 128)
    return launch_grad_k_dh<128>(ctx, s, kmap, vmap, dkmap, E, adj, beta, dbeta, dv, ld_dv);
  if (s.d == 64)
    return launch_grad_k_dh<64>(ctx, s, kmap, vmap, dkmap, E, adj, beta, dbeta, dv, ld_dv);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
