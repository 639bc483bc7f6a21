// VDA read-out ("Video DeltaNet", 10100.com article, 方法概述 item 2; the
// bidirectional reading of the figure caption under 效率阶梯):
//
//     o_vda[t*N + i, h] = (S_fwd_t,h + S_bwd_t,h) q_i
//
// One CTA per (frame, head).  The summed state is rounded to bf16 once into
// a 128B-swizzled K-major tile (the UMMA B operand, rows = value dims), then
// the CTA streams the frame's query tiles [128 tokens x d] through TMA,
// issues tcgen05.mma (M = 128 tokens, N = d, K = d) into a double-buffered
// TMEM accumulator, and four epilogue warps convert rows to bf16 in a
// swizzled staging tile that a TMA store writes back.  Loads and stores use
// a 3-D frame view, so the ragged last tile of a frame reads zeros and its
// extra rows are not written.  HBM-bound: q is read once and o written once.
//
// The gradient pass reuses the kernel: with kTransS the B operand is read
// MN-major, giving x (S_fwd + S_bwd) instead of x (S_fwd + S_bwd)^T
// (dq = dO S).  With kGram (head dim 128) each stage also holds the q tile
// of the same tokens and the kernel accumulates G = dO^T q (the adjoint
// scans' input, sum over the frame's tokens of dO_i q_i^T) in a third TMEM
// region from the dO tile already there, so dO is read once for both.
#include "common.cuh"
#include "ptx.cuh"

namespace vdn {
namespace {

template <int DH, bool kGram = false>
struct ReadoutCfg {
  static constexpr int SLABS = DH / 64;
  static constexpr int QTILE_BYTES = SLABS * 128 * 128;  // 128 tokens x DH bf16
  static constexpr int STAGE_BYTES = (kGram ? 2 : 1) * QTILE_BYTES;  // x tile (then q tile)
  static constexpr int STAGES = kGram ? 2 : 3;
  static constexpr int S_BYTES = SLABS * DH * 128;       // DH rows x DH bf16
  static constexpr int OUT_BUFS = kGram ? 1 : 2;
  static constexpr int TMEM_COLS = kGram ? 4 * DH : 2 * DH;  // 2 output buffers (+ G)
  static constexpr int THREADS = 192;
  static constexpr int SMEM =
      1024 + STAGES * STAGE_BYTES + S_BYTES + OUT_BUFS * QTILE_BYTES + 256;
};


template <int DH, bool kTransS, bool kGram = false>
__global__ void __launch_bounds__(ReadoutCfg<DH, kGram>::THREADS, 1)
    vda_readout_kernel(const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap omap, const float* __restrict__ states,
                       int T, int N, int H, uint32_t* status,
                       uint64_t budget_ns, const __grid_constant__ CUtensorMap gmap,
                       float* __restrict__ G) {
  static_assert(!kGram || (DH == 128 && kTransS), "G is formed beside dq, head dim 128");
  using Cfg = ReadoutCfg<DH, kGram>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* qbuf = smem;
  uint8_t* sbuf = qbuf + Cfg::STAGES * Cfg::STAGE_BYTES;
  uint8_t* obuf = sbuf + Cfg::S_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(obuf + Cfg::OUT_BUFS * Cfg::QTILE_BYTES);
  uint64_t* empty = full + Cfg::STAGES;
  uint64_t* tfull = empty + Cfg::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint64_t* g_full = mma_done + 1;  // kGram: every product into G has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(g_full + 1);

  const int t = blockIdx.x / H;
  const int h = blockIdx.x % H;
  const int ntiles = (N + 127) / 128;
  const uint32_t warp = warp_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(mma_done, 1);
    mbar_init(g_full, 1);
    fence_mbar_init();
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&omap);
    if constexpr (kGram) tma_prefetch_desc(&gmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }

  // Summed state -> bf16, 128B-swizzled K-major tile (row v, 64-wide k slabs).
  {
    const int64_t mat = (static_cast<int64_t>(t) * H + h) * DH * DH;
    const float* Sf = states + mat;
    const float* Sb = states + static_cast<int64_t>(T) * H * DH * DH + mat;
    constexpr int CHUNKS = DH * DH / 8;
    for (int ci = threadIdx.x; ci < CHUNKS; ci += Cfg::THREADS) {
      const int v = ci / (DH / 8);
      const int cc = ci % (DH / 8);
      const float4* pf = reinterpret_cast<const float4*>(Sf + v * DH + cc * 8);
      const float4* pb = reinterpret_cast<const float4*>(Sb + v * DH + cc * 8);
      const float4 f0 = __ldg(pf), f1 = __ldg(pf + 1), b0 = __ldg(pb), b1 = __ldg(pb + 1);
      uint4 u;
      u.x = pack_bf16x2(f0.x + b0.x, f0.y + b0.y);
      u.y = pack_bf16x2(f0.z + b0.z, f0.w + b0.w);
      u.z = pack_bf16x2(f1.x + b1.x, f1.y + b1.y);
      u.w = pack_bf16x2(f1.z + b1.z, f1.w + b1.w);
      *reinterpret_cast<uint4*>(sbuf + (cc / 8) * (DH * 128) + sw128_offset(v, cc % 8)) = u;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

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
        mbar_arrive_expect_tx(&full[s], Cfg::STAGE_BYTES);
        for (int sl = 0; sl < Cfg::SLABS; ++sl) {
          tma_load_3d(qbuf + s * Cfg::STAGE_BYTES + sl * 16384, &qmap, &full[s],
                      h * DH + 64 * sl, j * 128, t);
          if constexpr (kGram)
            tma_load_3d(qbuf + s * Cfg::STAGE_BYTES + Cfg::QTILE_BYTES + sl * 16384, &gmap,
                        &full[s], h * DH + 64 * sl, j * 128, t);
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
      constexpr uint32_t idesc = idesc_bf16(128, DH, false, kTransS);
      const uint32_t sb = smem_u32(sbuf);
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
        const uint32_t qb = smem_u32(qbuf + s * Cfg::STAGE_BYTES);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          // K-major: rows of the tile are N, 64-wide K slabs; MN-major: rows
          // are K (16 per step), 64-wide N slabs DH * 128 bytes apart
          const uint64_t sdesc = kTransS ? sdesc_sw128(sb + kk * 2048, DH * 128, 1024)
                                         : sdesc_sw128(sb + (kk >> 2) * (DH * 128) + (kk & 3) * 32,
                                                       16, 1024);
          umma_ss(tmem + b * DH, sdesc_sw128(qb + koff, 16, 1024), sdesc, idesc, kk > 0);
        }
        if constexpr (kGram) {
          // G += dO^T q over the tile's 128 tokens: both operands MN-major
          // (16 token rows per step, the two 64-feature slabs 16 KB apart)
          constexpr uint32_t idesc_g = idesc_bf16(128, DH, true, true);
          const uint32_t gb = qb + Cfg::QTILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tmem + 2 * DH, sdesc_sw128(qb + kk * 2048, 16384, 1024),
                    sdesc_sw128(gb + kk * 2048, 16384, 1024), idesc_g, (j | kk) != 0);
        }
        umma_commit(&empty[s]);
        umma_commit(&tfull[b]);
      }
      if constexpr (kGram) umma_commit(g_full);
      umma_commit(mma_done);  // every MMA of this CTA, also after an early exit
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t quarter = warp & 3;
    const int row = quarter * 32 + lane_id();
    const bool leader = threadIdx.x == 64;
    for (int j = 0; j < ntiles; ++j) {
      const int b = j & 1;
      if (leader) bulk_wait_read<Cfg::OUT_BUFS - 1>();  // staging buffer b is free again
      const bool ok = mbar_wait(&tfull[b], (j >> 1) & 1, budget_ns);
      // collective decision (also the barrier that publishes "buffer free"),
      // so no thread is left waiting at a named barrier after a timeout
      if (!named_bar_and(1, 128, ok)) {
        if (!ok) record_status(status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      uint8_t* ob = obuf + (j % Cfg::OUT_BUFS) * Cfg::QTILE_BYTES;
      const uint32_t taddr = tmem + b * DH + ((quarter * 32) << 16);
#pragma unroll
      for (int c = 0; c < DH; c += 32) {
        uint32_t r[32];
        tmem_ld32(taddr + c, r);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 u;
          u.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
          u.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
          u.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
          u.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
          const int chunk = ((c & 63) >> 3) + q;  // 16-byte chunk within the 128-byte row
          *reinterpret_cast<uint4*>(ob + (c >> 6) * 16384 + sw128_offset(row, chunk)) = u;
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[b]);
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (leader) {
        for (int sl = 0; sl < Cfg::SLABS; ++sl)
          tma_store_3d(&omap, ob + sl * 16384, h * DH + 64 * sl, j * 128, t);
        bulk_commit();
      }
    }
    if (leader) bulk_wait<0>();
    if constexpr (kGram) {
      // G: row m of the fp32 matrix from TMEM lane m (warp-uniform wait)
      if (__all_sync(0xffffffffu, mbar_wait(g_full, 0, budget_ns))) {
        tc_fence_after();
        float* dst = G + ((static_cast<int64_t>(t) * H + h) * DH + row) * DH;
        const uint32_t gaddr = tmem + 2 * DH + ((quarter * 32) << 16);
#pragma unroll 1
        for (int c = 0; c < DH; c += 32) {
          uint32_t r[32];
          tmem_ld32(gaddr + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + c + e) =
                make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                            __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
        }
      } else {
        record_status(status, kStatusTimeout);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    mbar_wait(mma_done, 0, 200000000ull);
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

template <int DH, bool kTransS, bool kGram = false>
cudaError_t launch_readout_dh(const Launch& ctx, const vdn_shape& s, const CUtensorMap& qmap,
                              const CUtensorMap& omap, const float* states,
                              const CUtensorMap* gmap = nullptr, float* G = nullptr) {
  using Cfg = ReadoutCfg<DH, kGram>;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_once(vda_readout_kernel<DH, kTransS, kGram>, Cfg::SMEM, smem_set))
    return e;
  vda_readout_kernel<DH, kTransS, kGram><<<s.T * s.H, Cfg::THREADS, Cfg::SMEM, ctx.stream>>>(
      qmap, omap, states, s.T, s.N, s.H, ctx.status, ctx.budget_ns, gmap ? *gmap : qmap, G);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_vda_readout(const Launch& ctx, const vdn_shape& s, const CUtensorMap& qmap,
                               const CUtensorMap& omap, const float* states) {
  if (s.d == 128) return launch_readout_dh<128, false>(ctx, s, qmap, omap, states);
  if (s.d == 64) return launch_readout_dh<64, false>(ctx, s, qmap, omap, states);
  return cudaErrorInvalidValue;
}

cudaError_t launch_vda_readout_dq_gram(const Launch& ctx, const vdn_shape& s,
                                       const CUtensorMap& domap, const CUtensorMap& dqmap,
                                       const CUtensorMap& qmap, const float* states, float* G) {
  if (s.d != 128) return cudaErrorInvalidValue;
  return launch_readout_dh<128, true, true>(ctx, s, domap, dqmap, states, &qmap, G);
}

cudaError_t launch_vda_readout_ex(const Launch& ctx, const vdn_shape& s, const CUtensorMap& xmap,
                                  const CUtensorMap& omap, const float* states, bool trans_s) {
  if (s.d == 128)
    return trans_s ? launch_readout_dh<128, true>(ctx, s, xmap, omap, states)
                   : launch_readout_dh<128, false>(ctx, s, xmap, omap, states);
  if (s.d == 64)
    return trans_s ? launch_readout_dh<64, true>(ctx, s, xmap, omap, states)
                   : launch_readout_dh<64, false>(ctx, s, xmap, omap, states);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
