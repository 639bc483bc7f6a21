// VDA-prep: per (frame t, head h) form
//     A_t,h = sum_i beta_i k_i k_i^T      B_t,h = sum_i beta_i v_i k_i^T
// over the N spatial tokens of frame t ("Video DeltaNet", 10100.com article,
// 方法概述 item 2: A_t gathers key correlations, B_t value-key writes).
//
// Design (sm_100a):
//  * one CTA per (t, h); the token dimension is the GEMM reduction;
//  * TMA streams [BK tokens x d] tiles of k and v into 128B-swizzled shared
//    memory through a 3-D frame view, so rows past the frame read as zero,
//    over a ring of 4 stages (6 in gram mode);
//  * four "scaler" warps write beta_i * k_i as a bf16 pair hi + lo (hi the
//    rounded product, lo the rounded remainder; their sum carries ~16
//    mantissa bits) into a ring of their own (2 stages), so the k/v ring
//    keeps more of its bytes in flight from HBM;
//  * one thread issues tcgen05.mma with both operands MN-major (token rows,
//    feature columns), fp32 accumulation in TMEM.  For d = 128 the K and V
//    tiles of a stage sit in adjacent 64-column slabs, so [K | V] is one
//    N = 256 operand: D += hi^T [K | V] + lo^T [K | V], two instructions per
//    16 tokens, with columns 0..127 of D holding A and 128..255 holding B^T
//    (the shared-memory operand reads are 24 KB per 16 tokens instead of
//    32 KB for four N = 128 products).  For d = 64 the stacked [K | V]
//    feature block is the M = 128 operand against hi and lo, so D holds A
//    (rows 0..63) and B (rows 64..127);
//  * the scaler warps then drain TMEM to global fp32 A and B (B^T columns
//    are stored transposed: per column, a warp writes 32 consecutive floats
//    of one row of B).
// The stage is HBM-bound (k and v are read once); the split doubles the
// tensor-core work, which stays below the HBM time.
//
// Gram mode (kGram) serves the gradient pass: with q in place of k and
// dL/do in place of v it forms G_t,h = sum_i dO_i q_i^T (no beta, no split:
// q is already bf16) and writes only that matrix.
#include "common.cuh"
#include "ptx.cuh"

namespace vdn {
namespace {

template <int DH, bool kGram>
struct PrepCfg {
  static constexpr int BK = DH == 128 ? 32 : 64;  // tokens per pipeline stage
  static constexpr int SLABS = DH / 64;           // 64-column slabs per tile
  static constexpr int SLAB_BYTES = BK * 128;
  static constexpr int TILE_BYTES = SLABS * SLAB_BYTES;
  static constexpr int KV_BYTES = 2 * TILE_BYTES;  // K then V (adjacent slabs)
  static constexpr int HL_BYTES = 2 * TILE_BYTES;  // (beta*K)_hi then (beta*K)_lo
  static constexpr int KV_STAGES = kGram ? 6 : 4;
  static constexpr int HL_STAGES = kGram ? 0 : 2;
  static constexpr int TMEM_COLS = DH == 128 ? 256 : 64;
  static constexpr int THREADS = 192;  // warp0 TMA, warp1 MMA, warps2-5 scale+epilogue
  static constexpr int SMEM = 1024 + KV_STAGES * KV_BYTES + HL_STAGES * HL_BYTES + 256;
  static constexpr int CHUNKS_PER_THREAD = TILE_BYTES / 16 / 128;
};

template <int DH, bool kGram>
__global__ void __launch_bounds__(PrepCfg<DH, kGram>::THREADS, 1)
    vda_prep_kernel(const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap, const float* __restrict__ beta,
                    float* __restrict__ A, float* __restrict__ B, int T, int N, int H,
                    uint32_t* status, uint64_t budget_ns) {
  using C = PrepCfg<DH, kGram>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* kv_ring = smem;
  uint8_t* hl_ring = smem + C::KV_STAGES * C::KV_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(hl_ring + C::HL_STAGES * C::HL_BYTES);
  uint64_t* empty = full + C::KV_STAGES;    // [KV_STAGES]
  uint64_t* scaled = empty + C::KV_STAGES;  // [HL_STAGES] hi/lo written
  uint64_t* hl_free = scaled + 2;           // [HL_STAGES] hi/lo consumed
  uint64_t* accum_full = hl_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_full + 1);

  const int th = blockIdx.x;  // = t * H + h
  const int t = th / H;
  const int h = th % H;
  const int nk = (N + C::BK - 1) / C::BK;
  const uint32_t warp = warp_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::KV_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < C::HL_STAGES; ++s) {
      mbar_init(&scaled[s], 128);
      mbar_init(&hl_free[s], 1);
    }
    mbar_init(accum_full, 1);
    fence_mbar_init();
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto stage_k = [&](int s) { return kv_ring + s * C::KV_BYTES; };
  auto stage_v = [&](int s) { return kv_ring + s * C::KV_BYTES + C::TILE_BYTES; };
  auto stage_hi = [&](int s) { return hl_ring + s * C::HL_BYTES; };
  auto stage_lo = [&](int s) { return hl_ring + s * C::HL_BYTES + C::TILE_BYTES; };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      int issued = 0;
      bool ok = true;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % C::KV_STAGES;
        if (kb >= C::KV_STAGES) {
          if (!mbar_wait(&empty[s], ((kb / C::KV_STAGES) & 1) ^ 1, budget_ns)) {
            record_status(status, kStatusTimeout);
            ok = false;
            break;
          }
        }
        mbar_arrive_expect_tx(&full[s], 2 * C::TILE_BYTES);
        for (int j = 0; j < C::SLABS; ++j) {
          tma_load_3d(stage_k(s) + j * C::SLAB_BYTES, &kmap, &full[s], h * DH + 64 * j,
                      kb * C::BK, t);
          tma_load_3d(stage_v(s) + j * C::SLAB_BYTES, &vmap, &full[s], h * DH + 64 * j,
                      kb * C::BK, t);
        }
        ++issued;
      }
      // Drain: the last loads of every stage must have landed before exit.
      for (int kb = (issued > C::KV_STAGES ? issued - C::KV_STAGES : 0); kb < issued; ++kb) {
        const int s = kb % C::KV_STAGES;
        if (!mbar_wait(&full[s], (kb / C::KV_STAGES) & 1, 200000000ull)) {
          record_status(status, kStatusTimeout);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_bf16(128, DH, true, true);
      constexpr uint32_t idesc_kv = idesc_bf16(128, 2 * DH, true, true);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % C::KV_STAGES;
        const int hs = kGram ? 0 : kb % C::HL_STAGES;
        // the k/v stage has landed, and (scaled) its hi/lo tiles are written
        if (!mbar_wait(&full[s], (kb / C::KV_STAGES) & 1, budget_ns) ||
            (!kGram && !mbar_wait(&scaled[hs], (kb / (kGram ? 1 : C::HL_STAGES)) & 1,
                                  budget_ns))) {
          record_status(status, kStatusTimeout);
          break;
        }
        tc_fence_after();
        const uint32_t kbase = smem_u32(stage_k(s));
        const uint32_t vbase = smem_u32(stage_v(s));
        const uint32_t hbase = smem_u32(stage_hi(hs));
        const uint32_t lbase = smem_u32(stage_lo(hs));
#pragma unroll
        for (int kk = 0; kk < C::BK / 16; ++kk) {
          const uint32_t acc = (kb | kk) != 0;
          const uint64_t hdesc = sdesc_sw128(hbase + kk * 2048, C::SLAB_BYTES, 1024);
          const uint64_t ldesc = sdesc_sw128(lbase + kk * 2048, C::SLAB_BYTES, 1024);
          const uint64_t kdesc = sdesc_sw128(kbase + kk * 2048, C::SLAB_BYTES, 1024);
          if constexpr (kGram) {
            if constexpr (DH == 128) {
              // G = dO^T q: dO features along M, q features along N
              umma_ss(tmem + 128, sdesc_sw128(vbase + kk * 2048, C::SLAB_BYTES, 1024), kdesc,
                      idesc, acc);
            } else {
              // [q | dO] stacked along M against q: rows 64..127 hold G
              umma_ss(tmem, kdesc, kdesc, idesc, acc);
            }
          } else if constexpr (DH == 128) {
            // kdesc spans the four slabs K0 K1 V0 V1 (N = 256)
            umma_ss(tmem, hdesc, kdesc, idesc_kv, acc);
            umma_ss(tmem, ldesc, kdesc, idesc_kv, 1);
          } else {
            // [K | V] stacked along M: the V slab sits one slab after K.
            umma_ss(tmem, kdesc, hdesc, idesc, acc);
            umma_ss(tmem, kdesc, ldesc, idesc, 1);
          }
        }
        umma_commit(&empty[s]);
        if constexpr (!kGram) umma_commit(&hl_free[hs]);
      }
      umma_commit(accum_full);
    }
  } else {
    // ------------------------------------------------------------ scalers
    const int tid = threadIdx.x - 64;  // 0..127
    bool ok = true;
    for (int kb = 0; kb < (kGram ? 0 : nk); ++kb) {
      const int s = kb % C::KV_STAGES;
      const int hs = kb % (kGram ? 1 : C::HL_STAGES);
      // beta for the rows this thread touches in this stage
      float bv[C::CHUNKS_PER_THREAD];
#pragma unroll
      for (int j = 0; j < C::CHUNKS_PER_THREAD; ++j) {
        const int off = (tid + 128 * j) * 16;
        const int row = (off % C::SLAB_BYTES) / 128;
        const int i = kb * C::BK + row;
        bv[j] = i < N ? __ldg(beta + (static_cast<int64_t>(t) * N + i) * H + h) : 0.f;
      }
      // the hi/lo stage must have been consumed by the MMAs of kb - HL_STAGES
      const bool got = mbar_wait(&full[s], (kb / C::KV_STAGES) & 1, budget_ns) &&
                       (kb < C::HL_STAGES ||
                        mbar_wait(&hl_free[hs], ((kb / (kGram ? 1 : C::HL_STAGES)) & 1) ^ 1,
                                  budget_ns));
      if (!__all_sync(0xffffffffu, got)) {
        record_status(status, kStatusTimeout);
        ok = false;
        break;
      }
      const uint8_t* ks = stage_k(s);
      uint8_t* his = stage_hi(hs);
      uint8_t* los = stage_lo(hs);
#pragma unroll
      for (int j = 0; j < C::CHUNKS_PER_THREAD; ++j) {
        const int off = (tid + 128 * j) * 16;
        uint4 u = *reinterpret_cast<const uint4*>(ks + off);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack_bf16x2(w[e]);
          const float px = f.x * bv[j], py = f.y * bv[j];
          hi[e] = pack_bf16x2(px, py);
          const float2 fh = unpack_bf16x2(hi[e]);
          lo[e] = pack_bf16x2(px - fh.x, py - fh.y);
        }
        *reinterpret_cast<uint4*>(his + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(los + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&scaled[hs]);
    }
    // ------------------------------------------------------------ epilogue
    // warp-uniform: the TMEM loads below are warp-collective
    if (__all_sync(0xffffffffu, ok && mbar_wait(accum_full, 0, budget_ns))) {
      tc_fence_after();
      const uint32_t quarter = warp & 3;  // TMEM lane quarter this warp may access
      const int m = quarter * 32 + lane_id();
      const uint32_t lane_base = tmem + ((quarter * 32) << 16);
      const int64_t mat = (static_cast<int64_t>(t) * H + h) * DH * DH;
      if constexpr (DH == 128) {
        // columns 0..127: row m of A (gram: unused); 128..255: row m of G
        // (gram) or column m of B
#pragma unroll 1
        for (int half = kGram ? 1 : 0; half < 2; ++half) {
          const bool rows = half == 0 || kGram;
          float* dst = (half == 0 ? A : B) + mat + static_cast<int64_t>(m) * (rows ? DH : 1);
#pragma unroll 1
          for (int c = 0; c < DH; c += 32) {
            uint32_t r[32];
            tmem_ld32(lane_base + half * 128 + c, r);
            tmem_ld_wait();
            if (rows) {
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4*>(dst + c + e) =
                    make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                dst[static_cast<int64_t>(c + e) * DH] = __uint_as_float(r[e]);
            }
          }
        }
      } else if (!kGram || quarter >= 2) {  // warp-uniform: rows 0..63 are q^T q
        float* dst = (m < 64 ? A + mat + static_cast<int64_t>(m) * DH
                             : B + mat + static_cast<int64_t>(m - 64) * DH);
#pragma unroll 1
        for (int c = 0; c < DH; c += 32) {
          uint32_t r[32];
          tmem_ld32(lane_base + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + c + e) =
                make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                            __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
        }
      }
    } else if (ok) {
      record_status(status, kStatusTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    // All MMAs were committed to accum_full; make sure they finished before
    // the columns are released (no-op on the normal path).
    mbar_wait(accum_full, 0, 200000000ull);
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int DH, bool kGram>
cudaError_t launch_prep_dh(const Launch& ctx, const vdn_shape& s, const CUtensorMap& kmap,
                           const CUtensorMap& vmap, const float* beta, float* A, float* B) {
  using C = PrepCfg<DH, kGram>;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_once(vda_prep_kernel<DH, kGram>, C::SMEM, smem_set)) return e;
  const int grid = s.T * s.H;
  vda_prep_kernel<DH, kGram><<<grid, C::THREADS, C::SMEM, ctx.stream>>>(
      kmap, vmap, beta, A, B, s.T, s.N, s.H, ctx.status, ctx.budget_ns);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_vda_prep(const Launch& ctx, const vdn_shape& s, const CUtensorMap& kmap,
                            const CUtensorMap& vmap, const float* beta, float* A, float* B) {
  if (s.d == 128) return launch_prep_dh<128, false>(ctx, s, kmap, vmap, beta, A, B);
  if (s.d == 64) return launch_prep_dh<64, false>(ctx, s, kmap, vmap, beta, A, B);
  return cudaErrorInvalidValue;
}

cudaError_t launch_vda_gram(const Launch& ctx, const vdn_shape& s, const CUtensorMap& qmap,
                            const CUtensorMap& domap, float* G) {
  if (s.d == 128) return launch_prep_dh<128, true>(ctx, s, qmap, domap, nullptr, nullptr, G);
  if (s.d == 64) return launch_prep_dh<64, true>(ctx, s, qmap, domap, nullptr, nullptr, G);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
