// Branch calibration and output projections ("Video DeltaNet", 10100.com
// article, 方法概述 item 3: the Softmax branch gets a content-dependent
// sigmoid gate, the linear branch RMSNorm and its own sigmoid output gate,
// each branch its own output projection, and the two are added):
//
//   GEMM 1  G = x [W_gs; W_gl]^T                    (M = L, N = 2D, K = D)
//           epilogue: Z[:, :D] = sigmoid(G[:, :D]) * o_s
//                     Z[:, D:] = sigmoid(G[:, D:]) * RMSNorm_head(o_vda) * gamma
//   GEMM 2  y = Z [W_os | W_ol]^T                   (M = L, N = D, K = 2D)
//           (the sum of the two projections happens in the accumulator)
//
// One persistent tcgen05 GEMM kernel serves both: 128 x 256 output tiles,
// TMA-fed 4-stage ring of [128 x 64] A and [256 x 64] B tiles (K-major,
// 128B swizzle), one MMA-issuing thread, two 256-column TMEM accumulators so
// the four epilogue warps drain tile i while the tensor core runs tile i+1.
// Tiles are walked m-major (all N blocks of one M block in turn) so the A
// rows are reused from L2 and the weights stay L2-resident.
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "mxfp8.cuh"
#include "ptx.cuh"
#include "repack.cuh"

namespace vdn {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
// warp 0 TMA, warp 1 MMA, warps 2-9 epilogue: two warps per TMEM lane quarter,
// each draining half of the tile's columns
constexpr int EPI_THREADS = 256;
constexpr int GEMM_THREADS = 64 + EPI_THREADS;
constexpr int GEMM_SMEM = 1024 + STAGES * STAGE_BYTES + 256;

enum class BSplit { kByN, kByK };

struct GateArgs {
  const __nv_bfloat16* o_s;
  const __nv_bfloat16* o_vda;
  const float* gamma;
  float eps;
  int D, d;      // hidden size and head stride (columns per head)
  float inv_d;   // 1 / (true head dim): the RMS divisor (padded columns are 0)
  __nv_bfloat16* Z;  // [M, 2D]
};

struct StoreArgs {
  __nv_bfloat16* y;  // [M, N]
};

struct StoreF32Args {
  float* y;  // [M, N] fp32 (partial sums of a head shard)
};

// GEMM fused with a reduce-scatter: row r of the fp32 partial is added into
// owner[r / rows] at row r % rows (peer memory of the rank that owns the
// row block), with system-scope atomics, so the partials of all shards
// arrive summed in their owners' buffers without a separate collective.
struct RedScatterArgs {
  float* owner[8];
  int rows;   // rows of each owner's block
  int count;  // owners
};

__device__ __forceinline__ float sigmoidf_fast(float x) {
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-x * 1.4426950408889634f));
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.f + e));
  return r;
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* p, float (&f)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = __ldg(q + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 v = unpack_bf16x2(w[e]);
      f[8 * i + 2 * e] = v.x;
      f[8 * i + 2 * e + 1] = v.y;
    }
  }
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* p, const float (&f)[32]) {
  uint4* q = reinterpret_cast<uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    q[i] = make_uint4(pack_bf16x2(f[8 * i], f[8 * i + 1]), pack_bf16x2(f[8 * i + 2], f[8 * i + 3]),
                      pack_bf16x2(f[8 * i + 4], f[8 * i + 5]),
                      pack_bf16x2(f[8 * i + 6], f[8 * i + 7]));
}

// Gated branch inputs z for one 32-column chunk of row r starting at
// column n of GEMM 1's output (gate logits in acc); rinv carries the head's
// 1 / RMS from its first chunk to the next ones (fresh: the thread's first
// chunk of a tile, which may start inside a head).
template <class A>
__device__ __forceinline__ void gate_values(const A& a, int64_t r, int n, const uint32_t (&acc)[32],
                                            float& rinv, float (&z)[32], bool fresh) {
  if (n < a.D) {
    float os[32];
    load_bf16x32(a.o_s + r * a.D + n, os);
#pragma unroll
    for (int e = 0; e < 32; ++e) z[e] = sigmoidf_fast(__uint_as_float(acc[e])) * os[e];
  } else {
    const int c = n - a.D;
    const __nv_bfloat16* orow = a.o_vda + r * a.D;
    if (fresh || c % a.d == 0) {  // the head's RMS over its d channels
      const int hs = c - c % a.d;
      float ss = 0.f;
      for (int k = 0; k < a.d; k += 32) {
        float f[32];
        load_bf16x32(orow + hs + k, f);
#pragma unroll
        for (int e = 0; e < 32; ++e) ss = fmaf(f[e], f[e], ss);
      }
      rinv = rsqrtf(ss * a.inv_d + a.eps);
    }
    float ov[32];
    load_bf16x32(orow + c, ov);
#pragma unroll
    for (int e = 0; e < 32; ++e)
      z[e] = sigmoidf_fast(__uint_as_float(acc[e])) * (ov[e] * rinv * __ldg(a.gamma + c + e));
  }
}

// Epilogue for GEMM 1 on one 32-column chunk of row r starting at column n.
__device__ __forceinline__ void gate_chunk(const GateArgs& a, int64_t r, int n,
                                           const uint32_t (&acc)[32], float& rinv, bool fresh) {
  float z[32];
  gate_values(a, r, n, acc, rinv, z, fresh);
  store_bf16x32(a.Z + r * (2 * static_cast<int64_t>(a.D)) + n, z);
}

template <BSplit SPLIT, class Args>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap b0map,
                const __grid_constant__ CUtensorMap b1map, int M, int N, int K, int split_at,
                Args args, uint32_t* status, uint64_t budget_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int mblocks = (M + BM - 1) / BM;
  const int nblocks = (N + BN - 1) / BN;
  const int ntiles = mblocks * nblocks;
  const int nk = K / BK;
  const uint32_t warp = warp_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], EPI_THREADS);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&amap);
    tma_prefetch_desc(&b0map);
    tma_prefetch_desc(&b1map);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int mb = tile / nblocks, nb = tile % nblocks;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          if (it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, budget_ns)) {
            record_status(status, kStatusTimeout);
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(sa, &amap, &full[s], kb * BK, mb * BM);
          // B tile in two 128-row halves, so a split between the two B
          // matrices may fall on any multiple of 128 rows
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            int brow = nb * BN + hb * (BN / 2), bcol = kb * BK;
            const CUtensorMap* bm = &b0map;
            if (SPLIT == BSplit::kByN && brow >= split_at) {
              bm = &b1map;
              brow -= split_at;
            }
            if (SPLIT == BSplit::kByK && bcol >= split_at) {
              bm = &b1map;
              bcol -= split_at;
            }
            tma_load_2d(sa + A_BYTES + hb * (B_BYTES / 2), bm, &full[s], bcol, brow);
          }
        }
      }
      // drain the last loads
      const uint32_t first = it > STAGES ? it - STAGES : 0;
      for (uint32_t j = first; j < it; ++j)
        if (!mbar_wait(&full[j % STAGES], (j / STAGES) & 1, 200000000ull))
          record_status(status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_bf16(BM, BN, false, false);
      uint32_t it = 0;
      int lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++lt) {
        const int b = lt & 1;
        if (lt >= 2 && !mbar_wait(&tempty[b], ((lt >> 1) & 1) ^ 1, budget_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc_addr = tmem + b * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1, budget_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_ss(acc_addr, sdesc_sw128(sa + kk * 32, 16, 1024),
                    sdesc_sw128(sa + A_BYTES + kk * 32, 16, 1024), idesc, (kb | kk) != 0);
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&tfull[b]);
      }
      if (!ok) record_status(status, kStatusTimeout);
      umma_commit(mma_done);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t quarter = warp & 3;
    const int row = quarter * 32 + lane_id();
    const int c0 = static_cast<int>((warp - 2) >> 2) * (BN / 2);  // this warp's column half
    int lt = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++lt) {
      const int b = lt & 1;
      // warp-uniform: the TMEM loads below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[b], (lt >> 1) & 1, budget_ns))) {
        record_status(status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      const int mb = tile / nblocks, nb = tile % nblocks;
      const int64_t r = static_cast<int64_t>(mb) * BM + row;
      const uint32_t taddr = tmem + b * BN + ((quarter * 32) << 16);
      float rinv = 0.f;
#pragma unroll 1
      for (int c = c0; c < c0 + BN / 2; c += 32) {
        uint32_t acc[32];
        tmem_ld32(taddr + c, acc);
        tmem_ld_wait();
        const int n = nb * BN + c;
        if (r < M && n < N) {
          if constexpr (SPLIT == BSplit::kByN) {
            gate_chunk(args, r, n, acc, rinv, c == c0);
          } else if constexpr (std::is_same<Args, RedScatterArgs>::value) {
            const int o = static_cast<int>(r / args.rows);
            // the owning rank's block, and the row within it (checked in
            // debug builds)
            if (in_bounds(status, o, args.count, n, 32, N) &&
                in_bounds(status, r - static_cast<int64_t>(o) * args.rows, args.rows, n, 32, N)) {
              float4* dst = reinterpret_cast<float4*>(
                  args.owner[o] + (r - static_cast<int64_t>(o) * args.rows) * N + n);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                atomicAdd_system(dst + e, make_float4(__uint_as_float(acc[4 * e]),
                                                      __uint_as_float(acc[4 * e + 1]),
                                                      __uint_as_float(acc[4 * e + 2]),
                                                      __uint_as_float(acc[4 * e + 3])));
            }
          } else if constexpr (sizeof(args.y[0]) == 4) {
            float4* dst = reinterpret_cast<float4*>(args.y + r * N + n);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(acc[4 * e]), __uint_as_float(acc[4 * e + 1]),
                                   __uint_as_float(acc[4 * e + 2]),
                                   __uint_as_float(acc[4 * e + 3]));
          } else {
            float f[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(acc[e]);
            store_bf16x32(args.y + r * N + n, f);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    mbar_wait(mma_done, 0, 200000000ull);
    tmem_dealloc(tmem, 512);
  }
}

template <BSplit SPLIT, class Args>
cudaError_t launch_gemm(const Launch& ctx, const CUtensorMap& a, const CUtensorMap& b0,
                        const CUtensorMap& b1, int M, int N, int K, int split_at, const Args& args,
                        int sm_count) {
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_once(gemm_kernel<SPLIT, Args>, GEMM_SMEM, smem_set)) return e;
  const int ntiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = ntiles < sm_count ? ntiles : sm_count;
  gemm_kernel<SPLIT, Args><<<grid, GEMM_THREADS, GEMM_SMEM, ctx.stream>>>(
      a, b0, b1, M, N, K, split_at, args, ctx.status, ctx.budget_ns);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- MXFP8 GEMM
//
// C[M, N] = A[M, K] B[N, K]^T with both operands MXFP8 (E4M3 codes, K-major,
// one UE8M0 scale per 32 elements of K in the tile layout of mxfp8.cuh).
// Same persistent structure as gemm_kernel, with 128 x 128 output tiles: a
// 6-stage ring of [128 x 128]-byte A and B tiles (TMA, 128B swizzle) plus
// the two 512-byte scale blocks of the stage (bulk copies); the MMA thread
// copies a stage's scales into TMEM (tcgen05.cp, replicated into all lane
// quarters) and issues four block-scaled MMAs (K = 32 each, the scale byte
// chosen by the instruction's scale id).  TMEM: two 128-column accumulators
// and 8 scale columns per stage.
constexpr int MX_BM = 128, MX_BN = 128, MX_BK = 128, MX_STAGES = 6;
constexpr int MX_TILE = 128 * MX_BK;                 // 16 KB of codes
constexpr int MX_STAGE = 2 * MX_TILE + 1024;         // A, B, their scale blocks
constexpr int MX_SMEM = 1024 + MX_STAGES * MX_STAGE + 256;
constexpr int MX_SF_COL = 2 * MX_BN;                 // first scale column in TMEM

struct GateMXArgs {
  const __nv_bfloat16* o_s;
  const __nv_bfloat16* o_vda;
  const float* gamma;
  float eps;
  int D, d;
  float inv_d;
  uint8_t* zq;   // [M, 2D] E4M3 codes
  uint8_t* zsf;  // scales of Z, tile layout (2D / 128 column tiles)
};

template <class Args>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_mx_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                   const uint8_t* __restrict__ a_sf, const uint8_t* __restrict__ b_sf, int M, int N,
                   int K, Args args, uint32_t* status, uint64_t budget_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + MX_STAGES * MX_STAGE);
  uint64_t* empty = full + MX_STAGES;
  uint64_t* tfull = empty + MX_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int mblocks = (M + MX_BM - 1) / MX_BM;
  const int nblocks = (N + MX_BN - 1) / MX_BN;
  const int ntiles = mblocks * nblocks;
  const int nk = K / MX_BK;
  const uint32_t warp = warp_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < MX_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], EPI_THREADS);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&amap);
    tma_prefetch_desc(&bmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int mb = tile / nblocks, nb = tile % nblocks;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % MX_STAGES;
          if (it >= MX_STAGES && !mbar_wait(&empty[s], ((it / MX_STAGES) & 1) ^ 1, budget_ns)) {
            record_status(status, kStatusTimeout);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * MX_STAGE;
          mbar_arrive_expect_tx(&full[s], MX_STAGE);
          tma_load_2d(st, &amap, &full[s], kb * MX_BK, mb * MX_BM);
          tma_load_2d(st + MX_TILE, &bmap, &full[s], kb * MX_BK, nb * MX_BN);
          bulk_load(st + 2 * MX_TILE, a_sf + (static_cast<int64_t>(mb) * nk + kb) * 512, 512,
                    &full[s]);
          bulk_load(st + 2 * MX_TILE + 512, b_sf + (static_cast<int64_t>(nb) * nk + kb) * 512, 512,
                    &full[s]);
        }
      }
      const uint32_t first = it > MX_STAGES ? it - MX_STAGES : 0;
      for (uint32_t j = first; j < it; ++j)
        if (!mbar_wait(&full[j % MX_STAGES], (j / MX_STAGES) & 1, 200000000ull))
          record_status(status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_mxf8(MX_BM, MX_BN);
      uint32_t it = 0;
      int lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++lt) {
        const int b = lt & 1;
        if (lt >= 2 && !mbar_wait(&tempty[b], ((lt >> 1) & 1) ^ 1, budget_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc_addr = tmem + b * MX_BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % MX_STAGES;
          if (!mbar_wait(&full[s], (it / MX_STAGES) & 1, budget_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * MX_STAGE);
          const uint32_t sfa = tmem + MX_SF_COL + 8 * s;
          const uint32_t sfb = sfa + 4;
          // 32 rows x 16 bytes per block: 8-row groups 128 bytes apart
          tmem_cp_32x128b_x4(sfa, sdesc_none(st + 2 * MX_TILE, 16, 128));
          tmem_cp_32x128b_x4(sfb, sdesc_none(st + 2 * MX_TILE + 512, 16, 128));
#pragma unroll
          for (int j = 0; j < MX_BK / 32; ++j) {
            const uint32_t id = idesc | (static_cast<uint32_t>(j) << 29) | (static_cast<uint32_t>(j) << 4);
            umma_mx_ss(acc_addr, sdesc_sw128(st + j * 32, 16, 1024),
                       sdesc_sw128(st + MX_TILE + j * 32, 16, 1024), id,
                       sfa | (static_cast<uint32_t>(j) << 30), sfb | (static_cast<uint32_t>(j) << 30),
                       (kb | j) != 0);
          }
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&tfull[b]);
      }
      if (!ok) record_status(status, kStatusTimeout);
      umma_commit(mma_done);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t quarter = warp & 3;
    const int row = quarter * 32 + lane_id();
    const int c0 = static_cast<int>((warp - 2) >> 2) * (MX_BN / 2);  // this warp's column half
    int lt = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++lt) {
      const int b = lt & 1;
      // warp-uniform: the TMEM loads below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[b], (lt >> 1) & 1, budget_ns))) {
        record_status(status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      const int mb = tile / nblocks, nb = tile % nblocks;
      const int64_t r = static_cast<int64_t>(mb) * MX_BM + row;
      const uint32_t taddr = tmem + b * MX_BN + ((quarter * 32) << 16);
      float rinv = 0.f;
#pragma unroll 1
      for (int c = c0; c < c0 + MX_BN / 2; c += 32) {
        uint32_t acc[32];
        tmem_ld32(taddr + c, acc);
        tmem_ld_wait();
        const int n = nb * MX_BN + c;
        if (r < M && n < N) {
          if constexpr (std::is_same<Args, GateMXArgs>::value) {
            float z[32];
            gate_values(args, r, n, acc, rinv, z, c == c0);
            uint4 codes[2];
            const uint8_t sb = mx_quantize_block(z, codes);
            const int64_t ldz = 2 * static_cast<int64_t>(args.D);
            uint4* dst = reinterpret_cast<uint4*>(args.zq + r * ldz + n);
            dst[0] = codes[0];
            dst[1] = codes[1];
            args.zsf[mx_sf_offset(r, n / 32, static_cast<int>(ldz / 128))] = sb;
          } else if constexpr (sizeof(args.y[0]) == 4) {
            float4* dst = reinterpret_cast<float4*>(args.y + r * N + n);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(acc[4 * e]), __uint_as_float(acc[4 * e + 1]),
                                   __uint_as_float(acc[4 * e + 2]),
                                   __uint_as_float(acc[4 * e + 3]));
          } else {
            float f[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(acc[e]);
            store_bf16x32(args.y + r * N + n, f);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    mbar_wait(mma_done, 0, 200000000ull);
    tmem_dealloc(tmem, 512);
  }
}

template <class Args>
cudaError_t launch_gemm_mx(const Launch& ctx, const CUtensorMap& a, const CUtensorMap& b,
                           const uint8_t* a_sf, const uint8_t* b_sf, int M, int N, int K,
                           const Args& args, int sm_count) {
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_once(gemm_mx_kernel<Args>, MX_SMEM, smem_set)) return e;
  const int ntiles = ((M + MX_BM - 1) / MX_BM) * ((N + MX_BN - 1) / MX_BN);
  const int grid = ntiles < sm_count ? ntiles : sm_count;
  gemm_mx_kernel<Args><<<grid, GEMM_THREADS, MX_SMEM, ctx.stream>>>(
      a, b, a_sf, b_sf, M, N, K, args, ctx.status, ctx.budget_ns);
  return cudaGetLastError();
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The head shard's fuse; Out is the output GEMM's epilogue (an fp32
// partial, or the reduce-scatter into the owners' buffers).
template <class Out>
vdn_status fuse_shard_impl(int L, int D, int H_local, int d, int head0, const void* x,
                           const void* o_s, const void* o_vda, int64_t ld_o, const void* W_gs,
                           const void* W_gl, const float* gamma, float eps, const void* W_os,
                           const void* W_ol, const Out& out, const void* out_ptr, void* ws,
                           size_t ws_bytes, void* stream) {
  const int64_t Dl = static_cast<int64_t>(H_local) * d;
  if (L < 1 || D < 1 || H_local < 1 || d < 1 || head0 < 0) return VDN_ERR_INVALID_ARG;
  if (D % d != 0 || static_cast<int64_t>(head0 + H_local) * d > D) return VDN_ERR_INVALID_ARG;
  if (!x || !o_s || !o_vda || !W_gs || !W_gl || !gamma || !W_os || !W_ol || !out_ptr)
    return VDN_ERR_INVALID_ARG;
  if (!a16(x) || !a16(o_s) || !a16(o_vda) || !a16(W_gs) || !a16(W_gl) || !a16(W_os) ||
      !a16(W_ol) || !a16(out_ptr) || (reinterpret_cast<uintptr_t>(gamma) & 3u))
    return VDN_ERR_INVALID_ARG;
  if (ld_o < Dl || ld_o % 8 || !(eps >= 0.f)) return VDN_ERR_INVALID_ARG;
  // row-parallel fuse: full-D reduction for the gates, local head columns in
  // Z, a partial y over the full output width
  if (d % 128 != 0 || D % 256 != 0 || Dl % 128 != 0) return VDN_ERR_UNSUPPORTED;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) ||
      ws_bytes < vdn_hybrid_fuse_shard_workspace(L, D, H_local, d))
    return VDN_ERR_WORKSPACE;
  __nv_bfloat16* Z = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + kStatusBytes);
  const int64_t c0 = static_cast<int64_t>(head0) * d;  // first local hidden column
  const __nv_bfloat16* bgs = static_cast<const __nv_bfloat16*>(W_gs) + c0 * D;  // local rows
  const __nv_bfloat16* bgl = static_cast<const __nv_bfloat16*>(W_gl) + c0 * D;
  const __nv_bfloat16* bos = static_cast<const __nv_bfloat16*>(W_os) + c0;      // local columns
  const __nv_bfloat16* bol = static_cast<const __nv_bfloat16*>(W_ol) + c0;
  constexpr int BH = BN / 2;
  CUtensorMap xmap, m_gs, m_gl, zmap, m_os, m_ol;
  if (!make_rows_map(&xmap, x, D, D, L, BM) || !make_rows_map(&m_gs, bgs, D, D, Dl, BH) ||
      !make_rows_map(&m_gl, bgl, D, D, Dl, BH) ||
      !make_rows_map(&zmap, Z, 2 * Dl, 2 * Dl, L, BM) ||
      !make_rows_map(&m_os, bos, Dl, D, D, BH) || !make_rows_map(&m_ol, bol, Dl, D, D, BH))
    return VDN_ERR_CUDA;
  // o_s / o_vda: local head columns with row stride ld_o
  if (ld_o != Dl) return VDN_ERR_UNSUPPORTED;
  Launch ctx{static_cast<cudaStream_t>(stream), static_cast<uint32_t*>(ws),
             current_wait_budget_ns()};
  const int sms = sm_count_of_current_device();
  GateArgs g{static_cast<const __nv_bfloat16*>(o_s), static_cast<const __nv_bfloat16*>(o_vda),
             gamma + c0, eps, static_cast<int>(Dl), d, 1.f / static_cast<float>(d), Z};
  if (launch_gemm<BSplit::kByN>(ctx, xmap, m_gs, m_gl, L, static_cast<int>(2 * Dl), D,
                                static_cast<int>(Dl), g, sms) != cudaSuccess)
    return VDN_ERR_CUDA;
  if (launch_gemm<BSplit::kByK>(ctx, zmap, m_os, m_ol, L, D, static_cast<int>(2 * Dl),
                                static_cast<int>(Dl), out, sms) != cudaSuccess)
    return VDN_ERR_CUDA;
  return VDN_OK;
}

}  // namespace
}  // namespace vdn

using namespace vdn;

extern "C" {

namespace {

// Fuse layout.  Hidden sizes that 256-wide tiles divide, with head dims that
// are multiples of 32, run as given: [status][Z].  Others run on heads padded
// to dp columns (the smallest multiple of 32 >= d with H * dp a multiple of
// 256): [status][Z][x' o_s' o_vda' y'][W_gs' W_gl' W_os' W_ol'][gamma'].
struct FusePlan {
  bool padded;
  int d, dp, Dp;
  size_t z, act, w, g, total;
};

size_t r256(size_t x) { return (x + 255) / 256 * 256; }

FusePlan fuse_plan(int L, int D, int H) {
  FusePlan p{};
  p.d = D / H;
  p.padded = (D % 256 != 0) || (p.d % 32 != 0);
  p.dp = p.d;
  if (p.padded) {
    p.dp = (p.d + 31) / 32 * 32;
    while ((static_cast<int64_t>(H) * p.dp) % 256 != 0) p.dp += 32;
  }
  p.Dp = H * p.dp;
  p.z = r256(static_cast<size_t>(L) * 2 * p.Dp * 2);
  p.act = p.padded ? r256(static_cast<size_t>(L) * p.Dp * 2) : 0;
  p.w = p.padded ? r256(static_cast<size_t>(p.Dp) * p.Dp * 2) : 0;
  p.g = p.padded ? r256(static_cast<size_t>(p.Dp) * 4) : 0;
  p.total = kStatusBytes + p.z + 4 * p.act + 4 * p.w + p.g;
  return p;
}

}  // namespace

size_t vdn_hybrid_fuse_workspace(int L, int D, int H) {
  if (L < 1 || D < 1 || H < 1 || D % H != 0) return 0;
  return fuse_plan(L, D, H).total;
}

vdn_status vdn_hybrid_fuse(int L, int D, int H, const void* x, const void* o_s,
                           const void* o_vda, const void* W_gs, const void* W_gl,
                           const float* gamma, float eps, const void* W_os, const void* W_ol,
                           void* y, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("vdn_hybrid_fuse");
  if (L < 1 || D < 1 || H < 1 || D % H != 0) return VDN_ERR_INVALID_ARG;
  if (!x || !o_s || !o_vda || !W_gs || !W_gl || !gamma || !W_os || !W_ol || !y)
    return VDN_ERR_INVALID_ARG;
  if (!a16(x) || !a16(o_s) || !a16(o_vda) || !a16(W_gs) || !a16(W_gl) || !a16(W_os) ||
      !a16(W_ol) || !a16(y) || (reinterpret_cast<uintptr_t>(gamma) & 3u))
    return VDN_ERR_INVALID_ARG;
  if (!(eps >= 0.f)) return VDN_ERR_INVALID_ARG;
  if (D % 8 != 0) return VDN_ERR_UNSUPPORTED;  // rows must stay 16-byte aligned
  const FusePlan pl = fuse_plan(L, D, H);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < pl.total)
    return VDN_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws) + kStatusBytes;
  __nv_bfloat16* Z = reinterpret_cast<__nv_bfloat16*>(base);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int Dp = pl.Dp, d = pl.d, dp = pl.dp;

  // operands of the two GEMMs: the caller's, or zero-padded copies per head
  const void *xg = x, *osg = o_s, *ovg = o_vda, *wgs = W_gs, *wgl = W_gl, *wos = W_os,
             *wol = W_ol;
  const float* gg = gamma;
  void* yg = y;
  if (pl.padded) {
    uint8_t* p = base + pl.z;
    void* xp = p;
    void* osp = p + pl.act;
    void* ovp = p + 2 * pl.act;
    void* yp = p + 3 * pl.act;
    uint8_t* wp = p + 4 * pl.act;
    float* gp = reinterpret_cast<float*>(wp + 4 * pl.w);
    const void* wsrc[4] = {W_gs, W_gl, W_os, W_ol};
    bool ok = launch_repack_bf16(st, xp, Dp, x, D, 1, L, L, H, dp, d) == cudaSuccess &&
              launch_repack_bf16(st, osp, Dp, o_s, D, 1, L, L, H, dp, d) == cudaSuccess &&
              launch_repack_bf16(st, ovp, Dp, o_vda, D, 1, L, L, H, dp, d) == cudaSuccess &&
              launch_repack_f32(st, gp, Dp, gamma, D, 1, 1, 1, H, dp, d) == cudaSuccess;
    for (int i = 0; i < 4 && ok; ++i)
      ok = launch_repack_bf16(st, wp + i * pl.w, Dp, wsrc[i], D, H, dp, d, H, dp, d) ==
           cudaSuccess;
    if (!ok) return VDN_ERR_CUDA;
    xg = xp;
    osg = osp;
    ovg = ovp;
    yg = yp;
    wgs = wp;
    wgl = wp + pl.w;
    wos = wp + 2 * pl.w;
    wol = wp + 3 * pl.w;
    gg = gp;
  }

  CUtensorMap xmap, m_gs, m_gl, zmap, m_os, m_ol;
  constexpr int BH = BN / 2;  // B boxes are 128-row halves
  if (!make_rows_map(&xmap, xg, Dp, Dp, L, BM) || !make_rows_map(&m_gs, wgs, Dp, Dp, Dp, BH) ||
      !make_rows_map(&m_gl, wgl, Dp, Dp, Dp, BH) ||
      !make_rows_map(&zmap, Z, 2 * Dp, 2 * Dp, L, BM) ||
      !make_rows_map(&m_os, wos, Dp, Dp, Dp, BH) || !make_rows_map(&m_ol, wol, Dp, Dp, Dp, BH))
    return VDN_ERR_CUDA;

  Launch ctx{st, static_cast<uint32_t*>(ws), current_wait_budget_ns()};
  const int sms = sm_count_of_current_device();
  GateArgs g{static_cast<const __nv_bfloat16*>(osg), static_cast<const __nv_bfloat16*>(ovg),
             gg, eps, Dp, dp, 1.f / static_cast<float>(d), Z};
  if (launch_gemm<BSplit::kByN>(ctx, xmap, m_gs, m_gl, L, 2 * Dp, Dp, Dp, g, sms) != cudaSuccess)
    return VDN_ERR_CUDA;
  StoreArgs so{static_cast<__nv_bfloat16*>(yg)};
  if (launch_gemm<BSplit::kByK>(ctx, zmap, m_os, m_ol, L, Dp, 2 * Dp, Dp, so, sms) != cudaSuccess)
    return VDN_ERR_CUDA;
  if (pl.padded && launch_repack_bf16(st, y, D, yg, Dp, 1, L, L, H, d, dp) != cudaSuccess)
    return VDN_ERR_CUDA;
  return VDN_OK;
}

size_t vdn_hybrid_fuse_shard_workspace(int L, int D, int H_local, int d) {
  if (L < 1 || D < 1 || H_local < 1 || d < 1) return 0;
  return kStatusBytes + static_cast<size_t>(L) * 2 * static_cast<size_t>(H_local) * d * 2;
}

vdn_status vdn_hybrid_fuse_shard(int L, int D, int H_local, int d, int head0, const void* x,
                                 const void* o_s, const void* o_vda, int64_t ld_o,
                                 const void* W_gs, const void* W_gl, const float* gamma, float eps,
                                 const void* W_os, const void* W_ol, float* y_partial, void* ws,
                                 size_t ws_bytes, void* stream) {
  NvtxRange nvtx("vdn_hybrid_fuse_shard");
  return fuse_shard_impl(L, D, H_local, d, head0, x, o_s, o_vda, ld_o, W_gs, W_gl, gamma, eps,
                         W_os, W_ol, StoreF32Args{y_partial}, y_partial, ws, ws_bytes, stream);
}

vdn_status vdn_hybrid_fuse_shard_rs(int L, int D, int H_local, int d, int head0, const void* x,
                                    const void* o_s, const void* o_vda, int64_t ld_o,
                                    const void* W_gs, const void* W_gl, const float* gamma,
                                    float eps, const void* W_os, const void* W_ol,
                                    float* const* y_owners, int G, void* ws, size_t ws_bytes,
                                    void* stream) {
  NvtxRange nvtx("vdn_hybrid_fuse_shard_rs");
  if (y_owners == nullptr || G < 1 || G > 8 || L < 1) return VDN_ERR_INVALID_ARG;
  RedScatterArgs out{};
  for (int o = 0; o < G; ++o) {
    if (y_owners[o] == nullptr || !a16(y_owners[o])) return VDN_ERR_INVALID_ARG;
    out.owner[o] = y_owners[o];
  }
  out.rows = (L + G - 1) / G;
  out.count = G;
  return fuse_shard_impl(L, D, H_local, d, head0, x, o_s, o_vda, ld_o, W_gs, W_gl, gamma, eps,
                         W_os, W_ol, out, y_owners[0], ws, ws_bytes, stream);
}

// ----------------------------------------------------------------- MXFP8

vdn_status vdn_gemm_mxfp8(int M, int N, int K, const void* a, const void* a_sf, const void* b,
                          const void* b_sf, void* c, int c_is_f32, void* ws, size_t ws_bytes,
                          void* stream) {
  NvtxRange nvtx("vdn_gemm_mxfp8");
  if (M < 1 || N < 1 || K < 1 || !a || !a_sf || !b || !b_sf || !c) return VDN_ERR_INVALID_ARG;
  if (K % 128 != 0 || N % 32 != 0) return VDN_ERR_UNSUPPORTED;
  if (!a16(a) || !a16(a_sf) || !a16(b) || !a16(b_sf) || !a16(c)) return VDN_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < kStatusBytes)
    return VDN_ERR_WORKSPACE;
  CUtensorMap amap, bmap;
  if (!make_rows_map_u8(&amap, a, K, K, M, MX_BM) || !make_rows_map_u8(&bmap, b, K, K, N, MX_BN))
    return VDN_ERR_CUDA;
  Launch ctx{static_cast<cudaStream_t>(stream), static_cast<uint32_t*>(ws),
             current_wait_budget_ns()};
  const int sms = sm_count_of_current_device();
  const uint8_t* asf = static_cast<const uint8_t*>(a_sf);
  const uint8_t* bsf = static_cast<const uint8_t*>(b_sf);
  cudaError_t e;
  if (c_is_f32)
    e = launch_gemm_mx(ctx, amap, bmap, asf, bsf, M, N, K, StoreF32Args{static_cast<float*>(c)},
                       sms);
  else
    e = launch_gemm_mx(ctx, amap, bmap, asf, bsf, M, N, K,
                       StoreArgs{static_cast<__nv_bfloat16*>(c)}, sms);
  return e == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

namespace {

// MXFP8 fuse workspace: [status][x codes L x D][x scales][Z codes L x 2D][Z scales]
struct MxFusePlan {
  size_t xq, xsf, zq, zsf, total;
};

MxFusePlan mx_fuse_plan(int L, int D) {
  MxFusePlan p;
  p.xq = kStatusBytes;
  p.xsf = p.xq + r256(static_cast<size_t>(L) * D);
  p.zq = p.xsf + r256(vdn_mxfp8_scale_bytes(L, D));
  p.zsf = p.zq + r256(static_cast<size_t>(L) * 2 * D);
  p.total = p.zsf + r256(vdn_mxfp8_scale_bytes(L, 2 * static_cast<int64_t>(D)));
  return p;
}

}  // namespace

size_t vdn_hybrid_fuse_mxfp8_workspace(int L, int D, int H) {
  if (L < 1 || D < 128 || H < 1 || D % H != 0 || D % 128 != 0) return 0;
  return mx_fuse_plan(L, D).total;
}

vdn_status vdn_hybrid_fuse_mxfp8(int L, int D, int H, const void* x, const void* o_s,
                                 const void* o_vda, const void* wg_q, const void* wg_sf,
                                 const float* gamma, float eps, const void* wo_q,
                                 const void* wo_sf, void* y, void* ws, size_t ws_bytes,
                                 void* stream) {
  NvtxRange nvtx("vdn_hybrid_fuse_mxfp8");
  if (L < 1 || D < 1 || H < 1 || D % H != 0) return VDN_ERR_INVALID_ARG;
  if (!x || !o_s || !o_vda || !wg_q || !wg_sf || !gamma || !wo_q || !wo_sf || !y)
    return VDN_ERR_INVALID_ARG;
  if (!a16(x) || !a16(o_s) || !a16(o_vda) || !a16(wg_q) || !a16(wg_sf) || !a16(wo_q) ||
      !a16(wo_sf) || !a16(y) || (reinterpret_cast<uintptr_t>(gamma) & 3u) || !(eps >= 0.f))
    return VDN_ERR_INVALID_ARG;
  const int d = D / H;
  // 128-column tiles: heads must not cross a tile (d divides 128) and the
  // RMSNorm reads whole 32-column chunks
  if (D % 128 != 0 || d % 32 != 0 || 128 % d != 0) return VDN_ERR_UNSUPPORTED;
  const MxFusePlan pl = mx_fuse_plan(L, D);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < pl.total)
    return VDN_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* xq = base + pl.xq;
  uint8_t* xsf = base + pl.xsf;
  uint8_t* zq = base + pl.zq;
  uint8_t* zsf = base + pl.zsf;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (launch_mx_quantize(st, x, D, L, D, xq, xsf) != cudaSuccess) return VDN_ERR_CUDA;

  CUtensorMap xmap, gmap, zmap, omap;
  if (!make_rows_map_u8(&xmap, xq, D, D, L, MX_BM) ||
      !make_rows_map_u8(&gmap, wg_q, D, D, 2 * static_cast<int64_t>(D), MX_BN) ||
      !make_rows_map_u8(&zmap, zq, 2 * static_cast<int64_t>(D), 2 * static_cast<int64_t>(D), L,
                        MX_BM) ||
      !make_rows_map_u8(&omap, wo_q, 2 * static_cast<int64_t>(D), 2 * static_cast<int64_t>(D), D,
                        MX_BN))
    return VDN_ERR_CUDA;
  Launch ctx{st, static_cast<uint32_t*>(ws), current_wait_budget_ns()};
  const int sms = sm_count_of_current_device();
  GateMXArgs g{static_cast<const __nv_bfloat16*>(o_s), static_cast<const __nv_bfloat16*>(o_vda),
               gamma, eps, D, d, 1.f / static_cast<float>(d), zq, zsf};
  if (launch_gemm_mx(ctx, xmap, gmap, xsf, static_cast<const uint8_t*>(wg_sf), L, 2 * D, D, g,
                     sms) != cudaSuccess)
    return VDN_ERR_CUDA;
  if (launch_gemm_mx(ctx, zmap, omap, zsf, static_cast<const uint8_t*>(wo_sf), L, D, 2 * D,
                     StoreArgs{static_cast<__nv_bfloat16*>(y)}, sms) != cudaSuccess)
    return VDN_ERR_CUDA;
  return VDN_OK;
}

}  // extern "C"

