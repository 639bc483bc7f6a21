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

#include "common.cuh"
#include "ptx.cuh"
#include "repack.cuh"

namespace vdn {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int GEMM_THREADS = 192;  // warp0 TMA, warp1 MMA, warps2-5 epilogue
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

// Epilogue for GEMM 1 on one 32-column chunk of row r starting at column n.
__device__ __forceinline__ void gate_chunk(const GateArgs& a, int64_t r, int n,
                                           const uint32_t (&acc)[32], float& rinv) {
  float z[32];
  if (n < a.D) {
    float os[32];
    load_bf16x32(a.o_s + r * a.D + n, os);
#pragma unroll
    for (int e = 0; e < 32; ++e) z[e] = sigmoidf_fast(__uint_as_float(acc[e])) * os[e];
  } else {
    const int c = n - a.D;
    const __nv_bfloat16* orow = a.o_vda + r * a.D;
    if (c % a.d == 0) {  // first chunk of a head: its RMS over d channels
      float ss = 0.f;
      for (int k = 0; k < a.d; k += 32) {
        float f[32];
        load_bf16x32(orow + c + k, f);
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
      mbar_init(&tempty[b], 128);
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
      for (int c = 0; c < BN; c += 32) {
        uint32_t acc[32];
        tmem_ld32(taddr + c, acc);
        tmem_ld_wait();
        const int n = nb * BN + c;
        if (r < M && n < N) {
          if constexpr (SPLIT == BSplit::kByN) {
            gate_chunk(args, r, n, acc, rinv);
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
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<SPLIT, Args>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM_SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int ntiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = ntiles < sm_count ? ntiles : sm_count;
  gemm_kernel<SPLIT, Args><<<grid, GEMM_THREADS, GEMM_SMEM, ctx.stream>>>(
      a, b0, b1, M, N, K, split_at, args, ctx.status, ctx.budget_ns);
  return cudaGetLastError();
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count_of_current_device() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n > 0 ? n : 148;
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
  const int64_t Dl = static_cast<int64_t>(H_local) * d;
  if (L < 1 || D < 1 || H_local < 1 || d < 1 || head0 < 0) return VDN_ERR_INVALID_ARG;
  if (D % d != 0 || static_cast<int64_t>(head0 + H_local) * d > D) return VDN_ERR_INVALID_ARG;
  if (!x || !o_s || !o_vda || !W_gs || !W_gl || !gamma || !W_os || !W_ol || !y_partial)
    return VDN_ERR_INVALID_ARG;
  if (!a16(x) || !a16(o_s) || !a16(o_vda) || !a16(W_gs) || !a16(W_gl) || !a16(W_os) ||
      !a16(W_ol) || !a16(y_partial) || (reinterpret_cast<uintptr_t>(gamma) & 3u))
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
  StoreF32Args so{y_partial};
  if (launch_gemm<BSplit::kByK>(ctx, zmap, m_os, m_ol, L, D, static_cast<int>(2 * Dl),
                                static_cast<int>(Dl), so, sms) != cudaSuccess)
    return VDN_ERR_CUDA;
  return VDN_OK;
}

}  // extern "C"
