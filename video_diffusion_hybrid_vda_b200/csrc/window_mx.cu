// Window-and-anchor Softmax with both products on MXFP8 operands ("Video
// DeltaNet", 10100.com article: the window Softmax of 方法概述 item 1 and the
// MXFP8 inference of 实验结果 / 效率阶梯).  The pages name MXFP8 only; the OCP
// Microscaling definition is taken: E4M3 elements, one power-of-two UE8M0
// scale per 32 consecutive elements along the contraction of each product.
//
//   q, k : blocks of 32 along the head dim, per token and head      (S = q k^T)
//   v    : blocks of 32 consecutive token rows, per column           (O = P V)
//   P    : blocks of 32 consecutive keys of a row, formed in the kernel
//
// With s = q^ . k^ * scale and an integer running maximum m of the row (in
// the log2 domain), P = 2^(s log2 e - m); the row sum l adds the unquantized
// P, O accumulates P^ V^ and the output is O / l.  Because m is an integer,
// the block quantization of P commutes with the lazy rescale (it moves P by
// a power of two), so the result does not depend on the order in which the
// kernel meets the keys.
//
// Layout: the quantized operands live in the workspace: codes q8, k8, v8 as
// [L, H*d] bytes (v8 keeps v's row-major layout: the PV product reads it
// MN-major), the scales of q and k as [L, H*d/32] bytes (row-major) and the
// scales of v as [ceil(L/32), H*d] bytes.  Key tiles hold 96 keys, so that
// TMEM has room for the scale factors beside S0 S1 O0 O1:
//   S0 [0, 96)  SFA(Q0) 96  SFA(Q1) 100  SFA(P0) 104  SFA(P1) 108
//   S1 [128, 224)  SFB(K, stage s) 224 + 4 s  SFB(V, stage s) 240 + 4 s
//   O0 [256, 384)  O1 [384, 512)
// P goes through shared memory (the block-scaled MMA reads both operands
// from there); S_i is released as soon as the softmax has loaded it, so the
// next S_i product runs during this tile's exponentials.
//
// Warps: 0 TMA and scale gathers (all lanes), 1 MMA issue, 4-7 softmax of
// query tile 0, 8-11 of tile 1 (one thread per query row).  A quarter of the
// exponentials run on the FMA pipe (see VDN_MX_EXP2_FMA_PAIRS).
#include <math.h>

#include "common.cuh"
#include "exp2_fma.cuh"
#include "mxfp8.cuh"
#include "ptx.cuh"
#include "window_sched.cuh"

namespace vdn {
namespace {

struct WinMxCfg {
  static constexpr int KT = 96;                 // keys per tile
  static constexpr int Q_TILE = 128 * 128;      // 128 query rows x 128 code bytes
  static constexpr int P_TILE = 128 * 128;      // 128 rows x 96 code bytes (128-byte rows)
  static constexpr int K_TILE = KT * 128;       // 96 keys x 128 code bytes
  static constexpr int V_TILE = KT * 128;       // 96 key rows x 128 value-column bytes
  static constexpr int STAGE = K_TILE + V_TILE;
  static constexpr int STAGES = 4;
  static constexpr int SF = 512;                // one scale block in the tcgen05.cp layout
  static constexpr int THREADS = 384;
  static constexpr int SMEM =
      1024 + 2 * Q_TILE + 2 * P_TILE + STAGES * STAGE + (4 + 2 * STAGES) * SF + 512;
  // TMEM columns
  static constexpr uint32_t SFA_Q = 96, SFA_P = 104, SFB_K = 224, SFB_V = 240;
  static constexpr uint32_t O_COL = 256;
};
static_assert(WinMxCfg::SMEM <= 232448, "shared memory of one CTA");
static_assert(WinMxCfg::STAGE % 1024 == 0, "stages keep 1024-byte alignment");

// Instruction descriptor of the block-scaled MMA with B MN-major (bit 16).
__host__ __device__ constexpr uint32_t idesc_mxf8_bmn(int M, int N) {
  return idesc_mxf8(M, N) | (1u << 16);
}

// Of every 16 score pairs of a 32-key block, this many take the FMA-pipe
// exponential (exp2_fma.cuh; relative error 7.5e-5, far below the E4M3 step
// P is rounded to) and the rest the MUFU.  With the tensor work halved by
// FP8 the MUFU is this kernel's busiest unit; measured at 102 frames x 4032 x
// 24 x 128 (CUDA events, one B200): 0 -> 326.0 ms, 4 -> 308.0 ms, 6 -> 319.7
// ms, 8 -> 332.6 ms.
#ifndef VDN_MX_EXP2_FMA_PAIRS
#define VDN_MX_EXP2_FMA_PAIRS 4
#endif
static_assert(VDN_MX_EXP2_FMA_PAIRS == 0 || VDN_MX_EXP2_FMA_PAIRS == 4 ||
                  VDN_MX_EXP2_FMA_PAIRS == 8,
              "VDN_MX_EXP2_FMA_PAIRS: 0, 4 or 8 of 16 pairs");

__device__ __forceinline__ bool mx_exp2_on_fma(int pair) {
  if (VDN_MX_EXP2_FMA_PAIRS == 4) return (pair & 3) == 3;
  if (VDN_MX_EXP2_FMA_PAIRS == 8) return (pair & 1) == 1;
  return false;
}

// Scale bytes 0..2 of a row (or column) packed with byte 3 unused (unit scale).
__device__ __forceinline__ uint32_t pack_sf3(uint32_t b0, uint32_t b1, uint32_t b2) {
  return b0 | (b1 << 8) | (b2 << 16) | (127u << 24);
}

// One softmax warpgroup of the MXFP8 kernel (query tile i, one thread per
// row).  Per key tile: load S_i (96 columns), report it loaded, take the row
// maximum, rescale O_i when the maximum grew by more than 2^8 (warp-uniform,
// exact powers of two), form P in 32-key blocks, add P to the row sum,
// quantize each block (its scale byte goes to the tile's scale block), wait
// until the previous tile's PV product has read P_i, store P_i's codes and
// scales, and report them.
__device__ __forceinline__ void softmax_mx(int i, uint32_t tmem, uint64_t* s_full,
                                           uint64_t* s_free, uint64_t* p_ready, uint64_t* o_done,
                                           uint8_t* pbuf, uint8_t* psf, const KvRange& kr, int nkv,
                                           float scale_log2, int q0, int q_end, int h, int H,
                                           int L, __nv_bfloat16* __restrict__ out, int64_t ld_o,
                                           float* __restrict__ lse, uint32_t* status,
                                           uint64_t budget_ns) {
  using Cfg = WinMxCfg;
  const uint32_t quarter = warp_id() & 3;
  const uint32_t lane = lane_id();
  const int row = quarter * 32 + lane;
  const uint32_t lane_off = (quarter * 32) << 16;
  const uint32_t s_addr = tmem + (i ? 128u : 0u) + lane_off;
  const uint32_t o_addr = tmem + Cfg::O_COL + 128 * i + lane_off;
  float m_used = -INFINITY;  // running maximum, log2 domain, an integer once set
  float l = 0.f;
  KvCursorT<Cfg::KT> cur;
  cur.init(kr);
  bool ok = true;
  for (int j = 0; j < nkv; ++j) {
    const int valid = cur.valid();
    cur.next(kr);
    if (!__all_sync(0xffffffffu, mbar_wait(&s_full[i], j & 1, budget_ns))) {
      ok = false;
      break;
    }
    tc_fence_after();
    uint32_t sr[96];
    uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
    uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
    uint32_t (&s2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[64]);
    tmem_ld32(s_addr, s0);
    tmem_ld32(s_addr + 32, s1);
    tmem_ld32(s_addr + 64, s2);
    tmem_ld_wait();
    reg_fence(s0);
    reg_fence(s1);
    reg_fence(s2);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s_free[i]);  // S_i may be overwritten now
    if (valid < Cfg::KT) {
#pragma unroll
      for (int c = 0; c < Cfg::KT; ++c)
        if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
    }
    // maxima of the three 32-key blocks (raw scores), and of the row
    float bm[3];
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      float m4[4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
        m4[a] = fmax3(__uint_as_float(sr[32 * q + a]), __uint_as_float(sr[32 * q + 4 + a]),
                      __uint_as_float(sr[32 * q + 8 + a]));
#pragma unroll
      for (int c = 12; c < 28; c += 8)
#pragma unroll
        for (int a = 0; a < 4; ++a)
          m4[a] = fmax3(m4[a], __uint_as_float(sr[32 * q + c + a]),
                        __uint_as_float(sr[32 * q + c + 4 + a]));
#pragma unroll
      for (int a = 0; a < 4; ++a) m4[a] = fmaxf(m4[a], __uint_as_float(sr[32 * q + 28 + a]));
      bm[q] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
    }
    const float mt = fmax3(bm[0], bm[1], bm[2]) * scale_log2;
    if (__any_sync(0xffffffffu, mt > m_used + 8.f)) {
      const float m_new = fmaxf(m_used, ceilf(mt));
      // 2^(m_used - m_new): an exact power of two (0 before the first tile)
      const float dm = m_used - m_new;
      const float factor =
          dm < -126.f ? 0.f : __uint_as_float(static_cast<uint32_t>(127 + static_cast<int>(dm)) << 23);
      l *= factor;
      if (j > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(&o_done[i], (j - 1) & 1, budget_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t o[32];
          tmem_ld32(o_addr + c, o);
          tmem_ld_wait();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
          tmem_st32(o_addr + c, o);
        }
      }
      m_used = m_new;
    }
    // Per 32-key block b with x = s * scale_log2 - m (P = 2^x): the block's
    // scale exponent is e = floor(max x) - 8 (= floor(log2 max P) - 8,
    // clamped at -127), the E4M3 codes are those of y = 2^(x - e) (the
    // exponential is evaluated there directly), and the row sum adds
    // 2^e * sum(y) = sum(P), unquantized.
    const uint64_t cc = f32x2_pack(scale_log2, scale_log2);
    uint4 codes[6];
    uint32_t sbytes[3];
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      const float xb = fmaf(bm[q], scale_log2, -m_used);
      const int e = xb == -INFINITY ? -127 : max(-127, static_cast<int>(floorf(xb)) - 8);
      const float ne = -(m_used + static_cast<float>(e));
      const uint64_t nb = f32x2_pack(ne, ne);
      uint64_t acc2[2] = {0ull, 0ull};
      uint32_t w[8];
#pragma unroll
      for (int e2 = 0; e2 < 16; e2 += 2) {
        uint32_t h2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c0 = 32 * q + 2 * (e2 + u);
          const uint64_t xs =
              f32x2_fma((static_cast<uint64_t>(sr[c0 + 1]) << 32) | sr[c0], cc, nb);
          float y0, y1;
          if (mx_exp2_on_fma(e2 + u)) {
            const uint64_t yy = exp2_fma_x2(xs);
            y0 = f32x2_lo(yy);
            y1 = f32x2_hi(yy);
          } else {
            y0 = exp2_mufu(f32x2_lo(xs));
            y1 = exp2_mufu(f32x2_hi(xs));
          }
          acc2[u] = f32x2_add(acc2[u], f32x2_pack(y0, y1));
          h2[u] = static_cast<uint32_t>(
              __nv_cvt_float2_to_fp8x2(make_float2(y0, y1), __NV_SATFINITE, __NV_E4M3));
        }
        w[e2 >> 1] = h2[0] | (h2[1] << 16);
      }
      codes[2 * q] = make_uint4(w[0], w[1], w[2], w[3]);
      codes[2 * q + 1] = make_uint4(w[4], w[5], w[6], w[7]);
      sbytes[q] = static_cast<uint32_t>(e + 127);
      const uint64_t ys = f32x2_add(acc2[0], acc2[1]);
      // 2^e exactly (0 for the clamped exponent -127: such a block's P are below 2^-118)
      l = fmaf(f32x2_lo(ys) + f32x2_hi(ys), __uint_as_float(static_cast<uint32_t>(e + 127) << 23),
               l);
    }
    // P_i and its scale block are read by the previous tile's PV product
    if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(&o_done[i], (j - 1) & 1, budget_ns))) {
      ok = false;
      break;
    }
    // codes of keys 16c .. 16c+15: 16-byte chunk c of the row (128-byte swizzle)
    uint8_t* prow = pbuf + row * 128;
#pragma unroll
    for (int c = 0; c < 6; ++c) *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) = codes[c];
    // scale byte of (row, key block kb) at (row % 32) * 16 + (row / 32) * 4 + kb
    *reinterpret_cast<uint32_t*>(psf + lane * 16 + quarter * 4) =
        pack_sf3(sbytes[0], sbytes[1], sbytes[2]);
    fence_proxy_async_smem();  // read by the tensor core through the async proxy
    __syncwarp();
    if (lane == 0) mbar_arrive(&p_ready[i]);
  }
  // ------------------------------------------------------------ epilogue
  if (__all_sync(0xffffffffu, ok && mbar_wait(&o_done[i], (nkv - 1) & 1, budget_ns))) {
    tc_fence_after();
    const int r = q0 + 128 * i + row;
    // rows past the segment are not stored (bounds checked in debug builds)
    const bool live = r < q_end && in_bounds(status, r, L, static_cast<int64_t>(h) * 128, 128,
                                             static_cast<int64_t>(H) * 128);
    const float inv = 1.f / l;
    __nv_bfloat16* dst = out + static_cast<int64_t>(r) * ld_o + h * 128;
#pragma unroll 1
    for (int c = 0; c < 128; c += 32) {
      uint32_t o[32];
      tmem_ld32(o_addr + c, o);
      tmem_ld_wait();
      if (live) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 u;
          u.x = pack_bf16x2(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
          u.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
          u.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
          u.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
          *reinterpret_cast<uint4*>(dst + c + e) = u;
        }
      }
    }
    if (live && lse != nullptr)
      lse[static_cast<int64_t>(h) * L + r] = (m_used + log2f(l)) * 0.69314718055994531f;
  } else {
    record_status(status, kStatusTimeout);
  }
}

__global__ void __launch_bounds__(WinMxCfg::THREADS, 1)
    window_attn_mx_kernel(const __grid_constant__ CUtensorMap qmap,
                          const __grid_constant__ CUtensorMap kmap,
                          const __grid_constant__ CUtensorMap vmap,
                          const uint8_t* __restrict__ qsc, const uint8_t* __restrict__ ksc,
                          const uint8_t* __restrict__ vsc,
                          const __grid_constant__ WinSched sched, int H, int L,
                          float scale_log2, __nv_bfloat16* __restrict__ out, int64_t ld_o,
                          float* __restrict__ lse, uint32_t* status, uint64_t budget_ns) {
  using Cfg = WinMxCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* qbuf = smem;                                 // Q0, Q1 codes
  uint8_t* pbuf = qbuf + 2 * Cfg::Q_TILE;               // P0, P1 codes
  uint8_t* kvbuf = pbuf + 2 * Cfg::P_TILE;              // stage s: K tile, V tile
  uint8_t* qsf = kvbuf + Cfg::STAGES * Cfg::STAGE;      // [2] scale blocks
  uint8_t* psf = qsf + 2 * Cfg::SF;                     // [2]
  uint8_t* ksf = psf + 2 * Cfg::SF;                     // [STAGES]
  uint8_t* vsf = ksf + Cfg::STAGES * Cfg::SF;           // [STAGES]
  uint64_t* bars = reinterpret_cast<uint64_t*>(vsf + Cfg::STAGES * Cfg::SF);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;                          // [STAGES]
  uint64_t* v_full = k_full + Cfg::STAGES;              // [STAGES]
  uint64_t* k_empty = v_full + Cfg::STAGES;             // [STAGES]
  uint64_t* v_empty = k_empty + Cfg::STAGES;            // [STAGES]
  uint64_t* s_full = v_empty + Cfg::STAGES;             // [2]
  uint64_t* s_free = s_full + 2;                        // [2], 4 warps
  uint64_t* p_ready = s_free + 2;                       // [2], 4 warps
  uint64_t* o_done = p_ready + 2;                       // [2]
  uint64_t* mma_done = o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int lin = blockIdx.x;
  const int h = lin / sched.total_tiles;
  const int tile = lin % sched.total_tiles;
  int si = 0;
  while (si + 1 < sched.nseg && tile >= sched.seg[si + 1].tile_base) ++si;
  const WinSeg& seg = sched.seg[si];
  const int q0 = seg.q0 + (tile - seg.tile_base) * 256;
  const int q_end = seg.q1;
  KvRange kr;
  kr.load(seg, 0);
  int nkv = 0;
  for (int iv = 0; iv < kr.nint; ++iv) nkv += (kr.end(iv) - kr.start(iv) + Cfg::KT - 1) / Cfg::KT;
  const uint32_t warp = warp_id();
  const int D = H * 128;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&p_ready[i], 4);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 96;\n" ::: "memory");
  }
  if (warp == 0) {
    // ================================================================ TMA and scales
    const uint32_t lane = lane_id();
    const bool leader = elect_one();
    // scale block of 128 rows of q or k (head h) starting at row r0: lane l
    // holds rows r0 + 32 c + l, c = 0..3, four block bytes each
    auto gather_rows = [&](const uint8_t* sc, int r0, int nrows, uint8_t* dst) {
      uint32_t w[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int r = r0 + 32 * c + static_cast<int>(lane);
        w[c] = (32 * c + static_cast<int>(lane) < nrows && r < L)
                   ? __ldg(reinterpret_cast<const uint32_t*>(sc + static_cast<int64_t>(r) * (D / 32) + 4 * h))
                   : 0x7F7F7F7Fu;
      }
      *reinterpret_cast<uint4*>(dst + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    };
    gather_rows(qsc, q0, 128, qsf);
    gather_rows(qsc, q0 + 128, 128, qsf + Cfg::SF);
    fence_proxy_async_smem();
    __syncwarp();
    if (leader) {
      mbar_arrive_expect_tx(q_full, 2 * Cfg::Q_TILE);
      tma_load_2d(qbuf, &qmap, q_full, h * 128, q0);
      tma_load_2d(qbuf + Cfg::Q_TILE, &qmap, q_full, h * 128, q0 + 128);
    }
    KvCursorT<Cfg::KT> cur;
    cur.init(kr);
    int issued = 0;
    const int vblocks = (L + 31) / 32;
    for (int j = 0; j < nkv; ++j) {
      const int s = j % Cfg::STAGES;
      const uint32_t par = ((j / Cfg::STAGES) & 1) ^ 1;
      uint8_t* kb = kvbuf + s * Cfg::STAGE;
      if (j >= Cfg::STAGES &&
          !__all_sync(0xffffffffu, mbar_wait(&k_empty[s], par, budget_ns))) {
        if (leader) record_status(status, kStatusTimeout);
        break;
      }
      // key scales: 96 keys, four d-blocks each (rows 96..127 unused)
      gather_rows(ksc, cur.pos, Cfg::KT, ksf + s * Cfg::SF);
      fence_proxy_async_smem();
      __syncwarp();
      if (leader) {
        mbar_arrive_expect_tx(&k_full[s], Cfg::K_TILE);
        tma_load_2d(kb, &kmap, &k_full[s], h * 128, cur.pos);
      }
      if (j >= Cfg::STAGES &&
          !__all_sync(0xffffffffu, mbar_wait(&v_empty[s], par, budget_ns))) {
        if (leader) record_status(status, kStatusTimeout);
        break;
      }
      // value scales: value column 32 c + lane of head h, key blocks 0..2
      {
        const int b0 = cur.pos / 32;
        uint32_t w[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint8_t* col = vsc + h * 128 + 32 * c + lane;
          uint32_t b[3];
#pragma unroll
          for (int kb2 = 0; kb2 < 3; ++kb2)
            b[kb2] = (b0 + kb2 < vblocks) ? __ldg(col + static_cast<int64_t>(b0 + kb2) * D) : 127u;
          w[c] = pack_sf3(b[0], b[1], b[2]);
        }
        *reinterpret_cast<uint4*>(vsf + s * Cfg::SF + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (leader) {
        mbar_arrive_expect_tx(&v_full[s], Cfg::V_TILE);
        tma_load_2d(kb + Cfg::K_TILE, &vmap, &v_full[s], h * 128, cur.pos);
      }
      ++issued;
      cur.next(kr);
    }
    if (leader) {
      mbar_wait(q_full, 0, 200000000ull);
      for (int j = (issued > Cfg::STAGES ? issued - Cfg::STAGES : 0); j < issued; ++j) {
        if (!mbar_wait(&k_full[j % Cfg::STAGES], (j / Cfg::STAGES) & 1, 200000000ull) ||
            !mbar_wait(&v_full[j % Cfg::STAGES], (j / Cfg::STAGES) & 1, 200000000ull))
          record_status(status, kStatusTimeout);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    if (elect_one()) {
      constexpr uint32_t idesc_s = idesc_mxf8(128, Cfg::KT);
      constexpr uint32_t idesc_o = idesc_mxf8_bmn(128, 128);
      const uint32_t qb = smem_u32(qbuf);
      const uint32_t pb = smem_u32(pbuf);
      // scale blocks: 32 rows x 16 bytes, 8-row groups 128 bytes apart
      auto cp_sf = [&](uint32_t col, const uint8_t* src) {
        tmem_cp_32x128b_x4(tmem + col, sdesc_none(smem_u32(src), 16, 128));
      };
      bool ok = mbar_wait(q_full, 0, budget_ns);
      if (ok) {
        tc_fence_after();
        cp_sf(Cfg::SFA_Q, qsf);
        cp_sf(Cfg::SFA_Q + 4, qsf + Cfg::SF);
      }
      // S_i = Q_i K^T over the tile's 96 keys: four K = 32 steps (head dim 128)
      auto issue_s = [&](int i, int j) {
        const int s = j % Cfg::STAGES;
        const uint32_t kb = smem_u32(kvbuf + s * Cfg::STAGE);
        const uint32_t sfa = tmem + Cfg::SFA_Q + 4 * i, sfb = tmem + Cfg::SFB_K + 4 * s;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const uint32_t id = idesc_s | (static_cast<uint32_t>(t) << 29) |
                              (static_cast<uint32_t>(t) << 4);
          umma_mx_ss(tmem + (i ? 128u : 0u), sdesc_sw128(qb + i * Cfg::Q_TILE + t * 32, 16, 1024),
                     sdesc_sw128(kb + t * 32, 16, 1024), id,
                     sfa | (static_cast<uint32_t>(t) << 30), sfb | (static_cast<uint32_t>(t) << 30),
                     t > 0);
        }
        umma_commit(&s_full[i]);
      };
      // O_i += P_i V over the tile's 96 keys: three K = 32 steps, V MN-major
      auto issue_o = [&](int i, int j) {
        const int s = j % Cfg::STAGES;
        const uint32_t vb = smem_u32(kvbuf + s * Cfg::STAGE + Cfg::K_TILE);
        const uint32_t sfa = tmem + Cfg::SFA_P + 4 * i, sfb = tmem + Cfg::SFB_V + 4 * s;
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          const uint32_t id = idesc_o | (static_cast<uint32_t>(t) << 29) |
                              (static_cast<uint32_t>(t) << 4);
          umma_mx_ss(tmem + Cfg::O_COL + 128 * i,
                     sdesc_sw128(pb + i * Cfg::P_TILE + t * 32, 16, 1024),
                     sdesc_sw128(vb + t * 4096, 16384, 1024), id,
                     sfa | (static_cast<uint32_t>(t) << 30), sfb | (static_cast<uint32_t>(t) << 30),
                     (j > 0 || t > 0));
        }
        umma_commit(&o_done[i]);
      };
      if (ok && (ok = mbar_wait(&k_full[0], 0, budget_ns))) {
        tc_fence_after();
        cp_sf(Cfg::SFB_K, ksf);
        issue_s(0, 0);
        issue_s(1, 0);
        umma_commit(&k_empty[0]);
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j % Cfg::STAGES;
        if (j + 1 < nkv) {
          const int sn = (j + 1) % Cfg::STAGES;
          if (!(ok = mbar_wait(&k_full[sn], ((j + 1) / Cfg::STAGES) & 1, budget_ns))) break;
          tc_fence_after();
          cp_sf(Cfg::SFB_K + 4 * sn, ksf + sn * Cfg::SF);
          if (!(ok = mbar_wait(&s_free[0], j & 1, budget_ns))) break;
          tc_fence_after();
          issue_s(0, j + 1);
          if (!(ok = mbar_wait(&s_free[1], j & 1, budget_ns))) break;
          tc_fence_after();
          issue_s(1, j + 1);
          umma_commit(&k_empty[sn]);
        }
        if (!(ok = mbar_wait(&v_full[s], (j / Cfg::STAGES) & 1, budget_ns))) break;
        tc_fence_after();
        cp_sf(Cfg::SFB_V + 4 * s, vsf + s * Cfg::SF);
        if (!(ok = mbar_wait(&p_ready[0], j & 1, budget_ns))) break;
        tc_fence_after();
        cp_sf(Cfg::SFA_P, psf);
        issue_o(0, j);
        if (!(ok = mbar_wait(&p_ready[1], j & 1, budget_ns))) break;
        tc_fence_after();
        cp_sf(Cfg::SFA_P + 4, psf + Cfg::SF);
        issue_o(1, j);
        umma_commit(&v_empty[s]);
      }
      if (!ok) record_status(status, kStatusTimeout);
      umma_commit(mma_done);
    }
  } else if (warp >= 4) {
    // ================================================================ softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 200;\n" ::: "memory");
    const int i = (warp - 4) >> 2;
    softmax_mx(i, tmem, s_full, s_free, p_ready, o_done, pbuf + i * Cfg::P_TILE,
               psf + i * Cfg::SF, kr, nkv, scale_log2, q0, q_end, h, H, L, out, ld_o, lse,
               status, budget_ns);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    mbar_wait(mma_done, 0, 200000000ull);
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- quantizers

// q and k: one thread per (row, 32-element block of the hidden columns);
// codes [R, D], scale bytes [R, D / 32].
__global__ void mx_quant_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t ld, int R, int D,
                                     uint8_t* __restrict__ q8, uint8_t* __restrict__ sc) {
  const int kblocks = D / 32;
  const int64_t total = static_cast<int64_t>(R) * kblocks;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = t / kblocks;
    const int kb = static_cast<int>(t % kblocks);
    const uint4* src = reinterpret_cast<const uint4*>(x + r * ld + 32 * kb);
    float v[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 u = __ldg(src + c);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack_bf16x2(w[e]);
        v[8 * c + 2 * e] = f.x;
        v[8 * c + 2 * e + 1] = f.y;
      }
    }
    uint4 codes[2];
    sc[r * kblocks + kb] = mx_quantize_block(v, codes);
    uint4* dst = reinterpret_cast<uint4*>(q8 + r * D + 32 * kb);
    dst[0] = codes[0];
    dst[1] = codes[1];
  }
}

// v: one thread per (32-row block, column); codes keep v's [R, D] layout,
// scale bytes [ceil(R / 32), D]; rows past R count as zeros.
__global__ void mx_quant_cols_kernel(const __nv_bfloat16* __restrict__ x, int64_t ld, int R, int D,
                                     uint8_t* __restrict__ v8, uint8_t* __restrict__ sc) {
  const int rblocks = (R + 31) / 32;
  const int64_t total = static_cast<int64_t>(rblocks) * D;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t rb = t / D;
    const int c = static_cast<int>(t % D);
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int64_t r = 32 * rb + e;
      v[e] = r < R ? __bfloat162float(x[r * ld + c]) : 0.f;
    }
    uint4 codes[2];
    sc[rb * D + c] = mx_quantize_block(v, codes);
    const uint32_t w[8] = {codes[0].x, codes[0].y, codes[0].z, codes[0].w,
                           codes[1].x, codes[1].y, codes[1].z, codes[1].w};
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int64_t r = 32 * rb + e;
      if (r < R) v8[r * D + c] = static_cast<uint8_t>(w[e >> 2] >> (8 * (e & 3)));
    }
  }
}

int quant_blocks(int64_t total) {
  const int64_t want = (total + 255) / 256;
  return static_cast<int>(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace: [status][q8][k8][v8][q scales][k scales][v scales].
struct MxPlan {
  size_t codes, rsc, vsc, q8, k8, v8, qs, ks, vs, total;
};

MxPlan mx_plan(const vdn_shape& s) {
  MxPlan p;
  const size_t L = static_cast<size_t>(s.T) * s.N, D = static_cast<size_t>(s.H) * s.d;
  p.codes = round256(L * D);
  p.rsc = round256(L * (D / 32));
  p.vsc = round256((L + 31) / 32 * D);
  p.q8 = kStatusBytes;
  p.k8 = p.q8 + p.codes;
  p.v8 = p.k8 + p.codes;
  p.qs = p.v8 + p.codes;
  p.ks = p.qs + p.rsc;
  p.vs = p.ks + p.rsc;
  p.total = p.vs + p.vsc;
  return p;
}

}  // namespace
}  // namespace vdn

using namespace vdn;

extern "C" {

size_t vdn_window_attn_mxfp8_workspace(const vdn_shape* shape) {
  if (shape == nullptr || shape->T < 1 || shape->N < 1 || shape->H < 1 || shape->d < 1) return 0;
  return mx_plan(*shape).total;
}

vdn_status vdn_window_attn_mxfp8(const vdn_shape* shape, const void* q, const void* k,
                                 const void* v, int64_t ld, int chunk_frames, int window_chunks,
                                 unsigned anchors, float scale, void* o, int64_t ld_o,
                                 float* lse_opt, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("vdn_window_attn_mxfp8");
  if (shape == nullptr || shape->T < 1 || shape->N < 1 || shape->H < 1 || shape->d < 1)
    return VDN_ERR_INVALID_ARG;
  const vdn_shape s = *shape;
  if (static_cast<int64_t>(s.T) * s.N >= (int64_t(1) << 31) - 512) return VDN_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return VDN_ERR_INVALID_ARG;
  const auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(q) || !a16(k) || !a16(v) || !a16(o) ||
      (lse_opt && (reinterpret_cast<uintptr_t>(lse_opt) & 3u)))
    return VDN_ERR_INVALID_ARG;
  if (chunk_frames < 1 || window_chunks < 0 || anchors > 3u) return VDN_ERR_INVALID_ARG;
  // head dim 128; key intervals (whole frames) on 32-token block boundaries
  if (s.d != 128 || s.N % 32 != 0) return VDN_ERR_UNSUPPORTED;
  const int64_t D = static_cast<int64_t>(s.H) * s.d;
  if (ld < D || ld % 8 || ld_o < D || ld_o % 8) return VDN_ERR_INVALID_ARG;
  const MxPlan pl = mx_plan(s);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < pl.total)
    return VDN_ERR_WORKSPACE;
  thread_local WinSched sched;
  if (!build_schedule(s, chunk_frames, window_chunks, anchors, &sched)) return VDN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(sched.total_tiles) * s.H >= (int64_t(1) << 31))
    return VDN_ERR_UNSUPPORTED;
  const int L = s.T * s.N;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t *q8 = base + pl.q8, *k8 = base + pl.k8, *v8 = base + pl.v8;
  uint8_t *qs = base + pl.qs, *ks = base + pl.ks, *vs = base + pl.vs;
  CUtensorMap qmap, kmap, vmap;
  if (!make_rows_map_u8(&qmap, q8, D, D, L, 128) || !make_rows_map_u8(&kmap, k8, D, D, L, WinMxCfg::KT) ||
      !make_rows_map_u8(&vmap, v8, D, D, L, WinMxCfg::KT))
    return VDN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t rows_total = static_cast<int64_t>(L) * (D / 32);
  mx_quant_rows_kernel<<<quant_blocks(rows_total), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(q), ld, L, static_cast<int>(D), q8, qs);
  mx_quant_rows_kernel<<<quant_blocks(rows_total), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(k), ld, L, static_cast<int>(D), k8, ks);
  mx_quant_cols_kernel<<<quant_blocks(static_cast<int64_t>((L + 31) / 32) * D), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(v), ld, L, static_cast<int>(D), v8, vs);
  if (cudaGetLastError() != cudaSuccess) return VDN_ERR_CUDA;
  static std::atomic<uint64_t> smem_set{0};
  if (set_smem_once(window_attn_mx_kernel, WinMxCfg::SMEM, smem_set) != cudaSuccess)
    return VDN_ERR_CUDA;
  const float sc = scale > 0.f ? scale : 1.f / sqrtf(static_cast<float>(s.d));
  window_attn_mx_kernel<<<sched.total_tiles * s.H, WinMxCfg::THREADS, WinMxCfg::SMEM, st>>>(
      qmap, kmap, vmap, qs, ks, vs, sched, s.H, L, sc * 1.4426950408889634f,
      static_cast<__nv_bfloat16*>(o), ld_o, lse_opt, static_cast<uint32_t*>(ws),
      current_wait_budget_ns());
  return cudaGetLastError() == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

}  // extern "C"
