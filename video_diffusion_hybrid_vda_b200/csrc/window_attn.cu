// Window-and-anchor Softmax attention ("Video DeltaNet", 10100.com article,
// 方法概述 item 1): latent frames form chunks of `chunk_frames`; a query frame
// attends to the frames of its own chunk and `window_chunks` chunks on each
// side, plus the anchor frames 0 and T-1, and the anchor frames attend to
// every frame.  All spatial tokens of a frame share its mask.
//
// Schedule (host): consecutive query frames with the same visible key set
// form a segment; a segment's keys are at most three contiguous token
// intervals (the window, frame 0, frame T-1).  Every CTA takes 256 query rows
// (two 128-row tiles) of one segment and one head and loops over the
// segment's key tiles (128 keys; the last tile of an interval is masked by
// column).  CTAs are ordered heaviest segment first so the long anchor rows
// start early.
//
// Kernel (sm_100a, one CTA per SM):
//   warp 0      TMA: Q0/Q1 once, then K and V tiles through a 2-stage ring
//               (K and V slots released separately)
//   warp 1      tcgen05.mma issue: S_i = Q_i K^T into TMEM, O_i += P_i V with
//               P_i read from TMEM (the A operand) and V MN-major in smem
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: one thread
//               per query row; online max/sum in the exp2 domain, P written
//               back over S as packed bf16; O rescaled in TMEM only when the
//               running max grows by more than 2^8 (lazy rescale)
// TMEM: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512) columns.
// The two softmax groups alternate with the tensor core: while one converts
// S_i to P_i, the MMA warp runs the other tile's products.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "common.cuh"
#include "exp2_fma.cuh"
#include "ptx.cuh"
#include "repack.cuh"
#include "window_sched.cuh"

namespace vdn {

namespace {


// P is stored in four 32-key chunks; the PV product of the first this-many
// chunks is issued as soon as they are stored, the rest once the row is done.
#ifndef VDN_P_EARLY_CHUNKS
#define VDN_P_EARLY_CHUNKS 2
#endif
static_assert(VDN_P_EARLY_CHUNKS >= 1 && VDN_P_EARLY_CHUNKS <= 3, "1..3 of the 4 chunks");

// Head dim 128 runs on the CTA-pair kernel (2-SM MMAs) unless this is 0,
// which selects the one-CTA kernel (kept for head dim 64 and comparisons).
#ifndef VDN_WINDOW_PAIR
#define VDN_WINDOW_PAIR 1
#endif

// Of every 16 score pairs in a 32-column chunk, this many take the FMA-pipe
// exponential and the rest the MUFU (measured on B200: see profiles/).
#ifndef VDN_EXP2_FMA_PAIRS
#define VDN_EXP2_FMA_PAIRS 0
#endif
static_assert(VDN_EXP2_FMA_PAIRS == 0 || VDN_EXP2_FMA_PAIRS == 2 || VDN_EXP2_FMA_PAIRS == 4 ||
                  VDN_EXP2_FMA_PAIRS == 8,
              "VDN_EXP2_FMA_PAIRS must divide 16 pairs evenly");

template <int DH>
struct WinCfg {
  static constexpr int SLABS = DH / 64;
  static constexpr int TILE_BYTES = SLABS * 128 * 128;  // 128 rows x DH bf16
  static constexpr int STAGES = 2;
  static constexpr int THREADS = 384;
  static constexpr int SMEM = 1024 + 2 * TILE_BYTES + STAGES * 2 * TILE_BYTES + 512;
};

// One softmax warpgroup (tile i of the CTA's two 128-row query tiles): one
// thread per query row.  For every key tile it waits for S_i, takes the row
// max, rescales O_i in TMEM when the max grew by more than 2^8 (warp-uniform
// decision), writes P = 2^(s - m) over S as bf16 in two halves (reporting
// each half through arrive_half / arrive_ready), and at the end normalises
// O_i by the row sum and stores the row (and its log-sum-exp).
//
// P_SMEM: P goes to this warpgroup's tile `pbuf` in shared memory (bf16,
// K-major, 128-byte swizzle, two 64-key slabs) instead of back over S in
// TMEM, so S_i is free once it has been loaded (reported through s_free)
// and the next S_i product overlaps this tile's exponentials; before writing
// P the warpgroup waits for the previous tile's PV product (it reads pbuf).
template <int DH, bool P_SMEM, class ArriveHalf, class ArriveReady, class SFree>
__device__ __forceinline__ void softmax_warpgroup(
    int i, uint32_t tmem, uint64_t* s_full, uint64_t* o_done, ArriveHalf arrive_half,
    ArriveReady arrive_ready, SFree s_free, uint8_t* pbuf, const KvRange& kr, int nkv,
    float scale_log2, int q0, int q_end, int h, int H, int L, __nv_bfloat16* __restrict__ out,
    int64_t ld_o, float* __restrict__ lse, uint32_t* status, uint64_t budget_ns) {
  const uint32_t quarter = warp_id() & 3;
  const int row = quarter * 32 + lane_id();
  const uint32_t lane_off = (quarter * 32) << 16;
  const uint32_t s_addr = tmem + 128 * i + lane_off;
  const uint32_t o_addr = tmem + 256 + 128 * i + lane_off;
  float m_used = -INFINITY;  // running max, log2 domain (scaled)
  float l = 0.f;
  KvCursor cur;
  cur.init(kr);
  bool ok = true;
  for (int j = 0; j < nkv; ++j) {
    const int valid = cur.valid();
    cur.next(kr);
    // warp-uniform decision: tcgen05.ld/st below are warp-collective
    if (!__all_sync(0xffffffffu, mbar_wait(&s_full[i], j & 1, budget_ns))) {
      ok = false;
      break;
    }
    tc_fence_after();
    uint32_t sr[128];
    uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
    uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
    uint32_t (&s2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[64]);
    uint32_t (&s3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[96]);
    // first half of the row, then start loading the second half while the
    // first half's max is taken
    tmem_ld32(s_addr, s0);
    tmem_ld32(s_addr + 32, s1);
    tmem_ld_wait();
    reg_fence(s0);
    reg_fence(s1);
    tmem_ld32(s_addr + 64, s2);
    tmem_ld32(s_addr + 96, s3);
    if (valid < 64) {
#pragma unroll
      for (int c = 0; c < 64; ++c)
        if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
    }
    // row max over eight running maxima, two scores per three-input max
    auto sv = [&](int c) { return __uint_as_float(sr[c]); };
    float mx8[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) mx8[a] = fmax3(sv(a), sv(a + 8), sv(a + 16));
#pragma unroll
    for (int c = 24; c < 56; c += 16)
#pragma unroll
      for (int a = 0; a < 8; ++a) mx8[a] = fmax3(mx8[a], sv(c + a), sv(c + 8 + a));
#pragma unroll
    for (int a = 0; a < 8; ++a) mx8[a] = fmaxf(mx8[a], sv(56 + a));
    tmem_ld_wait();
    reg_fence(s2);
    reg_fence(s3);
    if constexpr (P_SMEM) {
      tc_fence_before();
      s_free();  // all of S_i is in registers: the next S_i may overwrite it
    }
    if (valid < 128) {
#pragma unroll
      for (int c = 64; c < 128; ++c)
        if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
    }
#pragma unroll
    for (int c = 64; c < 128; c += 16)
#pragma unroll
      for (int a = 0; a < 8; ++a) mx8[a] = fmax3(mx8[a], sv(c + a), sv(c + 8 + a));
    const float mt = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                           fmaxf(mx8[6], mx8[7])) *
                     scale_log2;
    // Lazy rescale: only when some row's max grew by more than 2^8.  The
    // decision is taken per warp (the O accesses are warp-collective); rows
    // of a rescaling warp move to max(m_used, mt), a factor of 1 for rows
    // whose max did not grow.
    if (__any_sync(0xffffffffu, mt > m_used + 8.f)) {
      const float m_new = fmaxf(m_used, mt);
      const float factor = exp2_mufu(m_used - m_new);  // 0 on the first tile
      l *= factor;
      if (j > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(&o_done[i], (j - 1) & 1, budget_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < DH; c += 32) {
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
    // p = 2^(s * scale_log2 - m) with the argument by packed f32x2 FMA and
    // four packed partial sums; one pair in four takes the FMA-pipe
    // exponential, the rest the MUFU.  P goes back over S as bf16 in two
    // halves, so the PV product can start on keys 0..63.
    const uint64_t cc = f32x2_pack(scale_log2, scale_log2);
    const uint64_t nm = f32x2_pack(-m_used, -m_used);
    uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
    // P_SMEM: the row's 128 probabilities stay in registers (64 packed
    // words, reusing the scores' registers as they die) until the previous
    // tile's PV product has read pbuf, which is waited for only after the
    // exponentials
    uint32_t pall[P_SMEM ? 64 : 1];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const uint64_t xs = f32x2_fma(
            (static_cast<uint64_t>(sr[32 * q + 2 * e + 1]) << 32) | sr[32 * q + 2 * e], cc, nm);
        uint64_t pp;
        if (VDN_EXP2_FMA_PAIRS > 0 &&
            (e % (16 / (VDN_EXP2_FMA_PAIRS > 0 ? VDN_EXP2_FMA_PAIRS : 1))) ==
                (16 / (VDN_EXP2_FMA_PAIRS > 0 ? VDN_EXP2_FMA_PAIRS : 1)) - 1) {
          pp = exp2_fma_x2(xs);
        } else {
          pp = f32x2_pack(exp2_mufu(f32x2_lo(xs)), exp2_mufu(f32x2_hi(xs)));
        }
        acc2[e & 3] = f32x2_add(acc2[e & 3], pp);
        pk[e] = pack_bf16x2(f32x2_lo(pp), f32x2_hi(pp));
      }
      if constexpr (P_SMEM) {
#pragma unroll
        for (int e = 0; e < 16; ++e) pall[16 * q + e] = pk[e];
      } else {
        tmem_st16(s_addr + 16 * q, pk);
        if (q == VDN_P_EARLY_CHUNKS - 1) {
          tmem_st_wait();
          tc_fence_before();
          arrive_half();
        }
      }
    }
    acc2[0] = f32x2_add(f32x2_add(acc2[0], acc2[1]), f32x2_add(acc2[2], acc2[3]));
    l += f32x2_lo(acc2[0]) + f32x2_hi(acc2[0]);
    if constexpr (P_SMEM) {
      // pbuf is read by the previous tile's PV product
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(&o_done[i], (j - 1) & 1, budget_ns))) {
        ok = false;
        break;
      }
      // keys 32q .. 32q+31 of this row: four 16-byte chunks of slab q / 2
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint8_t* slab = pbuf + (q >> 1) * 16384 + row * 128;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t c = 4 * (q & 1) + m;
          *reinterpret_cast<uint4*>(slab + ((c ^ (row & 7)) << 4)) =
              make_uint4(pall[16 * q + 4 * m], pall[16 * q + 4 * m + 1],
                         pall[16 * q + 4 * m + 2], pall[16 * q + 4 * m + 3]);
        }
      }
      fence_proxy_async_smem();  // the tensor core reads pbuf through the async proxy
    } else {
      tmem_st_wait();
      tc_fence_before();
    }
    arrive_ready();
  }
  // ------------------------------------------------------------ epilogue
  if (__all_sync(0xffffffffu, ok && mbar_wait(&o_done[i], (nkv - 1) & 1, budget_ns))) {
    tc_fence_after();
    const int r = q0 + 128 * i + row;
    // rows past the segment are not stored; a stored row lies in [0, L) and
    // its head's columns in [0, H d) (checked in debug builds)
    const bool live = r < q_end && in_bounds(status, r, L, static_cast<int64_t>(h) * DH, DH,
                                             static_cast<int64_t>(H) * DH);
    const float inv = 1.f / l;
    __nv_bfloat16* dst = out + static_cast<int64_t>(r) * ld_o + h * DH;
#pragma unroll 1
    for (int c = 0; c < DH; c += 32) {
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

template <int DH>
__global__ void __launch_bounds__(WinCfg<DH>::THREADS, 1)
    window_attn_kernel(const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap,
                       const __grid_constant__ CUtensorMap ckmap,
                       const __grid_constant__ CUtensorMap cvmap, int m_ctx,
                       const __grid_constant__ WinSched sched, int H, int L, float scale_log2,
                       __nv_bfloat16* __restrict__ out, int64_t ld_o, float* __restrict__ lse,
                       uint32_t* status, uint64_t budget_ns) {
  using Cfg = WinCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* qbuf = smem;                              // Q0, Q1
  uint8_t* kvbuf = smem + 2 * Cfg::TILE_BYTES;       // stage s: K then V
  uint64_t* bars = reinterpret_cast<uint64_t*>(kvbuf + Cfg::STAGES * 2 * Cfg::TILE_BYTES);
  uint64_t* q_full = bars;
  // K and V of a stage have their own barriers: K is free once both S
  // products of its tile are done, half a period before V (free after both
  // PV products), so the next K load starts that much earlier
  uint64_t* k_full = bars + 1;                       // [STAGES]
  uint64_t* v_full = k_full + Cfg::STAGES;           // [STAGES]
  uint64_t* k_empty = v_full + Cfg::STAGES;          // [STAGES]
  uint64_t* v_empty = k_empty + Cfg::STAGES;         // [STAGES]
  uint64_t* s_full = v_empty + Cfg::STAGES;          // [2]
  uint64_t* p_half = s_full + 2;                     // [2] P for keys 0..63 stored
  uint64_t* p_ready = p_half + 2;                    // [2] all of P stored
  uint64_t* o_done = p_ready + 2;                    // [2]
  uint64_t* mma_done = o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  // ---- which segment / tile / head
  // head-major launch order: the CTAs resident at any time mostly share one
  // head, so the K/V rows they stream stay in L2 across query tiles
  const int lin = blockIdx.x;
  const int h = lin / sched.total_tiles;
  const int tile = lin % sched.total_tiles;
  int si = 0;
  while (si + 1 < sched.nseg && tile >= sched.seg[si + 1].tile_base) ++si;
  const WinSeg& seg = sched.seg[si];
  const int q0 = seg.q0 + (tile - seg.tile_base) * 256;
  const int q_end = seg.q1;
  const int nkv = seg.nkv + (m_ctx + 127) / 128;
  KvRange kr;
  kr.load(seg, m_ctx);
  const uint32_t warp = warp_id();

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
      mbar_init(&p_half[i], 128);
      mbar_init(&p_ready[i], 128);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
    if (m_ctx > 0) {
      tma_prefetch_desc(&ckmap);
      tma_prefetch_desc(&cvmap);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Register split (launched with 168 x 384 = 64512): the TMA/MMA warpgroup
  // drops to 96, the two softmax warpgroups rise to 200
  // (128 * 96 + 256 * 200 = 63488 <= 64512).
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 96;\n" ::: "memory");
  }
  if (warp == 0) {
    // ================================================================ TMA
    if (elect_one()) {
      mbar_arrive_expect_tx(q_full, 2 * Cfg::TILE_BYTES);
      for (int i = 0; i < 2; ++i)
        for (int sl = 0; sl < Cfg::SLABS; ++sl)
          tma_load_2d(qbuf + i * Cfg::TILE_BYTES + sl * 16384, &qmap, q_full, h * DH + 64 * sl,
                      q0 + 128 * i);
      KvCursor cur;
      cur.init(kr);
      int k_issued = 0, v_issued = 0;
      // K(j) waits for the S products of tile j - STAGES, V(j) for its PV
      // products; the MMA warp retires them in that order
      for (int j = 0; j < nkv; ++j) {
        const int s = j % Cfg::STAGES;
        const uint32_t par = ((j / Cfg::STAGES) & 1) ^ 1;
        uint8_t* kb = kvbuf + s * 2 * Cfg::TILE_BYTES;
        const CUtensorMap* km = cur.ctx ? &ckmap : &kmap;
        const CUtensorMap* vm = cur.ctx ? &cvmap : &vmap;
        if (j >= Cfg::STAGES && !mbar_wait(&k_empty[s], par, budget_ns)) {
          record_status(status, kStatusTimeout);
          break;
        }
        mbar_arrive_expect_tx(&k_full[s], Cfg::TILE_BYTES);
        for (int sl = 0; sl < Cfg::SLABS; ++sl)
          tma_load_2d(kb + sl * 16384, km, &k_full[s], h * DH + 64 * sl, cur.pos);
        ++k_issued;
        if (j >= Cfg::STAGES && !mbar_wait(&v_empty[s], par, budget_ns)) {
          record_status(status, kStatusTimeout);
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], Cfg::TILE_BYTES);
        for (int sl = 0; sl < Cfg::SLABS; ++sl)
          tma_load_2d(kb + Cfg::TILE_BYTES + sl * 16384, vm, &v_full[s], h * DH + 64 * sl,
                      cur.pos);
        ++v_issued;
        cur.next(kr);
      }
      // drain loads still in flight
      mbar_wait(q_full, 0, 200000000ull);
      for (int j = (k_issued > Cfg::STAGES ? k_issued - Cfg::STAGES : 0); j < k_issued; ++j)
        if (!mbar_wait(&k_full[j % Cfg::STAGES], (j / Cfg::STAGES) & 1, 200000000ull))
          record_status(status, kStatusTimeout);
      for (int j = (v_issued > Cfg::STAGES ? v_issued - Cfg::STAGES : 0); j < v_issued; ++j)
        if (!mbar_wait(&v_full[j % Cfg::STAGES], (j / Cfg::STAGES) & 1, 200000000ull))
          record_status(status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    if (elect_one()) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(128, DH, false, true);
      const uint32_t qb = smem_u32(qbuf);
      bool ok = mbar_wait(q_full, 0, budget_ns);
      auto issue_s = [&](int i, int j) {
        const uint32_t kb = smem_u32(kvbuf + (j % Cfg::STAGES) * 2 * Cfg::TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tmem + 128 * i, sdesc_sw128(qb + i * Cfg::TILE_BYTES + off, 16, 1024),
                  sdesc_sw128(kb + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(&s_full[i]);
      };
      // O_i += P_i V for keys [16 k0, 16 k1) of the tile
      auto issue_o = [&](int i, int j, int k0, int k1) {
        const uint32_t vb =
            smem_u32(kvbuf + (j % Cfg::STAGES) * 2 * Cfg::TILE_BYTES + Cfg::TILE_BYTES);
        for (int kk = k0; kk < k1; ++kk)
          umma_ts(tmem + 256 + 128 * i, tmem + 128 * i + kk * 8,
                  sdesc_sw128(vb + kk * 2048, 16384, 1024), idesc_o, (j > 0 || kk > 0));
      };
      if (ok && (ok = mbar_wait(&k_full[0], 0, budget_ns))) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        umma_commit(&k_empty[0]);
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j % Cfg::STAGES;
        const bool more = j + 1 < nkv;
        if (!(ok = mbar_wait(&v_full[s], (j / Cfg::STAGES) & 1, budget_ns))) break;
        if (!(ok = mbar_wait(&p_half[0], j & 1, budget_ns))) break;
        tc_fence_after();
        issue_o(0, j, 0, 2 * VDN_P_EARLY_CHUNKS);
        if (!(ok = mbar_wait(&p_ready[0], j & 1, budget_ns))) break;
        tc_fence_after();
        issue_o(0, j, 2 * VDN_P_EARLY_CHUNKS, 8);
        umma_commit(&o_done[0]);
        if (more) {
          const int sn = (j + 1) % Cfg::STAGES;
          if (!(ok = mbar_wait(&k_full[sn], ((j + 1) / Cfg::STAGES) & 1, budget_ns))) break;
          tc_fence_after();
          issue_s(0, j + 1);
        }
        if (!(ok = mbar_wait(&p_half[1], j & 1, budget_ns))) break;
        tc_fence_after();
        issue_o(1, j, 0, 2 * VDN_P_EARLY_CHUNKS);
        if (!(ok = mbar_wait(&p_ready[1], j & 1, budget_ns))) break;
        tc_fence_after();
        issue_o(1, j, 2 * VDN_P_EARLY_CHUNKS, 8);
        umma_commit(&o_done[1]);
        umma_commit(&v_empty[s]);
        if (more) {
          issue_s(1, j + 1);
          umma_commit(&k_empty[(j + 1) % Cfg::STAGES]);
        }
      }
      if (!ok) record_status(status, kStatusTimeout);
      umma_commit(mma_done);
    }
  } else if (warp >= 4) {
    // ================================================================ softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 200;\n" ::: "memory");
    const int i = (warp - 4) >> 2;  // query tile of this warpgroup
    softmax_warpgroup<DH, false>(
        i, tmem, s_full, o_done, [&] { mbar_arrive(&p_half[i]); },
        [&] { mbar_arrive(&p_ready[i]); }, [] {}, nullptr, kr, nkv, scale_log2, q0, q_end, h, H,
        L, out, ld_o, lse, status, budget_ns);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    mbar_wait(mma_done, 0, 200000000ull);
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- CTA-pair kernel
//
// Head dim 128 on the 2-SM MMA.  A cluster of two CTAs takes 512 query rows
// of one segment and head (256 each: two 128-row tiles per CTA, as above).
// S_i = Q_i K^T and O_i += P_i V are issued by the even CTA (the leader) as
// cta_group::2 MMAs of M = 256: rows 0..127 are the leader's tile i, rows
// 128..255 the odd CTA's, and each CTA receives its own rows in its own TMEM
// (the same S0 S1 O0 O1 columns as the one-CTA kernel).  B is split between
// the pair by N: per key tile the leader holds keys 0..63 and the odd CTA keys
// 64..127 (all head dims) for S, and for PV the leader holds V columns 0..63
// and the odd CTA columns 64..127 (all 128 keys).  Each CTA therefore loads
// 32 KB per key tile instead of 64 KB, and each MMA reads its A rows and half
// of B from each SM's shared memory: 6 KB per K = 16 step of S instead of
// 8 KB, 2 KB per step of PV instead of 4 KB.
//
// Synchronisation: every TMA load of both CTAs completes on the leader's
// full barriers (cta_group::2 loads, no multicast); the leader's MMA commits
// arrive on both CTAs' barriers (S ready, O done, stage free, all done); the
// softmax warps of both CTAs report P to the leader's barriers, one arrival
// per warp.  Both CTAs initialise all barriers and meet at a cluster barrier
// before the first load, and again before TMEM is released and they exit, so
// neither leaves while the other may still touch its barriers or memory.
template <int DH>
struct WinPairCfg {
  static_assert(DH == 128, "the pair kernel serves head dim 128");
  static constexpr int SLABS = DH / 64;                 // 64-column slabs of a row
  static constexpr int Q_TILE = SLABS * 128 * 128;      // 128 query rows x DH bf16
  static constexpr int K_HALF = SLABS * 64 * 128;       // 64 keys x DH bf16
  static constexpr int V_HALF = 128 * 128;              // 128 keys x 64 columns bf16
  static constexpr int STAGE = K_HALF + V_HALF;
  static constexpr int STAGES = 4;
  static constexpr int THREADS = 384;
  static constexpr int SMEM = 1024 + 2 * Q_TILE + STAGES * STAGE + 512;
};

template <int DH>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(WinPairCfg<DH>::THREADS, 1)
    window_attn_pair_kernel(const __grid_constant__ CUtensorMap qmap,
                            const __grid_constant__ CUtensorMap kmap,
                            const __grid_constant__ CUtensorMap vmap,
                            const __grid_constant__ CUtensorMap ckmap,
                            const __grid_constant__ CUtensorMap cvmap, int m_ctx,
                            const __grid_constant__ WinSched sched, int H, int L,
                            float scale_log2, __nv_bfloat16* __restrict__ out, int64_t ld_o,
                            float* __restrict__ lse, uint32_t* status, uint64_t budget_ns) {
  using Cfg = WinPairCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* qbuf = smem;                              // Q0, Q1 of this CTA
  uint8_t* kvbuf = smem + 2 * Cfg::Q_TILE;           // stage s: K half, then V half
  uint64_t* bars = reinterpret_cast<uint64_t*>(kvbuf + Cfg::STAGES * Cfg::STAGE);
  uint64_t* q_full = bars;                           // leader: Q of both CTAs
  uint64_t* k_full = bars + 1;                       // leader: [STAGES] both K halves
  uint64_t* v_full = k_full + Cfg::STAGES;           // leader: [STAGES] both V halves
  uint64_t* k_empty = v_full + Cfg::STAGES;          // both: [STAGES]
  uint64_t* v_empty = k_empty + Cfg::STAGES;         // both: [STAGES]
  uint64_t* s_full = v_empty + Cfg::STAGES;          // both: [2]
  uint64_t* p_half = s_full + 2;                     // leader: [2], 8 warps
  uint64_t* p_ready = p_half + 2;                    // leader: [2], 8 warps
  uint64_t* o_done = p_ready + 2;                    // both: [2]
  uint64_t* mma_done = o_done + 2;                   // both
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const uint32_t rank = cluster_ctarank();           // 0: leader, 1: its partner
  const int pair_lin = blockIdx.x >> 1;
  const int h = pair_lin / sched.total_pairs;
  const int pair = pair_lin % sched.total_pairs;
  int si = 0;
  while (si + 1 < sched.nseg && pair >= sched.seg[si + 1].pair_base) ++si;
  const WinSeg& seg = sched.seg[si];
  // rows past the segment (the odd CTA of a segment's last pair may have
  // none) are computed but never stored
  const int q0 = seg.q0 + (pair - seg.pair_base) * 512 + static_cast<int>(rank) * 256;
  const int q_end = seg.q1;
  const int nkv = seg.nkv + (m_ctx + 127) / 128;
  KvRange kr;
  kr.load(seg, m_ctx);
  const uint32_t warp = warp_id();

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
      mbar_init(&p_half[i], 8);
      mbar_init(&p_ready[i], 8);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
    if (m_ctx > 0) {
      tma_prefetch_desc(&ckmap);
      tma_prefetch_desc(&cvmap);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any load or remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 96;\n" ::: "memory");
  }
  if (warp == 0) {
    // ================================================================ TMA (both CTAs)
    if (elect_one()) {
      const uint32_t lq_full = mapa_shared(smem_u32(q_full), 0);
      if (rank == 0) mbar_arrive_expect_tx(q_full, 4 * Cfg::Q_TILE);
      for (int i = 0; i < 2; ++i)
        for (int sl = 0; sl < Cfg::SLABS; ++sl)
          tma_load_2d_pair(qbuf + i * Cfg::Q_TILE + sl * 16384, &qmap, lq_full,
                           h * DH + 64 * sl, q0 + 128 * i);
      KvCursor cur;
      cur.init(kr);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int s = j % Cfg::STAGES;
        const uint32_t par = ((j / Cfg::STAGES) & 1) ^ 1;
        uint8_t* kb = kvbuf + s * Cfg::STAGE;
        const CUtensorMap* km = cur.ctx ? &ckmap : &kmap;
        const CUtensorMap* vm = cur.ctx ? &cvmap : &vmap;
        if (j >= Cfg::STAGES && !mbar_wait(&k_empty[s], par, budget_ns)) {
          record_status(status, kStatusTimeout);
          break;
        }
        // this CTA's 64 keys of the tile, every head-dim slab
        if (rank == 0) mbar_arrive_expect_tx(&k_full[s], 2 * Cfg::K_HALF);
        for (int sl = 0; sl < Cfg::SLABS; ++sl)
          tma_load_2d_pair(kb + sl * 8192, km, mapa_shared(smem_u32(&k_full[s]), 0),
                           h * DH + 64 * sl, cur.pos + 64 * static_cast<int>(rank));
        if (j >= Cfg::STAGES && !mbar_wait(&v_empty[s], par, budget_ns)) {
          record_status(status, kStatusTimeout);
          break;
        }
        // all 128 keys of the tile, this CTA's 64 value columns
        if (rank == 0) mbar_arrive_expect_tx(&v_full[s], 2 * Cfg::V_HALF);
        tma_load_2d_pair(kb + Cfg::K_HALF, vm, mapa_shared(smem_u32(&v_full[s]), 0),
                         h * DH + 64 * static_cast<int>(rank), cur.pos);
        ++issued;
        cur.next(kr);
      }
      // the leader's full barriers count both CTAs' bytes: wait for the last
      // phases so that no load is in flight when the pair exits
      if (rank == 0) {
        mbar_wait(q_full, 0, 200000000ull);
        for (int j = (issued > Cfg::STAGES ? issued - Cfg::STAGES : 0); j < issued; ++j) {
          if (!mbar_wait(&k_full[j % Cfg::STAGES], (j / Cfg::STAGES) & 1, 200000000ull) ||
              !mbar_wait(&v_full[j % Cfg::STAGES], (j / Cfg::STAGES) & 1, 200000000ull))
            record_status(status, kStatusTimeout);
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA (leader)
    if (rank == 0 && elect_one()) {
      constexpr uint32_t idesc_s = idesc_bf16(256, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(256, DH, false, true);
      constexpr uint16_t kBoth = 3;
      const uint32_t qb = smem_u32(qbuf);
      bool ok = mbar_wait(q_full, 0, budget_ns);
      auto issue_s = [&](int i, int j) {
        const uint32_t kb = smem_u32(kvbuf + (j % Cfg::STAGES) * Cfg::STAGE);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t qoff = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
          umma_ss_pair(tmem + 128 * i, sdesc_sw128(qb + i * Cfg::Q_TILE + qoff, 16, 1024),
                       sdesc_sw128(kb + koff, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit_pair(&s_full[i], kBoth);
      };
      // O_i += P_i V for keys [16 k0, 16 k1) of the tile
      auto issue_o = [&](int i, int j, int k0, int k1) {
        const uint32_t vb = smem_u32(kvbuf + (j % Cfg::STAGES) * Cfg::STAGE + Cfg::K_HALF);
        for (int kk = k0; kk < k1; ++kk)
          umma_ts_pair(tmem + 256 + 128 * i, tmem + 128 * i + kk * 8,
                       sdesc_sw128(vb + kk * 2048, 16384, 1024), idesc_o, (j > 0 || kk > 0));
      };
      if (ok && (ok = mbar_wait(&k_full[0], 0, budget_ns))) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        umma_commit_pair(&k_empty[0], kBoth);
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j % Cfg::STAGES;
        const bool more = j + 1 < nkv;
        if (!(ok = mbar_wait(&v_full[s], (j / Cfg::STAGES) & 1, budget_ns))) break;
        if (!(ok = mbar_wait(&p_half[0], j & 1, budget_ns))) break;
        tc_fence_after();
        issue_o(0, j, 0, 2 * VDN_P_EARLY_CHUNKS);
        if (!(ok = mbar_wait(&p_ready[0], j & 1, budget_ns))) break;
        tc_fence_after();
        issue_o(0, j, 2 * VDN_P_EARLY_CHUNKS, 8);
        umma_commit_pair(&o_done[0], kBoth);
        if (more) {
          const int sn = (j + 1) % Cfg::STAGES;
          if (!(ok = mbar_wait(&k_full[sn], ((j + 1) / Cfg::STAGES) & 1, budget_ns))) break;
          tc_fence_after();
          issue_s(0, j + 1);
        }
        if (!(ok = mbar_wait(&p_half[1], j & 1, budget_ns))) break;
        tc_fence_after();
        issue_o(1, j, 0, 2 * VDN_P_EARLY_CHUNKS);
        if (!(ok = mbar_wait(&p_ready[1], j & 1, budget_ns))) break;
        tc_fence_after();
        issue_o(1, j, 2 * VDN_P_EARLY_CHUNKS, 8);
        umma_commit_pair(&o_done[1], kBoth);
        umma_commit_pair(&v_empty[s], kBoth);
        if (more) {
          issue_s(1, j + 1);
          umma_commit_pair(&k_empty[(j + 1) % Cfg::STAGES], kBoth);
        }
      }
      if (!ok) record_status(status, kStatusTimeout);
      umma_commit_pair(mma_done, kBoth);
    }
  } else if (warp >= 4) {
    // ================================================================ softmax (both CTAs)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 200;\n" ::: "memory");
    const int i = (warp - 4) >> 2;  // query tile of this warpgroup
    const uint32_t lp_half = mapa_shared(smem_u32(&p_half[i]), 0);
    const uint32_t lp_ready = mapa_shared(smem_u32(&p_ready[i]), 0);
    // one arrival per warp on the leader's barrier, after every lane's TMEM
    // stores have completed (tcgen05.wait::st and the fence precede it)
    softmax_warpgroup<DH, false>(
        i, tmem, s_full, o_done,
        [&] {
          __syncwarp();
          if (lane_id() == 0) mbar_arrive_cluster(lp_half);
        },
        [&] {
          __syncwarp();
          if (lane_id() == 0) mbar_arrive_cluster(lp_ready);
        },
        [] {}, nullptr, kr, nkv, scale_log2, q0, q_end, h, H, L, out, ld_o, lse, status,
        budget_ns);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // the leader's MMAs read this CTA's shared memory and write its TMEM
    tc_fence_after();
    mbar_wait(mma_done, 0, 200000000ull);
  }
  cluster_sync();  // neither CTA leaves while the other may still reach it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ---------------------------------------------------------------- host schedule

bool frame_visible(int tq, int tk, int T, int cf, int wc, unsigned anchors) {
  if ((anchors & 1u) && (tq == 0 || tk == 0)) return true;
  if ((anchors & 2u) && (tq == T - 1 || tk == T - 1)) return true;
  const int cq = tq / cf, ck = tk / cf;
  return (cq > ck ? cq - ck : ck - cq) <= wc;
}

// Visible key frames of query frame tq as maximal runs [a, b).
std::vector<std::pair<int, int>> key_runs(int tq, int T, int cf, int wc, unsigned anchors) {
  std::vector<std::pair<int, int>> runs;
  int a = -1;
  for (int tk = 0; tk <= T; ++tk) {
    const bool v = tk < T && frame_visible(tq, tk, T, cf, wc, anchors);
    if (v && a < 0) a = tk;
    if (!v && a >= 0) {
      runs.push_back({a, tk});
      a = -1;
    }
  }
  return runs;
}

template <int DH>
cudaError_t launch_window_dh(const Launch& ctx, const vdn_shape& s, const CUtensorMap& qmap,
                             const CUtensorMap& kmap, const CUtensorMap& vmap,
                             const CUtensorMap& ckmap, const CUtensorMap& cvmap, int m_ctx,
                             const WinSched& sched, float scale, void* o, int64_t ld_o,
                             float* lse) {
  using Cfg = WinCfg<DH>;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_once(window_attn_kernel<DH>, Cfg::SMEM, smem_set)) return e;
  const int grid = sched.total_tiles * s.H;
  window_attn_kernel<DH><<<grid, Cfg::THREADS, Cfg::SMEM, ctx.stream>>>(
      qmap, kmap, vmap, ckmap, cvmap, m_ctx, sched, s.H, s.T * s.N, scale * 1.4426950408889634f,
      static_cast<__nv_bfloat16*>(o), ld_o, lse, ctx.status, ctx.budget_ns);
  return cudaGetLastError();
}

// Head dim 128 on the CTA-pair kernel.  kmap_half / ckmap_half read 64-key
// boxes (each CTA of a pair loads half of a 128-key tile).
cudaError_t launch_window_pair(const Launch& ctx, const vdn_shape& s, const CUtensorMap& qmap,
                               const CUtensorMap& kmap_half, const CUtensorMap& vmap,
                               const CUtensorMap& ckmap_half, const CUtensorMap& cvmap,
                               int m_ctx, const WinSched& sched, float scale, void* o,
                               int64_t ld_o, float* lse) {
  using Cfg = WinPairCfg<128>;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_once(window_attn_pair_kernel<128>, Cfg::SMEM, smem_set)) return e;
  const int grid = 2 * sched.total_pairs * s.H;  // a multiple of the cluster size
  window_attn_pair_kernel<128><<<grid, Cfg::THREADS, Cfg::SMEM, ctx.stream>>>(
      qmap, kmap_half, vmap, ckmap_half, cvmap, m_ctx, sched, s.H, s.T * s.N,
      scale * 1.4426950408889634f, static_cast<__nv_bfloat16*>(o), ld_o, lse, ctx.status,
      ctx.budget_ns);
  return cudaGetLastError();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

bool build_schedule(const vdn_shape& s, int cf, int wc, unsigned anchors, WinSched* out) {
  struct Raw {
    int f0, f1;
    std::vector<std::pair<int, int>> runs;
    long work;
  };
  std::vector<Raw> raw;
  for (int t = 0; t < s.T; ++t) {
    auto runs = key_runs(t, s.T, cf, wc, anchors);
    if (!raw.empty() && raw.back().runs == runs && raw.back().f1 == t) {
      raw.back().f1 = t + 1;
    } else {
      raw.push_back({t, t + 1, runs, 0});
    }
  }
  if (static_cast<int>(raw.size()) > kMaxSegs) return false;
  for (auto& r : raw) {
    if (r.runs.size() > 3) return false;
    long keys = 0;
    for (auto& p : r.runs) keys += static_cast<long>(p.second - p.first) * s.N;
    r.work = keys;
  }
  std::stable_sort(raw.begin(), raw.end(), [](const Raw& a, const Raw& b) { return a.work > b.work; });
  memset(out, 0, sizeof(*out));
  out->nseg = static_cast<int>(raw.size());
  int base = 0, pbase = 0;
  for (size_t k = 0; k < raw.size(); ++k) {
    WinSeg& g = out->seg[k];
    g.q0 = raw[k].f0 * s.N;
    g.q1 = raw[k].f1 * s.N;
    g.ntiles = (g.q1 - g.q0 + 255) / 256;
    g.tile_base = base;
    base += g.ntiles;
    g.npairs = (g.ntiles + 1) / 2;
    g.pair_base = pbase;
    pbase += g.npairs;
    g.nint = static_cast<int>(raw[k].runs.size());
    g.nkv = 0;
    for (int v = 0; v < g.nint; ++v) {
      g.k0[v] = raw[k].runs[v].first * s.N;
      g.k1[v] = raw[k].runs[v].second * s.N;
      g.nkv += (g.k1[v] - g.k0[v] + 127) / 128;
    }
  }
  out->total_tiles = base;
  out->total_pairs = pbase;
  return true;
}

}  // namespace vdn

using namespace vdn;

extern "C" {

// Head dims 16 and 32 run on a zero-padded 64-wide copy of q, k, v and o
// kept in the workspace after the status word.
static size_t window_padded_act_bytes(const vdn_shape& s) {
  return (static_cast<size_t>(s.T) * s.N * s.H * 64 * 2 + 255) / 256 * 256;
}

size_t vdn_window_attn_workspace(const vdn_shape* shape) {
  if (shape == nullptr || shape->T < 1 || shape->N < 1 || shape->H < 1 || shape->d < 1) return 0;
  if (shape->d == 16 || shape->d == 32) return kStatusBytes + 4 * window_padded_act_bytes(*shape);
  return kStatusBytes;
}

vdn_status vdn_window_attn_ctx(const vdn_shape* shape, const void* q, const void* k,
                               const void* v, int64_t ld, const void* ctx_k, const void* ctx_v,
                               int64_t ld_ctx, int m_ctx, int chunk_frames, int window_chunks,
                               unsigned anchors, float scale, void* o, int64_t ld_o,
                               float* lse_opt, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("vdn_window_attn_ctx");
  if (shape == nullptr || shape->T < 1 || shape->N < 1 || shape->H < 1 || shape->d < 1)
    return VDN_ERR_INVALID_ARG;
  const vdn_shape s = *shape;
  if (static_cast<int64_t>(s.T) * s.N >= (int64_t(1) << 31) - 512) return VDN_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return VDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse_opt && (reinterpret_cast<uintptr_t>(lse_opt) & 3u)))
    return VDN_ERR_INVALID_ARG;
  if (chunk_frames < 1 || window_chunks < 0 || anchors > 3u) return VDN_ERR_INVALID_ARG;
  const bool padded = s.d == 16 || s.d == 32;
  if (s.d != 128 && s.d != 64 && !padded) return VDN_ERR_UNSUPPORTED;
  const int64_t D = static_cast<int64_t>(s.H) * s.d;
  if (ld < D || ld % 8 || ld_o < D || ld_o % 8) return VDN_ERR_INVALID_ARG;
  if (m_ctx < 0 || m_ctx >= (1 << 30)) return VDN_ERR_INVALID_ARG;
  if (m_ctx > 0 && (ctx_k == nullptr || ctx_v == nullptr || !aligned16(ctx_k) ||
                    !aligned16(ctx_v) || ld_ctx < D || ld_ctx % 8))
    return VDN_ERR_INVALID_ARG;
  if (m_ctx > 0 && padded) return VDN_ERR_UNSUPPORTED;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) ||
      ws_bytes < vdn_window_attn_workspace(shape))
    return VDN_ERR_WORKSPACE;
  const float sc = scale > 0.f ? scale : 1.f / sqrtf(static_cast<float>(s.d));
  if (padded) {
    // run on zero-padded 64-wide heads (exact: padded dims add nothing to a
    // score and give zero output columns), then copy the real columns back
    const int L = s.T * s.N;
    const int64_t D64 = static_cast<int64_t>(s.H) * 64;
    const size_t act = window_padded_act_bytes(s);
    uint8_t* qp = static_cast<uint8_t*>(ws) + kStatusBytes;
    uint8_t* kp = qp + act;
    uint8_t* vp = kp + act;
    uint8_t* op = vp + act;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (launch_repack_bf16(st, qp, D64, q, ld, 1, L, L, s.H, 64, s.d) != cudaSuccess ||
        launch_repack_bf16(st, kp, D64, k, ld, 1, L, L, s.H, 64, s.d) != cudaSuccess ||
        launch_repack_bf16(st, vp, D64, v, ld, 1, L, L, s.H, 64, s.d) != cudaSuccess)
      return VDN_ERR_CUDA;
    vdn_shape s64 = s;
    s64.d = 64;
    // the inner call sees a workspace that is just this call's status word
    const vdn_status r = vdn_window_attn_ctx(&s64, qp, kp, vp, D64, nullptr, nullptr, 0, 0,
                                             chunk_frames, window_chunks, anchors, sc, op, D64,
                                             lse_opt, ws, kStatusBytes, stream);
    if (r != VDN_OK) return r;
    if (launch_repack_bf16(st, o, ld_o, op, D64, 1, L, L, s.H, s.d, 64) != cudaSuccess)
      return VDN_ERR_CUDA;
    return VDN_OK;
  }
  thread_local WinSched sched;  // ~12 KB; copied into the launch's parameters
  if (!build_schedule(s, chunk_frames, window_chunks, anchors, &sched)) return VDN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(sched.total_tiles) * s.H >= (int64_t(1) << 31) ||
      2 * static_cast<int64_t>(sched.total_pairs) * s.H >= (int64_t(1) << 31))
    return VDN_ERR_UNSUPPORTED;
  const int64_t L = static_cast<int64_t>(s.T) * s.N;
  CUtensorMap qmap, kmap, vmap, ckmap, cvmap;
  if (!make_rows_map(&qmap, q, D, ld, L, 128) || !make_rows_map(&kmap, k, D, ld, L, 128) ||
      !make_rows_map(&vmap, v, D, ld, L, 128))
    return VDN_ERR_CUDA;
  if (m_ctx > 0) {
    if (!make_rows_map(&ckmap, ctx_k, D, ld_ctx, m_ctx, 128) ||
        !make_rows_map(&cvmap, ctx_v, D, ld_ctx, m_ctx, 128))
      return VDN_ERR_CUDA;
  } else {
    ckmap = kmap;  // unused
    cvmap = vmap;
  }
  Launch ctx{static_cast<cudaStream_t>(stream), static_cast<uint32_t*>(ws),
             current_wait_budget_ns()};
  if (VDN_WINDOW_PAIR && s.d == 128) {
    CUtensorMap kmap_half, ckmap_half;
    if (!make_rows_map(&kmap_half, k, D, ld, L, 64)) return VDN_ERR_CUDA;
    if (m_ctx > 0) {
      if (!make_rows_map(&ckmap_half, ctx_k, D, ld_ctx, m_ctx, 64)) return VDN_ERR_CUDA;
    } else {
      ckmap_half = kmap_half;  // unused
    }
    return launch_window_pair(ctx, s, qmap, kmap_half, vmap, ckmap_half, cvmap, m_ctx, sched, sc,
                              o, ld_o, lse_opt) == cudaSuccess
               ? VDN_OK
               : VDN_ERR_CUDA;
  }
  cudaError_t e = s.d == 128 ? launch_window_dh<128>(ctx, s, qmap, kmap, vmap, ckmap, cvmap, m_ctx,
                                                     sched, sc, o, ld_o, lse_opt)
                             : launch_window_dh<64>(ctx, s, qmap, kmap, vmap, ckmap, cvmap, m_ctx,
                                                    sched, sc, o, ld_o, lse_opt);
  return e == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

vdn_status vdn_window_attn_schedule(const vdn_shape* shape, int chunk_frames, int window_chunks,
                                   unsigned anchors, int* segs, int max_segs, int* nseg) {
  if (shape == nullptr || shape->T < 1 || shape->N < 1 || nseg == nullptr)
    return VDN_ERR_INVALID_ARG;
  if (chunk_frames < 1 || window_chunks < 0 || anchors > 3u || max_segs < 0 ||
      (max_segs > 0 && segs == nullptr))
    return VDN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(shape->T) * shape->N >= (int64_t(1) << 31) - 512)
    return VDN_ERR_INVALID_ARG;
  thread_local WinSched sched;
  if (!build_schedule(*shape, chunk_frames, window_chunks, anchors, &sched))
    return VDN_ERR_UNSUPPORTED;
  *nseg = sched.nseg;
  if (sched.nseg > max_segs) return VDN_ERR_INVALID_ARG;
  for (int g = 0; g < sched.nseg; ++g) {
    const WinSeg& w = sched.seg[g];
    int* o = segs + 12 * g;
    o[0] = w.q0;
    o[1] = w.q1;
    o[2] = w.tile_base;
    o[3] = w.ntiles;
    o[4] = w.nint;
    o[5] = w.nkv;
    for (int v = 0; v < 3; ++v) {
      o[6 + 2 * v] = v < w.nint ? w.k0[v] : 0;
      o[7 + 2 * v] = v < w.nint ? w.k1[v] : 0;
    }
  }
  return VDN_OK;
}

vdn_status vdn_window_attn(const vdn_shape* shape, const void* q, const void* k, const void* v,
                           int64_t ld, int chunk_frames, int window_chunks, unsigned anchors,
                           float scale, void* o, int64_t ld_o, float* lse_opt, void* ws,
                           size_t ws_bytes, void* stream) {
  return vdn_window_attn_ctx(shape, q, k, v, ld, nullptr, nullptr, 0, 0, chunk_frames,
                             window_chunks, anchors, scale, o, ld_o, lse_opt, ws, ws_bytes,
                             stream);
}

}  // extern "C"
