// Internal declarations shared by the libvdn translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include <nvtx3/nvToolsExt.h>

#include "../../include/vdn.h"

namespace vdn {

// Bits of the device status word (first 4 bytes of every workspace).
constexpr uint32_t kStatusNumeric = 1u << 0;
constexpr uint32_t kStatusTimeout = 1u << 1;
constexpr uint32_t kStatusBounds = 1u << 2;  // debug builds: an index outside its tensor

// Debug builds (VDN_DEBUG_BOUNDS=1) check the row and column range of every
// hand-computed global store, and the start of hand-computed tile
// coordinates, against the tensor's extents; a violation is recorded in the
// status word and the access skipped.  Release builds compile the checks out.
#ifndef VDN_DEBUG_BOUNDS
#define VDN_DEBUG_BOUNDS 0
#endif

// Workspace bytes reserved in front of every workspace for the status word.
constexpr size_t kStatusBytes = 256;

__device__ __forceinline__ void record_status(uint32_t* status, uint32_t bits) {
  if (status != nullptr) atomicOr(status, bits);
}

// Rows [r, r + 1) and columns [c, c + width) inside a rows x cols tensor?
// Always true in release builds; in debug builds a miss is recorded.
__device__ __forceinline__ bool in_bounds(uint32_t* status, int64_t r, int64_t rows, int64_t c,
                                          int64_t width, int64_t cols) {
  if constexpr (VDN_DEBUG_BOUNDS) {
    if (r < 0 || r >= rows || c < 0 || width < 0 || c + width > cols) {
      record_status(status, kStatusBounds);
      return false;
    }
  }
  return true;
}

// NVTX range around a C-ABI call (a no-op unless a profiler is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Launch context handed to every launcher.
struct Launch {
  cudaStream_t stream;
  uint32_t* status;     // device status word
  uint64_t budget_ns;   // bounded-wait budget
};

// SMs of the current device (148 on a B200; that figure if the query fails).
inline int sm_count_of_current_device() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n > 0 ? n : 148;
}

// Opt a kernel into `bytes` of dynamic shared memory on the current device,
// once per device (the attribute is per device; `done` is the kernel's own
// bit set of devices already done, safe under concurrent callers).
template <class Kernel>
cudaError_t set_smem_once(Kernel* kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Budget (ns) of the bounded device waits, set by vdn_set_wait_budget_ns.
uint64_t current_wait_budget_ns();

// Solver of the VDA closed form, set by vdn_set_vda_solver.
int current_vda_solver();

// vdn_vda_scan's validation and launch sequence on the workspace `ws`; with
// clear_status the workspace's status word is zeroed on the stream first.
vdn_status vda_scan_checked(const vdn_shape* shape, const void* q, const void* k, const void* v,
                            int64_t ld, const float* beta, const float* alpha, void* o_vda,
                            int64_t ld_o, float* states_opt, void* ws, size_t ws_bytes,
                            void* stream, bool clear_status);

// ---- tensor maps (built on the host with the driver's encoder) ----------

// 3-D bf16 view of a frame-major [T*N, ld] activation: dims {cols, N, T}.
// Rows past the end of a frame fall outside dim 1, so TMA loads read zeros
// there and TMA stores drop them.  Box {64, box_rows, 1}, 128-byte swizzle.
bool make_frame_map(CUtensorMap* map, const void* base, int64_t cols, int64_t ld, int N, int T,
                    int box_rows);

// 2-D bf16 map over a row-major [rows, ld] matrix with box {64, box_rows},
// 128-byte swizzle.
bool make_rows_map(CUtensorMap* map, const void* base, int64_t cols, int64_t ld, int64_t rows,
                   int box_rows);

// 2-D byte map over a row-major [rows, ld] matrix of 8-bit codes with box
// {128 bytes, box_rows}, 128-byte swizzle.
bool make_rows_map_u8(CUtensorMap* map, const void* base, int64_t cols, int64_t ld, int64_t rows,
                      int box_rows);

// ---- kernel launchers (return cudaSuccess or the launch error) ----------

cudaError_t launch_vda_prep(const Launch& ctx, const vdn_shape& s, const CUtensorMap& kmap,
                            const CUtensorMap& vmap, const float* beta, float* A, float* B);

// P = (I + (A + A^T)/2)^-1 per (frame, head).
cudaError_t launch_vda_solve(const Launch& ctx, const vdn_shape& s, const float* A, float* P);

// Both scans S_t = (alpha_t S_prev + B_t) P_t into states [2, T, H, d, d].
cudaError_t launch_vda_scan(const Launch& ctx, const vdn_shape& s, const float* P,
                            const float* B, const float* alpha, float* states);

cudaError_t launch_vda_readout(const Launch& ctx, const vdn_shape& s, const CUtensorMap& qmap,
                               const CUtensorMap& omap, const float* states);

// MXFP8 quantization of a bf16 [R, ld] operand (K = cols, a multiple of 128):
// codes [R, K] row-major and scale bytes in the MMA tile layout (mxfp8.cuh).
cudaError_t launch_mx_quantize(cudaStream_t st, const void* x, int64_t ld, int R, int K,
                               uint8_t* q, uint8_t* sf);

// ---- gradient pass (see vda_grad.cu) -------------------------------------

// G[t,h] = sum_i dO_i q_i^T (gram mode of the prep kernel; maps as for prep).
cudaError_t launch_vda_gram(const Launch& ctx, const vdn_shape& s, const CUtensorMap& qmap,
                            const CUtensorMap& domap, float* G);

// Adjoint scans D_t = (alpha_u D_u + G_t) P_t; adj is [2, T, H, d, d] with
// direction 0 forward in time (adjoint of the backward scan).
cudaError_t launch_vda_adjoint_scan(const Launch& ctx, const vdn_shape& s, const float* P,
                                    const float* G, const float* alpha, float* adj);

// Read-out variants: x (S0 + S1)^T, or x (S0 + S1) when trans_s.
cudaError_t launch_vda_readout_ex(const Launch& ctx, const vdn_shape& s, const CUtensorMap& xmap,
                                  const CUtensorMap& omap, const float* states, bool trans_s);

// Head dim 128: dq = dO (S0 + S1) (bf16 through dqmap) and, from the same dO
// tiles, G = sum_i dO_i q_i^T per (t, h) (fp32 [T, H, d, d]); the 128-row
// frame maps domap and qmap.
cudaError_t launch_vda_readout_dq_gram(const Launch& ctx, const vdn_shape& s,
                                       const CUtensorMap& domap, const CUtensorMap& dqmap,
                                       const CUtensorMap& qmap, const float* states, float* G);

// E = dA + dA^T with dA = -(S_fwd^T D_fwd + S_bwd^T D_bwd), and dalpha.
cudaError_t launch_vda_grad_combine(const Launch& ctx, const vdn_shape& s, const float* states,
                                    const float* adj, float* E, float* dalpha);

// dk = beta (K E + V dB) (bf16 through dkmap), dv = beta K dB^T (bf16 rows
// of dv, row stride ld_dv elements) and dbeta (fp32 [L, H]), in one pass
// over k and v.
cudaError_t launch_vda_grad_k(const Launch& ctx, const vdn_shape& s, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, const CUtensorMap& dkmap, const float* E,
                              const float* adj, const float* beta, float* dbeta, void* dv,
                              int64_t ld_dv);

}  // namespace vdn
