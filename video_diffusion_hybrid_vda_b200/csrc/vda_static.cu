// Allocation-free variant of vdn_vda_scan.
//
// Some callers cannot allocate device memory at all: a plugin that runs
// inside a host framework which owns every device allocation, or a loop with
// a fixed memory budget where a cudaMalloc (and the device synchronisation
// it can imply) is not allowed.  For them, vdn_vda_scan_static keeps its
// scratch (the per-(frame, head) A, B, P matrices and both scans' states)
// in a fixed-size array of this library's own device memory instead of a
// caller-provided workspace.  The array exists on every GPU that loads the
// library, until the process exits.
#include <mutex>

#include "common.cuh"

namespace vdn {
namespace {

// 64 MiB: room for T*H*d*d*4*5 bytes of scratch plus the status word, e.g.
// 204 (frame, head) pairs at d = 128 or 819 pairs at d = 64.
constexpr size_t kStaticScratchBytes = size_t(64) << 20;

static __device__ __align__(256) uint8_t g_vda_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
uint8_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_vda_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, once per device, with that device current.
cudaError_t scratch_on_current_device(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_vda_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

size_t round_up256(size_t x) { return (x + 255) / 256 * 256; }

bool ptr_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace vdn

using namespace vdn;

extern "C" vdn_status vdn_vda_scan_static(const vdn_shape* shape, const void* q, const void* k,
                                          const void* v, int64_t ld, const float* beta,
                                          const float* alpha, void* o_vda, int64_t ld_o,
                                          float* states_opt, unsigned* dev_status_opt,
                                          void* stream) {
  // ---- host-side validation, before any CUDA call
  if (shape == nullptr || shape->T < 1 || shape->N < 1 || shape->H < 1 || shape->d < 1)
    return VDN_ERR_INVALID_ARG;
  const vdn_shape s = *shape;
  if (static_cast<int64_t>(s.T) * s.N >= (int64_t(1) << 31)) return VDN_ERR_INVALID_ARG;
  if (s.d != 64 && s.d != 128) return VDN_ERR_UNSUPPORTED;
  const int64_t D = static_cast<int64_t>(s.H) * s.d;
  if (!q || !k || !v || !beta || !alpha || !o_vda) return VDN_ERR_INVALID_ARG;
  if (!ptr_aligned(q, 16) || !ptr_aligned(k, 16) || !ptr_aligned(v, 16) ||
      !ptr_aligned(o_vda, 16) || !ptr_aligned(beta, 4) || !ptr_aligned(alpha, 4) ||
      (states_opt && !ptr_aligned(states_opt, 16)) ||
      (dev_status_opt && !ptr_aligned(dev_status_opt, 4)))
    return VDN_ERR_INVALID_ARG;
  if (ld < D || ld % 8 || ld_o < D || ld_o % 8) return VDN_ERR_INVALID_ARG;
  // scratch: [status 256 B][A][B][P][states x2], as in the workspace path
  const size_t mat = round_up256(static_cast<size_t>(s.T) * s.H * s.d * s.d * sizeof(float));
  const size_t need = kStatusBytes + 5 * mat;
  if (need > kStaticScratchBytes) return VDN_ERR_WORKSPACE;  // beyond the fixed maximum

  uint8_t* base = nullptr;
  if (scratch_on_current_device(&base) != cudaSuccess) return VDN_ERR_CUDA;
  float* A = reinterpret_cast<float*>(base + kStatusBytes);
  float* B = reinterpret_cast<float*>(base + kStatusBytes + mat);
  float* P = reinterpret_cast<float*>(base + kStatusBytes + 2 * mat);
  float* states =
      states_opt ? states_opt : reinterpret_cast<float*>(base + kStatusBytes + 3 * mat);

  CUtensorMap kmap, vmap, qmap, omap;
  const int prep_rows = s.d == 128 ? 32 : 64;
  if (!make_frame_map(&kmap, k, D, ld, s.N, s.T, prep_rows) ||
      !make_frame_map(&vmap, v, D, ld, s.N, s.T, prep_rows) ||
      !make_frame_map(&qmap, q, D, ld, s.N, s.T, 128) ||
      !make_frame_map(&omap, o_vda, D, ld_o, s.N, s.T, 128))
    return VDN_ERR_CUDA;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the array keeps the previous call's contents: the status word must start at 0
  if (cudaMemsetAsync(base, 0, sizeof(uint32_t), st) != cudaSuccess) return VDN_ERR_CUDA;
  Launch ctx{st, reinterpret_cast<uint32_t*>(base), current_wait_budget_ns()};
  if (launch_vda_prep(ctx, s, kmap, vmap, beta, A, B) != cudaSuccess) return VDN_ERR_CUDA;
  if (launch_vda_solve(ctx, s, A, P) != cudaSuccess) return VDN_ERR_CUDA;
  if (launch_vda_scan(ctx, s, P, B, alpha, states) != cudaSuccess) return VDN_ERR_CUDA;
  if (launch_vda_readout(ctx, s, qmap, omap, states) != cudaSuccess) return VDN_ERR_CUDA;
  if (dev_status_opt != nullptr &&
      cudaMemcpyAsync(dev_status_opt, base, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st) !=
          cudaSuccess)
    return VDN_ERR_CUDA;
  return VDN_OK;
}
