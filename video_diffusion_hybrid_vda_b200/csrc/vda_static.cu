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

// 64 MiB: room for the workspace vdn_vda_scan would need, 256 + 5*T*H*d*d*4
// bytes at d = 64 or 128 (e.g. 204 (frame, head) pairs at d = 128, 819 at
// d = 64), plus four padded bf16 copies of [T*N, H*64] at d = 16 and 32.
constexpr size_t kStaticScratchBytes = size_t(64) << 20;

static __device__ __align__(256) uint8_t g_vda_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
uint8_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_vda_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, once per device, with that device current.  The
// cached address belongs to the context it was looked up in: it is not valid
// across cudaDeviceReset.
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

}  // namespace
}  // namespace vdn

using namespace vdn;

extern "C" vdn_status vdn_vda_scan_static(const vdn_shape* shape, const void* q, const void* k,
                                          const void* v, int64_t ld, const float* beta,
                                          const float* alpha, void* o_vda, int64_t ld_o,
                                          float* states_opt, unsigned* dev_status_opt,
                                          void* stream) {
  NvtxRange nvtx("vdn_vda_scan_static");
  // ---- host-side checks of what the shared path does not see, before any
  // CUDA call: the status pointer and the scratch array's fixed size (the
  // same bytes vdn_vda_scan would ask of a workspace, head dims 16 and 32
  // included through their padded copies)
  if (dev_status_opt != nullptr && (reinterpret_cast<uintptr_t>(dev_status_opt) & 3u))
    return VDN_ERR_INVALID_ARG;
  const size_t need = vdn_vda_scan_workspace(shape);
  if (need == 0) return VDN_ERR_INVALID_ARG;                 // invalid shape
  if (need > kStaticScratchBytes) return VDN_ERR_WORKSPACE;  // beyond the fixed maximum

  uint8_t* base = nullptr;
  if (scratch_on_current_device(&base) != cudaSuccess) return VDN_ERR_CUDA;
  // the array keeps the previous call's contents: the shared path clears the
  // status word on the stream before its first launch
  const vdn_status r = vda_scan_checked(shape, q, k, v, ld, beta, alpha, o_vda, ld_o, states_opt,
                                        base, kStaticScratchBytes, stream, true);
  if (r != VDN_OK) return r;
  if (dev_status_opt != nullptr &&
      cudaMemcpyAsync(dev_status_opt, base, sizeof(uint32_t), cudaMemcpyDeviceToDevice,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return VDN_ERR_CUDA;
  return VDN_OK;
}
