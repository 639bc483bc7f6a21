// C ABI of libvdn: host-side validation, workspace layout, TMA descriptor
// construction and kernel sequencing.  Every entry point validates all of
// its arguments before it enqueues anything, then launches asynchronously on
// the caller's stream.  Nothing here allocates, frees or synchronises (except
// vdn_get_device_status, whose job is to read the status word back).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "repack.cuh"

namespace vdn {

namespace {

std::atomic<uint64_t> g_budget_ns{2000000000ull};
std::atomic<int> g_solver{VDN_SOLVER_GAUSS_JORDAN};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool shape_ok(const vdn_shape* s) {
  return s != nullptr && s->T >= 1 && s->N >= 1 && s->H >= 1 && s->d >= 1 &&
         static_cast<int64_t>(s->T) * s->N < (int64_t(1) << 31) &&
         static_cast<int64_t>(s->H) * s->d < (int64_t(1) << 24);
}

bool head_dim_supported(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

bool head_dim_padded(int d) { return d == 16 || d == 32; }

bool ld_ok(int64_t ld, int64_t D) { return ld >= D && ld % 8 == 0; }

// VDA workspace: [status 256 B][A][B][P][states (2x)]([X]), each region
// 256-byte aligned, every matrix fp32 [T, H, d, d]; the gradient pass adds
// the slot X (for G, then E) at the end.
struct VdaLayout {
  size_t mat_bytes, A, B, P, states, X, total;
};

VdaLayout vda_layout(const vdn_shape& s, bool with_x) {
  VdaLayout l;
  l.mat_bytes = round_up(static_cast<size_t>(s.T) * s.H * s.d * s.d * sizeof(float), 256);
  l.A = kStatusBytes;
  l.B = l.A + l.mat_bytes;
  l.P = l.B + l.mat_bytes;
  l.states = l.P + l.mat_bytes;
  l.X = l.states + 2 * l.mat_bytes;
  l.total = l.X + (with_x ? l.mat_bytes : 0);
  return l;
}

// Workspace of a VDA call.  Head dims 16 and 32 run through a 64-wide padded
// copy: [status][q' k' v' o' bf16 L x H*64][the layout above for d = 64]
// and, for the gradient pass, [dq' dk' dv'] after it (o' holds dO' there).
// The forward's workspace is therefore a prefix of the gradient pass's, so
// one workspace can carry the forward's P and states into the gradient pass.
struct VdaPlan {
  bool padded;
  vdn_shape inner;  // shape the kernels run on
  size_t act;       // bytes of one padded activation
  size_t inner_off; // where the d = 64 layout (after its status word) starts
  VdaLayout lay;    // layout of the inner shape
  size_t extra;     // gradient pass: dq' dk' dv'
  size_t total;
};

VdaPlan vda_plan(const vdn_shape& s, bool backward = false) {
  VdaPlan p;
  p.padded = head_dim_padded(s.d);
  p.inner = s;
  if (p.padded) p.inner.d = 64;
  p.lay = vda_layout(p.inner, backward);
  p.act = p.padded ? round_up(static_cast<size_t>(s.T) * s.N * s.H * 64 * 2, 256) : 0;
  p.inner_off = 4 * p.act;
  p.extra = p.inner_off + p.lay.total;
  p.total = p.extra + (backward ? 3 * p.act : 0);
  return p;
}

// The four VDA kernels on head dim 64 or 128.
vdn_status run_vda(const Launch& ctx, const vdn_shape& s, const void* q, const void* k,
                   const void* v, int64_t ld, const float* beta, const float* alpha, void* o,
                   int64_t ld_o, float* A, float* B, float* P, float* states) {
  const int64_t D = static_cast<int64_t>(s.H) * s.d;
  const int prep_rows = s.d == 128 ? 32 : 64;
  CUtensorMap kmap, vmap, qmap, omap;
  if (!make_frame_map(&kmap, k, D, ld, s.N, s.T, prep_rows) ||
      !make_frame_map(&vmap, v, D, ld, s.N, s.T, prep_rows) ||
      !make_frame_map(&qmap, q, D, ld, s.N, s.T, 128) ||
      !make_frame_map(&omap, o, D, ld_o, s.N, s.T, 128))
    return VDN_ERR_CUDA;
  if (launch_vda_prep(ctx, s, kmap, vmap, beta, A, B) != cudaSuccess) return VDN_ERR_CUDA;
  if (launch_vda_solve(ctx, s, A, P) != cudaSuccess) return VDN_ERR_CUDA;
  if (launch_vda_scan(ctx, s, P, B, alpha, states) != cudaSuccess) return VDN_ERR_CUDA;
  if (launch_vda_readout(ctx, s, qmap, omap, states) != cudaSuccess) return VDN_ERR_CUDA;
  return VDN_OK;
}

// The gradient pass on head dim 64 or 128.  Workspace slots (in memory
// order A, B, P, X, states) are reused as their contents die: G goes to X,
// the adjoint states to A and B (dead after the forward scan; adjacent, so
// they form one [2, T, H, d, d] array), E to X (G is dead after the adjoint
// scan).  P is read by both adjoint directions until the adjoint scan ends,
// so nothing is written there.
vdn_status run_vda_backward(const Launch& ctx, const vdn_shape& s, const void* q, const void* k,
                            const void* v, int64_t ld, const float* beta, const float* alpha,
                            const void* d_o, int64_t ld_do, void* dq, void* dk, void* dv,
                            int64_t ld_g, float* dbeta, float* dalpha, float* A, float* B,
                            float* P, float* X, float* states, bool reuse_forward) {
  const int64_t D = static_cast<int64_t>(s.H) * s.d;
  const int prep_rows = s.d == 128 ? 32 : 64;
  CUtensorMap kmap_p, vmap_p, qmap_p, domap_p, domap, dqmap, kmap, vmap, dkmap, qmap;
  if (!make_frame_map(&kmap_p, k, D, ld, s.N, s.T, prep_rows) ||
      !make_frame_map(&vmap_p, v, D, ld, s.N, s.T, prep_rows) ||
      !make_frame_map(&qmap_p, q, D, ld, s.N, s.T, prep_rows) ||
      !make_frame_map(&domap_p, d_o, D, ld_do, s.N, s.T, prep_rows) ||
      !make_frame_map(&domap, d_o, D, ld_do, s.N, s.T, 128) ||
      !make_frame_map(&dqmap, dq, D, ld_g, s.N, s.T, 128) ||
      !make_frame_map(&kmap, k, D, ld, s.N, s.T, 128) ||
      !make_frame_map(&qmap, q, D, ld, s.N, s.T, 128) ||
      !make_frame_map(&vmap, v, D, ld, s.N, s.T, 128) ||
      !make_frame_map(&dkmap, dk, D, ld_g, s.N, s.T, 128))
    return VDN_ERR_CUDA;
  float* G = X;
  float* adj = A;
  float* E = X;
  if (!reuse_forward &&
      (launch_vda_prep(ctx, s, kmap_p, vmap_p, beta, A, B) != cudaSuccess ||
       launch_vda_solve(ctx, s, A, P) != cudaSuccess ||
       launch_vda_scan(ctx, s, P, B, alpha, states) != cudaSuccess))
    return VDN_ERR_CUDA;
  // dq and G: one pass over dO for head dim 128 (G beside the dq read-out),
  // the gram mode of the prep kernel and the transposed read-out otherwise
  if (s.d == 128) {
    if (launch_vda_readout_dq_gram(ctx, s, domap, dqmap, qmap, states, G) != cudaSuccess)
      return VDN_ERR_CUDA;
  } else if (launch_vda_gram(ctx, s, qmap_p, domap_p, G) != cudaSuccess ||
             launch_vda_readout_ex(ctx, s, domap, dqmap, states, true) != cudaSuccess) {
    return VDN_ERR_CUDA;
  }
  if (launch_vda_adjoint_scan(ctx, s, P, G, alpha, adj) != cudaSuccess ||
      launch_vda_grad_combine(ctx, s, states, adj, E, dalpha) != cudaSuccess ||
      launch_vda_grad_k(ctx, s, kmap, vmap, dkmap, E, adj, beta, dbeta, dv, ld_g) != cudaSuccess)
    return VDN_ERR_CUDA;
  return VDN_OK;
}

}  // namespace

uint64_t current_wait_budget_ns() { return g_budget_ns.load(); }

__global__ void bounds_selftest_kernel(uint32_t* status, int64_t r, int64_t rows, int64_t c,
                                       int64_t width, int64_t cols) {
  in_bounds(status, r, rows, c, width, cols);
}

int current_vda_solver() { return g_solver.load(); }

bool make_frame_map(CUtensorMap* map, const void* base, int64_t cols, int64_t ld, int N, int T,
                    int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 2,
                                 static_cast<cuuint64_t>(ld) * 2 * static_cast<cuuint64_t>(N)};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_rows_map(CUtensorMap* map, const void* base, int64_t cols, int64_t ld, int64_t rows,
                   int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_rows_map_u8(CUtensorMap* map, const void* base, int64_t cols, int64_t ld, int64_t rows,
                      int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld)};
  const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace vdn

using namespace vdn;

extern "C" {

const char* vdn_version(void) { return "vdn-b200 0.1 (sm_100a)"; }

const char* vdn_status_string(vdn_status s) {
  switch (s) {
    case VDN_OK: return "ok";
    case VDN_ERR_INVALID_ARG: return "invalid argument (null/misaligned pointer, bad size or stride)";
    case VDN_ERR_UNSUPPORTED: return "unsupported configuration";
    case VDN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case VDN_ERR_CUDA: return "CUDA runtime or driver call failed";
    case VDN_ERR_NUMERIC: return "numeric failure on the device (non-positive pivot or NaN)";
    case VDN_ERR_TIMEOUT: return "a bounded wait on the device ran out of time";
    case VDN_ERR_BOUNDS: return "an index outside its tensor (debug bounds check)";
  }
  return "unknown status";
}

void vdn_set_wait_budget_ns(uint64_t ns) { g_budget_ns.store(ns); }

vdn_status vdn_set_vda_solver(int solver) {
  if (solver != VDN_SOLVER_CHOLESKY && solver != VDN_SOLVER_GAUSS_JORDAN)
    return VDN_ERR_INVALID_ARG;
  g_solver.store(solver);
  return VDN_OK;
}

vdn_status vdn_reset_device_status(void* ws, void* stream) {
  if (ws == nullptr || !aligned(ws, 256)) return VDN_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return VDN_ERR_CUDA;
  return VDN_OK;
}

vdn_status vdn_copy2d_async(void* dst, size_t dst_pitch, const void* src, size_t src_pitch,
                            size_t width_bytes, size_t rows, void* stream) {
  if (dst == nullptr || src == nullptr || width_bytes > dst_pitch || width_bytes > src_pitch)
    return VDN_ERR_INVALID_ARG;
  if (width_bytes == 0 || rows == 0) return VDN_OK;
  return cudaMemcpy2DAsync(dst, dst_pitch, src, src_pitch, width_bytes, rows, cudaMemcpyDefault,
                           static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? VDN_OK
             : VDN_ERR_CUDA;
}

vdn_status vdn_get_device_status(const void* ws, void* stream) {
  if (ws == nullptr || !aligned(ws, 256)) return VDN_ERR_WORKSPACE;
  uint32_t word = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return VDN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return VDN_ERR_CUDA;
  if (word & kStatusTimeout) return VDN_ERR_TIMEOUT;
  if (word & kStatusNumeric) return VDN_ERR_NUMERIC;
  if (word & kStatusBounds) return VDN_ERR_BOUNDS;
  return VDN_OK;
}

int vdn_debug_bounds_enabled(void) { return VDN_DEBUG_BOUNDS ? 1 : 0; }

vdn_status vdn_selftest_bounds(void* ws, int64_t r, int64_t rows, int64_t c, int64_t width,
                               int64_t cols, void* stream) {
  if (ws == nullptr || !aligned(ws, 256)) return VDN_ERR_WORKSPACE;
  bounds_selftest_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint32_t*>(ws), r, rows, c, width, cols);
  return cudaGetLastError() == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

// ----------------------------------------------------------------- VDA

size_t vdn_vda_scan_workspace(const vdn_shape* shape) {
  if (!shape_ok(shape)) return 0;
  return vda_plan(*shape).total;
}

vdn_status vdn_vda_debug_buffers(const vdn_shape* shape, void* ws, float** A, float** B,
                                 float** P) {
  if (!shape_ok(shape) || ws == nullptr) return VDN_ERR_INVALID_ARG;
  const VdaPlan pl = vda_plan(*shape);
  uint8_t* base = static_cast<uint8_t*>(ws) + pl.inner_off;
  if (A) *A = reinterpret_cast<float*>(base + pl.lay.A);
  if (B) *B = reinterpret_cast<float*>(base + pl.lay.B);
  if (P) *P = reinterpret_cast<float*>(base + pl.lay.P);
  return VDN_OK;
}

vdn_status vdn_vda_scan(const vdn_shape* shape, const void* q, const void* k, const void* v,
                        int64_t ld, const float* beta, const float* alpha, void* o_vda,
                        int64_t ld_o, float* states_opt, void* ws, size_t ws_bytes,
                        void* stream) {
  NvtxRange nvtx("vdn_vda_scan");
  return vdn::vda_scan_checked(shape, q, k, v, ld, beta, alpha, o_vda, ld_o, states_opt, ws,
                               ws_bytes, stream, false);
}

}  // extern "C"

// Validation and launch sequence of vdn_vda_scan, shared with the
// allocation-free entry point (which passes its fixed scratch array as the
// workspace and asks for the status word to be cleared first).
vdn_status vdn::vda_scan_checked(const vdn_shape* shape, const void* q, const void* k,
                                 const void* v, int64_t ld, const float* beta,
                                 const float* alpha, void* o_vda, int64_t ld_o,
                                 float* states_opt, void* ws, size_t ws_bytes, void* stream,
                                 bool clear_status) {
  if (!shape_ok(shape)) return VDN_ERR_INVALID_ARG;
  const vdn_shape s = *shape;
  if (!head_dim_supported(s.d)) return VDN_ERR_UNSUPPORTED;
  const int64_t D = static_cast<int64_t>(s.H) * s.d;
  if (q == nullptr || k == nullptr || v == nullptr || beta == nullptr || alpha == nullptr ||
      o_vda == nullptr)
    return VDN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o_vda, 16) ||
      !aligned(beta, 4) || !aligned(alpha, 4) || (states_opt && !aligned(states_opt, 16)))
    return VDN_ERR_INVALID_ARG;
  if (!ld_ok(ld, D) || !ld_ok(ld_o, D)) return VDN_ERR_INVALID_ARG;
  const VdaPlan pl = vda_plan(s);
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < pl.total) return VDN_ERR_WORKSPACE;

  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* inner = base + pl.inner_off;
  float* A = reinterpret_cast<float*>(inner + pl.lay.A);
  float* B = reinterpret_cast<float*>(inner + pl.lay.B);
  float* P = reinterpret_cast<float*>(inner + pl.lay.P);
  float* states_ws = reinterpret_cast<float*>(inner + pl.lay.states);
  Launch ctx{static_cast<cudaStream_t>(stream), reinterpret_cast<uint32_t*>(ws),
             g_budget_ns.load()};
  if (clear_status && cudaMemsetAsync(ws, 0, sizeof(uint32_t), ctx.stream) != cudaSuccess)
    return VDN_ERR_CUDA;
  if (!pl.padded)
    return run_vda(ctx, s, q, k, v, ld, beta, alpha, o_vda, ld_o, A, B, P,
                   states_opt ? states_opt : states_ws);

  // d = 16 or 32: run on a zero-padded 64-wide copy of every head
  const int L = s.T * s.N, H = s.H, d = s.d;
  const int64_t D64 = static_cast<int64_t>(H) * 64;
  uint8_t* qp = base + kStatusBytes;
  uint8_t* kp = qp + pl.act;
  uint8_t* vp = kp + pl.act;
  uint8_t* op = vp + pl.act;
  cudaStream_t st = ctx.stream;
  if (launch_repack_bf16(st, qp, D64, q, ld, 1, L, L, H, 64, d) != cudaSuccess ||
      launch_repack_bf16(st, kp, D64, k, ld, 1, L, L, H, 64, d) != cudaSuccess ||
      launch_repack_bf16(st, vp, D64, v, ld, 1, L, L, H, 64, d) != cudaSuccess)
    return VDN_ERR_CUDA;
  const vdn_status r =
      run_vda(ctx, pl.inner, qp, kp, vp, D64, beta, alpha, op, D64, A, B, P, states_ws);
  if (r != VDN_OK) return r;
  if (launch_repack_bf16(st, o_vda, ld_o, op, D64, 1, L, L, H, d, 64) != cudaSuccess)
    return VDN_ERR_CUDA;
  if (states_opt != nullptr &&
      launch_repack_f32(st, states_opt, d, states_ws, 64, 2 * s.T * H, d, 64, 1, d, 64) !=
          cudaSuccess)
    return VDN_ERR_CUDA;
  return VDN_OK;
}

extern "C" {

// ----------------------------------------------------------------- VDA gradients

size_t vdn_vda_backward_workspace(const vdn_shape* shape) {
  if (!shape_ok(shape)) return 0;
  return vda_plan(*shape, true).total;
}

vdn_status vdn_vda_backward_debug_buffers(const vdn_shape* shape, void* ws, float** states,
                                          float** adj, float** E) {
  if (!shape_ok(shape) || ws == nullptr) return VDN_ERR_INVALID_ARG;
  const VdaPlan pl = vda_plan(*shape, true);
  uint8_t* base = static_cast<uint8_t*>(ws) + pl.inner_off;
  if (states) *states = reinterpret_cast<float*>(base + pl.lay.states);
  if (adj) *adj = reinterpret_cast<float*>(base + pl.lay.A);
  if (E) *E = reinterpret_cast<float*>(base + pl.lay.X);
  return VDN_OK;
}

vdn_status vdn_vda_backward(const vdn_shape* shape, const void* q, const void* k, const void* v,
                            int64_t ld, const float* beta, const float* alpha, const void* d_o,
                            int64_t ld_do, void* dq, void* dk, void* dv, int64_t ld_g,
                            float* dbeta, float* dalpha, int reuse_forward, void* ws,
                            size_t ws_bytes, void* stream) {
  NvtxRange nvtx("vdn_vda_backward");
  if (!shape_ok(shape)) return VDN_ERR_INVALID_ARG;
  const vdn_shape s = *shape;
  if (!head_dim_supported(s.d)) return VDN_ERR_UNSUPPORTED;
  const int64_t D = static_cast<int64_t>(s.H) * s.d;
  if (q == nullptr || k == nullptr || v == nullptr || beta == nullptr || alpha == nullptr ||
      d_o == nullptr || dq == nullptr || dk == nullptr || dv == nullptr || dbeta == nullptr ||
      dalpha == nullptr)
    return VDN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(d_o, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(beta, 4) ||
      !aligned(alpha, 4) || !aligned(dbeta, 4) || !aligned(dalpha, 4))
    return VDN_ERR_INVALID_ARG;
  if (!ld_ok(ld, D) || !ld_ok(ld_do, D) || !ld_ok(ld_g, D)) return VDN_ERR_INVALID_ARG;
  const VdaPlan pl = vda_plan(s, true);
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < pl.total) return VDN_ERR_WORKSPACE;

  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* inner = base + pl.inner_off;
  float* A = reinterpret_cast<float*>(inner + pl.lay.A);
  float* B = reinterpret_cast<float*>(inner + pl.lay.B);
  float* P = reinterpret_cast<float*>(inner + pl.lay.P);
  float* X = reinterpret_cast<float*>(inner + pl.lay.X);
  float* states = reinterpret_cast<float*>(inner + pl.lay.states);
  Launch ctx{static_cast<cudaStream_t>(stream), reinterpret_cast<uint32_t*>(ws),
             g_budget_ns.load()};
  if (!pl.padded)
    return run_vda_backward(ctx, s, q, k, v, ld, beta, alpha, d_o, ld_do, dq, dk, dv, ld_g,
                            dbeta, dalpha, A, B, P, X, states, reuse_forward != 0);

  // d = 16 or 32: every head zero-padded to 64 columns (exact, see repack.cu)
  const int L = s.T * s.N, H = s.H, d = s.d;
  const int64_t D64 = static_cast<int64_t>(H) * 64;
  // q' k' v' dO' (the forward's slots; o' takes dO'), then dq' dk' dv'
  uint8_t* pad[7];
  for (int i = 0; i < 4; ++i) pad[i] = base + kStatusBytes + i * pl.act;
  for (int i = 0; i < 3; ++i) pad[4 + i] = base + pl.extra + i * pl.act;
  const void* src[4] = {q, k, v, d_o};
  const int64_t lds[4] = {ld, ld, ld, ld_do};
  cudaStream_t st = ctx.stream;
  for (int i = reuse_forward ? 3 : 0; i < 4; ++i)  // a reused forward left q' k' v' in place
    if (launch_repack_bf16(st, pad[i], D64, src[i], lds[i], 1, L, L, H, 64, d) != cudaSuccess)
      return VDN_ERR_CUDA;
  const vdn_status r = run_vda_backward(ctx, pl.inner, pad[0], pad[1], pad[2], D64, beta, alpha,
                                        pad[3], D64, pad[4], pad[5], pad[6], D64, dbeta, dalpha,
                                        A, B, P, X, states, reuse_forward != 0);
  if (r != VDN_OK) return r;
  void* dst[3] = {dq, dk, dv};
  for (int i = 0; i < 3; ++i)
    if (launch_repack_bf16(st, dst[i], ld_g, pad[4 + i], D64, 1, L, L, H, d, 64) != cudaSuccess)
      return VDN_ERR_CUDA;
  return VDN_OK;
}

}  // extern "C"
