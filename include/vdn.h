/*
 * vdn.h -- C ABI of libvdn, the B200 (sm_100a) Video DeltaNet hybrid
 * attention layer.
 *
 * The layer replaces video-to-video Softmax attention inside a video DiT by
 * two branches ("Video DeltaNet", article on 10100.com, section 方法概述):
 *   1. window-and-anchor Softmax (方法概述 item 1): each query chunk of 5
 *      latent frames attends to itself and one chunk on each side; the first
 *      and last latent frames are anchors that every frame sees and that see
 *      every frame;                                   -> vdn_window_attn
 *   2. Video Delta Attention (方法概述 item 2): a frame-level delta rule whose
 *      state is S_t = (S_bar_t + B_t)(I + A_t)^-1 with S_bar_t = alpha_t S_{t-1},
 *      A_t = sum_i beta_i k_i k_i^T, B_t = sum_i beta_i v_i k_i^T over the
 *      tokens of frame t, run forward and backward over the frames (figure
 *      caption under 效率阶梯: forward and backward scans);         -> vdn_vda_scan
 *   3. branch calibration (方法概述 item 3): content-dependent sigmoid gate on
 *      the Softmax branch, RMSNorm then a sigmoid output gate on the linear
 *      branch, a separate output projection per branch, summed.
 *                                                     -> vdn_hybrid_fuse
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tokens are frame-major: token row r = t*N + i (frame t, spatial token i).
 *    Activations are row-major [L, ld] bf16 with L = T*N; head h occupies
 *    columns [h*d, (h+1)*d).  bf16 arrays are passed as `const void*`
 *    (IEEE bfloat16, 2 bytes per element).
 *  - Every pointer is DEVICE memory owned by the caller.  The library never
 *    allocates, frees or synchronises; every call only enqueues kernels on
 *    `stream` (a cudaStream_t; NULL = the legacy default stream) and returns.
 *  - Inputs are read-only; outputs are overwritten in full.
 *  - Pointers must be 16-byte aligned; leading dimensions (elements) must be
 *    multiples of 8 and >= H*d.
 *  - Workspaces are caller-allocated device memory of at least the size the
 *    matching *_workspace() query returns, 256-byte aligned.  The first 256
 *    bytes of every workspace hold the device status word (see
 *    vdn_get_device_status); call vdn_reset_device_status once after
 *    allocating a workspace.
 *  - Host-side argument errors return VDN_ERR_INVALID_ARG or
 *    VDN_ERR_UNSUPPORTED before anything is enqueued.  A failed launch
 *    returns VDN_ERR_CUDA.  Errors detected on the device (a non-positive
 *    Cholesky pivot or NaN, a wait that ran out of time, and in debug builds
 *    an index outside its tensor) are OR-ed into the workspace status word;
 *    no kernel traps.
 *  - Head dims: 64 and 128 run directly; 16 and 32 run on zero-padded
 *    64-wide copies of every head in the workspace (exact).  N, T, H >= 1.
 */
#ifndef VDN_H_
#define VDN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VDN_API __attribute__((visibility("default")))
#else
#define VDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VDN_OK = 0,
  VDN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or stride     */
  VDN_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head dim 96)    */
  VDN_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required      */
  VDN_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed               */
  VDN_ERR_NUMERIC = 5,     /* device: non-positive pivot or NaN in a solve    */
  VDN_ERR_TIMEOUT = 6,     /* device: a bounded wait ran out                   */
  VDN_ERR_BOUNDS = 7       /* device, debug builds: an index outside its tensor */
} vdn_status;

/* Problem shape: T latent frames, N tokens per frame, H heads, head dim d
 * (dk == dv == d). */
typedef struct {
  int T, N, H, d;
} vdn_shape;

/* ------------------------------------------------------------------------
 * Video Delta Attention (10100.com article, 方法概述 item 2; the scan
 * direction from the figure caption under 效率阶梯).
 *
 *   A_t,h = sum_{i in frame t} beta[i,h] k_i k_i^T
 *   B_t,h = sum_{i in frame t} beta[i,h] v_i k_i^T            ([v_dim, k_dim])
 *   P_t,h = (I + A_t,h)^-1   (Cholesky of the SPD matrix I + A)
 *   S_fwd_t = (alpha_t S_fwd_{t-1} + B_t) P_t,   S_fwd_{-1} = 0
 *   S_bwd_t = (alpha_t S_bwd_{t+1} + B_t) P_t,   S_bwd_T   = 0
 *   o_vda[t*N+i, h*d:(h+1)*d] = (S_fwd_t,h + S_bwd_t,h) q_i     (no q scale)
 *
 * q, k, v   : [L, ld] bf16 (keys are taken as given; normalise beforehand)
 * beta      : [L, H] fp32, row-major          (per-token write strength)
 * alpha     : [T, H] fp32, row-major          (per-frame decay)
 * o_vda     : [L, ld_o] bf16, output
 * states_opt: NULL, or fp32 [2, T, H, d, d] output: [0] = S_fwd, [1] = S_bwd,
 *             each state row-major [v_dim][k_dim]
 * ws        : >= vdn_vda_scan_workspace(shape) bytes.  After the call it
 *             also holds A, B and P (see vdn_vda_debug_buffers).
 * ------------------------------------------------------------------------ */
VDN_API size_t vdn_vda_scan_workspace(const vdn_shape* shape);

VDN_API vdn_status vdn_vda_scan(const vdn_shape* shape, const void* q, const void* k, const void* v,
                        int64_t ld, const float* beta, const float* alpha, void* o_vda,
                        int64_t ld_o, float* states_opt, void* ws, size_t ws_bytes,
                        void* stream);

/* Pointers into a VDA workspace to the per-(frame, head) fp32 matrices the
 * last vdn_vda_scan on that workspace produced, each [T, H, d, d]:
 * A, B (prep) and P = (I + A)^-1 (solve).  Any out pointer may be NULL.
 * Pure pointer arithmetic: enqueues nothing. */
VDN_API vdn_status vdn_vda_debug_buffers(const vdn_shape* shape, void* ws, float** A, float** B,
                                         float** P);

/* vdn_vda_scan without a workspace.  The paper has no counterpart: this
 * entry point exists for callers that cannot allocate device memory (for
 * example a plugin inside a host framework that owns every device
 * allocation, or a loop with a fixed memory budget where cudaMalloc is not
 * allowed).  It runs vdn_vda_scan's own validation and launch sequence, with
 * the same arguments minus ws/ws_bytes, on a fixed 64 MiB array of this
 * library's own device memory instead of a workspace; that array is present
 * on every GPU that loads the library until the process exits.  Every head
 * dim vdn_vda_scan takes (16, 32, 64, 128) is served; 16 and 32 run on
 * padded copies in the array, as they do in a workspace.
 *  - Limit: vdn_vda_scan_workspace(shape) must be <= 64 MiB (at d = 64 or
 *    128 that is 256 + 5 * T*H*d*d*4 bytes, e.g. T*H <= 204 at d = 128,
 *    <= 819 at d = 64); larger shapes return VDN_ERR_WORKSPACE before
 *    anything is enqueued.
 *  - The first call on a device looks up the array's device address (once
 *    per device, with that device current) and caches it; make that first
 *    call before any stream capture.  The cached address is not valid
 *    across cudaDeviceReset of that device.
 *  - Every call shares the one array: calls that overlap on the GPU (other
 *    streams, other host threads) race and corrupt each other's results.
 *    The array keeps the last call's contents; each call clears the status
 *    word it uses and overwrites everything else it reads.
 *  - dev_status_opt: NULL, or 4-byte aligned device memory that receives,
 *    as the call's last operation on `stream`, this call's device status
 *    bits (0 = ok, bit 0 = numeric failure, bit 1 = a wait ran out of time).
 * No cudaMalloc, cudaFree or allocating library routine is called. */
VDN_API vdn_status vdn_vda_scan_static(const vdn_shape* shape, const void* q, const void* k,
                                       const void* v, int64_t ld, const float* beta,
                                       const float* alpha, void* o_vda, int64_t ld_o,
                                       float* states_opt, unsigned* dev_status_opt,
                                       void* stream);

/* ------------------------------------------------------------------------
 * Gradients of Video Delta Attention, for training the branch (the staged
 * alignment of 10100.com article, 方法概述 item 3, trains it; the closed form
 * of item 2 is what is differentiated).
 *
 * Given dO = dLoss/do_vda, with G_t = sum_{i in t} dO_i q_i^T and the
 * adjoint states of the two scans
 *   D_fwd_t = (alpha_{t+1} D_fwd_{t+1} + G_t) P_t   (t = T-1 .. 0)
 *   D_bwd_t = (alpha_{t-1} D_bwd_{t-1} + G_t) P_t   (t = 0 .. T-1)
 * and dB_t = D_fwd_t + D_bwd_t, E_t = dA_t + dA_t^T with
 * dA_t = -(S_fwd_t^T D_fwd_t + S_bwd_t^T D_bwd_t):
 *   dq_i     = (S_fwd_t + S_bwd_t)^T dO_i
 *   dk_i     = beta_i (E_t k_i + dB_t^T v_i)
 *   dv_i     = beta_i dB_t k_i
 *   dbeta_i  = k_i . (E_t k_i / 2 + dB_t^T v_i)
 *   dalpha_t = <D_fwd_t, S_fwd_{t-1}> + <D_bwd_t, S_bwd_{t+1}>
 *
 * q, k, v, beta, alpha, ld: the forward's inputs (as for vdn_vda_scan).
 * d_o       : [L, ld_do] bf16, dLoss/do_vda
 * dq, dk, dv: [L, ld_g] bf16, outputs (columns past H*d are not written)
 * dbeta     : [L, H] fp32 output;  dalpha: [T, H] fp32 output
 * ws        : >= vdn_vda_backward_workspace(shape) bytes.
 * reuse_forward: 0 -> the call recomputes the forward's A, B, P and states
 *             in its workspace (about a third of its time at d = 128) and
 *             needs nothing kept from the forward call.  Non-zero -> ws
 *             already holds them: the last vdn_vda_scan on this same
 *             workspace ran on the same q, k, v, beta, alpha with
 *             states_opt == NULL (a forward workspace is a prefix of a
 *             gradient-pass workspace, so one allocation of the larger size
 *             serves both), and prep, solve and scan are skipped.  Stale
 *             contents give wrong gradients; nothing checks this.
 * Errors as for vdn_vda_scan.
 * ------------------------------------------------------------------------ */
VDN_API size_t vdn_vda_backward_workspace(const vdn_shape* shape);

VDN_API vdn_status vdn_vda_backward(const vdn_shape* shape, const void* q, const void* k,
                                    const void* v, int64_t ld, const float* beta,
                                    const float* alpha, const void* d_o, int64_t ld_do, void* dq,
                                    void* dk, void* dv, int64_t ld_g, float* dbeta, float* dalpha,
                                    int reuse_forward, void* ws, size_t ws_bytes, void* stream);

/* Pointers into a backward workspace, after vdn_vda_backward on it, to fp32
 * [2, T, H, d, d] arrays: states ([0] = S_fwd, [1] = S_bwd), adjoint
 * states ([0] = D_bwd, [1] = D_fwd), and E [T, H, d, d].  For head dims 16
 * and 32 the arrays are those of the zero-padded 64-wide problem.  Any out
 * pointer may be NULL.  Pure pointer arithmetic: enqueues nothing. */
VDN_API vdn_status vdn_vda_backward_debug_buffers(const vdn_shape* shape, void* ws,
                                                  float** states, float** adj, float** E);

/* ------------------------------------------------------------------------
 * MXFP8 projections (10100.com article, 实验结果 / 效率阶梯 times the
 * denoiser under MXFP8; the format is the OCP Microscaling one).
 *
 * An MXFP8 operand [R, K] (K-major, K a multiple of 128) is a pair:
 *  - codes: R x K bytes, row-major, E4M3 (bias 7, no infinities, +-448 max);
 *  - scales: vdn_mxfp8_scale_bytes(R, K) bytes of UE8M0 (2^(byte - 127)),
 *    one per 32 consecutive elements of a row, in the tile layout the
 *    block-scaled tensor-core MMA reads: per 128-row x 128-column tile one
 *    512-byte block; the scale of (row r, column block kb = k / 32) is byte
 *    (r % 32) * 16 + ((r % 128) / 32) * 4 + kb % 4 of block number
 *    (r / 128) * (K / 128) + k / 128; rows past R up to the next multiple
 *    of 128 hold 127 (scale 1).
 * Quantization: per block e = floor(log2(max|v|)) - 8 clamped to
 * [-127, 127] (-127 for a zero block); code = E4M3(v * 2^-e), round to
 * nearest even, saturated at +-448; scale byte = e + 127.
 * ------------------------------------------------------------------------ */
VDN_API size_t vdn_mxfp8_scale_bytes(int64_t rows, int64_t cols);

/* x bf16 [rows, ld] -> q codes [rows, cols] and sf scales (sizes above).
 * cols a multiple of 128, ld >= cols and a multiple of 8; x, q 16-byte
 * aligned.  One kernel on `stream`. */
VDN_API vdn_status vdn_mxfp8_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                      void* q, void* sf, void* stream);

/* C [M, N] = A [M, K] B [N, K]^T on MXFP8 operands (codes and scales as
 * above, row stride K bytes), fp32 accumulation; C row-major with row
 * stride N, bf16 (c_is_f32 = 0) or fp32 (c_is_f32 != 0).  K a multiple of
 * 128, N a multiple of 32; pointers 16-byte aligned; ws >= 256 bytes
 * (status word).  VDN_ERR_UNSUPPORTED for other shapes. */
VDN_API vdn_status vdn_gemm_mxfp8(int M, int N, int K, const void* a, const void* a_sf,
                                  const void* b, const void* b_sf, void* c, int c_is_f32,
                                  void* ws, size_t ws_bytes, void* stream);

/* vdn_hybrid_fuse with both projection GEMMs in MXFP8: x is quantized on
 * the device; the gate GEMM's epilogue forms Z = [g_s o_s | g_l RMSNorm(o_vda)
 * gamma] in fp32 and writes it quantized; y = Z [W_os | W_ol]^T.
 * wg_q / wg_sf: MXFP8 of the stacked gate weights [W_gs; W_gl] ([2D, D]);
 * wo_q / wo_sf: MXFP8 of [W_os | W_ol] ([D, 2D]) (vdn_mxfp8_quantize).
 * Shapes: D a multiple of 128, head dim d = D / H a multiple of 32 that
 * divides 128.  ws >= vdn_hybrid_fuse_mxfp8_workspace(L, D, H). */
VDN_API size_t vdn_hybrid_fuse_mxfp8_workspace(int L, int D, int H);

VDN_API vdn_status vdn_hybrid_fuse_mxfp8(int L, int D, int H, const void* x, const void* o_s,
                                         const void* o_vda, const void* wg_q, const void* wg_sf,
                                         const float* gamma, float eps, const void* wo_q,
                                         const void* wo_sf, void* y, void* ws, size_t ws_bytes,
                                         void* stream);

/* ------------------------------------------------------------------------
 * Window-and-anchor Softmax (10100.com article, 方法概述 item 1).
 *
 * Chunk c(t) = floor(t / chunk_frames).  Query frame tq sees key frame tk iff
 * |c(tq) - c(tk)| <= window_chunks, or (anchors & 1) and 0 in {tq, tk}, or
 * (anchors & 2) and T-1 in {tq, tk}.  All tokens of a frame share its mask.
 *   o[r, h] = softmax_{visible keys}(q_r k^T * scale) v,  per head
 *
 * q, k, v  : [L, ld] bf16;  o: [L, ld_o] bf16 output
 * scale    : <= 0 selects 1/sqrt(d)
 * lse_opt  : NULL, or fp32 [H, L] output: natural-log sum of exp(scaled
 *            scores) over the visible keys of each query row
 * ws       : >= vdn_window_attn_workspace(shape) bytes
 * chunk_frames >= 1, window_chunks >= 0, anchors in 0..3.
 * ------------------------------------------------------------------------ */
VDN_API size_t vdn_window_attn_workspace(const vdn_shape* shape);

VDN_API vdn_status vdn_window_attn(const vdn_shape* shape, const void* q, const void* k, const void* v,
                           int64_t ld, int chunk_frames, int window_chunks, unsigned anchors,
                           float scale, void* o, int64_t ld_o, float* lse_opt, void* ws,
                           size_t ws_bytes, void* stream);

/* Window-and-anchor Softmax with context keys.  The pages keep every
 * interaction with text or audio tokens as full Softmax (10100.com 方法概述
 * item 1; ai-feeds.com 方法).  Here every video query attends, in the same
 * softmax as its visible video keys, to all m_ctx context keys/values:
 *   o[r, h] = softmax over {visible video keys} U {context keys}.
 * ctx_k, ctx_v : [m_ctx, ld_ctx] bf16 (head h at columns [h*d, (h+1)*d)),
 *                may be NULL when m_ctx == 0.  Everything else as for
 *                vdn_window_attn, which is this call with m_ctx = 0. */
VDN_API vdn_status vdn_window_attn_ctx(const vdn_shape* shape, const void* q, const void* k,
                                       const void* v, int64_t ld, const void* ctx_k,
                                       const void* ctx_v, int64_t ld_ctx, int m_ctx,
                                       int chunk_frames, int window_chunks, unsigned anchors,
                                       float scale, void* o, int64_t ld_o, float* lse_opt,
                                       void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Window-and-anchor Softmax with MXFP8 products (10100.com article: the
 * window Softmax of 方法概述 item 1, run under the MXFP8 inference of
 * 实验结果 / 效率阶梯; the pages name the format only, the OCP Microscaling
 * definition is taken: E4M3 elements, one UE8M0 power-of-two scale per 32
 * elements along each product's contraction).
 *
 * Same mask and arguments as vdn_window_attn, and the same bf16 output; the
 * call quantizes into the workspace, then runs the attention:
 *   q, k : blocks of 32 along the head dim, per token and head;
 *   v    : blocks of 32 consecutive token rows (from row 0), per column;
 *   P    : blocks of 32 consecutive keys of a row, with P = 2^(s log2 e - m)
 *          for an integer row maximum m; the row sum adds the unquantized P,
 *          the output is sum(P^ v^) / sum(P).
 * lse_opt: NULL or fp32 [H, L], the natural log of the row sum of exp(s).
 * Supported: head dim 128 and N (tokens per frame) a multiple of 32, so
 * every visible key interval starts on a value block (else
 * VDN_ERR_UNSUPPORTED); no context keys.
 * ws: >= vdn_window_attn_mxfp8_workspace(shape) bytes, 256-byte aligned:
 *   status word, the E4M3 codes of q, k, v (3 x L x H*d bytes) and their
 *   scale bytes (2 x L x H*d/32 + ceil(L/32) x H*d).
 * Errors as for vdn_window_attn.
 * ------------------------------------------------------------------------ */
VDN_API size_t vdn_window_attn_mxfp8_workspace(const vdn_shape* shape);

VDN_API vdn_status vdn_window_attn_mxfp8(const vdn_shape* shape, const void* q, const void* k,
                                         const void* v, int64_t ld, int chunk_frames,
                                         int window_chunks, unsigned anchors, float scale,
                                         void* o, int64_t ld_o, float* lse_opt, void* ws,
                                         size_t ws_bytes, void* stream);

/* The window Softmax's work plan, as the kernel launch uses it (host only:
 * no CUDA call, no device memory).  Consecutive query frames with the same
 * visible key frames (the mask of vdn_window_attn) form a segment; segments
 * are listed heaviest first (most visible keys), the order their CTAs are
 * launched in.  Per segment, 12 ints into segs[12*g ..]:
 *   q0, q1        query token rows [q0, q1) (whole frames);
 *   tile_base     index of its first 256-row CTA tile in launch order;
 *   ntiles        its 256-row CTA tiles, ceil((q1 - q0) / 256);
 *   nint          key intervals (1..3: the window, frame 0, frame T-1);
 *   nkv           128-key tiles over those intervals (each rounded up);
 *   k0, k1 x 3    key token intervals [k0, k1), unused ones 0.
 * *nseg receives the number of segments.  Returns VDN_ERR_INVALID_ARG for
 * a bad argument or when max_segs < *nseg (nothing written to segs then),
 * VDN_ERR_UNSUPPORTED when the plan does not fit the kernel's fixed table
 * (more than 256 segments or 3 intervals), which vdn_window_attn reports
 * the same way. */
VDN_API vdn_status vdn_window_attn_schedule(const vdn_shape* shape, int chunk_frames,
                                            int window_chunks, unsigned anchors, int* segs,
                                            int max_segs, int* nseg);

/* ------------------------------------------------------------------------
 * Branch calibration and output projections (10100.com article, 方法概述
 * item 3; hotpaper.ai summary, 기술적 접근법).
 *
 *   g_s = sigmoid(x W_gs^T),  g_l = sigmoid(x W_gl^T)              (elementwise)
 *   n   = per-token, per-head RMSNorm of o_vda over d channels:
 *         n = o / sqrt(mean_d(o^2) + eps) * gamma
 *   y   = (g_s * o_s) W_os^T + (g_l * n) W_ol^T
 *
 * x, o_s, o_vda, y : [L, D] bf16, contiguous (ld = D), D = H*d
 * W_gs, W_gl, W_os, W_ol : [D, D] bf16 row-major, W[out][in] (y = z W^T)
 * gamma    : [D] fp32
 * ws       : >= vdn_hybrid_fuse_workspace(L, D, H) bytes (holds the gated
 *            branch outputs [L, 2D] bf16 between the two GEMMs)
 * D must be a multiple of 8 and of H; L >= 1.  Hidden sizes that are not a
 * multiple of 256, or head dims not a multiple of 32, run on zero-padded
 * copies of every head in the workspace (exact; the RMS divides by the true
 * head dim).
 * ------------------------------------------------------------------------ */
VDN_API size_t vdn_hybrid_fuse_workspace(int L, int D, int H);

VDN_API vdn_status vdn_hybrid_fuse(int L, int D, int H, const void* x, const void* o_s,
                           const void* o_vda, const void* W_gs, const void* W_gl,
                           const float* gamma, float eps, const void* W_os, const void* W_ol,
                           void* y, void* ws, size_t ws_bytes, void* stream);

/* One head shard of the fuse, for head-parallel multi-GPU runs of one video
 * (rank r of G owns heads [head0, head0 + H_local)).  The gates are
 * elementwise, so a shard computes its own hidden columns
 * c in [head0*d, (head0 + H_local)*d): Z_r = [sigmoid(x W_gs[c]^T) o_s_r |
 * sigmoid(x W_gl[c]^T) RMSNorm(o_vda_r) gamma[c]], and the partial
 *   y_partial = Z_r [W_os[:, c] | W_ol[:, c]]^T           (fp32, [L, D])
 * whose sum over the shards is y (the caller's all-reduce).
 * x: [L, D] bf16 (full); o_s, o_vda: [L, ld_o] bf16, this shard's heads only
 * (ld_o == H_local*d); W_*: the full [D, D] bf16 weights; gamma: full [D].
 * Requires d % 128 == 0 and D % 256 == 0.
 * ws: >= vdn_hybrid_fuse_shard_workspace(L, D, H_local, d) bytes. */
VDN_API size_t vdn_hybrid_fuse_shard_workspace(int L, int D, int H_local, int d);

VDN_API vdn_status vdn_hybrid_fuse_shard(int L, int D, int H_local, int d, int head0,
                                         const void* x, const void* o_s, const void* o_vda,
                                         int64_t ld_o, const void* W_gs, const void* W_gl,
                                         const float* gamma, float eps, const void* W_os,
                                         const void* W_ol, float* y_partial, void* ws,
                                         size_t ws_bytes, void* stream);

/* vdn_hybrid_fuse_shard with the reduce-scatter fused into the output
 * GEMM: instead of writing an fp32 partial, the GEMM's epilogue adds row r
 * of this shard's partial into y_owners[r / R] at row r % R, R = ceil(L / G),
 * with system-scope atomic adds (so the owners may be other GPUs' memory
 * reached through a peer mapping: CUDA IPC, a symmetric-memory allocation).
 * After every shard's call the owners hold the summed rows of y.
 *  - y_owners: host array of G device pointers (1 <= G <= 8), each fp32
 *    [R, D] (the last [L - (G-1) R, D]), 16-byte aligned.
 *  - The caller zeroes the owners' buffers before any shard's call and reads
 *    them only after every shard's call has finished (a barrier across the
 *    ranks' streams on both sides).  The sum's order is not fixed.
 *  - Other arguments, shapes and errors as for vdn_hybrid_fuse_shard.
 * Head-parallel runs were not possible here (one GPU); the single-GPU test
 * runs G shards into G owner buffers on one device. */
VDN_API vdn_status vdn_hybrid_fuse_shard_rs(int L, int D, int H_local, int d, int head0,
                                            const void* x, const void* o_s, const void* o_vda,
                                            int64_t ld_o, const void* W_gs, const void* W_gl,
                                            const float* gamma, float eps, const void* W_os,
                                            const void* W_ol, float* const* y_owners, int G,
                                            void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Status and diagnostics.
 * ------------------------------------------------------------------------ */

/* Static, human-readable message for a status code. */
VDN_API const char* vdn_status_string(vdn_status s);

/* Synchronise `stream`, then read the device status word of a workspace
 * (VDN_OK if no kernel recorded an error since the last reset). */
VDN_API vdn_status vdn_get_device_status(const void* ws, void* stream);

/* Enqueue a clear of the workspace's device status word on `stream`. */
VDN_API vdn_status vdn_reset_device_status(void* ws, void* stream);

/* 1 if this library was built with VDN_DEBUG_BOUNDS=1: every hand-computed
 * global store (and tile start) is checked against its tensor's extents,
 * and a miss is recorded as VDN_ERR_BOUNDS in the status word and the
 * access skipped, instead of faulting; 0 for release builds, where the
 * checks are compiled out.  Debug scaffolding (the paper has no
 * counterpart). */
VDN_API int vdn_debug_bounds_enabled(void);

/* Self-test of the bounds check: one device thread checks row `r` and
 * columns [c, c + width) against a rows x cols tensor, touching no memory
 * but the status word of `ws`.  In a debug build an out-of-range index sets
 * VDN_ERR_BOUNDS (read it with vdn_get_device_status); a release build
 * records nothing.  Enqueued on `stream`. */
VDN_API vdn_status vdn_selftest_bounds(void* ws, int64_t r, int64_t rows, int64_t c,
                                       int64_t width, int64_t cols, void* stream);

/* Pitched copy, enqueued on `stream` (cudaMemcpy2DAsync, the direction taken
 * from the pointers): `rows` rows of `width_bytes` bytes, rows `src_pitch`
 * bytes apart in the source and `dst_pitch` in the destination.  Data
 * movement only (the paper has no counterpart): it lets a caller stream a
 * block of columns of a row-major host activation, for example the heads of
 * one group, into a device buffer, so that work on those heads can start
 * before the rest has arrived.  Host memory must be pinned for the copy to
 * be asynchronous.  VDN_ERR_INVALID_ARG for null pointers or a width above
 * either pitch; VDN_ERR_CUDA if the copy cannot be enqueued. */
VDN_API vdn_status vdn_copy2d_async(void* dst, size_t dst_pitch, const void* src,
                                    size_t src_pitch, size_t width_bytes, size_t rows,
                                    void* stream);

/* Wall-clock budget (ns) of every bounded wait inside the kernels launched
 * after this call (default 2e9).  0 makes any wait that is not already
 * satisfied fail at once with VDN_ERR_TIMEOUT: a test hook for the timeout
 * path.  Process-wide; not thread-safe against concurrent launches. */
VDN_API void vdn_set_wait_budget_ns(uint64_t ns);

/* Diagnostic: y_fma[i] = 2^x[i] by the FMA-pipe exponential the Softmax uses
 * for part of its scores (range reduction x = n + f, cubic for 2^f, 2^n added
 * to the exponent; inputs below -125 are clamped there), and y_mufu[i] =
 * 2^x[i] by the hardware ex2.approx.  Device pointers, n >= 0 floats;
 * enqueued on `stream`. */
VDN_API vdn_status vdn_selftest_exp2(const float* x, float* y_fma, float* y_mufu, int n,
                                     void* stream);

/* Solver for (I + A_t)^-1 in the VDA path, process-wide, for calls enqueued
 * after this one: VDN_SOLVER_GAUSS_JORDAN (default: an in-register
 * Gauss-Jordan sweep, the variant the 10100.com article's 消融 section
 * reports for its own kernels) or VDN_SOLVER_CHOLESKY (blocked Cholesky,
 * W = L^-1, P = W^T W).  Both give P to within a few 1e-5 of the exact
 * inverse (relative to max |P|).  Returns VDN_ERR_INVALID_ARG for other
 * values.  Not thread-safe against concurrent launches. */
#define VDN_SOLVER_CHOLESKY 0
#define VDN_SOLVER_GAUSS_JORDAN 1
VDN_API vdn_status vdn_set_vda_solver(int solver);

/* Library version string. */
VDN_API const char* vdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VDN_H_ */
