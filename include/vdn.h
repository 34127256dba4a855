/*
 * vdn.h - C ABI of the B200 (sm_100a) forward pass of VideoDeltaNet's hybrid
 * attention layer (VDN-MiniMax-H3).
 *
 * The layer, as the pages describe it:
 *  - latent frames are grouped into blocks of 5 consecutive frames; a block
 *    attends exactly (softmax) with itself and its two neighbouring blocks,
 *    and the first and last frames are boundary anchors visible to every
 *    block ["VDN-MiniMax-H3" (openi.cn), section 技术原理：局部精确、远程压缩;
 *    "VDN-MiniMax-H3 - OpenVDN's Open-Source Video Generation Acceleration
 *    Solution" (nav.superapi.store), Technical Principles, Local Softmax
 *    Branch];
 *  - text tokens are visible to every frame in the softmax branch and are
 *    written once into the linear state at initialisation [nav.superapi.store
 *    page, Technical Principles, Text Dual-Branch Injection];
 *  - Video Delta Attention (VDA): one joint normal-equation solve per frame
 *    replaces the token-by-token delta rule [nav.superapi.store page,
 *    Technical Principles, Video Delta Attention];
 *  - the linear branch sums the context before and after the current window,
 *    leaving out the window frames and the anchors [openi.cn page, same
 *    section];
 *  - each branch has a content-dependent sigmoid gate and the linear output
 *    is RMS-normalised before its gate [openi.cn page, same section, last
 *    paragraph; nav.superapi.store page, Gated Fusion Mechanism].
 *
 * The pages print no formulas; this library implements one fixed reading:
 *   o_soft = softmax(q K^T / sqrt(d)) V over the keys of frames in
 *            {window of the query's block} U {0, F-1} and all text tokens;
 *   k_hat  = k / max(||k||_2, 1e-12)  (VDA only, video and text keys);
 *   S_text = (lambda I + Kt^T Kt)^-1 Kt^T Vt;
 *   S_f    = (lambda I + K_f^T K_f)^-1 (lambda S_prev + K_f^T V_f);
 *   forward scan over frames 1..F-2 and backward scan over F-2..1, both
 *   starting from S_text; block b reads R_b = Sfwd[max(w0-1,0)] +
 *   Sbwd[min(w1+1,F-1)] where [w0, w1] is its window, Sfwd[0] = Sbwd[F-1] =
 *   S_text; o_lin = q^T R_b;
 *   out = sigmoid(g_s) o_soft + sigmoid(g_l) * w_h * o_lin / sqrt(mean(o_lin^2) + eps).
 *
 * Conventions for every entry point
 *  - Token-major packed layouts, row-major and contiguous:
 *      q, k, v, out, o_soft : [N, H, d]       (N = off_host[F])
 *      kt, vt               : [T, H, d]
 *      g_s, g_l             : [N, H]
 *      rms_w                : [H, d] fp32
 *      states               : [.., H, d, d] fp32, S[key dim][value dim]
 *    Element type of q, k, v, kt, vt, g_s, g_l and out is shape->dtype
 *    (bf16 or fp32). fp32 inputs are narrowed to bf16 on entry (the tensor
 *    cores compute in bf16 with fp32 accumulation); d < 128 is zero-padded to
 *    128 internally.
 *  - All tensor pointers are DEVICE pointers, 16-byte aligned, owned by the
 *    caller; except shape->off_host, which is a host pointer. The library
 *    never allocates, frees or synchronises on the caller's behalf: it
 *    enqueues kernels on `stream` (a cudaStream_t, NULL = legacy default
 *    stream) and returns. `workspace` must hold at least
 *    vdn_workspace_bytes(shape) bytes and stay valid until the work
 *    completes; calls that share a workspace must be ordered on one stream.
 *  - Errors: every argument is validated on the host before anything is
 *    launched, so a call that returns an error has written nothing.
 *    Return value 0 = VDN_OK, otherwise one of the negative VDN_ERR_* codes.
 *    VDN_ERR_CUDA reports a launch failure (cudaGetLastError). Device-side
 *    failures (a bounded wait that expired) are reported by
 *    vdn_get_device_error() after the caller synchronises.
 *  - Sizes: 2 <= F <= 4096, 0 <= T, 1 <= H, d in {32, 64, 128},
 *    block_frames >= 1, lambda > 0, rms_eps >= 0, frame sizes
 *    off[f+1] - off[f] >= 0, N * H * 128 < 2^31.
 */
#ifndef VDN_H_
#define VDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VDN_OK 0
#define VDN_ERR_INVALID_ARG (-1)
#define VDN_ERR_UNSUPPORTED (-2)
#define VDN_ERR_WORKSPACE_TOO_SMALL (-3)
#define VDN_ERR_MISALIGNED (-4)
#define VDN_ERR_CUDA (-5)
#define VDN_ERR_DEVICE_TIMEOUT (-6)
#define VDN_ERR_DEVICE (-7)

typedef enum { VDN_BF16 = 0, VDN_F32 = 1 } vdn_dtype_t;

/* Arithmetic of the per-branch output projections. */
#define VDN_PROJ_BF16 0 /* bf16 operands, fp32 accumulation                  */
#define VDN_PROJ_FP8 1  /* e4m3 operands with per-row scales, fp32 accumulation */

typedef struct vdn_shape {
  int32_t F;            /* latent frames                                   */
  int32_t T;            /* text tokens (0 allowed: S_text = 0)             */
  int32_t H;            /* heads                                           */
  int32_t d;            /* head dim: 32, 64 or 128                         */
  int32_t block_frames; /* frames per block; 5 on the pages                */
  float lambda;         /* VDA ridge weight; 1.0                           */
  float rms_eps;        /* RMSNorm epsilon; 1e-6                           */
  int32_t dtype;        /* vdn_dtype_t of the activations                  */
  const int32_t* off_host; /* [F+1] host copy of frame offsets (off[0]=0)   */
  const int32_t* off_dev;  /* [F+1] device copy of the same offsets         */
} vdn_shape_t;

/* Bytes of workspace every entry point below needs for this shape
 * (the maximum over entry points). Returns 0 if the shape is invalid. */
size_t vdn_workspace_bytes(const vdn_shape_t* shape);

/* Whole layer: softmax branch, VDA scans, readout, RMSNorm and gated merge.
 * Writes out [N, H, d] (dtype). rms_w may not be NULL. kt/vt may be NULL iff
 * T == 0. */
int vdn_hybrid_attn_fwd(const vdn_shape_t* shape, const void* q, const void* k,
                        const void* v, const void* kt, const void* vt,
                        const void* g_s, const void* g_l, const float* rms_w,
                        void* out, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Per-branch output projections. Each branch has its own sigmoid gate and its
 * own output projection before the merge [nav.superapi.store page, Technical
 * Principles, Gated Fusion Mechanism; openi.cn page, 技术原理, last
 * paragraph]; the pages run these linears in FP8. Reading implemented (gates
 * are per token and head, so they act before the projection):
 *   a_s = sigmoid(g_s) o_soft,  a_l = sigmoid(g_l) RMSNorm(o_lin)   [N, H, d]
 *   y   = W_s a_s + W_l a_l = [a_s | a_l] w_o^T,  w_o = [W_s | W_l] [D, 2 H d]
 * (heads flattened as h * d + j; w_o = [I | I] gives vdn_hybrid_attn_fwd's
 * output). These entry points need bf16 activations with d = 128
 * (VDN_ERR_UNSUPPORTED otherwise).
 * ------------------------------------------------------------------------- */

/* Workspace bytes of vdn_hybrid_attn_proj_fwd (0 if the arguments are
 * invalid): the layer's workspace plus the gated branches [N, 2H, 128] bf16
 * and, for VDN_PROJ_FP8, their e4m3 codes [N, 2H, 128] and row scales [N]. */
size_t vdn_proj_workspace_bytes(const vdn_shape_t* shape, int D, int precision);

/* The layer up to the merge, with the two gated branches kept apart:
 * branches [N, 2H, d] bf16 gets a_s in heads 0..H-1 and a_l in heads
 * H..2H-1 (so row n is the [2 H d] input of the projection). */
int vdn_hybrid_attn_branches(const vdn_shape_t* shape, const void* q, const void* k,
                             const void* v, const void* kt, const void* vt,
                             const void* g_s, const void* g_l, const float* rms_w,
                             void* branches, void* workspace, size_t ws_bytes,
                             void* stream);

/* y [M, D] bf16 = a [M, K] w [D, K]^T, fp32 accumulation (row-major, K
 * contiguous in both operands; w is laid out like a linear layer's weight).
 * VDN_PROJ_BF16: a, w bf16, scales ignored (may be NULL).
 * VDN_PROJ_FP8: a, w e4m3 codes (1 byte each), y[m, n] = a_scale[m] *
 * w_scale[n] * sum_k a[m, k] w[n, k]; a_scale [M], w_scale [D] fp32.
 * K % 16 == 0, K >= 16, D % 8 == 0, D >= 8, M >= 0. */
int vdn_linear(const void* a, const float* a_scale, const void* w, const float* w_scale,
               int64_t M, int K, int D, int precision, void* y, void* stream);

/* Per-row e4m3 quantisation of x [rows, K] bf16 (K % 16 == 0):
 * scales[r] = amax_r / 448 (1 for an all-zero row) and codes[r, k] =
 * e4m3(x[r, k] * (448 / amax_r)) rounded to nearest even with saturation,
 * all in fp32. Used for the weights (once, per output channel) and, inside
 * vdn_hybrid_attn_proj_fwd, for the gated branches (per token). */
int vdn_quantize_rows_e4m3(const void* x, int64_t rows, int K, void* codes, float* scales,
                           void* stream);

/* Whole layer with the per-branch output projections: y [N, D] bf16.
 * VDN_PROJ_BF16: w_o [D, 2 H d] bf16, w_scale NULL. VDN_PROJ_FP8: w_o holds
 * e4m3 codes [D, 2 H d] and w_scale [D] as written by vdn_quantize_rows_e4m3;
 * the gated branches are quantised per token on the fly. workspace must hold
 * vdn_proj_workspace_bytes(shape, D, precision). */
int vdn_hybrid_attn_proj_fwd(const vdn_shape_t* shape, const void* q, const void* k,
                             const void* v, const void* kt, const void* vt,
                             const void* g_s, const void* g_l, const float* rms_w,
                             const void* w_o, const float* w_scale, int D, int precision,
                             void* y, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * FP8 softmax branch. The pages pair FlashAttention-4 with FP8 on B200
 * [agentlenshq.com page, core-ideas table; aigc.douyoubuy.cn page, section
 * 07]. Reading implemented: QK^T and PV as e4m3 x e4m3 contractions with fp32
 * accumulation; q has one scale per (token, head) row, k and v one scale per
 * head over all video and text tokens (scale = amax / 448, codes rounded to
 * nearest even in fp32); P is rounded to e4m3 after the exponential (P <= 256
 * by the kernel's lazy rescale, so it needs no scale); the row sums use the
 * unrounded P. Same shapes and layouts as vdn_bsa_fwd / vdn_hybrid_attn_fwd;
 * bf16 activations with d = 128 only (VDN_ERR_UNSUPPORTED otherwise).
 * ------------------------------------------------------------------------- */

/* Workspace bytes of the two entry points below (0 if unsupported): the
 * layer's workspace plus the e4m3 codes of q, k, v, kt, vt, the q row scales
 * and the per-head amax words. */
size_t vdn_fp8_workspace_bytes(const vdn_shape_t* shape);

/* Softmax branch in e4m3: o_soft [N, H, d] bf16, lse [H, N] optional. */
int vdn_bsa_fwd_fp8(const vdn_shape_t* shape, const void* q, const void* k, const void* v,
                    const void* kt, const void* vt, void* o_soft, float* lse, void* workspace,
                    size_t ws_bytes, void* stream);

/* Whole layer with the e4m3 softmax branch; the linear branch, readout,
 * RMSNorm and gated merge as in vdn_hybrid_attn_fwd (readout and merge fused
 * into the e4m3 softmax kernel's epilogue, the readout contraction on the
 * bf16 q). Writes out [N, H, d] bf16. */
int vdn_hybrid_attn_fwd_fp8(const vdn_shape_t* shape, const void* q, const void* k,
                            const void* v, const void* kt, const void* vt, const void* g_s,
                            const void* g_l, const float* rms_w, void* out, void* workspace,
                            size_t ws_bytes, void* stream);

/* Measurement helper (no paper counterpart). Runs vdn_hybrid_attn_fwd (same
 * arguments) `iters` times (1..256) on `stream` with CUDA events recorded on
 * that stream between its kernels, waits for the stream, and writes the mean
 * time per layer, in ms, of each launch group to kernel_ms[5]:
 *   [0] fp32 narrowing / head-dim padding (about 0 when not needed),
 *   [1] Gram matrices + inverses, [2] forward/backward scans,
 *   [3] read-state packing, [4] softmax branch with the fused readout,
 *   RMSNorm and gated merge.
 * Unlike every other entry point it synchronises the stream and creates and
 * destroys its own events (host-side only; no device memory is allocated).
 * The event records add a few microseconds between kernels. */
int vdn_hybrid_attn_fwd_profile(const vdn_shape_t* shape, const void* q, const void* k,
                                const void* v, const void* kt, const void* vt,
                                const void* g_s, const void* g_l, const float* rms_w,
                                void* out, void* workspace, size_t ws_bytes, void* stream,
                                int iters, float* kernel_ms);

/* The layer split at the read states, so that the two branches can run on
 * different GPUs (branch-specific placement: the pages place the softmax and
 * the linear branch on different devices [openi.cn page, 主要功能 item 5;
 * nav.superapi.store page, Main Features, Branch-Specific Parallelism]).
 * vdn_vda_read_images runs the linear branch (Grams, inverses, scans) and
 * writes R_b = Sfwd + Sbwd of every (block, head) as one 32 KB bf16 tile,
 * [nb][H] tiles in the layout the fused readout loads; vdn_read_images_bytes
 * gives the size (nb * H * 32768). vdn_bsa_merge_fwd runs the softmax branch
 * with the readout, RMSNorm and gated merge in its epilogue, reading those
 * tiles from `rimg` (device memory of the calling GPU: copy them there
 * first). The two calls in a row equal vdn_hybrid_attn_fwd. Both take the
 * workspace of vdn_workspace_bytes(shape). */
size_t vdn_read_images_bytes(const vdn_shape_t* shape);

int vdn_vda_read_images(const vdn_shape_t* shape, const void* k, const void* v,
                        const void* kt, const void* vt, void* rimg, void* workspace,
                        size_t ws_bytes, void* stream);

int vdn_bsa_merge_fwd(const vdn_shape_t* shape, const void* q, const void* k, const void* v,
                      const void* kt, const void* vt, const void* g_s, const void* g_l,
                      const float* rms_w, const void* rimg, void* out, void* workspace,
                      size_t ws_bytes, void* stream);

/* Linear branch states only. read_states [nb, H, d, d] fp32 (required;
 * nb = ceil(F / block_frames)) gets R_b. Optional (NULL to skip):
 * text_state [H, d, d]; fwd_states [F, H, d, d] gets Sfwd[i] for
 * i = 0..F-2 (entry F-1 is not written); bwd_states [F, H, d, d] gets
 * Sbwd[j] for j = 1..F-1 (entry 0 is not written). */
int vdn_vda_scan(const vdn_shape_t* shape, const void* k, const void* v,
                 const void* kt, const void* vt, float* read_states,
                 float* text_state, float* fwd_states, float* bwd_states,
                 void* workspace, size_t ws_bytes, void* stream);

/* Readout and merge only: o_lin = q^T R_b, RMSNorm, sigmoid gates.
 * read_states [nb, H, d, d] fp32 as written by vdn_vda_scan; o_soft
 * [N, H, d] bf16 as written by vdn_bsa_fwd. Writes out [N, H, d] (dtype). */
int vdn_gate_merge(const vdn_shape_t* shape, const void* q,
                   const float* read_states, const void* o_soft,
                   const void* g_s, const void* g_l, const float* rms_w,
                   void* out, void* workspace, size_t ws_bytes, void* stream);

/* Softmax branch only. Writes o_soft [N, H, d] bf16 and, if lse != NULL,
 * lse [H, N] fp32 = log(sum_j exp(q.k_j / sqrt(d))) over the allowed keys. */
int vdn_bsa_fwd(const vdn_shape_t* shape, const void* q, const void* k,
                const void* v, const void* kt, const void* vt, void* o_soft,
                float* lse, void* workspace, size_t ws_bytes, void* stream);

/* Audit of the block schedule the kernels run: soft_pairs [F, F+1] int64
 * (device) counts the (query token, key token) pairs the softmax kernel
 * visits, per (query frame, key frame), with column F counting text keys;
 * lin_pairs [F, F] int64 (device) counts the pairs folded into the read
 * states the readout uses. Both are zeroed first. */
int vdn_pair_audit(const vdn_shape_t* shape, int64_t* soft_pairs,
                   int64_t* lin_pairs, void* stream);

/* Same results as vdn_vda_scan, for callers that cannot provide a workspace
 * (no paper counterpart: this is a deployment variant). Such callers are,
 * for instance, serving loops that cannot absorb the device-wide
 * synchronisation cudaMalloc / cudaFree imply, or plug-ins whose process
 * memory belongs to an allocator they have no handle to. Its scratch is a
 * 64 MiB array inside the library, resident on every GPU that loads the
 * library until the process exits; the call itself allocates nothing.
 * Limit: 128 KiB x H x (F - 1) for the per-frame matrices, plus
 * 128 KiB x H x ceil(F / block_frames) for the read states, plus (fp32 or
 * d < 128 inputs only) 256 B x H x (2N + 2T) of staged keys/values must fit
 * in 64 MiB; larger shapes return VDN_ERR_WORKSPACE_TOO_SMALL. The first call
 * in a CUDA context (normally once per device) looks up the array's device
 * address with cudaGetSymbolAddress, so make that first call before any
 * stream capture. All calls share the one array and every call overwrites
 * what it reads: calls that overlap on the GPU (other streams, other host
 * threads) race and must be ordered by the caller. Like every entry point
 * here it makes CUDA runtime calls, so it may not be called from a stream
 * host function (cudaLaunchHostFunc). */
int vdn_vda_scan_noalloc(const vdn_shape_t* shape, const void* k, const void* v,
                         const void* kt, const void* vt, float* read_states,
                         float* text_state, float* fwd_states, float* bwd_states,
                         void* stream);

/* Check of the library's failure detection (no paper counterpart). Launches
 * one CTA on `stream` that holds `tmem_cols` tensor-memory columns (0, or a
 * power of two from 32 to 512), waits on a shared-memory barrier phase that
 * nothing completes through the same bounded wait the kernels use, gives up
 * after limit_ns nanoseconds (1 <= limit_ns <= 1e9), frees the columns and
 * returns. Returns VDN_OK once launched (VDN_ERR_INVALID_ARG before any
 * launch for out-of-range arguments); vdn_get_device_error() then reports
 * VDN_ERR_DEVICE_TIMEOUT, and the device stays usable. */
int vdn_selftest_wait_timeout(int64_t limit_ns, int tmem_cols, void* stream);

/* Synchronises the current device, returns VDN_OK or the first device-side
 * error recorded since the last call (VDN_ERR_DEVICE_TIMEOUT for an expired
 * bounded wait), and clears it. */
int vdn_get_device_error(void);

/* Static string for a return code. */
const char* vdn_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* VDN_H_ */
