// C ABI of the hybrid attention layer (declared in include/vdn.h).
// Host side only: argument validation, workspace carving, TMA descriptor
// encoding and kernel launches on the caller's stream. Single translation
// unit (the kernels are header-only), so one device error word serves all
// kernels.
#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include "../../include/vdn.h"
#include "k_audit.cuh"
#include "k_bsa_fwd.cuh"
#include "k_linear.cuh"
#include "k_merge.cuh"
#include "k_prepare.cuh"
#include "k_quant_attn.cuh"
#include "k_vda.cuh"
#include "layer_plan.cuh"
#include "sm100_ptx.cuh"

namespace {

using namespace vdn;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [rows, H, 128] bf16 viewed as a 3-D tensor {128, H, rows}; box {64, 1, box_rows}.
bool map_act(CUtensorMap* m, const void* ptr, int64_t rows, int H, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kDPad, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)kDPad * 2, (cuuint64_t)H * kDPad * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, H, 128] e4m3 codes as a 3-D tensor {128, H, rows}; box {128, 1, box_rows}.
bool map_act8(CUtensorMap* m, const void* ptr, int64_t rows, int H, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kDPad, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)kDPad, (cuuint64_t)H * kDPad};
  cuuint32_t box[3] = {128, 1, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, 128] fp32 as a 2-D tensor; box {32, box_rows}.
bool map_mat(CUtensorMap* m, const void* ptr, int64_t rows, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)128, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)128 * 4};
  cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// [rows, inner] row-major matrix of 2-byte (bf16) or 1-byte (raw e4m3)
// elements; box {box_inner, box_rows}, 128-byte swizzle (box_inner x element
// size must be 128 B).
bool map_rows(CUtensorMap* m, const void* ptr, int64_t inner, int64_t rows, int esize,
              int box_inner, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(inner * esize)};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
             const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

__global__ void k_sum_states(const float* a, const float* b, float* out, int64_t n, int d) {
  // out[(bh, i, j)] = a[(bh, i, j)] + b[(bh, i, j)] with a, b padded to 128 x 128
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n) return;
  const int64_t bh = t / ((int64_t)d * d);
  const int r = (int)((t / d) % d), c = (int)(t % d);
  const int64_t src = (bh * 128 + r) * 128 + c;
  out[t] = a[src] + b[src];
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Plan {
  int F, T, H, d, bf, nb, N;
  float lambda, eps;
  int dtype;
  int max_qtiles;
  bool staged;  // inputs are narrowed / padded into the workspace
  size_t o_q, o_k, o_v, o_kt, o_vt, o_C, o_W, o_R, o_Rimg, total;
  const int32_t* off_dev;
};

int make_plan(const vdn_shape_t* s, Plan* P) {
  if (s == nullptr) return VDN_ERR_INVALID_ARG;
  if (s->F < 2 || s->F > 4096 || s->T < 0 || s->H < 1 || s->block_frames < 1)
    return VDN_ERR_INVALID_ARG;
  if (!(s->d == 32 || s->d == 64 || s->d == 128)) return VDN_ERR_UNSUPPORTED;
  if (!(s->lambda > 0.f) || !std::isfinite(s->lambda) || !(s->rms_eps >= 0.f) ||
      !std::isfinite(s->rms_eps))
    return VDN_ERR_INVALID_ARG;
  if (s->dtype != VDN_BF16 && s->dtype != VDN_F32) return VDN_ERR_UNSUPPORTED;
  if (s->off_host == nullptr || s->off_dev == nullptr) return VDN_ERR_INVALID_ARG;
  if (s->off_host[0] != 0) return VDN_ERR_INVALID_ARG;
  for (int f = 0; f < s->F; ++f)
    if (s->off_host[f + 1] < s->off_host[f]) return VDN_ERR_INVALID_ARG;
  const int64_t N = s->off_host[s->F];
  if (N * (int64_t)s->H * kDPad >= (int64_t(1) << 31)) return VDN_ERR_UNSUPPORTED;
  if ((int64_t)s->T * s->H * kDPad >= (int64_t(1) << 31)) return VDN_ERR_UNSUPPORTED;
  if ((int64_t)(s->F - 1) * s->H * 128 >= (int64_t(1) << 31)) return VDN_ERR_UNSUPPORTED;
  P->F = s->F;
  P->T = s->T;
  P->H = s->H;
  P->d = s->d;
  P->bf = s->block_frames;
  P->nb = num_blocks(s->F, s->block_frames);
  P->N = (int)N;
  P->lambda = s->lambda;
  P->eps = s->rms_eps;
  P->dtype = s->dtype;
  P->off_dev = s->off_dev;
  P->max_qtiles = 0;
  for (int b = 0; b < P->nb; ++b) {
    int q0, q1;
    block_rows(s->off_host, P->F, P->bf, b, q0, q1);
    P->max_qtiles = imax(P->max_qtiles, (q1 - q0 + kTile - 1) / kTile);
  }
  P->staged = (s->dtype != VDN_BF16) || (s->d != kDPad);
  const size_t act = (size_t)N * P->H * kDPad * 2;
  const size_t txt = (size_t)P->T * P->H * kDPad * 2;
  const size_t mat = (size_t)(P->F - 1) * P->H * 128 * 128 * 4;
  size_t o = 0;
  P->o_q = o; o += P->staged ? align256(act) : 0;
  P->o_k = o; o += P->staged ? align256(act) : 0;
  P->o_v = o; o += P->staged ? align256(act) : 0;
  P->o_kt = o; o += P->staged ? align256(txt) : 0;
  P->o_vt = o; o += P->staged ? align256(txt) : 0;
  P->o_C = o; o += align256(mat);
  P->o_W = o; o += align256(mat);
  P->o_R = o; o += align256((size_t)2 * P->nb * P->H * 128 * 128 * 4);
  P->o_Rimg = o; o += align256((size_t)P->nb * P->H * kRImageBytes);
  P->total = o;
  return VDN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Kernel attribute set-up, once per device.
bool set_smem_attrs() {
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (done[dev]) return true;
  bool ok = cudaFuncSetAttribute(k_bsa_fwd<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kBsaSmemBytes) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_bsa_fwd<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kBsaMergeSmemBytes) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_bsa_fwd<0, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kBsa8SmemBytes) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_bsa_fwd<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kBsa8MergeSmemBytes) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_bsa_fwd<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kBsaMergeSmemBytes) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_linear<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kLinSmemBytes) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_linear<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kLinSmemBytes) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_vda_gram_inv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kGramSmemBytes) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_vda_scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kScanSmemBytes) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_readout_merge, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kMergeSmemBytes) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_readout_merge_tma, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kMergeTmaSmemBytes) == cudaSuccess;
  done[dev] = ok;
  return ok;
}

// bf16 [rows, H, 128] views of the activations, staged into the workspace
// when the caller's tensors are fp32 or narrower than 128.
struct Acts {
  const __nv_bfloat16 *q, *k, *v, *kt, *vt;
};

int stage_one(const Plan& P, const void* src, int64_t rows, void* dst, cudaStream_t st) {
  if (rows == 0) return VDN_OK;
  const int64_t rh = rows * P.H;
  const int64_t units = rh * (kDPad / 8);
  const int threads = 256;
  const int blocks = (int)imin((int)((units + threads - 1) / threads), 148 * 16);
  if (P.dtype == VDN_F32)
    k_pad_to_bf16<float><<<blocks, threads, 0, st>>>(static_cast<const float*>(src),
                                                     static_cast<__nv_bfloat16*>(dst), rh, P.d);
  else
    k_pad_to_bf16<__nv_bfloat16><<<blocks, threads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(src), static_cast<__nv_bfloat16*>(dst), rh, P.d);
  return VDN_OK;
}

Acts stage_inputs(const Plan& P, const void* q, const void* k, const void* v, const void* kt,
                  const void* vt, uint8_t* ws, cudaStream_t st, bool need_q, bool need_kv) {
  Acts a;
  if (!P.staged) {
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.kt = static_cast<const __nv_bfloat16*>(kt);
    a.vt = static_cast<const __nv_bfloat16*>(vt);
    return a;
  }
  a.q = reinterpret_cast<const __nv_bfloat16*>(ws + P.o_q);
  a.k = reinterpret_cast<const __nv_bfloat16*>(ws + P.o_k);
  a.v = reinterpret_cast<const __nv_bfloat16*>(ws + P.o_v);
  a.kt = reinterpret_cast<const __nv_bfloat16*>(ws + P.o_kt);
  a.vt = reinterpret_cast<const __nv_bfloat16*>(ws + P.o_vt);
  if (need_q) stage_one(P, q, P.N, ws + P.o_q, st);
  if (need_kv) {
    stage_one(P, k, P.N, ws + P.o_k, st);
    stage_one(P, v, P.N, ws + P.o_v, st);
    stage_one(P, kt, P.T, ws + P.o_kt, st);
    stage_one(P, vt, P.T, ws + P.o_vt, st);
  }
  return a;
}

// TMA maps; empty tensors get a never-dereferenced map over the workspace.
bool act_map(CUtensorMap* m, const void* ptr, int64_t rows, const Plan& P, int box, void* dummy) {
  if (rows == 0) return map_act(m, dummy, 1, P.H, box);
  return map_act(m, ptr, rows, P.H, box);
}

int launch_vda(const Plan& P, const Acts& a, uint8_t* ws, cudaStream_t st, float* text_out,
               float* fwd_out, float* bwd_out, cudaEvent_t after_gram = nullptr) {
  CUtensorMap tk, tv, tkt, tvt, tw, tct;
  if (!act_map(&tk, a.k, P.N, P, 64, ws + P.o_C) || !act_map(&tv, a.v, P.N, P, 64, ws + P.o_C) ||
      !act_map(&tkt, a.kt, P.T, P, 64, ws + P.o_C) ||
      !act_map(&tvt, a.vt, P.T, P, 64, ws + P.o_C) ||
      !map_mat(&tw, ws + P.o_W, (int64_t)(P.F - 1) * P.H * 128, 128) ||
      !map_mat(&tct, ws + P.o_C, (int64_t)(P.F - 1) * P.H * 128, kScanHalf))
    return VDN_ERR_CUDA;
  // Frames the read states depend on (all of them when per-frame states are
  // requested): forward reads go up to fwd_last, backward reads down to bwd_first.
  int fwd_last = 0, bwd_first = P.F - 1;
  for (int b = 0; b < P.nb; ++b) {
    int i_f, i_b;
    block_read_indices(b, P.F, P.bf, i_f, i_b);
    fwd_last = imax(fwd_last, i_f);
    bwd_first = imin(bwd_first, i_b);
  }
  if (fwd_out != nullptr || bwd_out != nullptr) {
    fwd_last = P.F - 2;
    bwd_first = 1;
  }
  const int n_fwd = fwd_last;                                   // frames 1..fwd_last
  const int n_bwd = imax(0, (P.F - 2) - imax(bwd_first, fwd_last + 1) + 1);
  GramParams gp;
  gp.off = P.off_dev;
  gp.F = P.F;
  gp.T = P.T;
  gp.H = P.H;
  gp.fwd_last = fwd_last;
  gp.bwd_first = bwd_first;
  gp.lambda = P.lambda;
  gp.Cmat = reinterpret_cast<float*>(ws + P.o_C);
  gp.Wmat = reinterpret_cast<float*>(ws + P.o_W);
  k_vda_gram_inv<<<dim3(1 + n_fwd + n_bwd, P.H), kGramThreads, kGramSmemBytes, st>>>(tk, tv, tkt,
                                                                                   tvt, gp);
  if (after_gram != nullptr) cudaEventRecord(after_gram, st);
  ScanParams sp;
  sp.F = P.F;
  sp.H = P.H;
  sp.bf = P.bf;
  sp.nb = P.nb;
  sp.steps_fwd = 1 + fwd_last;
  sp.steps_bwd = 1 + (P.F - 1 - bwd_first);
  sp.lambda = P.lambda;
  sp.Rpart = reinterpret_cast<float*>(ws + P.o_R);
  sp.text_out = text_out;
  sp.fwd_out = fwd_out;
  sp.bwd_out = bwd_out;
  sp.d_out = P.d;
  k_vda_scan<<<dim3(2, P.H, 128 / kScanHalf), kScanThreads, kScanSmemBytes, st>>>(tw, tct, sp);
  return VDN_OK;
}

struct MergeArgs {
  const void* g_s;
  const void* g_l;
  const float* rms_w;
  void* out;
  bool branches = false;  // out is [N][2H][128] bf16: the two gated branches
  const uint8_t* rimg = nullptr;  // packed R_b tiles; nullptr: the workspace's own
};

// Softmax branch; with `merge` set, the readout + gated merge run in its
// epilogue (R_b packed images at ws + o_Rimg must be ready) and `out` is
// written instead of o_soft.
int launch_bsa(const Plan& P, const Acts& a, uint8_t* ws, __nv_bfloat16* o, int64_t o_row,
               int d_store, float* lse, cudaStream_t st, const MergeArgs* merge) {
  if (P.N == 0) return VDN_OK;
  CUtensorMap tq, tk, tv, tkt, tvt, tout;
  if (!act_map(&tq, a.q, P.N, P, 128, ws + P.o_C) || !act_map(&tk, a.k, P.N, P, 128, ws + P.o_C) ||
      !act_map(&tv, a.v, P.N, P, 128, ws + P.o_C) ||
      !act_map(&tkt, a.kt, P.T, P, 128, ws + P.o_C) ||
      !act_map(&tvt, a.vt, P.T, P, 128, ws + P.o_C))
    return VDN_ERR_CUDA;
  // the merged output leaves by TMA stores when it is bf16 with d = 128
  const bool tma_out = merge != nullptr && P.dtype == VDN_BF16 && P.d == kDPad;
  if (merge != nullptr && merge->branches) {
    if (!map_act(&tout, merge->out, P.N, 2 * P.H, 128)) return VDN_ERR_CUDA;
  } else if (!act_map(&tout, tma_out ? merge->out : a.q, P.N, P, 128, ws + P.o_C)) {
    return VDN_ERR_CUDA;
  }
  BsaParams bp;
  memset(&bp, 0, sizeof(bp));
  bp.off = P.off_dev;
  bp.F = P.F;
  bp.T = P.T;
  bp.H = P.H;
  bp.bf = P.bf;
  bp.N = P.N;
  bp.scale_log2 = 1.4426950408889634f / sqrtf((float)P.d);
  bp.o = o;
  bp.o_row_stride = o_row;
  bp.d_store = d_store;
  bp.lse = lse;
  bp.d = P.d;
  // heads on z (one head after the other), blocks on y visited interior-first
  const dim3 grid((P.max_qtiles + 1) / 2, P.nb, P.H);
  if (merge == nullptr) {
    k_bsa_fwd<0><<<grid, kBsaThreads, kBsaSmemBytes, st>>>(tq, tk, tv, tkt, tvt, tout, tq, bp);
  } else {
    bp.rimg = merge->rimg != nullptr ? merge->rimg : ws + P.o_Rimg;
    bp.g_s = merge->g_s;
    bp.g_l = merge->g_l;
    bp.gate_f32 = (P.dtype == VDN_F32);
    bp.rms_w = merge->rms_w;
    bp.eps = P.eps;
    bp.out = merge->out;
    bp.out_f32 = (P.dtype == VDN_F32);
    bp.tma_out = tma_out ? 1 : 0;
    if (merge->branches)
      k_bsa_fwd<2><<<grid, kBsaThreads, kBsaMergeSmemBytes, st>>>(tq, tk, tv, tkt, tvt, tout, tq,
                                                                bp);
    else
      k_bsa_fwd<1><<<grid, kBsaThreads, kBsaMergeSmemBytes, st>>>(tq, tk, tv, tkt, tvt, tout, tq,
                                                                bp);
  }
  return VDN_OK;
}

int launch_merge(const Plan& P, const __nv_bfloat16* qb, const float* RA, const float* RB, int r_d,
                 const __nv_bfloat16* o_soft, int64_t os_row, int os_head, const void* g_s,
                 const void* g_l, const float* rms_w, void* out, uint8_t* ws, cudaStream_t st) {
  if (P.N == 0) return VDN_OK;
  CUtensorMap tq;
  if (!act_map(&tq, qb, P.N, P, 128, ws + P.o_C)) return VDN_ERR_CUDA;
  MergeParams mp;
  mp.off = P.off_dev;
  mp.F = P.F;
  mp.H = P.H;
  mp.bf = P.bf;
  mp.N = P.N;
  mp.d = P.d;
  mp.RA = RA;
  mp.RB = RB;
  mp.r_d = r_d;
  mp.o_soft = o_soft;
  mp.os_row = os_row;
  mp.os_head = os_head;
  mp.g_s = g_s;
  mp.g_l = g_l;
  mp.gate_f32 = (P.dtype == VDN_F32);
  mp.rms_w = rms_w;
  mp.eps = P.eps;
  mp.out = out;
  mp.out_f32 = (P.dtype == VDN_F32);
  // bf16 out, d = 128, packed o_soft [N, H, 128]: streamed variant (TMA in and out)
  if (P.dtype == VDN_BF16 && P.d == kDPad && r_d == kDPad && os_head == kDPad &&
      os_row == (int64_t)P.H * kDPad) {
    CUtensorMap tos, tout;
    if (!act_map(&tos, o_soft, P.N, P, 128, ws + P.o_C) ||
        !act_map(&tout, out, P.N, P, 128, ws + P.o_C))
      return VDN_ERR_CUDA;
    const int gx = (P.max_qtiles + kMergeTmaTiles - 1) / kMergeTmaTiles;
    k_readout_merge_tma<<<dim3(gx, P.nb, P.H), kMergeTmaThreads, kMergeTmaSmemBytes, st>>>(tq, tos,
                                                                                      tout, mp);
    return VDN_OK;
  }
  const int gx = (P.max_qtiles + kMergeTiles - 1) / kMergeTiles;
  k_readout_merge<<<dim3(gx, P.nb, P.H), kMergeThreads, kMergeSmemBytes, st>>>(tq, mp);
  return VDN_OK;
}

int finish(int rc) {
  if (rc != VDN_OK) return rc;
  return cudaGetLastError() == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

int common_checks(const Plan& P, void* ws, size_t ws_bytes) {
  if (ws == nullptr || ws_bytes < P.total) return VDN_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(ws)) return VDN_ERR_MISALIGNED;
  if (!set_smem_attrs()) return VDN_ERR_CUDA;
  if (!encode_fn()) return VDN_ERR_CUDA;
  return VDN_OK;
}

int check_ptrs(std::initializer_list<const void*> must, std::initializer_list<const void*> text,
               int T) {
  for (const void* p : must) {
    if (p == nullptr) return VDN_ERR_INVALID_ARG;
    if (!aligned16(p)) return VDN_ERR_MISALIGNED;
  }
  if (T > 0) {
    for (const void* p : text) {
      if (p == nullptr) return VDN_ERR_INVALID_ARG;
      if (!aligned16(p)) return VDN_ERR_MISALIGNED;
    }
  }
  return VDN_OK;
}

// ---------------------------------------------------------- projections --

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

int check_linear_args(const void* a, const float* a_scale, const void* w, const float* w_scale,
                      int64_t M, int K, int D, int precision, const void* y) {
  if (precision != VDN_PROJ_BF16 && precision != VDN_PROJ_FP8) return VDN_ERR_UNSUPPORTED;
  if (M < 0 || K < 16 || D < 8 || (K % 16) != 0 || (D % 8) != 0) return VDN_ERR_INVALID_ARG;
  if (M > ((int64_t)1 << 31) - 1 || (int64_t)D * K > ((int64_t)1 << 40)) return VDN_ERR_UNSUPPORTED;
  for (const void* p : {a, w, y}) {
    if (p == nullptr) return VDN_ERR_INVALID_ARG;
    if (!aligned16(p)) return VDN_ERR_MISALIGNED;
  }
  if (precision == VDN_PROJ_FP8) {
    if (a_scale == nullptr || w_scale == nullptr) return VDN_ERR_INVALID_ARG;
    if (!aligned16(a_scale) || !aligned16(w_scale)) return VDN_ERR_MISALIGNED;
  }
  return VDN_OK;
}

// y [M, D] bf16 = A [M, K] W [D, K]^T (times the row / column scales for e4m3)
int launch_linear(const void* a, const float* a_scale, const void* w, const float* w_scale,
                  int64_t M, int K, int D, int precision, void* y, cudaStream_t st) {
  if (M == 0) return VDN_OK;
  const bool fp8 = precision == VDN_PROJ_FP8;
  const int es = fp8 ? 1 : 2;
  const int bk = fp8 ? 128 : 64;
  CUtensorMap ta, tw, ty;
  if (!map_rows(&ta, a, K, M, es, bk, kLinBM) || !map_rows(&tw, w, K, D, es, bk, kLinBN) ||
      !map_rows(&ty, y, D, M, 2, 64, kLinBM))
    return VDN_ERR_CUDA;
  LinParams lp;
  lp.M = (int)M;
  lp.K = K;
  lp.D = D;
  lp.tiles_m = (int)((M + kLinBM - 1) / kLinBM);
  lp.tiles_n = (D + kLinBN - 1) / kLinBN;
  lp.a_scale = a_scale;
  lp.w_scale = w_scale;
  const int tiles = lp.tiles_m * lp.tiles_n;
  const int sms = sm_count();
  if (sms <= 0) return VDN_ERR_CUDA;
  const int grid = imin(tiles, sms);
  if (fp8)
    k_linear<true><<<grid, kLinThreads, kLinSmemBytes, st>>>(ta, tw, ty, lp);
  else
    k_linear<false><<<grid, kLinThreads, kLinSmemBytes, st>>>(ta, tw, ty, lp);
  return VDN_OK;
}

void launch_quant(const void* x, int64_t rows, int K, void* codes, float* scales, cudaStream_t st) {
  if (rows == 0) return;
  const int warps = 8;
  k_quant_rows_e4m3<<<(unsigned)((rows + warps - 1) / warps), warps * 32, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), rows, K, static_cast<uint8_t*>(codes), scales);
}

// Workspace of the projected layer: the layer's own workspace, then the
// gated branches [N, 2H, 128] bf16 and, for e4m3, their codes and row scales.
struct ProjPlan {
  size_t o_branches, o_codes, o_scales, total;
};

int make_proj_plan(const Plan& P, int D, int precision, ProjPlan* Q) {
  if (P.dtype != VDN_BF16 || P.d != kDPad) return VDN_ERR_UNSUPPORTED;
  if (precision != VDN_PROJ_BF16 && precision != VDN_PROJ_FP8) return VDN_ERR_UNSUPPORTED;
  if (D < 8 || (D % 8) != 0) return VDN_ERR_INVALID_ARG;
  const size_t K = (size_t)2 * P.H * kDPad;
  size_t o = P.total;
  Q->o_branches = o;
  o += align256((size_t)P.N * K * 2);
  Q->o_codes = o;
  o += precision == VDN_PROJ_FP8 ? align256((size_t)P.N * K) : 0;
  Q->o_scales = o;
  o += precision == VDN_PROJ_FP8 ? align256((size_t)P.N * 4) : 0;
  Q->total = o;
  return VDN_OK;
}

// ------------------------------------------------------ e4m3 softmax --

// Workspace of the e4m3 softmax branch: the layer's own workspace, then the
// per-head amax words of k and v, the codes of q, k, v, kt, vt and the q row
// scales.
struct Fp8Plan {
  size_t o_amax, o_q8, o_k8, o_v8, o_kt8, o_vt8, o_qs, total;
};

int make_fp8_plan(const Plan& P, Fp8Plan* Q) {
  if (P.dtype != VDN_BF16 || P.d != kDPad) return VDN_ERR_UNSUPPORTED;
  const size_t act = (size_t)P.N * P.H * kDPad;
  const size_t txt = (size_t)P.T * P.H * kDPad;
  size_t o = P.total;
  Q->o_amax = o; o += align256((size_t)2 * P.H * 4);
  Q->o_q8 = o; o += align256(act);
  Q->o_k8 = o; o += align256(act);
  Q->o_v8 = o; o += align256(act);
  Q->o_kt8 = o; o += align256(txt);
  Q->o_vt8 = o; o += align256(txt);
  Q->o_qs = o; o += align256((size_t)P.N * P.H * 4);
  Q->total = o;
  return VDN_OK;
}

int grid_for(int64_t units, int threads) {
  return (int)std::min<int64_t>((units + threads - 1) / threads, (int64_t)148 * 8);
}

// amax of k, v per head (video and text together), then the e4m3 codes
int launch_fp8_prepass(const Plan& P, const Fp8Plan& Q, const void* q, const void* k,
                       const void* v, const void* kt, const void* vt, uint8_t* ws,
                       cudaStream_t st) {
  uint32_t* amax = reinterpret_cast<uint32_t*>(ws + Q.o_amax);
  if (cudaMemsetAsync(amax, 0, (size_t)2 * P.H * 4, st) != cudaSuccess) return VDN_ERR_CUDA;
  const int th = 256;
  const auto bf = [](const void* x) { return static_cast<const __nv_bfloat16*>(x); };
  if (P.N > 0) {
    const int64_t u = (int64_t)P.N * P.H * 16;
    k_attn_amax<<<grid_for(u, th), th, 0, st>>>(bf(k), bf(v), P.N, P.H, amax);
  }
  if (P.T > 0) {
    const int64_t u = (int64_t)P.T * P.H * 16;
    k_attn_amax<<<grid_for(u, th), th, 0, st>>>(bf(kt), bf(vt), P.T, P.H, amax);
  }
  if (P.N > 0) {
    const int64_t u = (int64_t)P.N * P.H * 16;
    k_attn_quant<<<grid_for(u, th), th, 0, st>>>(bf(q), bf(k), bf(v), P.N, P.H, amax,
                                                ws + Q.o_q8, reinterpret_cast<float*>(ws + Q.o_qs),
                                                ws + Q.o_k8, ws + Q.o_v8);
  }
  if (P.T > 0) {
    const int64_t u = (int64_t)P.T * P.H * 16;
    k_attn_quant<<<grid_for(u, th), th, 0, st>>>(nullptr, bf(kt), bf(vt), P.T, P.H, amax, nullptr,
                                                nullptr, ws + Q.o_kt8, ws + Q.o_vt8);
  }
  return VDN_OK;
}

// e4m3 softmax branch: o [N, H, 128] bf16 (row stride o_row), lse optional;
// with `merge` set, the merged layer output instead (readout, RMSNorm and
// gated merge in the epilogue, R_b tiles at ws + o_Rimg, q in bf16 `qb`).
int launch_bsa_fp8(const Plan& P, const Fp8Plan& Q, uint8_t* ws, __nv_bfloat16* o, int64_t o_row,
                   float* lse, cudaStream_t st, const MergeArgs* merge = nullptr,
                   const void* qb = nullptr) {
  if (P.N == 0) return VDN_OK;
  CUtensorMap tq, tk, tv, tkt, tvt, tout, tqb;
  void* dummy = ws + Q.o_q8;  // never dereferenced for an empty text
  const bool t = P.T > 0;
  if (!map_act8(&tq, ws + Q.o_q8, P.N, P.H, 128) || !map_act8(&tk, ws + Q.o_k8, P.N, P.H, 128) ||
      !map_act8(&tv, ws + Q.o_v8, P.N, P.H, 128) ||
      !map_act8(&tkt, t ? ws + Q.o_kt8 : dummy, t ? P.T : 1, P.H, 128) ||
      !map_act8(&tvt, t ? ws + Q.o_vt8 : dummy, t ? P.T : 1, P.H, 128))
    return VDN_ERR_CUDA;
  if (merge != nullptr && (!map_act(&tout, merge->out, P.N, P.H, 128) ||
                           !map_act(&tqb, qb, P.N, P.H, 128)))
    return VDN_ERR_CUDA;
  BsaParams bp;
  memset(&bp, 0, sizeof(bp));
  bp.off = P.off_dev;
  bp.F = P.F;
  bp.T = P.T;
  bp.H = P.H;
  bp.bf = P.bf;
  bp.N = P.N;
  bp.scale_log2 = 1.4426950408889634f / sqrtf((float)P.d);
  bp.o = o;
  bp.o_row_stride = o_row;
  bp.d_store = kDPad;
  bp.lse = lse;
  bp.d = P.d;
  bp.q_scale = reinterpret_cast<const float*>(ws + Q.o_qs);
  bp.kv_amax = reinterpret_cast<const uint32_t*>(ws + Q.o_amax);
  const dim3 grid((P.max_qtiles + 1) / 2, P.nb, P.H);
  if (merge == nullptr) {
    k_bsa_fwd<0, true><<<grid, kBsaThreads, kBsa8SmemBytes, st>>>(tq, tk, tv, tkt, tvt, tq, tq, bp);
  } else {
    bp.rimg = ws + P.o_Rimg;
    bp.g_s = merge->g_s;
    bp.g_l = merge->g_l;
    bp.gate_f32 = 0;
    bp.rms_w = merge->rms_w;
    bp.eps = P.eps;
    bp.out = merge->out;
    bp.out_f32 = 0;
    bp.tma_out = 1;
    k_bsa_fwd<1, true><<<grid, kBsaThreads, kBsa8MergeSmemBytes, st>>>(tq, tk, tv, tkt, tvt, tout,
                                                                       tqb, bp);
  }
  return VDN_OK;
}

// The layer's launches in order: staging (fp32 narrowing / d padding, when
// needed), Gram + inverse, scans, read-state packing, softmax kernel with the
// merge epilogue. With `ev` set, ev[0..kProfileGroups] are recorded on the
// stream at the boundaries of those five groups.
constexpr int kProfileGroups = 5;

int layer_launches(const Plan& P, const void* q, const void* k, const void* v, const void* kt,
                   const void* vt, const void* g_s, const void* g_l, const float* rms_w,
                   void* out, uint8_t* ws, cudaStream_t st, cudaEvent_t* ev,
                   bool branches = false) {
  if (ev != nullptr) cudaEventRecord(ev[0], st);
  const Acts a = stage_inputs(P, q, k, v, kt, vt, ws, st, true, true);
  if (ev != nullptr) cudaEventRecord(ev[1], st);
  int rc = launch_vda(P, a, ws, st, nullptr, nullptr, nullptr, ev != nullptr ? ev[2] : nullptr);
  if (rc != VDN_OK) return rc;
  if (ev != nullptr) cudaEventRecord(ev[3], st);
  const float* R = reinterpret_cast<const float*>(ws + P.o_R);
  k_pack_read_states<<<dim3(P.nb * P.H, kPackSplit), 128, 0, st>>>(
      R, R + (size_t)P.nb * P.H * 128 * 128, ws + P.o_Rimg);
  if (ev != nullptr) cudaEventRecord(ev[4], st);
  MergeArgs m{g_s, g_l, rms_w, out, branches};
  rc = launch_bsa(P, a, ws, nullptr, 0, kDPad, nullptr, st, &m);
  if (ev != nullptr) cudaEventRecord(ev[5], st);
  return rc;
}

}  // namespace

extern "C" {

size_t vdn_workspace_bytes(const vdn_shape_t* shape) {
  Plan P;
  if (make_plan(shape, &P) != VDN_OK) return 0;
  return P.total;
}

int vdn_hybrid_attn_fwd(const vdn_shape_t* shape, const void* q, const void* k, const void* v,
                        const void* kt, const void* vt, const void* g_s, const void* g_l,
                        const float* rms_w, void* out, void* workspace, size_t ws_bytes,
                        void* stream) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  if (P.N == 0) return VDN_OK;  // no query tokens: nothing to write
  rc = check_ptrs({q, k, v, g_s, g_l, rms_w, out}, {kt, vt}, P.T);
  if (rc != VDN_OK) return rc;
  rc = common_checks(P, workspace, ws_bytes);
  if (rc != VDN_OK) return rc;
  return finish(layer_launches(P, q, k, v, kt, vt, g_s, g_l, rms_w, out,
                               static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream),
                               nullptr));
}

int vdn_hybrid_attn_fwd_profile(const vdn_shape_t* shape, const void* q, const void* k,
                                const void* v, const void* kt, const void* vt, const void* g_s,
                                const void* g_l, const float* rms_w, void* out, void* workspace,
                                size_t ws_bytes, void* stream, int iters, float* kernel_ms) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  if (iters < 1 || iters > 256 || kernel_ms == nullptr) return VDN_ERR_INVALID_ARG;
  for (int i = 0; i < kProfileGroups; ++i) kernel_ms[i] = 0.f;
  if (P.N == 0) return VDN_OK;
  rc = check_ptrs({q, k, v, g_s, g_l, rms_w, out}, {kt, vt}, P.T);
  if (rc != VDN_OK) return rc;
  rc = common_checks(P, workspace, ws_bytes);
  if (rc != VDN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int ne = (kProfileGroups + 1) * iters;
  cudaEvent_t* ev = new cudaEvent_t[ne];
  int made = 0;
  for (; made < ne; ++made)
    if (cudaEventCreate(&ev[made]) != cudaSuccess) break;
  if (made == ne) {
    for (int it = 0; it < iters && rc == VDN_OK; ++it)
      rc = layer_launches(P, q, k, v, kt, vt, g_s, g_l, rms_w, out,
                          static_cast<uint8_t*>(workspace), st, ev + it * (kProfileGroups + 1));
    rc = finish(rc);
    if (rc == VDN_OK && cudaStreamSynchronize(st) != cudaSuccess) rc = VDN_ERR_CUDA;
    for (int it = 0; it < iters && rc == VDN_OK; ++it)
      for (int g = 0; g < kProfileGroups; ++g) {
        float ms = 0.f;
        cudaEvent_t* e = ev + it * (kProfileGroups + 1);
        if (cudaEventElapsedTime(&ms, e[g], e[g + 1]) != cudaSuccess) rc = VDN_ERR_CUDA;
        kernel_ms[g] += ms / (float)iters;
      }
  } else {
    rc = VDN_ERR_CUDA;
  }
  for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
  delete[] ev;
  return rc;
}

size_t vdn_proj_workspace_bytes(const vdn_shape_t* shape, int D, int precision) {
  Plan P;
  ProjPlan Q;
  if (make_plan(shape, &P) != VDN_OK || make_proj_plan(P, D, precision, &Q) != VDN_OK) return 0;
  return Q.total;
}

int vdn_hybrid_attn_branches(const vdn_shape_t* shape, const void* q, const void* k,
                             const void* v, const void* kt, const void* vt, const void* g_s,
                             const void* g_l, const float* rms_w, void* branches,
                             void* workspace, size_t ws_bytes, void* stream) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  if (P.dtype != VDN_BF16 || P.d != kDPad) return VDN_ERR_UNSUPPORTED;
  if (P.N == 0) return VDN_OK;
  rc = check_ptrs({q, k, v, g_s, g_l, rms_w, branches}, {kt, vt}, P.T);
  if (rc != VDN_OK) return rc;
  rc = common_checks(P, workspace, ws_bytes);
  if (rc != VDN_OK) return rc;
  return finish(layer_launches(P, q, k, v, kt, vt, g_s, g_l, rms_w, branches,
                               static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream),
                               nullptr, true));
}

int vdn_linear(const void* a, const float* a_scale, const void* w, const float* w_scale,
               int64_t M, int K, int D, int precision, void* y, void* stream) {
  int rc = check_linear_args(a, a_scale, w, w_scale, M, K, D, precision, y);
  if (rc != VDN_OK) return rc;
  if (!set_smem_attrs() || !encode_fn()) return VDN_ERR_CUDA;
  return finish(launch_linear(a, a_scale, w, w_scale, M, K, D, precision, y,
                              static_cast<cudaStream_t>(stream)));
}

int vdn_quantize_rows_e4m3(const void* x, int64_t rows, int K, void* codes, float* scales,
                           void* stream) {
  if (rows < 0 || K < 16 || (K % 16) != 0 || rows > ((int64_t)1 << 31) - 1)
    return VDN_ERR_INVALID_ARG;
  if (rows == 0) return VDN_OK;
  for (const void* p : {x, (const void*)codes, (const void*)scales}) {
    if (p == nullptr) return VDN_ERR_INVALID_ARG;
    if (!aligned16(p)) return VDN_ERR_MISALIGNED;
  }
  launch_quant(x, rows, K, codes, scales, static_cast<cudaStream_t>(stream));
  return finish(VDN_OK);
}

int vdn_hybrid_attn_proj_fwd(const vdn_shape_t* shape, const void* q, const void* k,
                             const void* v, const void* kt, const void* vt, const void* g_s,
                             const void* g_l, const float* rms_w, const void* w_o,
                             const float* w_scale, int D, int precision, void* y,
                             void* workspace, size_t ws_bytes, void* stream) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  ProjPlan Q;
  rc = make_proj_plan(P, D, precision, &Q);
  if (rc != VDN_OK) return rc;
  if (P.N == 0) return VDN_OK;
  rc = check_ptrs({q, k, v, g_s, g_l, rms_w, w_o, y}, {kt, vt}, P.T);
  if (rc != VDN_OK) return rc;
  if (precision == VDN_PROJ_FP8 && (w_scale == nullptr || !aligned16(w_scale)))
    return w_scale == nullptr ? VDN_ERR_INVALID_ARG : VDN_ERR_MISALIGNED;
  if (workspace == nullptr || ws_bytes < Q.total) return VDN_ERR_WORKSPACE_TOO_SMALL;
  rc = common_checks(P, workspace, ws_bytes);
  if (rc != VDN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* A = ws + Q.o_branches;
  const int K = 2 * P.H * kDPad;
  rc = layer_launches(P, q, k, v, kt, vt, g_s, g_l, rms_w, A, ws, st, nullptr, true);
  if (rc != VDN_OK) return finish(rc);
  if (precision == VDN_PROJ_FP8) {
    float* sa = reinterpret_cast<float*>(ws + Q.o_scales);
    launch_quant(A, P.N, K, ws + Q.o_codes, sa, st);
    rc = launch_linear(ws + Q.o_codes, sa, w_o, w_scale, P.N, K, D, precision, y, st);
  } else {
    rc = launch_linear(A, nullptr, w_o, nullptr, P.N, K, D, precision, y, st);
  }
  return finish(rc);
}

size_t vdn_fp8_workspace_bytes(const vdn_shape_t* shape) {
  Plan P;
  Fp8Plan Q;
  if (make_plan(shape, &P) != VDN_OK || make_fp8_plan(P, &Q) != VDN_OK) return 0;
  return Q.total;
}

int vdn_bsa_fwd_fp8(const vdn_shape_t* shape, const void* q, const void* k, const void* v,
                    const void* kt, const void* vt, void* o_soft, float* lse, void* workspace,
                    size_t ws_bytes, void* stream) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  Fp8Plan Q;
  rc = make_fp8_plan(P, &Q);
  if (rc != VDN_OK) return rc;
  if (P.N == 0) return VDN_OK;
  rc = check_ptrs({q, k, v, o_soft}, {kt, vt}, P.T);
  if (rc != VDN_OK) return rc;
  if (lse != nullptr && !aligned16(lse)) return VDN_ERR_MISALIGNED;
  if (workspace == nullptr || ws_bytes < Q.total) return VDN_ERR_WORKSPACE_TOO_SMALL;
  rc = common_checks(P, workspace, ws_bytes);
  if (rc != VDN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  rc = launch_fp8_prepass(P, Q, q, k, v, kt, vt, ws, st);
  if (rc == VDN_OK)
    rc = launch_bsa_fp8(P, Q, ws, static_cast<__nv_bfloat16*>(o_soft), (int64_t)P.H * kDPad, lse,
                        st);
  return finish(rc);
}

int vdn_hybrid_attn_fwd_fp8(const vdn_shape_t* shape, const void* q, const void* k,
                            const void* v, const void* kt, const void* vt, const void* g_s,
                            const void* g_l, const float* rms_w, void* out, void* workspace,
                            size_t ws_bytes, void* stream) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  Fp8Plan Q;
  rc = make_fp8_plan(P, &Q);
  if (rc != VDN_OK) return rc;
  if (P.N == 0) return VDN_OK;
  rc = check_ptrs({q, k, v, g_s, g_l, rms_w, out}, {kt, vt}, P.T);
  if (rc != VDN_OK) return rc;
  if (workspace == nullptr || ws_bytes < Q.total) return VDN_ERR_WORKSPACE_TOO_SMALL;
  rc = common_checks(P, workspace, ws_bytes);
  if (rc != VDN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  rc = launch_fp8_prepass(P, Q, q, k, v, kt, vt, ws, st);
  const Acts a = stage_inputs(P, q, k, v, kt, vt, ws, st, false, false);
  if (rc == VDN_OK) rc = launch_vda(P, a, ws, st, nullptr, nullptr, nullptr);
  if (rc == VDN_OK) {
    const float* R = reinterpret_cast<const float*>(ws + P.o_R);
    k_pack_read_states<<<dim3(P.nb * P.H, kPackSplit), 128, 0, st>>>(
        R, R + (size_t)P.nb * P.H * 128 * 128, ws + P.o_Rimg);
    MergeArgs m{g_s, g_l, rms_w, out};
    rc = launch_bsa_fp8(P, Q, ws, nullptr, 0, nullptr, st, &m, q);
  }
  return finish(rc);
}

size_t vdn_read_images_bytes(const vdn_shape_t* shape) {
  Plan P;
  if (make_plan(shape, &P) != VDN_OK) return 0;
  return (size_t)P.nb * P.H * kRImageBytes;
}

int vdn_vda_read_images(const vdn_shape_t* shape, const void* k, const void* v, const void* kt,
                        const void* vt, void* rimg, void* workspace, size_t ws_bytes,
                        void* stream) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  if (P.N > 0) rc = check_ptrs({k, v, rimg}, {kt, vt}, P.T);
  else rc = check_ptrs({rimg}, {kt, vt}, P.T);
  if (rc != VDN_OK) return rc;
  rc = common_checks(P, workspace, ws_bytes);
  if (rc != VDN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const Acts a = stage_inputs(P, nullptr, k, v, kt, vt, ws, st, false, true);
  rc = launch_vda(P, a, ws, st, nullptr, nullptr, nullptr);
  if (rc != VDN_OK) return finish(rc);
  const float* R = reinterpret_cast<const float*>(ws + P.o_R);
  k_pack_read_states<<<dim3(P.nb * P.H, kPackSplit), 128, 0, st>>>(
      R, R + (size_t)P.nb * P.H * 128 * 128, static_cast<uint8_t*>(rimg));
  return finish(VDN_OK);
}

int vdn_bsa_merge_fwd(const vdn_shape_t* shape, const void* q, const void* k, const void* v,
                      const void* kt, const void* vt, const void* g_s, const void* g_l,
                      const float* rms_w, const void* rimg, void* out, void* workspace,
                      size_t ws_bytes, void* stream) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  if (P.N == 0) return VDN_OK;
  rc = check_ptrs({q, k, v, g_s, g_l, rms_w, rimg, out}, {kt, vt}, P.T);
  if (rc != VDN_OK) return rc;
  rc = common_checks(P, workspace, ws_bytes);
  if (rc != VDN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const Acts a = stage_inputs(P, q, k, v, kt, vt, ws, st, true, true);
  MergeArgs m{g_s, g_l, rms_w, out, false, static_cast<const uint8_t*>(rimg)};
  return finish(launch_bsa(P, a, ws, nullptr, 0, kDPad, nullptr, st, &m));
}

int vdn_vda_scan(const vdn_shape_t* shape, const void* k, const void* v, const void* kt,
                 const void* vt, float* read_states, float* text_state, float* fwd_states,
                 float* bwd_states, void* workspace, size_t ws_bytes, void* stream) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  if (P.N > 0) rc = check_ptrs({k, v, read_states}, {kt, vt}, P.T);
  else rc = check_ptrs({read_states}, {kt, vt}, P.T);
  if (rc != VDN_OK) return rc;
  for (const void* p : {(const void*)text_state, (const void*)fwd_states, (const void*)bwd_states})
    if (p != nullptr && !aligned16(p)) return VDN_ERR_MISALIGNED;
  rc = common_checks(P, workspace, ws_bytes);
  if (rc != VDN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const Acts a = stage_inputs(P, nullptr, k, v, kt, vt, ws, st, false, true);
  rc = launch_vda(P, a, ws, st, text_state, fwd_states, bwd_states);
  if (rc != VDN_OK) return finish(rc);
  // read_states [nb][H][d][d] = fwd part + bwd part (leading d x d block)
  const float* R = reinterpret_cast<const float*>(ws + P.o_R);
  const size_t part = (size_t)P.nb * P.H * 128 * 128;
  const int d = P.d;
  const int64_t n = (int64_t)P.nb * P.H * d * d;
  k_sum_states<<<(int)((n + 255) / 256), 256, 0, st>>>(R, R + part, read_states, n, d);
  return finish(VDN_OK);
}

int vdn_gate_merge(const vdn_shape_t* shape, const void* q, const float* read_states,
                   const void* o_soft, const void* g_s, const void* g_l, const float* rms_w,
                   void* out, void* workspace, size_t ws_bytes, void* stream) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  if (P.N == 0) return VDN_OK;
  rc = check_ptrs({q, read_states, o_soft, g_s, g_l, rms_w, out}, {}, 0);
  if (rc != VDN_OK) return rc;
  rc = common_checks(P, workspace, ws_bytes);
  if (rc != VDN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const Acts a = stage_inputs(P, q, nullptr, nullptr, nullptr, nullptr, ws, st, true, false);
  rc = launch_merge(P, a.q, read_states, nullptr, P.d, static_cast<const __nv_bfloat16*>(o_soft),
                    (int64_t)P.H * P.d, P.d, g_s, g_l, rms_w, out, ws, st);
  return finish(rc);
}

int vdn_bsa_fwd(const vdn_shape_t* shape, const void* q, const void* k, const void* v,
                const void* kt, const void* vt, void* o_soft, float* lse, void* workspace,
                size_t ws_bytes, void* stream) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  if (P.N == 0) return VDN_OK;
  rc = check_ptrs({q, k, v, o_soft}, {kt, vt}, P.T);
  if (rc != VDN_OK) return rc;
  if (lse != nullptr && !aligned16(lse)) return VDN_ERR_MISALIGNED;
  rc = common_checks(P, workspace, ws_bytes);
  if (rc != VDN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const Acts a = stage_inputs(P, q, k, v, kt, vt, ws, st, true, true);
  rc = launch_bsa(P, a, ws, static_cast<__nv_bfloat16*>(o_soft), (int64_t)P.H * P.d, P.d, lse, st,
                  nullptr);
  return finish(rc);
}

int vdn_pair_audit(const vdn_shape_t* shape, int64_t* soft_pairs, int64_t* lin_pairs,
                   void* stream) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  if (soft_pairs == nullptr || lin_pairs == nullptr) return VDN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(soft_pairs, 0, sizeof(int64_t) * P.F * (P.F + 1), st) != cudaSuccess)
    return VDN_ERR_CUDA;
  if (P.max_qtiles > 0)
    k_pair_audit_soft<<<dim3(P.max_qtiles, P.nb), 128, 0, st>>>(
        P.off_dev, P.F, P.T, P.bf, reinterpret_cast<unsigned long long*>(soft_pairs));
  k_pair_audit_lin<<<P.F, 128, 0, st>>>(P.off_dev, P.F, P.bf,
                                         reinterpret_cast<unsigned long long*>(lin_pairs));
  return finish(VDN_OK);
}

int vdn_selftest_wait_timeout(int64_t limit_ns, int tmem_cols, void* stream) {
  if (limit_ns < 1 || limit_ns > 1000000000) return VDN_ERR_INVALID_ARG;
  if (!(tmem_cols == 0 || tmem_cols == 32 || tmem_cols == 64 || tmem_cols == 128 ||
        tmem_cols == 256 || tmem_cols == 512))
    return VDN_ERR_INVALID_ARG;
  vdn::k_selftest_wait_timeout<<<1, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      (uint64_t)limit_ns, tmem_cols);
  return cudaGetLastError() == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

int vdn_get_device_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return VDN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, vdn::g_device_error, sizeof(int)) != cudaSuccess)
    return VDN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(vdn::g_device_error, &zero, sizeof(int)) != cudaSuccess)
    return VDN_ERR_CUDA;
  if (v == kDevErrWaitTimeout) return VDN_ERR_DEVICE_TIMEOUT;
  return v == 0 ? VDN_OK : VDN_ERR_DEVICE;
}

const char* vdn_error_string(int code) {
  switch (code) {
    case VDN_OK: return "ok";
    case VDN_ERR_INVALID_ARG: return "invalid argument";
    case VDN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case VDN_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case VDN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case VDN_ERR_CUDA: return "CUDA launch or driver error";
    case VDN_ERR_DEVICE_TIMEOUT: return "device-side bounded wait expired";
    case VDN_ERR_DEVICE: return "device-side error";
    default: return "unknown error";
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Linear-branch states without a caller-provided workspace.
//
// Some callers cannot hand this library a workspace: a serving loop whose
// latency budget cannot absorb the implicit device synchronisation of
// cudaMalloc / cudaFree, or a plug-in living inside a process whose device
// memory is owned by another allocator it has no handle to. For them,
// vdn_vda_scan_noalloc keeps its scratch (per-frame C and W matrices,
// read-state halves and, for fp32 or d < 128 inputs, the staged bf16
// keys/values) in one file-scope device array of kNoAllocScratchBytes. Every
// GPU that loads this library holds that array until the process exits.
// The entry point itself makes CUDA runtime calls and launches kernels, so
// like every other entry point it must not be called from inside a stream
// host function (cudaLaunchHostFunc callbacks may not call CUDA at all).
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)64 << 20;  // 64 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context (0 if there is none
// yet). Context ids are never reused within a process, unlike device
// ordinals (a context torn down by cudaDeviceReset and created again keeps
// its ordinal but gets a new id and may map the array elsewhere).
int current_context_id(unsigned long long* id) {
  static const CtxGetCurrentFn get_cur = []() -> CtxGetCurrentFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
               ? reinterpret_cast<CtxGetCurrentFn>(p)
               : nullptr;
  }();
  static const CtxGetIdFn get_id = []() -> CtxGetIdFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
               ? reinterpret_cast<CtxGetIdFn>(p)
               : nullptr;
  }();
  if (get_cur == nullptr || get_id == nullptr) return VDN_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS) return VDN_ERR_CUDA;
  *id = 0;
  if (ctx != nullptr && get_id(ctx, id) != CUDA_SUCCESS) return VDN_ERR_CUDA;
  return VDN_OK;
}

// Device address of g_noalloc_scratch in the current context. In host code
// the symbol itself is only a host-side stand-in, so the address is looked up
// with cudaGetSymbolAddress once per context (in practice once per device:
// the runtime's primary context), with that device current, and cached under
// the context's id. A mutex guards the cache against concurrent host threads.
int noalloc_scratch_address(uint8_t** out) {
  struct Entry {
    unsigned long long ctx;
    uint8_t* addr;
  };
  static std::mutex mu;
  static Entry cache[64];
  static int used = 0;
  unsigned long long ctx = 0;
  if (current_context_id(&ctx) != VDN_OK) return VDN_ERR_CUDA;
  if (ctx != 0) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
      if (cache[i].ctx == ctx) {
        *out = cache[i].addr;
        return VDN_OK;
      }
  }
  // first call in this context (cudaGetSymbolAddress also creates the
  // runtime's primary context if no context is current yet)
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
    return VDN_ERR_CUDA;
  if (current_context_id(&ctx) != VDN_OK || ctx == 0) return VDN_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(mu);
    bool found = false;
    for (int i = 0; i < used && !found; ++i) found = (cache[i].ctx == ctx);
    if (!found && used < 64) cache[used++] = Entry{ctx, static_cast<uint8_t*>(p)};
  }
  *out = static_cast<uint8_t*>(p);
  return VDN_OK;
}

}  // namespace

extern "C" int vdn_vda_scan_noalloc(const vdn_shape_t* shape, const void* k, const void* v,
                                    const void* kt, const void* vt, float* read_states,
                                    float* text_state, float* fwd_states, float* bwd_states,
                                    void* stream) {
  Plan P;
  int rc = make_plan(shape, &P);
  if (rc != VDN_OK) return rc;
  if (P.N > 0) rc = check_ptrs({k, v, read_states}, {kt, vt}, P.T);
  else rc = check_ptrs({read_states}, {kt, vt}, P.T);
  if (rc != VDN_OK) return rc;
  for (const void* p : {(const void*)text_state, (const void*)fwd_states, (const void*)bwd_states})
    if (p != nullptr && !aligned16(p)) return VDN_ERR_MISALIGNED;
  // Scratch layout inside the static array: C, W, read-state halves, then
  // the staged keys/values when the inputs need narrowing or padding.
  Plan S = P;
  const size_t mat = align256((size_t)(P.F - 1) * P.H * 128 * 128 * 4);
  const size_t act = P.staged ? align256((size_t)P.N * P.H * kDPad * 2) : 0;
  const size_t txt = P.staged ? align256((size_t)P.T * P.H * kDPad * 2) : 0;
  S.o_C = 0;
  S.o_W = mat;
  S.o_R = 2 * mat;
  S.o_k = S.o_R + align256((size_t)2 * P.nb * P.H * 128 * 128 * 4);
  S.o_v = S.o_k + act;
  S.o_kt = S.o_v + act;
  S.o_vt = S.o_kt + txt;
  S.o_q = 0;  // not used by the scan
  S.total = S.o_vt + txt;
  if (S.total > kNoAllocScratchBytes) return VDN_ERR_WORKSPACE_TOO_SMALL;
  uint8_t* scratch = nullptr;
  rc = noalloc_scratch_address(&scratch);
  if (rc != VDN_OK) return rc;
  if (!set_smem_attrs() || !encode_fn()) return VDN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Nothing in the scratch has to start at zero: every region is written in
  // full by this call before it is read.
  const Acts a = stage_inputs(S, nullptr, k, v, kt, vt, scratch, st, false, true);
  rc = launch_vda(S, a, scratch, st, text_state, fwd_states, bwd_states);
  if (rc != VDN_OK) return finish(rc);
  const float* R = reinterpret_cast<const float*>(scratch + S.o_R);
  const size_t part = (size_t)P.nb * P.H * 128 * 128;
  const int64_t n = (int64_t)P.nb * P.H * P.d * P.d;
  k_sum_states<<<(int)((n + 255) / 256), 256, 0, st>>>(R, R + part, read_states, n, P.d);
  return finish(VDN_OK);
}
