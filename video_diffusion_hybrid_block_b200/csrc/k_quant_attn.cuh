// e4m3 operands of the FP8 softmax branch (the pages pair FlashAttention-4
// with FP8 on B200: agentlenshq.com page, core-ideas table; aigc.douyoubuy.cn
// page, section 07). Scales:
//   q: one scale per (token, head) row, s_q = amax_row / 448; each softmax
//      thread owns one query row, so the scale folds into its exponent scale;
//   k, v: one scale per head over all video and text tokens,
//      s_k = amax_k / 448, s_v = amax_v / 448; s_k folds into the exponent
//      scale, s_v into the output normalisation;
//   codes = e4m3_rn_satfinite(x * (448 / amax)) in fp32 (an all-zero row or
//   head gets scale 1).
// k_attn_amax: per-head amax of k, v over video and text tokens, as fp32
//   bit patterns combined with atomicMax (non-negative floats order like
//   their bits); the destination must be zeroed first.
// k_attn_quant: q rows (with their scales), k and v with the head scales;
//   one 16-lane half-warp per (token, head) row of 128 elements.
#pragma once

#include "sm100_ptx.cuh"

namespace vdn {

__device__ __forceinline__ float amax8(uint4 u) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  float m = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) m = fmaxf(m, fmaxf(fabsf(bf_lo(w[e])), fabsf(bf_hi(w[e]))));
  return m;
}

// 8 bf16 values times inv -> 8 e4m3 codes
__device__ __forceinline__ uint2 quant8(uint4 u, float inv) {
  return make_uint2(e4m3x4(__fmul_rn(bf_lo(u.x), inv), __fmul_rn(bf_hi(u.x), inv),
                           __fmul_rn(bf_lo(u.y), inv), __fmul_rn(bf_hi(u.y), inv)),
                    e4m3x4(__fmul_rn(bf_lo(u.z), inv), __fmul_rn(bf_hi(u.z), inv),
                           __fmul_rn(bf_lo(u.w), inv), __fmul_rn(bf_hi(u.w), inv)));
}

// k, v [rows, H, 128] bf16 -> amax bits [2][H] (k heads, then v heads)
__global__ void k_attn_amax(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                            int64_t rows, int H, uint32_t* __restrict__ amax_bits) {
  const int64_t units = rows * H * 16;  // 16-byte units
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int lane = threadIdx.x & 31;
  // blockDim and the grid stride are multiples of 32, so lanes 16 g .. 16 g + 15
  // of a warp always hold the 16 units of one (row, head)
  for (int64_t u0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); u0 < units;
       u0 += stride) {
    const int64_t u = u0 + lane;
    float mk = 0.f, mv = 0.f;
    if (u < units) {
      mk = amax8(__ldg(reinterpret_cast<const uint4*>(k) + u));
      mv = amax8(__ldg(reinterpret_cast<const uint4*>(v) + u));
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o));
      mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, o));
    }
    if ((lane & 15) == 0 && u < units) {
      const int h = (int)((u >> 4) % H);
      atomicMax(amax_bits + h, __float_as_uint(mk));
      atomicMax(amax_bits + H + h, __float_as_uint(mv));
    }
  }
}

__device__ __forceinline__ float head_inv(const uint32_t* bits, int i) {
  const float a = __uint_as_float(bits[i]);
  return a > 0.f ? __fdiv_rn(448.f, a) : 1.f;
}

// q (optional), k, v [rows, H, 128] bf16 -> codes [rows, H, 128] u8;
// q_scale [rows, H] fp32 (when q is given)
__global__ void k_attn_quant(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                             const __nv_bfloat16* __restrict__ v, int64_t rows, int H,
                             const uint32_t* __restrict__ amax_bits, uint8_t* __restrict__ q8,
                             float* __restrict__ q_scale, uint8_t* __restrict__ k8,
                             uint8_t* __restrict__ v8) {
  const int64_t units = rows * H * 16;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int lane = threadIdx.x & 31;
  for (int64_t u0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); u0 < units;
       u0 += stride) {
    const int64_t u = u0 + lane;
    const bool in = u < units;
    const int h = in ? (int)((u >> 4) % H) : 0;
    if (q != nullptr) {
      const uint4 x = in ? __ldg(reinterpret_cast<const uint4*>(q) + u) : make_uint4(0, 0, 0, 0);
      float m = amax8(x);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const float inv = m > 0.f ? __fdiv_rn(448.f, m) : 1.f;
      if (in) {
        reinterpret_cast<uint2*>(q8)[u] = quant8(x, inv);
        if ((lane & 15) == 0) q_scale[u >> 4] = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
      }
    }
    if (in) {
      reinterpret_cast<uint2*>(k8)[u] =
          quant8(__ldg(reinterpret_cast<const uint4*>(k) + u), head_inv(amax_bits, h));
      reinterpret_cast<uint2*>(v8)[u] =
          quant8(__ldg(reinterpret_cast<const uint4*>(v) + u), head_inv(amax_bits, H + h));
    }
  }
}

}  // namespace vdn
