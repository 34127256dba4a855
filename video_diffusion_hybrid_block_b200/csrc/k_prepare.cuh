// Input staging: narrows fp32 activations to bf16 and zero-pads head dims
// below 128, so the tensor-core kernels always see [rows, H, 128] bf16.
// Zero columns leave q.k, K^T K and K^T V unchanged; callers pass the real d
// for the softmax scale and the RMSNorm mean.
#pragma once

#include "layer_plan.cuh"
#include "sm100_ptx.cuh"

namespace vdn {

template <typename Tin>
__global__ void k_pad_to_bf16(const Tin* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                              int64_t rows_heads, int d) {
  // one thread per 8 output elements (16 bytes)
  const int64_t units = rows_heads * (kDPad / 8);
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t rh = u / (kDPad / 8);
    const int c0 = (int)(u % (kDPad / 8)) * 8;
    float x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = c0 + i;
      x[i] = (c < d) ? static_cast<float>(src[rh * d + c]) : 0.f;
    }
    uint4 v;
    v.x = pack_bf16x2(x[0], x[1]);
    v.y = pack_bf16x2(x[2], x[3]);
    v.z = pack_bf16x2(x[4], x[5]);
    v.w = pack_bf16x2(x[6], x[7]);
    *reinterpret_cast<uint4*>(dst + rh * kDPad + c0) = v;
  }
}

}  // namespace vdn
