// Linear-branch readout fused with RMSNorm and the gated merge:
//   o_lin = q^T R_b,  out = sigmoid(g_s) o_soft + sigmoid(g_l) w * o_lin / rms(o_lin)
// ["VDN-MiniMax-H3" (openi.cn), 技术原理, last paragraph: each branch has a
// content-dependent sigmoid gate and the linear output is RMS-normalised
// before its gate; nav.superapi.store page, Gated Fusion Mechanism].
//
// One CTA = one (block b, head h) and up to kMergeTiles query tiles of 128
// rows. R_b (fp32, from the scans) is summed and converted to bf16 once per
// CTA into a 128B-swizzled MN-major tile; each query tile is one
// M=128, N=128, K=128 bf16 tcgen05 contraction into a double-buffered TMEM
// accumulator, so the next tile's MMA overlaps this tile's epilogue. The
// epilogue runs one query row per thread (row = TMEM lane): sum of squares,
// normalisation, gates and 16-byte vector stores, no cross-thread reduction.
#pragma once

#include "layer_plan.cuh"
#include "sm100_ptx.cuh"

namespace vdn {

constexpr int kMergeThreads = 128;
constexpr int kMergeTiles = 4;
constexpr uint32_t kMergeSmemR = 0;          // 32 KB
constexpr uint32_t kMergeSmemQ = 32768;      // 2 x 32 KB
constexpr uint32_t kMergeSmemBytes = 3 * 32768 + 1024;

struct MergeParams {
  const int32_t* off;
  int F, H, bf, N, d;      // d = real head dim
  const float* RA;         // [nb][H][r_d][r_d]
  const float* RB;         // same layout or nullptr (added to RA)
  int r_d;
  const __nv_bfloat16* o_soft;
  int64_t os_row;          // elements between tokens of o_soft
  int os_head;             // elements between heads of o_soft
  const void* g_s;
  const void* g_l;
  int gate_f32;
  const float* rms_w;      // [H][d]
  float eps;
  void* out;               // [N][H][d]
  int out_f32;
};

__device__ __forceinline__ float load_gate(const void* g, int64_t i, int f32) {
  return f32 ? __ldg(reinterpret_cast<const float*>(g) + i)
             : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(g)[i]);
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + __expf(-x)); }

__global__ void __launch_bounds__(kMergeThreads, 2)
    k_readout_merge(const __grid_constant__ CUtensorMap tq, const MergeParams p) {
  const int b = blockIdx.y, h = blockIdx.z;
  int q0, q1;
  block_rows(p.off, p.F, p.bf, b, q0, q1);
  const int t_first = blockIdx.x * kMergeTiles;
  const int ntl = imin(kMergeTiles, (q1 - q0 + kTile - 1) / kTile - t_first);
  if (ntl <= 0) return;

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q[2], bar_m[2];
  __shared__ uint32_t tmem_slot;
  __shared__ float wsm[128];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sR = base + kMergeSmemR;
  const uint32_t sQ[2] = {base + kMergeSmemQ, base + kMergeSmemQ + 32768};
  const int i = threadIdx.x, warp = i >> 5;
  const uint32_t qf[2] = {smem_u32(&bar_q[0]), smem_u32(&bar_q[1])};
  const uint32_t mm[2] = {smem_u32(&bar_m[0]), smem_u32(&bar_m[1])};

  if (i == 0) {
    for (int k = 0; k < 2; ++k) {
      mbar_init(qf[k], 1);
      mbar_init(mm[k], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  auto load_q = [&](int t, int st) {
    mbar_arrive_expect_tx(qf[st], 32768);
    const int row = q0 + (t_first + t) * kTile;
    tma_load_3d(sQ[st], &tq, qf[st], 0, h, row);
    tma_load_3d(sQ[st] + 16384, &tq, qf[st], 64, h, row);
  };
  if (i == 0) {
    tma_prefetch_desc(&tq);
    load_q(0, 0);
    if (ntl > 1) load_q(1, 1);
  }

  // R_b -> bf16, row i (key dim), MN-major 128B-swizzled: chunk c holds value dims 64c..64c+63
  {
    const int64_t rbase = ((int64_t)b * p.H + h) * p.r_d * p.r_d;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int n = c * 64 + u * 8 + e;
          float v = 0.f;
          if (i < p.r_d && n < p.r_d) {
            v = __ldg(p.RA + rbase + (int64_t)i * p.r_d + n);
            if (p.RB) v += __ldg(p.RB + rbase + (int64_t)i * p.r_d + n);
          }
          x[e] = v;
        }
        st_shared_v4(sR + (uint32_t)(c * 16384) + sw128_off((uint32_t)i, (uint32_t)u),
                     pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                     pack_bf16x2(x[6], x[7]));
      }
    }
    wsm[i] = (i < p.d) ? __ldg(p.rms_w + (int64_t)h * p.d + i) : 0.f;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t idO = idesc_bf16(128, 128, false, true);
  auto issue = [&](int t) -> bool {
    const int st = t & 1;
    if (!mbar_wait(qf[st], (uint32_t)((t >> 1) & 1))) return false;
    tc_fence_after();
#pragma unroll
    for (int s = 0; s < 8; ++s)
      umma_bf16_ss(tmem + (uint32_t)(st * 128),
                   sdesc_sw128(sQ[st] + (uint32_t)((s >> 2) * 16384 + (s & 3) * 32), 16, 1024),
                   sdesc_sw128(sR + (uint32_t)(s * 2048), 16384, 1024), idO, s > 0 ? 1u : 0u);
    umma_commit(mm[st]);
    return true;
  };
  __shared__ int abort_flag;
  if (i == 0) abort_flag = 0;
  __syncthreads();
  volatile int* abort_v = &abort_flag;
  if (i == 0 && !issue(0)) *abort_v = 1;

  const float inv_d = 1.f / (float)p.d;
  for (int t = 0; t < ntl; ++t) {
    if (t > 0) {
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
    }
    if (*abort_v) break;
    if (i == 0 && t + 1 < ntl && !issue(t + 1)) *abort_v = 1;
    const int row = q0 + (t_first + t) * kTile + i;
    const bool valid = row < q1;
    // prefetch this row's o_soft and gates
    uint4 os[16];
    float gsv = 0.f, glv = 0.f;
    if (valid) {
      const uint4* src =
          reinterpret_cast<const uint4*>(p.o_soft + (int64_t)row * p.os_row + (int64_t)h * p.os_head);
#pragma unroll
      for (int u = 0; u < 16; ++u) os[u] = (u * 8 < p.d) ? __ldg(src + u) : make_uint4(0, 0, 0, 0);
      gsv = sigmoidf_(load_gate(p.g_s, (int64_t)row * p.H + h, p.gate_f32));
      glv = sigmoidf_(load_gate(p.g_l, (int64_t)row * p.H + h, p.gate_f32));
    }
    const int st = t & 1;
    if (!mbar_wait(mm[st], (uint32_t)((t >> 1) & 1))) { *abort_v = 1; break; }
    tc_fence_after();
    if (i == 0 && t + 2 < ntl) load_q(t + 2, st);
    uint32_t o[128];
    tmem_ld128(tmem + lane_base + (uint32_t)(st * 128), o);
    tmem_ld_wait128(o);
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 128; ++c) ss = fmaf(__uint_as_float(o[c]), __uint_as_float(o[c]), ss);
    const float nr = glv * rsqrtf(ss * inv_d + p.eps);
    if (valid) {
      const int64_t obase = ((int64_t)row * p.H + h) * p.d;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        if (u * 8 >= p.d) continue;
        const uint32_t w4[4] = {os[u].x, os[u].y, os[u].z, os[u].w};
        float y[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c0 = u * 8 + 2 * e;
          y[2 * e] = gsv * bf_lo(w4[e]) + nr * wsm[c0] * __uint_as_float(o[c0]);
          y[2 * e + 1] = gsv * bf_hi(w4[e]) + nr * wsm[c0 + 1] * __uint_as_float(o[c0 + 1]);
        }
        if (p.out_f32) {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + obase + u * 8);
          dst[0] = make_float4(y[0], y[1], y[2], y[3]);
          dst[1] = make_float4(y[4], y[5], y[6], y[7]);
        } else {
          *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + obase + u * 8) =
              make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]),
                         pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace vdn
