// Per-branch output projections: y = A W^T with A = [a_s | a_l] the two gated
// branch outputs of every head ([M, K], K = 2 H d) and W = [W_s | W_l]
// ([D, K], one row per output channel) ["VDN-MiniMax-H3 - OpenVDN's
// Open-Source Video Generation Acceleration Solution" (nav.superapi.store),
// Technical Principles, Gated Fusion Mechanism: each branch has its own gate
// and output projection before the merge]. The pages run these linears in
// FP8; this file has a bf16 and an e4m3 variant.
//
// k_linear<kFp8>: persistent GEMM, one CTA per SM walking 128 x 256 output
// tiles (row-block major, so the CTAs in flight share A row blocks and the
// whole of W in L2). Warp roles (192 threads):
//   warp 0     TMA producer: A and W K-slices (128 B per row) into a 4-stage
//              ring, 48 KB per stage
//   warp 1     MMA issuer: four M128 N256 contractions per stage (K16 bf16 or
//              K32 e4m3, both operands K-major), accumulating into one of two
//              256-column TMEM accumulators
//   warps 2-5  epilogue: TMEM -> registers (thread = output row) -> bf16
//              (times a_scale[row] * w_scale[col] for e4m3) -> swizzled shared
//              memory -> TMA store, 128 columns at a time, while the MMA warp
//              already fills the other accumulator.
// Ragged M, D and K edges are handled by the tensor maps: loads outside the
// tensor read zeros, stores outside it are dropped.
//
// k_quant_rows_e4m3: per-row e4m3 quantisation, one warp per row:
//   scale = amax / 448 (1 for an all-zero row), code = e4m3_rn_satfinite(x *
//   (448 / amax)), all in fp32 with IEEE rounding.
#pragma once

#include "sm100_ptx.cuh"

namespace vdn {

constexpr int kLinThreads = 192;
constexpr int kLinBM = 128;
constexpr int kLinBN = 256;
constexpr int kLinStages = 4;
constexpr uint32_t kLinStageA = 16384;                 // 128 rows x 128 B
constexpr uint32_t kLinStageB = 32768;                 // 256 rows x 128 B
constexpr uint32_t kLinStage = kLinStageA + kLinStageB;
constexpr uint32_t kLinSmemOut = kLinStages * kLinStage;           // 192 KB
constexpr uint32_t kLinSmemBytes = kLinSmemOut + 32768 + 1024;     // + 32 KB staging

struct LinParams {
  int M, K, D;            // A [M, K], W [D, K], Y [M, D]
  int tiles_m, tiles_n;
  const float* a_scale;   // e4m3 only: [M]
  const float* w_scale;   // e4m3 only: [D]
};

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1)
      : "memory");
}

template <bool kFp8>
__global__ void __launch_bounds__(kLinThreads, 1)
    k_linear(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tw,
             const __grid_constant__ CUtensorMap ty, const LinParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_full[kLinStages], bar_empty[kLinStages], bar_acc_full[2],
      bar_acc_empty[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sOut = base + kLinSmemOut;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.tiles_m * p.tiles_n;
  // K elements per stage: 64 bf16 or 128 e4m3 (128 bytes per row either way)
  constexpr int kBK = kFp8 ? 128 : 64;
  const int nk = (p.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < kLinStages; ++i) {
      mbar_init(smem_u32(&bar_full[i]), 1);
      mbar_init(smem_u32(&bar_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_acc_full[i]), 1);
      mbar_init(smem_u32(&bar_acc_empty[i]), 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_v = &abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      tma_prefetch_desc(&ta);
      tma_prefetch_desc(&tw);
      int it = 0;
      for (int t = blockIdx.x; t < ntiles && !*abort_v; t += gridDim.x) {
        const int m0 = (t / p.tiles_n) * kLinBM, n0 = (t % p.tiles_n) * kLinBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int st = it % kLinStages;
          const uint32_t ph = (uint32_t)((it / kLinStages) & 1);
          if (!mbar_wait(smem_u32(&bar_empty[st]), ph ^ 1)) { *abort_v = 1; break; }
          const uint32_t full = smem_u32(&bar_full[st]);
          const uint32_t sA = base + (uint32_t)st * kLinStage;
          mbar_arrive_expect_tx(full, kLinStage);
          tma_load_2d(sA, &ta, full, kb * kBK, m0);
          tma_load_2d(sA + kLinStageA, &tw, full, kb * kBK, n0);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t idesc = kFp8 ? idesc_e4m3(kLinBM, kLinBN, false, false) : idesc_bf16(kLinBM, kLinBN, false, false);
      int it = 0, tl = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tl) {
        const int buf = tl & 1;
        if (!mbar_wait(smem_u32(&bar_acc_empty[buf]), (uint32_t)(((tl >> 1) & 1) ^ 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dacc = tmem + (uint32_t)(buf * kLinBN);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int st = it % kLinStages;
          const uint32_t ph = (uint32_t)((it / kLinStages) & 1);
          if (!mbar_wait_spin(smem_u32(&bar_full[st]), ph)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sA = base + (uint32_t)st * kLinStage;
          const uint32_t sB = sA + kLinStageA;
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const uint64_t da = sdesc_sw128(sA + (uint32_t)(s * 32), 16, 1024);
            const uint64_t db = sdesc_sw128(sB + (uint32_t)(s * 32), 16, 1024);
            const uint32_t acc = (kb > 0 || s > 0) ? 1u : 0u;
            if (kFp8)
              umma_f8_ss(dacc, da, db, idesc, acc);
            else
              umma_bf16_ss(dacc, da, db, idesc, acc);
          }
          umma_commit(smem_u32(&bar_empty[st]));
        }
        if (!ok) break;
        umma_commit(smem_u32(&bar_acc_full[buf]));
      }
      if (!ok) *abort_v = 1;
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue --
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int r = q * 32 + lane;            // output row within the tile
    const int et = threadIdx.x - 64;        // 0..127
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    int tl = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++tl) {
      const int m0 = (t / p.tiles_n) * kLinBM, n0 = (t % p.tiles_n) * kLinBN;
      const int buf = tl & 1;
      const bool mine = mbar_wait(smem_u32(&bar_acc_full[buf]), (uint32_t)((tl >> 1) & 1));
      // uniform over the 128 epilogue threads: all leave or none does
      if (!named_barrier_and(1, 128, mine)) {
        *abort_v = 1;
        break;
      }
      tc_fence_after();
      float sa = 1.f;
      if (kFp8) sa = (m0 + r < p.M) ? __ldg(p.a_scale + m0 + r) : 0.f;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + (uint32_t)(buf * kLinBN + half * 128 + c * 32), v);
          tmem_ld_wait(v);
          const int col0 = n0 + half * 128 + c * 32;
          float f[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
          if (kFp8) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float ws = (col0 + e < p.D) ? __ldg(p.w_scale + col0 + e) : 0.f;
              f[e] *= sa * ws;
            }
          }
#pragma unroll
          for (int uu = 0; uu < 4; ++uu) {
            const int cc = c * 32 + uu * 8;   // column within the 128-column half
            st_shared_v4(sOut + (uint32_t)(cc >> 6) * 16384u +
                             sw128_off((uint32_t)r, (uint32_t)((cc & 63) >> 3)),
                         pack_bf16x2(f[uu * 8 + 0], f[uu * 8 + 1]),
                         pack_bf16x2(f[uu * 8 + 2], f[uu * 8 + 3]),
                         pack_bf16x2(f[uu * 8 + 4], f[uu * 8 + 5]),
                         pack_bf16x2(f[uu * 8 + 6], f[uu * 8 + 7]));
          }
        }
        if (half == 1) {
          // both halves of this accumulator are in registers / staging: the
          // MMA warp may refill it
          tc_fence_before();
        }
        fence_proxy_async_smem();
        named_barrier_sync(1, 128);
        if (et == 0) {
          if (half == 1) mbar_arrive(smem_u32(&bar_acc_empty[buf]));
          tma_store_2d(&ty, sOut, n0 + half * 128, m0);
          tma_store_2d(&ty, sOut + 16384u, n0 + half * 128 + 64, m0);
          bulk_commit_group();
          bulk_wait_read_all();  // staging is rewritten by the next half
        }
        named_barrier_sync(1, 128);
      }
    }
    if (et == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Per-row e4m3 quantisation of a bf16 matrix [rows, K] (K % 8 == 0), one warp
// per row: scales[row] = amax / 448, codes = e4m3(x * (448 / amax)).
// Rows of up to kQuantRegUnits x 32 16-byte units (K <= 6144) stay in
// registers between the amax and the code pass, so each row is read from
// memory once and all of a lane's loads are in flight together; longer rows
// are read twice.
constexpr int kQuantRegUnits = 24;

__device__ __forceinline__ float amax_bf16x8(uint4 u) {
  const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
  float m = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) m = fmaxf(m, fmaxf(fabsf(bf_lo(w4[e])), fabsf(bf_hi(w4[e]))));
  return m;
}

// 8 bf16 values times inv -> 8 e4m3 codes, in memory order
__device__ __forceinline__ uint2 codes_bf16x8(uint4 u, float inv) {
  const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
  uint32_t packed[2];
#pragma unroll
  for (int e = 0; e < 4; e += 2) {
    uint16_t lo, hi;
    // the first source lands in the upper byte: (x1, x0) puts x0 first in memory
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
        : "=h"(lo)
        : "f"(__fmul_rn(bf_hi(w4[e]), inv)), "f"(__fmul_rn(bf_lo(w4[e]), inv)));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
        : "=h"(hi)
        : "f"(__fmul_rn(bf_hi(w4[e + 1]), inv)), "f"(__fmul_rn(bf_lo(w4[e + 1]), inv)));
    packed[e >> 1] = (uint32_t)lo | ((uint32_t)hi << 16);
  }
  return make_uint2(packed[0], packed[1]);
}

__global__ void k_quant_rows_e4m3(const __nv_bfloat16* __restrict__ x, int64_t rows, int K,
                                  uint8_t* __restrict__ codes, float* __restrict__ scales) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + row * K);
  uint2* dst = reinterpret_cast<uint2*>(codes + row * K);
  const int nv = K >> 3;
  float amax = 0.f;
  if (nv <= kQuantRegUnits * 32) {
    uint4 xr[kQuantRegUnits];
#pragma unroll
    for (int u = 0; u < kQuantRegUnits; ++u) {
      const int i = lane + 32 * u;
      xr[u] = i < nv ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kQuantRegUnits; ++u) amax = fmaxf(amax, amax_bf16x8(xr[u]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
    if (lane == 0) scales[row] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
#pragma unroll
    for (int u = 0; u < kQuantRegUnits; ++u) {
      const int i = lane + 32 * u;
      if (i < nv) dst[i] = codes_bf16x8(xr[u], inv);
    }
    return;
  }
  for (int i = lane; i < nv; i += 32) amax = fmaxf(amax, amax_bf16x8(__ldg(src + i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
  if (lane == 0) scales[row] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  for (int i = lane; i < nv; i += 32) dst[i] = codes_bf16x8(__ldg(src + i), inv);
}

}  // namespace vdn
