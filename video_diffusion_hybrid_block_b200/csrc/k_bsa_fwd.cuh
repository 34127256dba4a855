// Softmax branch of the hybrid layer: block-sparse bidirectional attention.
//
// Each query block (5 latent frames) attends exactly to the keys of its own
// and its neighbouring blocks, the first and last frames (boundary anchors)
// and every text token, with softmax scale 1/sqrt(d) ["VDN-MiniMax-H3"
// (openi.cn), 技术原理：局部精确、远程压缩; nav.superapi.store page, Technical
// Principles, Local Softmax Branch / Text Dual-Branch Injection].
//
// One CTA = one 128-row query tile of one block and one head. Key tiles are
// enumerated from the block's key segments (layer_plan.cuh), so tiles outside
// the allowed set are never loaded; only the ragged last tile of each segment
// is masked column-wise. Warp roles:
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r); online
//              softmax in the exp2 domain with a lazily updated running max
//              (O and l are rescaled only when the max grows by > 2^8);
//              writes P (bf16) to shared memory; final 1/l and bf16 store.
//   warp 4     TMA producer: Q once, then K and V tiles (2-stage ring).
//   warp 5     MMA issuer: S = Q K^T into a double-buffered TMEM S, then
//              O += P V into TMEM O, committing to mbarriers.
// TMEM columns: S0 [0,128), S1 [128,256), O [256,384).
#pragma once

#include "layer_plan.cuh"
#include "sm100_ptx.cuh"

namespace vdn {

constexpr int kBsaThreads = 192;
constexpr uint32_t kBsaSmemQ = 0;
constexpr uint32_t kBsaSmemK = 32768;          // 2 stages x 32 KB
constexpr uint32_t kBsaSmemV = 32768 * 3;      // 2 stages x 32 KB
constexpr uint32_t kBsaSmemP = 32768 * 5;      // 32 KB
constexpr uint32_t kBsaSmemBytes = 32768 * 6 + 1024;  // + alignment slack

struct BsaParams {
  const int32_t* off;  // [F+1] device
  int F, T, H, bf, N;
  float scale_log2;    // log2(e) / sqrt(d)
  __nv_bfloat16* o;    // o_soft output base
  int64_t o_row_stride;  // elements between consecutive tokens
  int d_store;         // leading columns of each head row to store
  float* lse;          // optional [H][N]
};

__global__ void __launch_bounds__(kBsaThreads, 1)
    k_bsa_fwd(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tkt,
              const __grid_constant__ CUtensorMap tvt, const BsaParams p) {
  const int tile = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  int q0, q1;
  block_rows(p.off, p.F, p.bf, b, q0, q1);
  const int qs = q0 + tile * kTile;
  if (qs >= q1) return;  // uniform over the CTA, before any resource is taken
  const int qrows = imin(kTile, q1 - qs);
  const KeySegs segs = key_segments(p.off, p.F, p.bf, p.T, b);
  const int nkt = segs_tiles(segs);

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q, bar_kf[2], bar_ke[2], bar_vf[2], bar_ve[2], bar_sf[2],
      bar_sfree[2], bar_p, bar_o;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + kBsaSmemQ;
  const uint32_t sK[2] = {base + kBsaSmemK, base + kBsaSmemK + 32768};
  const uint32_t sV[2] = {base + kBsaSmemV, base + kBsaSmemV + 32768};
  const uint32_t sP = base + kBsaSmemP;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t q_full = smem_u32(&bar_q);
  const uint32_t k_full[2] = {smem_u32(&bar_kf[0]), smem_u32(&bar_kf[1])};
  const uint32_t k_empty[2] = {smem_u32(&bar_ke[0]), smem_u32(&bar_ke[1])};
  const uint32_t v_full[2] = {smem_u32(&bar_vf[0]), smem_u32(&bar_vf[1])};
  const uint32_t v_empty[2] = {smem_u32(&bar_ve[0]), smem_u32(&bar_ve[1])};
  const uint32_t s_full[2] = {smem_u32(&bar_sf[0]), smem_u32(&bar_sf[1])};
  const uint32_t s_free[2] = {smem_u32(&bar_sfree[0]), smem_u32(&bar_sfree[1])};
  const uint32_t p_full = smem_u32(&bar_p);
  const uint32_t o_done = smem_u32(&bar_o);

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(k_full[i], 1);
      mbar_init(k_empty[i], 1);
      mbar_init(v_full[i], 1);
      mbar_init(v_empty[i], 1);
      mbar_init(s_full[i], 1);
      mbar_init(s_free[i], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(&tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_v = &abort_flag;

  if (warp == 4) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      mbar_arrive_expect_tx(q_full, 32768);
      tma_load_3d(sQ, &tq, q_full, 0, h, qs);
      tma_load_3d(sQ + 16384, &tq, q_full, 64, h, qs);
      for (int j = 0; j < nkt; ++j) {
        if (*abort_v) break;
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        int src, row0, valid;
        segs_tile(segs, j, src, row0, valid);
        const CUtensorMap* mk = src ? &tkt : &tk;
        const CUtensorMap* mv = src ? &tvt : &tv;
        if (!mbar_wait(k_empty[st], ph ^ 1)) { *abort_v = 1; break; }
        mbar_arrive_expect_tx(k_full[st], 32768);
        tma_load_3d(sK[st], mk, k_full[st], 0, h, row0);
        tma_load_3d(sK[st] + 16384, mk, k_full[st], 64, h, row0);
        if (!mbar_wait(v_empty[st], ph ^ 1)) { *abort_v = 1; break; }
        mbar_arrive_expect_tx(v_full[st], 32768);
        tma_load_3d(sV[st], mv, v_full[st], 0, h, row0);
        tma_load_3d(sV[st] + 16384, mv, v_full[st], 64, h, row0);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // -------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(128, 128, false, false);
      const uint32_t idO = idesc_bf16(128, 128, false, true);
      bool ok = mbar_wait(q_full, 0);
      tc_fence_after();
      // S(j) = Q K(j)^T into TMEM buffer j&1
      auto issue_qk = [&](int j) -> bool {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(k_full[st], ph)) return false;
        if (!mbar_wait(s_free[st], ph ^ 1)) return false;
        tc_fence_after();
        const uint32_t dS = tmem + (uint32_t)(st * 128);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint32_t ko = (uint32_t)((s >> 2) * 16384 + (s & 3) * 32);
          umma_bf16_ss(dS, sdesc_sw128(sQ + ko, 16, 1024), sdesc_sw128(sK[st] + ko, 16, 1024),
                       idS, s > 0 ? 1u : 0u);
        }
        umma_commit(k_empty[st]);
        umma_commit(s_full[st]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int j = 0; ok && j < nkt; ++j) {
        if (*abort_v) { ok = false; break; }
        if (j + 1 < nkt && !issue_qk(j + 1)) { ok = false; break; }
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(p_full, (uint32_t)(j & 1))) { ok = false; break; }
        if (!mbar_wait(v_full[st], ph)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          umma_bf16_ss(tmem + 256, sdesc_sw128(sP + (uint32_t)((s >> 2) * 16384 + (s & 3) * 32), 16, 1024),
                       sdesc_sw128(sV[st] + (uint32_t)(s * 2048), 16384, 1024), idO,
                       (j > 0 || s > 0) ? 1u : 0u);
        }
        umma_commit(v_empty[st]);
        umma_commit(o_done);
      }
      if (!ok) *abort_v = 1;
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------- softmax warps --
    const int r = threadIdx.x;  // query row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m_use = 0.f, l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < nkt; ++j) {
      if (*abort_v) { ok = false; break; }
      const int st = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      int src, row0, valid;
      segs_tile(segs, j, src, row0, valid);
      if (!mbar_wait(s_full[st], ph)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[128];
      tmem_ld128(tmem + lane_base + (uint32_t)(st * 128), s);
      tmem_ld_wait128(s);
      tc_fence_before();
      mbar_arrive(s_free[st]);

      float mloc = -INFINITY;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        float x = __uint_as_float(s[i]) * p.scale_log2;
        x = (i < valid) ? x : -INFINITY;
        s[i] = __float_as_uint(x);
        mloc = fmaxf(mloc, x);
      }
      bool need = false;
      float factor = 1.f;
      if (j == 0) {
        m_use = mloc;
      } else if (mloc > m_use + 8.f) {
        need = true;
        factor = ex2_approx(m_use - mloc);
        m_use = mloc;
        l_sum *= factor;
      }
      float rs = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float e0 = ex2_approx(__uint_as_float(s[2 * i]) - m_use);
        const float e1 = ex2_approx(__uint_as_float(s[2 * i + 1]) - m_use);
        rs += e0 + e1;
        pk[i] = pack_bf16x2(e0, e1);
      }
      l_sum += rs;
      // PV(j-1) must be done: P buffer is reused and O may be rescaled.
      if (j > 0 && !mbar_wait(o_done, (uint32_t)((j - 1) & 1))) { ok = false; break; }
      tc_fence_after();
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + 256u + (uint32_t)(c * 32), o);
          tmem_ld_wait(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
          tmem_st32(tmem + lane_base + 256u + (uint32_t)(c * 32), o);
        }
        tmem_st_wait();
      }
      // P row r -> shared memory, 128B-swizzled K-major (two 64-key chunks)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = c * 32 + u * 4;
          st_shared_v4(sP + (uint32_t)(c * 16384) + sw128_off((uint32_t)r, (uint32_t)u), pk[i],
                       pk[i + 1], pk[i + 2], pk[i + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && !mbar_wait(o_done, (uint32_t)((nkt - 1) & 1))) ok = false;
    if (!ok) *abort_v = 1;
    tc_fence_after();
    uint32_t o[128];
    tmem_ld128(tmem + lane_base + 256u, o);
    tmem_ld_wait128(o);
    if (ok && r < qrows) {
      const float inv = 1.f / l_sum;
      __nv_bfloat16* dst = p.o + (int64_t)(qs + r) * p.o_row_stride + (int64_t)h * p.d_store;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        if (u * 8 < p.d_store) {
          uint4 val;
          val.x = pack_bf16x2(__uint_as_float(o[u * 8 + 0]) * inv, __uint_as_float(o[u * 8 + 1]) * inv);
          val.y = pack_bf16x2(__uint_as_float(o[u * 8 + 2]) * inv, __uint_as_float(o[u * 8 + 3]) * inv);
          val.z = pack_bf16x2(__uint_as_float(o[u * 8 + 4]) * inv, __uint_as_float(o[u * 8 + 5]) * inv);
          val.w = pack_bf16x2(__uint_as_float(o[u * 8 + 6]) * inv, __uint_as_float(o[u * 8 + 7]) * inv);
          *reinterpret_cast<uint4*>(dst + u * 8) = val;
        }
      }
      if (p.lse != nullptr)
        p.lse[(int64_t)h * p.N + qs + r] = (m_use + __log2f(l_sum)) * 0.69314718055994531f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace vdn
