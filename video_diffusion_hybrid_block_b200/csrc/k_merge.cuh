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

// Same operation for the common case (bf16 out, d = 128, o_soft [N, H, 128]
// bf16), streamed and warp-specialised, with separate rings for q and o_soft
// so that neither waits on the other's release:
//   warp 8 lane 0  issues o_lin = q R_b into a double-buffered TMEM
//                  accumulator; each contraction's commit frees its q stage
//   warp 8 lane 1  loads q tiles (3-stage ring), as soon as a stage is free
//   warp 8 lane 2  loads o_soft tiles (3-stage ring)
//   warp 8 lane 3  stores: once all epilogue threads have staged a full tile
//                  it sends it with one TMA store, waits until the store has
//                  read the stage and frees it for the o_soft loader
//   warps 0-7      epilogue: warp w reads TMEM lane quarter w % 4 and column
//                  half w / 4 (the RMSNorm sum of squares of a row is the sum
//                  of its halves, exchanged through shared memory); a full
//                  tile of `out` overwrites its o_soft tile in place (each
//                  thread rewrites the 16-byte units it read) and is handed
//                  to the store lane, so the epilogue moves on to the next
//                  tile without waiting for the store; a block's ragged last
//                  tile is stored row by row.
constexpr int kMergeTmaThreads = 288;          // 8 epilogue warps + the load / MMA warp
constexpr int kMergeTmaEpi = 256;
constexpr int kMergeTmaStages = 3;
constexpr int kMergeTmaTiles = 14;           // 3 CTAs cover a 40-tile block
constexpr uint32_t kMergeTmaSmemR = 0;       // 32 KB
constexpr uint32_t kMergeTmaSmemQ = 32768;   // q stage s at 32 KB + 32 KB s
constexpr uint32_t kMergeTmaSmemO = 32768 + kMergeTmaStages * 32768;  // o_soft stage s
constexpr uint32_t kMergeTmaSmemBytes = (1 + 2 * kMergeTmaStages) * 32768 + 1024;

__global__ void __launch_bounds__(kMergeTmaThreads, 1)
    k_readout_merge_tma(const __grid_constant__ CUtensorMap tq,
                        const __grid_constant__ CUtensorMap tos,
                        const __grid_constant__ CUtensorMap tout, const MergeParams p) {
  const int b = blockIdx.y, h = blockIdx.z;
  int q0, q1;
  block_rows(p.off, p.F, p.bf, b, q0, q1);
  const int t_first = blockIdx.x * kMergeTmaTiles;
  const int ntl = imin(kMergeTmaTiles, (q1 - q0 + kTile - 1) / kTile - t_first);
  if (ntl <= 0) return;

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full[kMergeTmaStages], q_empty[kMergeTmaStages], o_full[kMergeTmaStages],
      o_empty[kMergeTmaStages], o_staged[kMergeTmaStages], acc_full[2], acc_empty[2], r_ready;
  __shared__ uint32_t tmem_slot;
  __shared__ float wsm[128];
  __shared__ float ssh[2][128];  // per-row sums of squares of the two column halves
  __shared__ int abort_flag;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sR = base + kMergeTmaSmemR;
  const int i = threadIdx.x, warp = i >> 5;
  auto sQ = [&](int st) { return base + kMergeTmaSmemQ + (uint32_t)st * 32768u; };
  auto sO = [&](int st) { return base + kMergeTmaSmemO + (uint32_t)st * 32768u; };

  if (i == 0) {
    abort_flag = 0;
    for (int k = 0; k < kMergeTmaStages; ++k) {
      mbar_init(smem_u32(&q_full[k]), 1);
      mbar_init(smem_u32(&q_empty[k]), 1);
      mbar_init(smem_u32(&o_full[k]), 1);
      mbar_init(smem_u32(&o_empty[k]), 1);
      mbar_init(smem_u32(&o_staged[k]), kMergeTmaEpi);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(smem_u32(&acc_full[k]), 1);
      mbar_init(smem_u32(&acc_empty[k]), 1);
    }
    mbar_init(smem_u32(&r_ready), kMergeTmaEpi);
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
  volatile int* abort_v = &abort_flag;

  if (warp == 8) {
    const int lane = i & 31;
    if (lane == 1 || lane == 2) {
      // -------------------------------------------------------- loaders
      const CUtensorMap* m = lane == 1 ? &tq : &tos;
      tma_prefetch_desc(m);
      for (int t = 0; t < ntl; ++t) {
        if (*abort_v) break;
        const int st = t % kMergeTmaStages;
        const uint32_t ph = (uint32_t)((t / kMergeTmaStages) & 1);
        const uint32_t empty = smem_u32(lane == 1 ? &q_empty[st] : &o_empty[st]);
        const uint32_t full = smem_u32(lane == 1 ? &q_full[st] : &o_full[st]);
        if (!mbar_wait(empty, ph ^ 1)) { *abort_v = 1; break; }
        const uint32_t dst = lane == 1 ? sQ(st) : sO(st);
        const int row = q0 + (t_first + t) * kTile;
        mbar_arrive_expect_tx(full, 32768);
        tma_load_3d(dst, m, full, 0, h, row);
        tma_load_3d(dst + 16384, m, full, 64, h, row);
      }
    }
    if (lane == 3) {
      // ------------------------------------------------------------ stores
      tma_prefetch_desc(&tout);
      for (int t = 0; t < ntl; ++t) {
        if (*abort_v) break;
        const int st = t % kMergeTmaStages;
        if (!mbar_wait(smem_u32(&o_staged[st]), (uint32_t)((t / kMergeTmaStages) & 1))) {
          *abort_v = 1;
          break;
        }
        const int row0 = q0 + (t_first + t) * kTile;
        if (row0 + kTile <= q1) {
          tma_store_3d(&tout, sO(st), 0, h, row0);
          tma_store_3d(&tout, sO(st) + 16384, 64, h, row0);
          bulk_commit_group();
          bulk_wait_read_all();  // the stage may be refilled once the store has read it
        }
        mbar_arrive(smem_u32(&o_empty[st]));
      }
      bulk_wait_all();
    }
    // The four lanes run independently; none of them takes part in a named
    // barrier, so a lane blocked on a stage never holds up the others.
    if (lane == 0) {
      // ----------------------------------------------------- contractions
      const uint32_t idO = idesc_bf16(128, 128, false, true);
      // R_b is in shared memory once all epilogue threads have arrived
      if (!mbar_wait(smem_u32(&r_ready), 0)) *abort_v = 1;
      for (int t = 0; t < ntl; ++t) {
        if (*abort_v) break;
        const int st = t % kMergeTmaStages, ab = t & 1;
        if (!mbar_wait(smem_u32(&q_full[st]), (uint32_t)((t / kMergeTmaStages) & 1))) {
          *abort_v = 1;
          break;
        }
        if (t >= 2 && !mbar_wait(smem_u32(&acc_empty[ab]), (uint32_t)(((t - 2) >> 1) & 1))) {
          *abort_v = 1;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 8; ++s)
          umma_bf16_ss(tmem + (uint32_t)(ab * 128),
                       sdesc_sw128(sQ(st) + (uint32_t)((s >> 2) * 16384 + (s & 3) * 32), 16, 1024),
                       sdesc_sw128(sR + (uint32_t)(s * 2048), 16384, 1024), idO, s > 0 ? 1u : 0u);
        umma_commit(smem_u32(&acc_full[ab]));
        umma_commit(smem_u32(&q_empty[st]));  // the q stage is free once this has run
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // R_b (fwd + bwd) -> bf16, MN-major 128B-swizzled: thread i converts
    // chunk i / 128 (64 value dims) of row i % 128 (key dim)
    {
      const int rr = i & 127, c = i >> 7;
      const int64_t rbase = ((int64_t)b * p.H + h) * 128 * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4* ra = reinterpret_cast<const float4*>(p.RA + rbase + (int64_t)rr * 128 + c * 64 + u * 8);
        float4 x0 = __ldg(ra), x1 = __ldg(ra + 1);
        if (p.RB) {
          const float4* rb = reinterpret_cast<const float4*>(p.RB + rbase + (int64_t)rr * 128 + c * 64 + u * 8);
          const float4 y0 = __ldg(rb), y1 = __ldg(rb + 1);
          x0 = make_float4(x0.x + y0.x, x0.y + y0.y, x0.z + y0.z, x0.w + y0.w);
          x1 = make_float4(x1.x + y1.x, x1.y + y1.y, x1.z + y1.z, x1.w + y1.w);
        }
        st_shared_v4(sR + (uint32_t)(c * 16384) + sw128_off((uint32_t)rr, (uint32_t)u),
                     pack_bf16x2(x0.x, x0.y), pack_bf16x2(x0.z, x0.w), pack_bf16x2(x1.x, x1.y),
                     pack_bf16x2(x1.z, x1.w));
      }
    }
    if (i < 128) wsm[i] = __ldg(p.rms_w + (int64_t)h * 128 + i);
    fence_proxy_async_smem();
    mbar_arrive(smem_u32(&r_ready));      // R_b written (async-proxy visible)
    named_barrier_sync(2, kMergeTmaEpi);  // wsm written
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + (i & 31);   // row of the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    // gate logits one tile ahead, kept as raw bits until the next tile uses
    // them: a conversion right after the load would stall the warp for the
    // load's whole latency
    auto gate_bits = [&](const void* g, int row) -> uint32_t {
      if (row >= q1) return 0u;
      const int64_t gi = (int64_t)row * p.H + h;
      return p.gate_f32 ? __float_as_uint(__ldg(reinterpret_cast<const float*>(g) + gi))
                        : (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(g) + gi);
    };
    auto gate_val = [&](uint32_t bits) -> float {
      return sigmoidf_(p.gate_f32 ? __uint_as_float(bits) : __uint_as_float(bits << 16));
    };
    uint32_t gs_next = gate_bits(p.g_s, q0 + t_first * kTile + r);
    uint32_t gl_next = gate_bits(p.g_l, q0 + t_first * kTile + r);
    for (int t = 0; t < ntl; ++t) {
      const int st = t % kMergeTmaStages, ab = t & 1;
      const int row0 = q0 + (t_first + t) * kTile;
      const int row = row0 + r;
      const bool valid = row < q1;
      const bool full_tile = row0 + kTile <= q1;
      const uint32_t gs_bits = gs_next, gl_bits = gl_next;
      if (t + 1 < ntl) {
        gs_next = gate_bits(p.g_s, row + kTile);
        gl_next = gate_bits(p.g_l, row + kTile);
      }
      const bool mine = !*abort_v &&
                        mbar_wait(smem_u32(&acc_full[ab]), (uint32_t)((t >> 1) & 1)) &&
                        mbar_wait(smem_u32(&o_full[st]), (uint32_t)((t / kMergeTmaStages) & 1));
      // uniform over the 256 epilogue threads: all leave or none does
      if (!named_barrier_and(2, kMergeTmaEpi, mine)) {
        *abort_v = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tO = tmem + lane_base + (uint32_t)(ab * 128 + half * 64);
      uint32_t o[2][32];
      tmem_ld32(tO, o[0]);
      tmem_ld32(tO + 32u, o[1]);
      tmem_ld_wait(o[0]);
      tmem_ld_wait(o[1]);
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(o[c][e]), __uint_as_float(o[c][e]), ss);
      ssh[half][r] = ss;
      // both halves' sums are written; the TMEM buffer has been read
      tc_fence_before();
      named_barrier_sync(2, kMergeTmaEpi);
      if (i == 0) mbar_arrive(smem_u32(&acc_empty[ab]));
      ss = ssh[0][r] + ssh[1][r];
      const float gsv = valid ? gate_val(gs_bits) : 0.f;
      const float nr = (valid ? gate_val(gl_bits) : 0.f) * rsqrtf(ss * (1.f / 128.f) + p.eps);
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + ((int64_t)row * p.H + h) * 128;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c0 = half * 64 + c * 32 + u * 8;
          const uint32_t off = (uint32_t)half * 16384u + sw128_off((uint32_t)r, (uint32_t)((c0 & 63) >> 3));
          const uint4 ov = ld_shared_v4(sO(st) + off);
          const uint32_t w4[4] = {ov.x, ov.y, ov.z, ov.w};
          uint32_t y4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int cc = c0 + 2 * e;
            const float ylo = gsv * bf_lo(w4[e]) + nr * wsm[cc] * __uint_as_float(o[c][u * 8 + 2 * e]);
            const float yhi = gsv * bf_hi(w4[e]) + nr * wsm[cc + 1] * __uint_as_float(o[c][u * 8 + 2 * e + 1]);
            y4[e] = pack_bf16x2(ylo, yhi);
          }
          if (full_tile)
            st_shared_v4(sO(st) + off, y4[0], y4[1], y4[2], y4[3]);  // in place
          else if (valid)
            *reinterpret_cast<uint4*>(orow + c0) = make_uint4(y4[0], y4[1], y4[2], y4[3]);
        }
      }
      // this thread's part of the tile is staged (or, for a ragged tile,
      // its reads of the o_soft stage are done)
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&o_staged[st]));
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
