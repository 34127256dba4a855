// Video Delta Attention (linear branch): per-frame Grams, per-frame SPD
// inverses and the two text-initialised state scans.
//
// VDA replaces the token-by-token delta rule with one joint solve per frame:
// the normal equations of all spatial tokens of the frame determine the new
// state; the text writes the state once at initialisation; the branch sums
// the context before and after the current window
// [nav.superapi.store page, Technical Principles, Video Delta Attention and
// Text Dual-Branch Injection; "VDN-MiniMax-H3" (openi.cn), 技术原理].
// Reading implemented: k_hat = k / max(||k||, 1e-12),
//   M_f = lambda I + K_f^T K_f, C_f = K_f^T V_f,
//   S_f = M_f^-1 (lambda S_prev + C_f), S_text = M_t^-1 C_t.
//
// k_vda_gram_inv: one CTA per (matrix m, head): m = 0 is the text, m = f is
//   latent frame f (1 <= f <= F-2; anchors 0 and F-1 are never scanned).
//   Streams the frame's k, v rows in 64-token tiles (TMA, 3-stage ring),
//   L2-normalises k rows in shared memory, accumulates G = K^T K and
//   C^T = V^T K as two M=128 x N=128 bf16 tcgen05 contractions into TMEM,
//   writes C^T (fp32, the layout the scan loads as its X operand)
//   and then inverts M = lambda I + G (2 x 2 blocks of 64: two 64-pivot
//   Gauss-Jordan sweeps in registers, no pivoting since M is symmetric
//   positive definite with eigenvalues >= lambda, and four 64^3 products
//   through the Schur complement) and writes W = M^-1 (fp32, tf32-rounded).
// Only frames whose state some block reads are processed: the forward scan
//   stops at the largest forward read index, the backward scan at the
//   smallest backward one (the remaining frames always sit inside the window
//   of every block that could reach them), unless per-frame states are asked
//   for.
// k_vda_scan: one CTA per (direction, head, value-column half). Step 0
//   applies the text (S = W_t C_t), then one step per frame:
//   X = lambda S + C_f, S = W_f X as a tf32 tcgen05 contraction (W and C_f^T
//   via TMA, lambda S^T added in shared memory, D in TMEM). States a block
//   reads go to Rpart[dir][b]; optional per-frame / text outputs too.
#pragma once

#include "layer_plan.cuh"
#include "sm100_ptx.cuh"

namespace vdn {

// ------------------------------------------------------------ Gram + inverse

constexpr int kGramThreads = 256;
constexpr int kGramTok = 64;                // tokens per tile
constexpr int kGramStages = 3;
constexpr uint32_t kGramStage = 4 * 8192;  // k chunk0, k chunk1, v chunk0, v chunk1
// 3 stages (96 KB, reused for G once the Grams are done); at most two CTAs
// share an SM (two x 256 TMEM columns).
constexpr uint32_t kGramSmemBytes = kGramStages * kGramStage + 1024;

struct GramParams {
  const int32_t* off;  // [F+1] device
  int F, T, H;
  int fwd_last;        // frames 1..fwd_last feed the forward scan
  int bwd_first;       // frames bwd_first..F-2 feed the backward scan
  float lambda;
  float* Cmat;  // [F-1][H][128][128], C^T = V^T K_hat (row = value dim)
  float* Wmat;  // [F-1][H][128][128]
};

__global__ void __launch_bounds__(kGramThreads, 2)
    k_vda_gram_inv(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                   const __grid_constant__ CUtensorMap tkt, const __grid_constant__ CUtensorMap tvt,
                   const GramParams p) {
  // blockIdx.x enumerates the text (0), frames 1..fwd_last, then the frames
  // max(bwd_first, fwd_last+1)..F-2; matrices keep index m = frame.
  const int h = blockIdx.y;
  int m = blockIdx.x;
  if (m > p.fwd_last) m = imax(p.bwd_first, p.fwd_last + 1) + (m - p.fwd_last - 1);
  const bool text = (m == 0);
  const int r0 = text ? 0 : p.off[m];
  const int r1 = text ? p.T : p.off[m + 1];
  const int nrows = r1 - r0;
  const int ntiles = (nrows + kGramTok - 1) / kGramTok;
  const CUtensorMap* mk = text ? &tkt : &tk;
  const CUtensorMap* mv = text ? &tvt : &tv;

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_full[kGramStages], bar_empty[kGramStages], bar_done;
  __shared__ uint32_t tmem_slot;
  __shared__ __align__(16) float rowbuf[2][128];
  __shared__ __align__(16) float colbuf[2][128];
  __shared__ int abort_flag;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t done = smem_u32(&bar_done);
  volatile int* abort_v = &abort_flag;

  if (tid == 0) {
    abort_flag = 0;
    for (int i = 0; i < kGramStages; ++i) {
      mbar_init(smem_u32(&bar_full[i]), 1);
      mbar_init(smem_u32(&bar_empty[i]), 1);
    }
    mbar_init(done, 1);
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

  auto load_tile = [&](int i, int st) {
    const uint32_t dst = base + (uint32_t)st * kGramStage;
    const uint32_t bar = smem_u32(&bar_full[st]);
    const int row = r0 + i * kGramTok;
    mbar_arrive_expect_tx(bar, kGramStage);
    tma_load_3d(dst, mk, bar, 0, h, row);
    tma_load_3d(dst + 8192, mk, bar, 64, h, row);
    tma_load_3d(dst + 16384, mv, bar, 0, h, row);
    tma_load_3d(dst + 24576, mv, bar, 64, h, row);
  };
  if (tid == 0) {
    for (int i = 0; i < imin(kGramStages - 1, ntiles); ++i) load_tile(i, i);
  }

  const uint32_t idG = idesc_bf16(128, 128, true, true);
  bool ok = true;
  for (int i = 0; i < ntiles; ++i) {
    const int st = i % kGramStages;
    const uint32_t ph = (uint32_t)((i / kGramStages) & 1);
    if (*abort_v || !mbar_wait(smem_u32(&bar_full[st]), ph)) { ok = false; *abort_v = 1; }
    __syncthreads();
    if (*abort_v) { ok = false; break; }
    // L2-normalise k rows (zero rows beyond the frame, and their v rows):
    // 4 threads per token row, 32 elements (four 16-byte units) each
    const uint32_t stage = base + (uint32_t)st * kGramStage;
    const int row = tid >> 2, part = tid & 3;
    const uint32_t chunk = (uint32_t)(part >> 1);
    const uint32_t u0 = (uint32_t)((part & 1) * 4);
    uint4 kv[4];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      kv[u] = ld_shared_v4(stage + chunk * 8192 + sw128_off((uint32_t)row, u0 + u));
      const uint32_t w4[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf_lo(w4[e]), b = bf_hi(w4[e]);
        ss = fmaf(a, a, fmaf(b, b, ss));
      }
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    const bool valid = (i * kGramTok + row) < nrows;
    const float sc = valid ? 1.f / fmaxf(sqrtf(ss), 1e-12f) : 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t w4[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
      uint32_t o4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) o4[e] = pack_bf16x2(bf_lo(w4[e]) * sc, bf_hi(w4[e]) * sc);
      st_shared_v4(stage + chunk * 8192 + sw128_off((uint32_t)row, u0 + u), o4[0], o4[1], o4[2],
                   o4[3]);
      if (!valid)
        st_shared_v4(stage + 16384 + chunk * 8192 + sw128_off((uint32_t)row, u0 + u), 0u, 0u, 0u,
                     0u);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        // G = K^T K (A = K^T, B = K) and C^T = V^T K (A = V^T, B = K): all
        // operands MN-major straight from the TMA tiles
        const uint64_t dk = sdesc_sw128(stage + (uint32_t)(s * 2048), 8192, 1024);
        const uint64_t dv = sdesc_sw128(stage + 16384u + (uint32_t)(s * 2048), 8192, 1024);
        const uint32_t acc = (i > 0 || s > 0) ? 1u : 0u;
        umma_bf16_ss(tmem, dk, dk, idG, acc);
        umma_bf16_ss(tmem + 128u, dv, dk, idG, acc);
      }
      umma_commit(smem_u32(&bar_empty[st]));
      if (i == ntiles - 1) umma_commit(done);
      // refill the stage the previous tile used (its MMAs are most likely
      // done already) with the tile two ahead
      const int nxt = i + kGramStages - 1;
      if (nxt < ntiles) {
        const int sp = nxt % kGramStages;
        if (i > 0 && !mbar_wait(smem_u32(&bar_empty[sp]), (uint32_t)(((i - 1) / kGramStages) & 1))) {
          *abort_v = 1;
        } else {
          load_tile(nxt, sp);
        }
      }
    }
  }
  if (ok && ntiles > 0 && !mbar_wait(done, 0)) ok = false;
  if (!ok) *abort_v = 1;
  tc_fence_after();
  __syncthreads();

  // TMEM -> C^T (global, fp32) and G (shared, fp32, 16-byte units XOR-swizzled):
  // lane quarter = warp % 4; warps 0-3 read G, warps 4-7 read C^T.
  const uint32_t gs = base;  // reuses the (now idle) staging buffers: 64 KB
  {
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    float* cdst = p.Cmat + (((int64_t)m * p.H + h) * 128 + r) * 128;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t v[32];
      if (ntiles > 0) {
        tmem_ld32(tmem + ((uint32_t)(wq * 32) << 16) + (warp < 4 ? 0u : 128u) + (uint32_t)(c * 32), v);
        tmem_ld_wait(v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
#pragma unroll
      for (int uu = 0; uu < 8; ++uu) {
        const int u = c * 8 + uu;
        if (warp >= 4)
          reinterpret_cast<uint4*>(cdst)[u] =
              make_uint4(v[4 * uu], v[4 * uu + 1], v[4 * uu + 2], v[4 * uu + 3]);
        else
          st_shared_v4(gs + (uint32_t)r * 512u + (((uint32_t)u ^ (uint32_t)(r & 31)) << 4),
                       v[4 * uu], v[4 * uu + 1], v[4 * uu + 2], v[4 * uu + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }

  // Inverse of M = lambda I + G = [[A, B], [B^T, D]] (64 x 64 blocks) by the
  // Schur complement: X = A^-1 B, S = D - B^T X, Y = X S^-1, and
  //   W = M^-1 = [[A^-1 + Y X^T, -Y], [-Y^T, S^-1]].
  // A^-1 and S^-1 come from 64-pivot Gauss-Jordan sweeps (no pivoting: both
  // are symmetric positive definite with eigenvalues >= lambda) on 4 x 4
  // register tiles, thread (ty, tx) holding rows 4ty.., columns 4tx..; the
  // four 64 x 64 x 64 products are sums of rank-1 updates read from shared
  // memory as 16-byte vectors (A^-1 is symmetric; X and Y are also kept
  // transposed). W feeds only the scans' tf32 contractions and is stored
  // rounded to tf32.
  const int ty = tid >> 4, tx = tid & 15;
  // G element (r, c) in the swizzled copy: row r at 512 r, 16-byte unit c / 4
  auto g_addr = [&](int r, int c) -> uint32_t {
    return gs + (uint32_t)r * 512u + ((((uint32_t)(c >> 2)) ^ ((uint32_t)r & 31u)) << 4);
  };
  // 64 x 64 fp32 matrices, row-major (256 B rows): AI and X beyond G (bytes
  // 64K..96K of the staging area); SI, XT and YT over G once it is consumed
  const uint32_t mAI = base + 65536u, mX = base + 81920u;
  const uint32_t mSI = base, mXT = base + 16384u, mYT = base + 32768u;
  auto m_addr = [](uint32_t m, int r, int c) -> uint32_t { return m + (uint32_t)(r * 64 + c) * 4u; };
  auto ld4 = [](uint32_t addr) -> float4 {
    const uint4 v = ld_shared_v4(addr);
    return make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w));
  };
  auto st4 = [](uint32_t addr, float x0, float x1, float x2, float x3) {
    st_shared_v4(addr, __float_as_uint(x0), __float_as_uint(x1), __float_as_uint(x2), __float_as_uint(x3));
  };
  // in-place Gauss-Jordan inverse of a 64 x 64 SPD matrix held in 4 x 4 tiles
  auto gj64 = [&](float (&a)[4][4]) {
    for (int kb = 0; kb < 16; ++kb) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int k = kb * 4 + kk;
        const int buf = k & 1;
        if (ty == kb)
          *reinterpret_cast<float4*>(&rowbuf[buf][4 * tx]) = make_float4(a[kk][0], a[kk][1], a[kk][2], a[kk][3]);
        if (tx == kb)
          *reinterpret_cast<float4*>(&colbuf[buf][4 * ty]) = make_float4(a[0][kk], a[1][kk], a[2][kk], a[3][kk]);
        __syncthreads();
        // pivot >= lambda > 0: the MUFU reciprocal (within a couple of ulp) is
        // enough, and it shortens the per-pivot chain
        float ip;
        asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(ip) : "f"(rowbuf[buf][k]));
        const float4 r4 = *reinterpret_cast<const float4*>(&rowbuf[buf][4 * tx]);
        const float4 c4 = *reinterpret_cast<const float4*>(&colbuf[buf][4 * ty]);
        const float rj[4] = {r4.x * ip, r4.y * ip, r4.z * ip, r4.w * ip};
        const float ci[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 nc = make_float2(-ci[i], -ci[i]);
#pragma unroll
          for (int j = 0; j < 4; j += 2) {
            const float2 upd = ffma2(nc, make_float2(rj[j], rj[j + 1]), make_float2(a[i][j], a[i][j + 1]));
            a[i][j] = upd.x;
            a[i][j + 1] = upd.y;
          }
        }
        if (ty == kb) {
#pragma unroll
          for (int j = 0; j < 4; ++j) a[kk][j] = rj[j];
        }
        if (tx == kb) {
#pragma unroll
          for (int i = 0; i < 4; ++i) a[i][kk] = -ci[i] * ip;
        }
        if (ty == kb && tx == kb) a[kk][kk] = ip;
      }
    }
  };
  // acc[i][j] += sum_k P[4ty+i][k] Q[k][4tx+j], with colP(k) = P[4ty..4ty+3][k]
  // and rowQ(k) = Q[k][4tx..4tx+3] as 16-byte vectors
  auto mm_acc = [&](float (&acc)[4][4], auto colP, auto rowQ) {
#pragma unroll 8
    for (int k = 0; k < 64; ++k) {
      const float4 pv = colP(k);
      const float4 q = rowQ(k);
      const float pi[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 pp = make_float2(pi[i], pi[i]);
        const float2 u0 = ffma2(pp, make_float2(q.x, q.y), make_float2(acc[i][0], acc[i][1]));
        const float2 u1 = ffma2(pp, make_float2(q.z, q.w), make_float2(acc[i][2], acc[i][3]));
        acc[i][0] = u0.x;
        acc[i][1] = u0.y;
        acc[i][2] = u1.x;
        acc[i][3] = u1.y;
      }
    }
  };
  float* wdst = p.Wmat + ((int64_t)m * p.H + h) * 128 * 128;
  auto store_w = [&](int r, int c0, float x0, float x1, float x2, float x3) {
    *reinterpret_cast<float4*>(wdst + (int64_t)r * 128 + c0) =
        make_float4(round_tf32(x0), round_tf32(x1), round_tf32(x2), round_tf32(x3));
  };

  // 1. A^-1 (kept in registers for step 7 too)
  float ai[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 v = ld4(g_addr(4 * ty + i, 4 * tx));
    ai[i][0] = v.x; ai[i][1] = v.y; ai[i][2] = v.z; ai[i][3] = v.w;
  }
  if (ty == tx) {
#pragma unroll
    for (int i = 0; i < 4; ++i) ai[i][i] += p.lambda;
  }
  gj64(ai);
#pragma unroll
  for (int i = 0; i < 4; ++i) st4(m_addr(mAI, 4 * ty + i, 4 * tx), ai[i][0], ai[i][1], ai[i][2], ai[i][3]);
  __syncthreads();
  // 2. X = A^-1 B, B = G[0:64, 64:128]; column k of A^-1's row block = row k (symmetric)
  float xt[4][4] = {};
  mm_acc(xt, [&](int k) { return ld4(m_addr(mAI, k, 4 * ty)); },
         [&](int k) { return ld4(g_addr(k, 64 + 4 * tx)); });
#pragma unroll
  for (int i = 0; i < 4; ++i) st4(m_addr(mX, 4 * ty + i, 4 * tx), xt[i][0], xt[i][1], xt[i][2], xt[i][3]);
  __syncthreads();
  // 3. S = lambda I + G[64:128, 64:128] - B^T X; column k of B^T's row block = row k of B
  float sa[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 v = ld4(g_addr(64 + 4 * ty + i, 64 + 4 * tx));
    sa[i][0] = -v.x; sa[i][1] = -v.y; sa[i][2] = -v.z; sa[i][3] = -v.w;
  }
  if (ty == tx) {
#pragma unroll
    for (int i = 0; i < 4; ++i) sa[i][i] -= p.lambda;
  }
  mm_acc(sa, [&](int k) { return ld4(g_addr(k, 64 + 4 * ty)); },
         [&](int k) { return ld4(m_addr(mX, k, 4 * tx)); });
  // sa = B^T X - D; S = -sa
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) sa[i][j] = -sa[i][j];
  __syncthreads();  // G is consumed: SI, XT, YT may overwrite it
  // X^T tile (this thread's X tile, transposed)
#pragma unroll
  for (int j = 0; j < 4; ++j) st4(m_addr(mXT, 4 * tx + j, 4 * ty), xt[0][j], xt[1][j], xt[2][j], xt[3][j]);
  // 4. S^-1 = W[64:128, 64:128]
  gj64(sa);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    st4(m_addr(mSI, 4 * ty + i, 4 * tx), sa[i][0], sa[i][1], sa[i][2], sa[i][3]);
    store_w(64 + 4 * ty + i, 64 + 4 * tx, sa[i][0], sa[i][1], sa[i][2], sa[i][3]);
  }
  __syncthreads();
  // 5. Y = X S^-1; W[0:64, 64:128] = -Y, W[64:128, 0:64] = -Y^T
  float y[4][4] = {};
  mm_acc(y, [&](int k) { return ld4(m_addr(mXT, k, 4 * ty)); },
         [&](int k) { return ld4(m_addr(mSI, k, 4 * tx)); });
#pragma unroll
  for (int i = 0; i < 4; ++i) store_w(4 * ty + i, 64 + 4 * tx, -y[i][0], -y[i][1], -y[i][2], -y[i][3]);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    store_w(64 + 4 * tx + j, 4 * ty, -y[0][j], -y[1][j], -y[2][j], -y[3][j]);
    st4(m_addr(mYT, 4 * tx + j, 4 * ty), y[0][j], y[1][j], y[2][j], y[3][j]);
  }
  __syncthreads();
  // 6. W[0:64, 0:64] = A^-1 + Y X^T; column k of Y's row block = row k of Y^T,
  //    row k of X^T = X^T[k][..]
  mm_acc(ai, [&](int k) { return ld4(m_addr(mYT, k, 4 * ty)); },
         [&](int k) { return ld4(m_addr(mXT, k, 4 * tx)); });
#pragma unroll
  for (int i = 0; i < 4; ++i) store_w(4 * ty + i, 4 * tx, ai[i][0], ai[i][1], ai[i][2], ai[i][3]);
}

// --------------------------------------------------------------- scans ----

constexpr int kScanThreads = 128;
constexpr int kScanHalf = 64;                 // value columns of S per CTA
constexpr uint32_t kScanSmemW = 0;            // 2 stages x 64 KB (W, fp32 K-major)
constexpr uint32_t kScanSmemX = 2 * 65536;    // 2 stages x 32 KB (X^T half, fp32 K-major)
constexpr uint32_t kScanSmemBytes = 2 * 65536 + 2 * 32768 + 1024;

struct ScanParams {
  int F, H, bf, nb;
  int steps_fwd;      // text + frames 1..steps_fwd-1
  int steps_bwd;      // text + frames F-2 down to F-steps_bwd
  float lambda;
  float* Rpart;       // [2][nb][H][128][128]
  float* text_out;    // optional [H][d][d]
  float* fwd_out;     // optional [F][H][d][d]
  float* bwd_out;     // optional [F][H][d][d]
  int d_out;
};

// One CTA per (direction, head, half of the value columns): the columns of
// S evolve independently (S_f = W_f (lambda S_prev + C_f) acts column-wise),
// so two CTAs split a chain without exchanging anything. Per step the CTA
// TMA-loads W_f (128 x 128) and its 64 rows of C_f^T into two-stage rings,
// adds lambda S_prev^T in place (thread i owns key row i of S, TMEM lane i),
// and runs 16 tf32 MMAs (M128 N64 K8, both operands K-major).
__global__ void __launch_bounds__(kScanThreads, 1)
    k_vda_scan(const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap tct,
               const ScanParams p) {
  const int dir = blockIdx.x, h = blockIdx.y, g = blockIdx.z;
  const int F = p.F;
  const int nsteps = dir == 0 ? p.steps_fwd : p.steps_bwd;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_full[2], bar_mma;
  __shared__ uint32_t tmem_slot;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int i = threadIdx.x, warp = i >> 5;
  const uint32_t full[2] = {smem_u32(&bar_full[0]), smem_u32(&bar_full[1])};
  const uint32_t mma_bar = smem_u32(&bar_mma);

  if (i == 0) {
    mbar_init(full[0], 1);
    mbar_init(full[1], 1);
    mbar_init(mma_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  auto mat_of = [&](int s) -> int { return (s == 0) ? 0 : (dir == 0 ? s : F - 1 - s); };
  auto idx_of = [&](int s) -> int { return dir == 0 ? s : (s == 0 ? F - 1 : F - 1 - s); };
  auto load_step = [&](int s, int st) {
    const int row = (mat_of(s) * p.H + h) * 128;
    const uint32_t sW = base + kScanSmemW + (uint32_t)st * 65536u;
    const uint32_t sX = base + kScanSmemX + (uint32_t)st * 32768u;
    mbar_arrive_expect_tx(full[st], 65536 + 32768);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      tma_load_2d(sW + (uint32_t)(c * 16384), &tw, full[st], c * 32, row);
      tma_load_2d(sX + (uint32_t)(c * 8192), &tct, full[st], c * 32, row + g * kScanHalf);
    }
  };
  if (i == 0) {
    tma_prefetch_desc(&tw);
    tma_prefetch_desc(&tct);
    load_step(0, 0);
    if (nsteps > 1) load_step(1, 1);
  }

  // element (n, k = i) of the X^T half: chunk i/32, row n, 4-byte slot of unit (i%32)/4
  const uint32_t xcol = (uint32_t)(i >> 5) * 8192u + (uint32_t)((i & 3) * 4);
  const uint32_t xu = (uint32_t)((i & 31) >> 2);
  const uint32_t idW = idesc_tf32(128, kScanHalf, false, false);
  bool ok = true;

  for (int s = 0; s < nsteps && ok; ++s) {
    const int st = s & 1;
    const uint32_t sW = base + kScanSmemW + (uint32_t)st * 65536u;
    const uint32_t sX = base + kScanSmemX + (uint32_t)st * 32768u;
    if (!mbar_wait(full[st], (uint32_t)((s >> 1) & 1))) { ok = false; break; }
    {
      // X^T[n][i] = C^T[n][i] + lambda S_prev[i][n] (no state before the text
      // step), rounded to tf32 here so the contraction does not truncate it
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sv[32];
        if (s > 0) {
          tmem_ld32(tmem + lane_base + (uint32_t)(c * 32), sv);
          tmem_ld_wait(sv);
        }
        // all 32 loads first, so they overlap, then the updates and stores
        float xv[32];
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const uint32_t addr = sX + xcol + sw128_off((uint32_t)(c * 32 + jj), xu);
          asm volatile("ld.shared.f32 %0, [%1];" : "=f"(xv[jj]) : "r"(addr) : "memory");
        }
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const uint32_t addr = sX + xcol + sw128_off((uint32_t)(c * 32 + jj), xu);
          const float x = (s > 0) ? fmaf(p.lambda, __uint_as_float(sv[jj]), xv[jj]) : xv[jj];
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(round_tf32(x)) : "memory");
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    named_barrier_sync(1, kScanThreads);
    if (i == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const uint32_t ka = (uint32_t)((k >> 2) * 16384 + (k & 3) * 32);
        const uint32_t kb = (uint32_t)((k >> 2) * 8192 + (k & 3) * 32);
        umma_tf32_ss(tmem, sdesc_sw128(sW + ka, 16, 1024), sdesc_sw128(sX + kb, 16, 1024), idW,
                     k > 0 ? 1u : 0u);
      }
      umma_commit(mma_bar);
    }
    if (!mbar_wait(mma_bar, (uint32_t)(s & 1))) { ok = false; break; }
    tc_fence_after();
    if (i == 0 && s + 2 < nsteps) load_step(s + 2, st);

    // outputs of this state
    const int idx = idx_of(s);
    bool want = (dir == 0 && p.fwd_out != nullptr) || (dir == 1 && p.bwd_out != nullptr) ||
                (s == 0 && dir == 0 && p.text_out != nullptr);
    for (int b = 0; b < p.nb && !want; ++b) {
      int i_f, i_b;
      block_read_indices(b, F, p.bf, i_f, i_b);
      want = (dir == 0 ? i_f : i_b) == idx;
    }
    if (want) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sv[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(c * 32), sv);
        tmem_ld_wait(sv);
        const int col0 = g * kScanHalf + c * 32;
        for (int b = 0; b < p.nb; ++b) {
          int i_f, i_b;
          block_read_indices(b, F, p.bf, i_f, i_b);
          if ((dir == 0 ? i_f : i_b) != idx) continue;
          float* dst = p.Rpart + ((((int64_t)dir * p.nb + b) * p.H + h) * 128 + i) * 128 + col0;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            reinterpret_cast<uint4*>(dst)[u] =
                make_uint4(sv[4 * u], sv[4 * u + 1], sv[4 * u + 2], sv[4 * u + 3]);
        }
        if (i < p.d_out) {
          float* outs[3] = {nullptr, nullptr, nullptr};
          if (dir == 0 && p.fwd_out) outs[0] = p.fwd_out + (((int64_t)idx * p.H + h) * p.d_out + i) * p.d_out;
          if (dir == 1 && p.bwd_out) outs[1] = p.bwd_out + (((int64_t)idx * p.H + h) * p.d_out + i) * p.d_out;
          if (s == 0 && dir == 0 && p.text_out) outs[2] = p.text_out + ((int64_t)h * p.d_out + i) * p.d_out;
#pragma unroll
          for (int o = 0; o < 3; ++o) {
            if (outs[o] == nullptr) continue;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
              if (col0 + jj < p.d_out) outs[o][col0 + jj] = __uint_as_float(sv[jj]);
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

}  // namespace vdn
