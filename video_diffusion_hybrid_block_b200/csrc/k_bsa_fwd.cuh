// Softmax branch of the hybrid layer: block-sparse bidirectional attention.
//
// Each query block (5 latent frames) attends exactly to the keys of its own
// and its neighbouring blocks, the first and last frames (boundary anchors)
// and every text token, with softmax scale 1/sqrt(d) ["VDN-MiniMax-H3"
// (openi.cn), 技术原理：局部精确、远程压缩; nav.superapi.store page, Technical
// Principles, Local Softmax Branch / Text Dual-Branch Injection].
//
// One CTA = two 128-row query tiles (256 consecutive rows of one block) of one
// head. Key tiles are enumerated from the block's key segments
// (layer_plan.cuh), so tiles outside the allowed set are never loaded; only
// the ragged last tile of each segment is masked column-wise. Both query
// tiles share every K/V tile. Grid (query-row pairs, blocks, heads): heads
// sit on z and are dispatched one after the other, so the CTAs of one head's
// blocks run close together and share that head's K/V in L2 (a head's
// blocks overlap in most key frames); within a head the blocks are visited
// interior-first (block_in_visit_order), so the CTAs with the most key
// tiles start first and the tail of the grid is made of short ones. Warp roles (384 threads, 3
// warpgroups):
//   warps 0-3  softmax of query tile 0 (thread r owns row r = TMEM lane r)
//   warps 4-7  softmax of query tile 1
//   warp 8     TMA producer: Q0, Q1 once, then K and V tiles (2-stage rings)
//   warp 9     MMA issuer (one thread); warps 10-11 idle
// Registers: launched at 168 per thread (384 x 168 = 64512); the producer
// warpgroup drops to 72 and the two softmax warpgroups rise to 216
// (128 x (216 + 216 + 72) = 64512), enough to hold a full 128-column S row.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// P_i (bf16, packed in pairs) overwrites the first 64 columns of S_i and is
// consumed from TMEM by the PV contraction (A operand in TMEM), so P never
// touches shared memory. MMA issue order per key tile j:
//   PV0(j), QK0(j+1), PV1(j), QK1(j+1)
// so while softmax i works on S_i(j+1), the tensor core runs the other tile's
// PV and QK. Contractions issued by one thread execute in issue order, so
// QK_i(j+1) may overwrite S_i right after PV_i(j) read P_i from it; and the
// commit that signals S_i(j+1) also covers PV_i(j), so the softmax owns O_i
// (for a rescale) from then until it hands over P_i(j+1).
// Online softmax in the exp2 domain with a lazily updated running max: O and
// the row sum are rescaled only when the tile max exceeds the max in use by
// more than 8 (a factor 256), which keeps every P <= 256. The exp2 work is
// split between the MUFU unit (3 of 4 column pairs) and a polynomial on the
// FMA pipe (1 of 4); measured on pages-scale this beats all-MUFU (2.62 vs
// 2.68 ms) and both 1/8 and 1/2 splits, while packing P with integer ops
// instead of cvt.rn.bf16x2 was slower in every split.
//
// kMerge = true fuses the linear-branch readout and the gated merge into the
// epilogue: after the last PV_i the MMA thread issues o_lin_i = Q_i R_b into
// the (now free) S_i columns, with R_b a packed bf16 tile loaded once per CTA;
// each softmax thread then forms
//   out = sigmoid(g_s) O/l + sigmoid(g_l) w * o_lin / sqrt(mean(o_lin^2) + eps)
// for its row ["VDN-MiniMax-H3" (openi.cn), 技术原理, last paragraph;
// nav.superapi.store page, Gated Fusion Mechanism], so o_soft never goes to
// HBM and q is not read a second time.
#pragma once

#include "layer_plan.cuh"
#include "sm100_ptx.cuh"

namespace vdn {

constexpr int kBsaThreads = 384;
constexpr int kBsaRegsSoftmax = 216;
constexpr int kBsaRegsProducer = 72;
constexpr int kBsaMergeRegsSoftmax = 208;
constexpr int kBsaMergeRegsProducer = 88;  // 128 x (208 + 208 + 88) = 64512
constexpr uint32_t kBsaSmemQ = 0;               // Q0, Q1: 2 x 32 KB
constexpr uint32_t kBsaSmemK = 2 * 32768;       // 2 stages x 32 KB
constexpr uint32_t kBsaSmemV = 4 * 32768;       // 2 stages x 32 KB
constexpr uint32_t kBsaSmemR = 6 * 32768;       // packed R_b (merge variant), 32 KB
constexpr uint32_t kBsaSmemBytes = 6 * 32768 + 1024;       // + alignment slack
constexpr uint32_t kBsaMergeSmemBytes = 7 * 32768 + 1024;
constexpr uint32_t kRImageBytes = 32768;  // one packed R_b tile (bf16, 128B-swizzled MN-major)
// e4m3 layout (16 KB tiles): Q8 tiles 0 and 1, K8 and V8 two stages each,
// then (merge variant) the bf16 Q tiles of the readout, which also stage the
// output tiles, and the packed R_b.
constexpr uint32_t kBsa8SmemK = 2 * 16384;
constexpr uint32_t kBsa8SmemV = 4 * 16384;
constexpr uint32_t kBsa8SmemQb = 6 * 16384;
constexpr uint32_t kBsa8SmemR = 6 * 16384 + 2 * 32768;
constexpr uint32_t kBsa8SmemBytes = 6 * 16384 + 1024;
constexpr uint32_t kBsa8MergeSmemBytes = kBsa8SmemR + 32768 + 1024;
constexpr int kBsaRowsPerCta = 2 * kTile;

struct BsaParams {
  const int32_t* off;  // [F+1] device
  int F, T, H, bf, N;
  float scale_log2;      // log2(e) / sqrt(d)
  __nv_bfloat16* o;      // o_soft output base
  int64_t o_row_stride;  // elements between consecutive tokens
  int d_store;           // leading columns of each head row to store
  float* lse;            // optional [H][N]
  // merge variant only
  const uint8_t* rimg;   // [nb][H] packed R_b tiles of kRImageBytes
  const void* g_s;       // [N][H] gate logits
  const void* g_l;
  int gate_f32;
  const float* rms_w;    // [H][d]
  float eps;
  void* out;             // [N][H][d]
  int out_f32;
  int d;                 // real head dim
  int tma_out;           // out is bf16 [N][H][128]: full tiles leave through a TMA store
  // e4m3 variant only: per-(token, head) q scales [N][H] and the per-head
  // amax bit patterns of k and v ([2][H]; scale = amax / 448, 1 if zero)
  const float* q_scale;
  const uint32_t* kv_amax;
};

// kMode: 0 = softmax branch only (o_soft, lse); 1 = merged layer output;
// 2 = the two gated branches written side by side for the per-branch output
// projections (out is [N][2H][128] bf16: head h holds sigmoid(g_s) O / l,
// head H + h holds sigmoid(g_l) w * o_lin / rms).
//
// kFp8 (softmax branch, or with kMode 1 the merged layer output): q, k, v arrive as e4m3 codes ([rows][H][128]
// bytes, one 128-byte swizzle row per token) with a scale per (token, head)
// row of q and per head for k and v. QK^T and PV run as kind::f8f6f4
// contractions (K32 steps), P is rounded to e4m3 (P <= 256 < 448 needs no
// scale) and packed four per TMEM column, the q and k scales fold into each
// row's exponent scale and the v scale into the final 1 / l.
template <int kMode, bool kFp8 = false>
__global__ void __launch_bounds__(kBsaThreads, 1)
    k_bsa_fwd(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tkt,
              const __grid_constant__ CUtensorMap tvt, const __grid_constant__ CUtensorMap tout,
              const __grid_constant__ CUtensorMap tqb, const BsaParams p) {
  constexpr bool kMerge = kMode != 0;
  static_assert(!kFp8 || kMode <= 1, "the e4m3 variant has no gated-branches output");
  // shared-memory layout: tile strides and offsets of the two variants
  constexpr uint32_t kTileB = kFp8 ? 16384u : 32768u;          // Q / K / V tile bytes
  constexpr uint32_t kOffK = kFp8 ? kBsa8SmemK : kBsaSmemK;
  constexpr uint32_t kOffV = kFp8 ? kBsa8SmemV : kBsaSmemV;
  constexpr uint32_t kOffQb = kFp8 ? kBsa8SmemQb : kBsaSmemQ;   // bf16 Q (readout, out staging)
  constexpr uint32_t kOffR = kFp8 ? kBsa8SmemR : kBsaSmemR;
  const int pair = blockIdx.x, h = blockIdx.z;
  const int b = block_in_visit_order(blockIdx.y, num_blocks(p.F, p.bf));
  int q0, q1;
  block_rows(p.off, p.F, p.bf, b, q0, q1);
  const int qs = q0 + pair * kBsaRowsPerCta;
  if (qs >= q1) return;  // uniform over the CTA, before any resource is taken
  // A block whose query tile count is odd leaves one CTA with a single tile.
  // That CTA splits the key tiles instead: both warpgroups take the same
  // query rows (Q is loaded into both Q buffers), warpgroup i the key tiles
  // j = i, i + 2, ... into its own S_i and O_i, and warpgroup 0 combines the
  // two partial softmaxes (m_i, l_i, O_i) at the end. Uniform over the CTA.
  // Softmax branch alone (kMode 0), bf16 only. In the e4m3 variant each
  // warpgroup's own running max would change which P values e4m3 rounds and
  // how, so it keeps one running max per row; the merged epilogues keep
  // their register budget for the readout and merge (measured: the merged
  // kernel with split CTAs ran about 1 % slower on layouts without single
  // tiles and gained 2 % on vda-stress).
  const bool split = kMode == 0 && !kFp8 && qs + kTile >= q1;

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q, bar_kf[2], bar_ke[2], bar_vf[2], bar_ve[2], bar_sf[2], bar_pf[2],
      bar_of[2], bar_r;
  __shared__ float w_sm[128];
  __shared__ KeySegs segs;  // key segments of this block, shared by all roles
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + kBsaSmemQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t q_full = smem_u32(&bar_q);

  if (threadIdx.x == 0) {
    segs = key_segments(p.off, p.F, p.bf, p.T, b);
    abort_flag = 0;
    mbar_init(q_full, 1);
    mbar_init(smem_u32(&bar_r), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_kf[i]), 1);
      mbar_init(smem_u32(&bar_ke[i]), 1);
      mbar_init(smem_u32(&bar_vf[i]), 1);
      mbar_init(smem_u32(&bar_ve[i]), 1);
      mbar_init(smem_u32(&bar_sf[i]), 1);
      mbar_init(smem_u32(&bar_pf[i]), 128);
      mbar_init(smem_u32(&bar_of[i]), 1);
    }
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(&tmem_slot), 512);
    tmem_relinquish();
  }
  if (kMerge && threadIdx.x < 128)
    w_sm[threadIdx.x] = (threadIdx.x < p.d) ? __ldg(p.rms_w + (int64_t)h * p.d + threadIdx.x) : 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_v = &abort_flag;
  const int nkt = segs_tiles(segs);
  // Each role's code sits inside the branch that set its register budget, so
  // no path joins two budgets before the common teardown.
  if (warp >= 8) {
  regs_dealloc<kMerge ? kBsaMergeRegsProducer : kBsaRegsProducer>();
  if (warp == 8) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      // rows of the second Q buffer: the second tile, or the first again
      // when the CTA splits its key tiles
      const int qs1 = split ? qs : qs + kTile;
      if constexpr (kFp8) {
        // e4m3 Q tiles; the merge variant's readout also needs Q in bf16
        mbar_arrive_expect_tx(q_full, 2 * 16384 + (kMerge ? 2 * 32768 : 0));
        tma_load_3d(sQ, &tq, q_full, 0, h, qs);
        tma_load_3d(sQ + 16384, &tq, q_full, 0, h, qs1);
        if (kMerge) {
          const uint32_t sQb = base + kOffQb;
          tma_prefetch_desc(&tqb);
          tma_load_3d(sQb, &tqb, q_full, 0, h, qs);
          tma_load_3d(sQb + 16384, &tqb, q_full, 64, h, qs);
          tma_load_3d(sQb + 32768, &tqb, q_full, 0, h, qs1);
          tma_load_3d(sQb + 49152, &tqb, q_full, 64, h, qs1);
        }
      } else {
        mbar_arrive_expect_tx(q_full, 2 * 32768);
        tma_load_3d(sQ, &tq, q_full, 0, h, qs);
        tma_load_3d(sQ + 16384, &tq, q_full, 64, h, qs);
        tma_load_3d(sQ + 32768, &tq, q_full, 0, h, qs1);
        tma_load_3d(sQ + 49152, &tq, q_full, 64, h, qs1);
      }
      if (kMerge) {
        mbar_arrive_expect_tx(smem_u32(&bar_r), kRImageBytes);
        bulk_load(base + kOffR, p.rimg + ((int64_t)b * p.H + h) * kRImageBytes, kRImageBytes,
                  smem_u32(&bar_r));
      }
      for (int j = 0; j < nkt; ++j) {
        if (*abort_v) break;
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        int src, row0, valid;
        segs_tile(segs, j, src, row0, valid);
        const CUtensorMap* mk = src ? &tkt : &tk;
        const CUtensorMap* mv = src ? &tvt : &tv;
        const uint32_t sK = base + kOffK + (uint32_t)st * kTileB;
        const uint32_t sV = base + kOffV + (uint32_t)st * kTileB;
        const uint32_t kf = smem_u32(&bar_kf[st]), vf = smem_u32(&bar_vf[st]);
        if (!mbar_wait(smem_u32(&bar_ke[st]), ph ^ 1)) { *abort_v = 1; break; }
        if constexpr (kFp8) {
          mbar_arrive_expect_tx(kf, 16384);
          tma_load_3d(sK, mk, kf, 0, h, row0);
        } else {
          mbar_arrive_expect_tx(kf, 32768);
          tma_load_3d(sK, mk, kf, 0, h, row0);
          tma_load_3d(sK + 16384, mk, kf, 64, h, row0);
        }
        if (!mbar_wait(smem_u32(&bar_ve[st]), ph ^ 1)) { *abort_v = 1; break; }
        if constexpr (kFp8) {
          mbar_arrive_expect_tx(vf, 16384);
          tma_load_3d(sV, mv, vf, 0, h, row0);
        } else {
          mbar_arrive_expect_tx(vf, 32768);
          tma_load_3d(sV, mv, vf, 0, h, row0);
          tma_load_3d(sV + 16384, mv, vf, 64, h, row0);
        }
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // -------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(128, 128, false, false);
      const uint32_t idO = idesc_bf16(128, 128, false, true);
      const uint32_t idS8 = idesc_e4m3(128, 128, false, false);
      const uint32_t idO8 = idesc_e4m3(128, 128, false, true);
      // S_i = Q_i K^T for key tile in K stage st
      auto qk = [&](int i, int st) {
        const uint32_t sQi = sQ + (uint32_t)i * kTileB;
        const uint32_t sK = base + kOffK + (uint32_t)st * kTileB;
        const uint32_t dS = tmem + (uint32_t)(i * 128);
        if constexpr (kFp8) {
          // one 128-byte row per token: four K32 steps 32 bytes apart
#pragma unroll
          for (int s = 0; s < 4; ++s)
            umma_f8_ss(dS, sdesc_sw128(sQi + (uint32_t)(s * 32), 16, 1024),
                       sdesc_sw128(sK + (uint32_t)(s * 32), 16, 1024), idS8, s > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            const uint32_t ko = (uint32_t)((s >> 2) * 16384 + (s & 3) * 32);
            umma_bf16_ss(dS, sdesc_sw128(sQi + ko, 16, 1024), sdesc_sw128(sK + ko, 16, 1024), idS,
                         s > 0 ? 1u : 0u);
          }
        }
        umma_commit(smem_u32(&bar_sf[i]));
      };
      // O_i += P_i V with P_i read from the first 64 TMEM columns of S_i
      auto pv = [&](int i, int st, bool acc) {
        const uint32_t sV = base + kOffV + (uint32_t)st * kTileB;
        const uint32_t aP = tmem + (uint32_t)(i * 128);
        const uint32_t dO = tmem + 256u + (uint32_t)(i * 128);
        if constexpr (kFp8) {
          // P: four e4m3 per TMEM column (8 columns per K32 step); V MN-major,
          // 32 key rows of 128 bytes per step
#pragma unroll
          for (int s = 0; s < 4; ++s)
            umma_f8_ts(dO, aP + (uint32_t)(s * 8), sdesc_sw128(sV + (uint32_t)(s * 4096), 16384, 1024),
                       idO8, (acc || s > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int s = 0; s < 8; ++s)
            umma_bf16_ts(dO, aP + (uint32_t)(s * 8), sdesc_sw128(sV + (uint32_t)(s * 2048), 16384, 1024),
                         idO, (acc || s > 0) ? 1u : 0u);
        }
      };
      // o_lin_i = Q_i R_b into the S_i columns (merge variant, after PV_i's last tile)
      auto readout = [&](int i) {
        const uint32_t sQi = base + kOffQb + (uint32_t)i * 32768u;   // bf16 Q
        const uint32_t sR = base + kOffR;
#pragma unroll
        for (int s = 0; s < 8; ++s)
          umma_bf16_ss(tmem + (uint32_t)(i * 128),
                       sdesc_sw128(sQi + (uint32_t)((s >> 2) * 16384 + (s & 3) * 32), 16, 1024),
                       sdesc_sw128(sR + (uint32_t)(s * 2048), 16384, 1024), idO, s > 0 ? 1u : 0u);
      };
      bool ok = mbar_wait(q_full, 0) &&
                mbar_wait(smem_u32(&bar_kf[0]), 0);
      if (split) {
        // key tile j goes to warpgroup j & 1 through stage j & 1 (the stage
        // the producer filled with it): S_i = Q K_j, then O_i += P_i V_j, and
        // QK of key tile j + 2 into S_i right after (in issue order)
        if (ok) {
          tc_fence_after();
          qk(0, 0);
          umma_commit(smem_u32(&bar_ke[0]));
          if (nkt > 1) {
            ok = mbar_wait(smem_u32(&bar_kf[1]), 0);
            if (ok) {
              tc_fence_after();
              qk(1, 1);
              umma_commit(smem_u32(&bar_ke[1]));
            }
          }
        }
        for (int j = 0; ok && j < nkt; ++j) {
          const int i = j & 1;
          const uint32_t ph = (uint32_t)((j >> 1) & 1);
          if (!mbar_wait_spin(smem_u32(&bar_vf[i]), ph) ||
              !mbar_wait_spin(smem_u32(&bar_pf[i]), ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          pv(i, i, j >= 2);
          umma_commit(smem_u32(&bar_ve[i]));
          if (j + 2 < nkt) {
            if (!mbar_wait_spin(smem_u32(&bar_kf[i]), ph ^ 1u)) {
              ok = false;
              break;
            }
            tc_fence_after();
            qk(i, i);
            umma_commit(smem_u32(&bar_ke[i]));
          }
        }
        if (ok && kMerge) {
          ok = mbar_wait(smem_u32(&bar_r), 0);
          if (ok) {
            tc_fence_after();
            readout(0);
          }
        }
        // both commits cover every contraction issued above
        if (ok) {
          umma_commit(smem_u32(&bar_of[0]));
          umma_commit(smem_u32(&bar_of[1]));
        }
      }
      if (!split && ok) {
        tc_fence_after();
        qk(0, 0);
        qk(1, 0);
        umma_commit(smem_u32(&bar_ke[0]));
      }
      for (int j = 0; !split && ok && j < nkt; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int st1 = (j + 1) & 1;
        const uint32_t ph1 = ((j + 1) >> 1) & 1;
        const bool more = j + 1 < nkt;
        if (!mbar_wait_spin(smem_u32(&bar_vf[st]), ph)) { ok = false; break; }
        if (!mbar_wait_spin(smem_u32(&bar_pf[0]), (uint32_t)(j & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        pv(0, st, j > 0);
        if (!more) {
          if (kMerge) {
            if (!mbar_wait(smem_u32(&bar_r), 0)) { ok = false; break; }
            tc_fence_after();
            readout(0);
          }
          umma_commit(smem_u32(&bar_of[0]));
        }
        if (more) {
          if (!mbar_wait_spin(smem_u32(&bar_kf[st1]), ph1)) { ok = false; break; }
          tc_fence_after();
          qk(0, st1);
        }
        if (!mbar_wait_spin(smem_u32(&bar_pf[1]), (uint32_t)(j & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        pv(1, st, j > 0);
        umma_commit(smem_u32(&bar_ve[st]));
        if (!more) {
          if (kMerge) readout(1);
          umma_commit(smem_u32(&bar_of[1]));
        }
        if (more) {
          qk(1, st1);
          umma_commit(smem_u32(&bar_ke[st1]));
        }
      }
      if (!ok) *abort_v = 1;
    }
    __syncwarp();
  }
  } else {
    regs_alloc<kMerge ? kBsaMergeRegsSoftmax : kBsaRegsSoftmax>();
    // ---------------------------------------------------- softmax warps --
    const int tile = warp >> 2;             // query tile of this warpgroup
    const int r = threadIdx.x & 127;        // row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + (uint32_t)(tile * 128);
    const uint32_t tO = tmem + lane_base + 256u + (uint32_t)(tile * 128);
    const uint32_t s_full = smem_u32(&bar_sf[tile]);
    const uint32_t p_full = smem_u32(&bar_pf[tile]);
    float scale = p.scale_log2;
    float v_scale = 1.f;
    if constexpr (kFp8) {
      // e4m3 scores are q8 . k8: fold the row's q scale and the head's k scale
      // into the exponent scale, the head's v scale into 1 / l
      const int qrow = qs + (split ? 0 : tile * kTile) + r;
      const float sq = qrow < q1 ? __ldg(p.q_scale + (int64_t)qrow * p.H + h) : 1.f;
      const float ak = __uint_as_float(__ldg(p.kv_amax + h));
      const float av = __uint_as_float(__ldg(p.kv_amax + p.H + h));
      scale *= sq * (ak > 0.f ? __fdiv_rn(ak, 448.f) : 1.f);
      v_scale = av > 0.f ? __fdiv_rn(av, 448.f) : 1.f;
    }
    float m_use = 0.f;
    float2 lacc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
    bool ok = true;
    // this warpgroup's key tiles: all of them, or every other one when the
    // CTA splits its key tiles (tile 0: j = 0, 2, ...; tile 1: j = 1, 3, ...)
    const int nown = split ? (nkt + 1 - tile) / 2 : nkt;
    for (int jj = 0; jj < nown; ++jj) {
      const int j = split ? 2 * jj + tile : jj;
      int src, row0, valid;
      segs_tile(segs, j, src, row0, valid);
      // no per-tile abort poll: a failed (bounded) wait ends the loop
      if (!mbar_wait(s_full, (uint32_t)(jj & 1))) {
        ok = false;
        *abort_v = 1;
        break;
      }
      tc_fence_after();
      uint32_t s[128];
      tmem_ld128(tS, s);
      tmem_ld_wait128(s);
      if (valid < 128) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) s[c] = __float_as_uint(-INFINITY);
      }
      // tile row max of the raw scores (scale > 0 keeps the order); eight
      // independent chains of 3-input maxes, then a small tree
      float mq[8];
#pragma unroll
      for (int a = 0; a < 8; ++a)
        mq[a] = fmax3(__uint_as_float(s[a]), __uint_as_float(s[a + 8]), __uint_as_float(s[a + 16]));
#pragma unroll
      for (int c = 24; c < 120; c += 16)
#pragma unroll
        for (int a = 0; a < 8; ++a)
          mq[a] = fmax3(mq[a], __uint_as_float(s[c + a]), __uint_as_float(s[c + a + 8]));
#pragma unroll
      for (int a = 0; a < 8; ++a) mq[a] = fmaxf(mq[a], __uint_as_float(s[120 + a]));
      const float mx = fmaxf(fmax3(mq[0], mq[1], mq[2]), fmax3(fmax3(mq[3], mq[4], mq[5]), mq[6], mq[7]));
      const float m_tile = mx * scale;
      if (jj == 0) {
        m_use = m_tile;
      } else {
        const bool need = m_tile > m_use + 8.f;
        if (__any_sync(0xffffffffu, need)) {
          // O_i is idle here: PV_i(j-1) completed before S_i(j) was signalled.
          const float factor = need ? ex2_approx(m_use - m_tile) : 1.f;
          if (need) {
            m_use = m_tile;
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              lacc[a].x *= factor;
              lacc[a].y *= factor;
            }
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + (uint32_t)(c * 32), o);
            tmem_ld_wait(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st32(tO + (uint32_t)(c * 32), o);
          }
        }
      }
      // P = exp2(s * scale - m_use), packed to bf16 pairs, written into S_i's
      // first 64 TMEM columns
      const float2 sc2 = make_float2(scale, scale);
      const float2 nm2 = make_float2(-m_use, -m_use);
      if constexpr (kFp8) {
        // P as e4m3, four per TMEM column, into S_i's first 32 columns
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const int c = 2 * e;
          const float2 x0 = ffma2(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sc2, nm2);
          const float2 x1 = ffma2(make_float2(__uint_as_float(s[c + 2]), __uint_as_float(s[c + 3])), sc2, nm2);
          const float2 p0 = ((e & 3) == 3) ? exp2_poly2(x0)
                                           : make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
          const float2 p1 = (((e + 1) & 3) == 3) ? exp2_poly2(x1)
                                                 : make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
          lacc[e & 3] = fadd2(lacc[e & 3], p0);
          lacc[(e + 1) & 3] = fadd2(lacc[(e + 1) & 3], p1);
          pk[e >> 1] = e4m3x4(p0.x, p0.y, p1.x, p1.y);
        }
        tmem_st32(tS, pk);
      } else {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = half * 64 + 2 * e;
          const float2 x = ffma2(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sc2, nm2);
          // one pair in four goes to the FMA pipe, the rest to MUFU ex2
          const float2 pe = ((e & 3) == 3) ? exp2_poly2(x)
                                           : make_float2(ex2_approx(x.x), ex2_approx(x.y));
          lacc[e & 3] = fadd2(lacc[e & 3], pe);
          pk[e] = pack_bf16x2(pe.x, pe.y);
        }
        tmem_st32(tS + (uint32_t)(half * 32), pk);
      }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    const float l_sum = (lacc[0].x + lacc[0].y) + (lacc[1].x + lacc[1].y) +
                        (lacc[2].x + lacc[2].y) + (lacc[3].x + lacc[3].y);
    // merge variant: fetch this row's gate logits before waiting on the last
    // MMAs so the load latency overlaps them
    float gs = 0.f, gl = 0.f;
    if (kMerge) {
      const int grow = qs + tile * kTile + r;
      if (grow < q1) {
        const int64_t gi = (int64_t)grow * p.H + h;
        gs = p.gate_f32 ? __ldg(reinterpret_cast<const float*>(p.g_s) + gi)
                        : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.g_s)[gi]);
        gl = p.gate_f32 ? __ldg(reinterpret_cast<const float*>(p.g_l) + gi)
                        : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.g_l)[gi]);
      }
    }
    if (ok && !mbar_wait(smem_u32(&bar_of[tile]), 0)) ok = false;
    if (!ok) *abort_v = 1;
    tc_fence_after();
    // split CTA: warpgroup 1 hands its rows' (m, l) to warpgroup 0 through
    // the second Q buffer (idle once every contraction has completed);
    // warpgroup 0 weights the two partial outputs by 2^(m_i - m) and adds
    // them. Warpgroup 1's own rows lie past the block, so it stores nothing.
    float m_fin = m_use, l_fin = l_sum, oa0 = 1.f, oa1 = 0.f;
    const bool combine = split && tile == 0;
    if (split) {
      float* xch = reinterpret_cast<float*>(smem_raw + (base + kTileB - smem_u32(smem_raw)));
      if (tile == 1) {
        xch[r] = m_use;
        xch[128 + r] = l_sum;  // 0 if the warpgroup had no key tile
      }
      named_barrier_sync(4, 256);
      if (tile == 0) {
        const float m1 = xch[r], l1 = xch[128 + r];
        if (l1 > 0.f) {
          m_fin = fmaxf(m_use, m1);
          oa0 = ex2_approx(m_use - m_fin);
          oa1 = ex2_approx(m1 - m_fin);
          l_fin = l_sum * oa0 + l1 * oa1;
        }
      }
    }
    const uint32_t tO1 = tmem + lane_base + 384u;  // O_1: same lanes, next 128 columns
    // chunk c of this row's O (already loaded from O_0): the weighted sum
    // with O_1's chunk in a split CTA
    auto combine_o = [&](int c, uint32_t (&o)[32]) {
      if (!combine) return;
      uint32_t o1[32];
      tmem_ld32(tO1 + (uint32_t)(c * 32), o1);
      tmem_ld_wait(o1);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float x = __uint_as_float(o[e]) * oa0;
        o[e] = __float_as_uint(oa1 != 0.f ? fmaf(__uint_as_float(o1[e]), oa1, x) : x);
      }
    };
    const int row = qs + tile * kTile + r;
    const bool store = ok && row < q1;
    const float inv = v_scale / l_fin;
    if (!kMerge) {
      __nv_bfloat16* dst = p.o + (int64_t)row * p.o_row_stride + (int64_t)h * p.d_store;
      // the TMEM loads are warp-collective: every thread runs them, only the
      // stores depend on the row
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + (uint32_t)(c * 32), o);
        tmem_ld_wait(o);
        combine_o(c, o);
        if (store) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (c * 32 + u * 8 < p.d_store) {
              uint4 val;
              val.x = pack_bf16x2(__uint_as_float(o[u * 8 + 0]) * inv, __uint_as_float(o[u * 8 + 1]) * inv);
              val.y = pack_bf16x2(__uint_as_float(o[u * 8 + 2]) * inv, __uint_as_float(o[u * 8 + 3]) * inv);
              val.z = pack_bf16x2(__uint_as_float(o[u * 8 + 4]) * inv, __uint_as_float(o[u * 8 + 5]) * inv);
              val.w = pack_bf16x2(__uint_as_float(o[u * 8 + 6]) * inv, __uint_as_float(o[u * 8 + 7]) * inv);
              *reinterpret_cast<uint4*>(dst + c * 32 + u * 8) = val;
            }
          }
        }
      }
      if (store && p.lse != nullptr)
        p.lse[(int64_t)h * p.N + row] = (m_fin + __log2f(l_fin)) * 0.69314718055994531f;
    } else {
      // gated merge of O / l with RMSNorm(o_lin); o_lin sits in the S_i columns
      const int64_t gi = (int64_t)row * p.H + h;
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t z[32];
        tmem_ld32(tS + (uint32_t)(c * 32), z);
        tmem_ld_wait(z);
#pragma unroll
        for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(z[e]), __uint_as_float(z[e]), ss);
      }
      const float a_s = inv / (1.f + __expf(-gs));
      const float a_l = rsqrtf(ss / (float)p.d + p.eps) / (1.f + __expf(-gl));
      const int64_t obase = gi * p.d;
      // a full tile of a bf16 d=128 output leaves through the (now idle) Q_i
      // buffer and one TMA store; otherwise each thread stores its row
      const bool via_tma = p.tma_out && (qs + tile * kTile + kTile <= q1);
      const uint32_t stage = base + kOffQb + (uint32_t)tile * 32768u;
      if constexpr (kMode == 2) {
        // pass 0: soft branch into head h, pass 1: linear branch into head H + h
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t x[32];
            tmem_ld32((pass == 0 ? tO : tS) + (uint32_t)(c * 32), x);
            tmem_ld_wait(x);
            if (pass == 0) combine_o(c, x);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int c0 = c * 32 + u * 8;
              float y[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                y[e] = pass == 0 ? a_s * __uint_as_float(x[u * 8 + e])
                                 : a_l * w_sm[c0 + e] * __uint_as_float(x[u * 8 + e]);
              const uint32_t w0 = pack_bf16x2(y[0], y[1]), w1 = pack_bf16x2(y[2], y[3]);
              const uint32_t w2 = pack_bf16x2(y[4], y[5]), w3 = pack_bf16x2(y[6], y[7]);
              if (via_tma) {
                st_shared_v4(stage + (uint32_t)(c0 >> 6) * 16384u +
                                 sw128_off((uint32_t)r, (uint32_t)((c0 & 63) >> 3)),
                             w0, w1, w2, w3);
              } else if (store) {
                const int64_t ob = ((int64_t)row * 2 * p.H + pass * p.H + h) * kDPad + c0;
                *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + ob) =
                    make_uint4(w0, w1, w2, w3);
              }
            }
          }
          if (via_tma) {
            fence_proxy_async_smem();
            named_barrier_sync(2 + tile, 128);
            if (r == 0 && ok) {
              const int row0 = qs + tile * kTile;
              tma_store_3d(&tout, stage, 0, pass * p.H + h, row0);
              tma_store_3d(&tout, stage + 16384u, 64, pass * p.H + h, row0);
              bulk_commit_group();
              bulk_wait_all();  // the staging buffer is refilled by the next pass
            }
            named_barrier_sync(2 + tile, 128);
          }
        }
      } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32], z[32];
        tmem_ld32(tO + (uint32_t)(c * 32), o);
        tmem_ld32(tS + (uint32_t)(c * 32), z);
        tmem_ld_wait(o);
        tmem_ld_wait(z);
        combine_o(c, o);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c0 = c * 32 + u * 8;
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            y[e] = a_s * __uint_as_float(o[u * 8 + e]) + a_l * w_sm[c0 + e] * __uint_as_float(z[u * 8 + e]);
          if (via_tma) {
            st_shared_v4(stage + (uint32_t)(c0 >> 6) * 16384u + sw128_off((uint32_t)r, (uint32_t)((c0 & 63) >> 3)),
                         pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                         pack_bf16x2(y[6], y[7]));
          } else if (store && c0 < p.d) {
            if (p.out_f32) {
              float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + obase + c0);
              dst[0] = make_float4(y[0], y[1], y[2], y[3]);
              dst[1] = make_float4(y[4], y[5], y[6], y[7]);
            } else {
              *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + obase + c0) =
                  make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]),
                             pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7]));
            }
          }
        }
      }
      if (via_tma) {
        fence_proxy_async_smem();
        named_barrier_sync(2 + tile, 128);
        if (r == 0 && ok) {
          const int row0 = qs + tile * kTile;
          tma_store_3d(&tout, stage, 0, h, row0);
          tma_store_3d(&tout, stage + 16384u, 64, h, row0);
          bulk_commit_group();
          bulk_wait_all();
        }
      }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// R_b = Rfwd + Rbwd (fp32, padded 128 x 128) -> bf16 tile image laid out
// exactly as the merge variant's shared-memory B operand (128B-swizzled,
// MN-major: row k of 128 B per 64 value dims, two 16 KB chunks), so the CTA
// fetches it with one bulk copy. Grid (block x head, kPackSplit row groups),
// 128 threads; a unit is 8 consecutive values of one row (32 B of each
// input, one 16-byte unit of the image), consecutive threads take
// consecutive units, so each warp reads whole 512-byte rows; all of a
// thread's loads are issued before its stores.
constexpr int kPackSplit = 4;
constexpr int kPackUnits = 128 * 16 / kPackSplit / 128;  // units per thread

__global__ void k_pack_read_states(const float* __restrict__ ra, const float* __restrict__ rb,
                                   uint8_t* __restrict__ img) {
  const int64_t bh = blockIdx.x;
  const float4* a = reinterpret_cast<const float4*>(ra + bh * 128 * 128);
  const float4* c4 = reinterpret_cast<const float4*>(rb + bh * 128 * 128);
  uint8_t* dst = img + bh * kRImageBytes;
  const int u0 = (int)blockIdx.y * (128 * 16 / kPackSplit) + (int)threadIdx.x;
  float4 x[kPackUnits][2], y[kPackUnits][2];
#pragma unroll
  for (int j = 0; j < kPackUnits; ++j) {
    const int u = u0 + j * 128;  // row u / 16, values 8 (u % 16) ..
    x[j][0] = __ldg(a + 2 * u);
    x[j][1] = __ldg(a + 2 * u + 1);
    y[j][0] = __ldg(c4 + 2 * u);
    y[j][1] = __ldg(c4 + 2 * u + 1);
  }
#pragma unroll
  for (int j = 0; j < kPackUnits; ++j) {
    const int u = u0 + j * 128;
    const int row = u >> 4, c8 = u & 15;
    const float4 p0 = x[j][0], p1 = x[j][1], q0 = y[j][0], q1 = y[j][1];
    *reinterpret_cast<uint4*>(dst + (c8 >> 3) * 16384 + sw128_off((uint32_t)row, (uint32_t)(c8 & 7))) =
        make_uint4(pack_bf16x2(p0.x + q0.x, p0.y + q0.y), pack_bf16x2(p0.z + q0.z, p0.w + q0.w),
                   pack_bf16x2(p1.x + q1.x, p1.y + q1.y), pack_bf16x2(p1.z + q1.z, p1.w + q1.w));
  }
}

}  // namespace vdn
