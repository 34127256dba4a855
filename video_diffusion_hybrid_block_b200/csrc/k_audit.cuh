// Audit of the schedules the layer kernels run, for verification: counts the
// (query token, key token) pairs per (query frame, key frame) that the
// softmax kernel visits (same key_segments / segs_tile enumeration, same
// valid-row and valid-column masks), and the pairs folded into the linear
// read states (same block_read_indices the scans use). Integer counts, so the
// comparison with the oracle's pair classes is exact. Also the check of the
// bounded-wait failure path (k_selftest_wait_timeout).
#pragma once

#include "layer_plan.cuh"
#include "sm100_ptx.cuh"

namespace vdn {

__device__ __forceinline__ int frame_of_row(const int32_t* off, int F, int row) {
  int lo = 0, hi = F - 1;  // last f with off[f] <= row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void k_pair_audit_soft(const int32_t* off, int F, int T, int bf,
                                  unsigned long long* soft) {
  const int tile = blockIdx.x, b = blockIdx.y;
  int q0, q1;
  block_rows(off, F, bf, b, q0, q1);
  const int qs = q0 + tile * kTile;
  if (qs >= q1) return;
  const int qe = imin(qs + kTile, q1);
  const KeySegs segs = key_segments(off, F, bf, T, b);
  const int nkt = segs_tiles(segs);
  for (int j = threadIdx.x; j < nkt; j += blockDim.x) {
    int src, row0, valid;
    segs_tile(segs, j, src, row0, valid);
    for (int fq = frame_of_row(off, F, qs); fq < F && off[fq] < qe; ++fq) {
      const long long nq = imin(off[fq + 1], qe) - imax(off[fq], qs);
      if (nq <= 0) continue;
      if (src == 1) {
        atomicAdd(&soft[(int64_t)fq * (F + 1) + F], (unsigned long long)(nq * valid));
        continue;
      }
      const int k1 = row0 + valid;
      for (int fk = frame_of_row(off, F, row0); fk < F && off[fk] < k1; ++fk) {
        const long long nk = imin(off[fk + 1], k1) - imax(off[fk], row0);
        if (nk > 0) atomicAdd(&soft[(int64_t)fq * (F + 1) + fk], (unsigned long long)(nq * nk));
      }
    }
  }
}

__global__ void k_pair_audit_lin(const int32_t* off, int F, int bf, unsigned long long* lin) {
  const int fq = blockIdx.x;
  const int b = fq / bf;
  int i_f, i_b;
  block_read_indices(b, F, bf, i_f, i_b);
  const long long nq = off[fq + 1] - off[fq];
  for (int g = threadIdx.x; g < F; g += blockDim.x) {
    // forward state i_f holds frames 1..i_f, backward state i_b frames i_b..F-2
    const bool in = (g >= 1 && g <= i_f) || (g >= i_b && g <= F - 2);
    lin[(int64_t)fq * F + g] = in ? (unsigned long long)(nq * (off[g + 1] - off[g])) : 0ull;
  }
}

// Failure-path check of the bounded waits: one CTA (optionally holding TMEM)
// waits on an mbarrier phase that nothing completes, through the same
// routine the kernels use, gives up after limit_ns (recording
// kDevErrWaitTimeout), frees its TMEM and returns, leaving the context usable.
__global__ void k_selftest_wait_timeout(uint64_t limit_ns, int tmem_cols) {
  __shared__ uint64_t bar;
  __shared__ uint32_t slot;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  if (tmem_cols > 0 && warp == 0) {
    tmem_alloc(smem_u32(&slot), (uint32_t)tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) (void)mbar_wait_limit(smem_u32(&bar), 0u, limit_ns);
  tc_fence_before();
  __syncthreads();
  if (tmem_cols > 0 && warp == 0) {
    tc_fence_after();
    tmem_dealloc(slot, (uint32_t)tmem_cols);
  }
}

}  // namespace vdn
