// Integer structure of the hybrid layer, shared by host and device code:
// frame blocks, softmax windows with boundary anchors, key segments of a
// query block, the scan states a block reads.
//
// Blocks of `bf` consecutive latent frames; block b's softmax window is
// blocks b-1..b+1 (clipped), plus frames 0 and F-1 as boundary anchors, plus
// every text token ["VDN-MiniMax-H3" (openi.cn), 技术原理：局部精确、远程压缩;
// nav.superapi.store page, Technical Principles, Local Softmax Branch and
// Text Dual-Branch Injection]. The linear branch of block b reads the forward
// state just before its window and the backward state just after it, both
// excluding window frames and anchors [openi.cn page, same section].
#pragma once

#include <stdint.h>

namespace vdn {

constexpr int kTile = 128;   // query rows / key rows per softmax tile
constexpr int kDPad = 128;   // head dim the kernels run at (smaller d is zero-padded)
constexpr int kMaxSegs = 4;  // text + at most three video ranges

__host__ __device__ inline int imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ inline int imax(int a, int b) { return a > b ? a : b; }

__host__ __device__ inline int num_blocks(int F, int bf) { return (F + bf - 1) / bf; }

// First and last frame of block b's window (blocks b-1, b, b+1, clipped).
__host__ __device__ inline void block_window(int b, int F, int bf, int& w0, int& w1) {
  w0 = bf * imax(b - 1, 0);
  w1 = imin(bf * (b + 2), F) - 1;
}

// Scan-state indices block b reads: forward state after frame w0-1 (index 0
// is the text-initialised state) and backward state after frame w1+1 (index
// F-1 is the text-initialised state).
__host__ __device__ inline void block_read_indices(int b, int F, int bf, int& i_fwd,
                                                   int& i_bwd) {
  int w0, w1;
  block_window(b, F, bf, w0, w1);
  i_fwd = imax(w0 - 1, 0);
  i_bwd = imin(w1 + 1, F - 1);
}

// Order in which the softmax kernel's CTAs visit blocks: interior blocks
// (three blocks of window, the most key tiles) before the two edge blocks, so
// the last CTAs to start are the short ones (longest-first list scheduling).
__host__ __device__ inline int block_in_visit_order(int z, int nb) {
  if (nb <= 2) return z;
  if (z < nb - 2) return z + 1;
  return z == nb - 2 ? 0 : nb - 1;
}

// Query rows of block b: [q0, q1).
__host__ __device__ inline void block_rows(const int32_t* off, int F, int bf, int b, int& q0,
                                           int& q1) {
  q0 = off[bf * b];
  q1 = off[imin(bf * b + bf, F)];
}

// Key segments of block b in visiting order: text first, then the video
// frame ranges {0}, [w0, w1], {F-1} merged where they touch.
struct KeySegs {
  int n;
  int src[kMaxSegs];    // 0 = video k/v rows, 1 = text kt/vt rows
  int start[kMaxSegs];  // first row in its source
  int len[kMaxSegs];    // rows
  int first_tile[kMaxSegs + 1];
};

// Appends a segment. The loops run over compile-time indices only, so a
// KeySegs value can live in registers (no dynamically indexed local array).
__host__ __device__ inline void segs_push(KeySegs& s, int src, int a, int e) {
  if (e > a) {
#pragma unroll
    for (int q = 0; q < kMaxSegs; ++q) {
      if (q == s.n) {
        s.src[q] = src;
        s.start[q] = a;
        s.len[q] = e - a;
        s.first_tile[q + 1] = s.first_tile[q] + (e - a + kTile - 1) / kTile;
      }
    }
    s.n++;
  }
}

__host__ __device__ inline KeySegs key_segments(const int32_t* off, int F, int bf, int T,
                                                int b) {
  KeySegs s;
  s.n = 0;
#pragma unroll
  for (int q = 0; q < kMaxSegs; ++q) {
    s.src[q] = 0;
    s.start[q] = 0;
    s.len[q] = 0;
    s.first_tile[q + 1] = 0;
  }
  s.first_tile[0] = 0;
  segs_push(s, 1, 0, T);
  int w0, w1;
  block_window(b, F, bf, w0, w1);
  // frame ranges, inclusive, in increasing order
  int ra[3] = {0, w0, F - 1};
  int rb[3] = {0, w1, F - 1};
  int ca = ra[0], cb = rb[0];
#pragma unroll
  for (int i = 1; i < 3; ++i) {
    if (ra[i] <= cb + 1) {
      cb = imax(cb, rb[i]);
    } else {
      segs_push(s, 0, off[ca], off[cb + 1]);
      ca = ra[i];
      cb = rb[i];
    }
  }
  segs_push(s, 0, off[ca], off[cb + 1]);
  return s;
}

__host__ __device__ inline int segs_tiles(const KeySegs& s) {
  int t = 0;
#pragma unroll
  for (int q = 1; q <= kMaxSegs; ++q)
    if (q == s.n) t = s.first_tile[q];
  return t;
}

// Key tile j of the list: source, first row, number of valid rows (1..128).
__host__ __device__ inline void segs_tile(const KeySegs& s, int j, int& src, int& row0,
                                          int& valid) {
  int sel_src = s.src[0], sel_start = s.start[0], sel_len = s.len[0], sel_ft = 0;
#pragma unroll
  for (int q = 1; q < kMaxSegs; ++q) {
    if (q < s.n && j >= s.first_tile[q]) {
      sel_src = s.src[q];
      sel_start = s.start[q];
      sel_len = s.len[q];
      sel_ft = s.first_tile[q];
    }
  }
  src = sel_src;
  row0 = sel_start + (j - sel_ft) * kTile;
  valid = imin(kTile, sel_start + sel_len - row0);
}

}  // namespace vdn
