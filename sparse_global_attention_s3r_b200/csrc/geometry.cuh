// geometry.cuh -- which tokens each key block holds (the block <-> token map).
//
// Speed3R (gist.science summary, "Methodologie" §1 "Compressie-tak"): the compression branch
// summarises the tokens by spatial average pooling. Two geometries:
//   1-D   block j = tokens [j*b, min((j+1)*b, L)) of the flattened sequence;
//   2-D   the sequence is N views of P = special + gh*gw tokens (special tokens first, then the
//         patch grid row by row). Each view contributes one block of its special tokens (when
//         special > 0), then windows of wh x ww patches (wh*ww = b) tiling its grid from the
//         top-left, row by row, cut at the right and bottom edges.
// A block has b slots; slot o of a 2-D window is patch (o / ww, o % ww) of the window, slot o of
// the special block is special token o. slot_token() gives the token of a slot, or -1 for a slot
// that holds no token (past L, past the special tokens, or outside the grid).
#pragma once

#include <stdint.h>

namespace s3r {

struct BlockGeo {
  int64_t L;
  int b;
  int two_d;     // 0: 1-D blocks
  int64_t P;     // tokens per view (2-D)
  int special;   // special tokens per view (2-D)
  int gh, gw;    // patch grid (2-D)
  int wh, lww;   // window height; log2 of the window width (b and its divisors are powers of 2)
  int cols;      // windows per grid row
  int per_view;  // blocks per view
};

// Where block j starts: its first token (1-D), the view's first token (special block), or the
// first patch of the window together with the window's first grid row and column.
struct BlockOrigin {
  int64_t first;  // token of slot 0 when that slot holds one
  int kind;       // 0: 1-D run, 1: special tokens of a view, 2: window
  int r0, c0;     // window: grid row and column of slot 0
};

// (Block indices are below S3R_MAX_BLOCKS, so 32-bit division suffices.)
__host__ __device__ __forceinline__ BlockOrigin block_origin(const BlockGeo& g, int64_t j) {
  if (!g.two_d) return BlockOrigin{j * g.b, 0, 0, 0};
  const int jj = static_cast<int>(j);
  const int view = jj / g.per_view;
  int m = jj - view * g.per_view;
  const int64_t first = static_cast<int64_t>(view) * g.P;
  if (g.special > 0) {
    if (m == 0) return BlockOrigin{first, 1, 0, 0};
    m -= 1;
  }
  const int wr = m / g.cols, wc = m - wr * g.cols;
  const int r0 = wr * g.wh, c0 = wc << g.lww;
  return BlockOrigin{first + g.special + static_cast<int64_t>(r0) * g.gw + c0, 2, r0, c0};
}

// Token of slot o (0 <= o < b) of the block that starts at bo, or -1.
__host__ __device__ __forceinline__ int64_t origin_token(const BlockGeo& g, const BlockOrigin& bo,
                                                         int o) {
  if (bo.kind == 0) return bo.first + o < g.L ? bo.first + o : -1;
  if (bo.kind == 1) return o < g.special ? bo.first + o : -1;
  const int dr = o >> g.lww, dc = o & ((1 << g.lww) - 1);
  return (bo.r0 + dr < g.gh && bo.c0 + dc < g.gw)
             ? bo.first + static_cast<int64_t>(dr) * g.gw + dc
             : -1;
}

// Token of slot o (0 <= o < b) of key block j, or -1.
__host__ __device__ __forceinline__ int64_t slot_token(const BlockGeo& g, int64_t j, int o) {
  return origin_token(g, block_origin(g, j), o);
}

// True when every slot of the block that starts at bo holds a token.
__host__ __device__ __forceinline__ bool origin_full(const BlockGeo& g, const BlockOrigin& bo) {
  if (bo.kind == 0) return bo.first + g.b <= g.L;
  if (bo.kind == 1) return g.special == g.b;
  return bo.r0 + g.wh <= g.gh && bo.c0 + (1 << g.lww) <= g.gw;
}

__host__ __device__ __forceinline__ bool block_full(const BlockGeo& g, int64_t j) {
  return origin_full(g, block_origin(g, j));
}

// Bits of the slots o0 .. o0+n-1 (n <= 64) of the block that starts at bo: bit i set when slot
// o0 + i holds a token. A window contributes, for each of its patch rows that lies in the grid,
// the run of its first cv slots (cv = columns of the window inside the grid).
__host__ __device__ __forceinline__ uint64_t range_bits(int lo, int hi) {  // bits lo .. hi-1
  if (hi <= lo) return 0ull;
  const uint64_t upto_hi = hi >= 64 ? ~0ull : ((1ull << hi) - 1ull);
  const uint64_t below_lo = (1ull << lo) - 1ull;
  return upto_hi & ~below_lo;
}

__host__ __device__ __forceinline__ uint64_t slot_bits(const BlockGeo& g, const BlockOrigin& bo,
                                                       int o0, int n) {
  if (bo.kind == 0) {  // tokens first .. L-1 of the run
    const int64_t cnt = g.L - bo.first - o0;
    return range_bits(0, cnt < 0 ? 0 : (cnt > n ? n : static_cast<int>(cnt)));
  }
  if (bo.kind == 1) return range_bits(0, g.special - o0 > n ? n : g.special - o0);
  const int ww = 1 << g.lww;
  const int rv = g.gh - bo.r0 < g.wh ? g.gh - bo.r0 : g.wh;  // window rows inside the grid
  const int cv = g.gw - bo.c0 < ww ? g.gw - bo.c0 : ww;      // window columns inside the grid
  uint64_t bits = 0ull;
  for (int r = o0 >> g.lww; r < rv && (r << g.lww) < o0 + n; ++r) {
    const int lo = (r << g.lww) > o0 ? (r << g.lww) : o0;
    const int hi = (r << g.lww) + cv < o0 + n ? (r << g.lww) + cv : o0 + n;
    bits |= range_bits(lo - o0, hi - o0);
  }
  return bits;
}

}  // namespace s3r
