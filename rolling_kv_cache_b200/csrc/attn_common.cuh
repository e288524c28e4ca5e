// Pieces shared by the attention and score kernels: the KV tile walk over the
// plan's segment list and the shared-memory tile geometry.
#pragma once

#include "kernels.cuh"

namespace rc {

constexpr int kTileRows = 128;
constexpr uint32_t kSubTileBytes = 128 * 64 * 2;  // 128 rows x 64 bf16 = one 128-byte-swizzle box

struct Tile {
  int tok, nvalid, rank;
};

// Yields, in segment order, the 128-token KV tiles that a query block whose
// highest mask class is rq_hi can see: a segment of a later chunk frame is
// skipped whole, a segment's ragged end gives a tile with nvalid < 128.
// Every warp role walks the same sequence.
struct TileWalker {
  const KvSegment* seg;
  int n_segs, rq_hi;
  int s = 0, off = 0;
  __device__ bool next(Tile& t) {
    while (s < n_segs) {
      const KvSegment& g = seg[s];
      if ((g.rank >= 0 && g.rank > rq_hi) || off >= g.len) {
        ++s;
        off = 0;
        continue;
      }
      t.tok = g.tok_start + off;
      t.nvalid = min(kTileRows, g.len - off);
      t.rank = g.rank;
      off += kTileRows;
      return true;
    }
    return false;
  }
  // Skips the first k tiles of the walk.
  __device__ void seek(int k) {
    while (k > 0 && s < n_segs) {
      const KvSegment& g = seg[s];
      if (g.rank >= 0 && g.rank > rq_hi) {
        ++s;
        continue;
      }
      const int nt = (g.len - off + kTileRows - 1) / kTileRows;
      if (k < nt) {
        off += k * kTileRows;
        return;
      }
      k -= nt;
      ++s;
      off = 0;
    }
  }
};

__device__ __forceinline__ int count_tiles(const KvSegment* seg, int n, int rq_hi) {
  int c = 0;
  for (int s = 0; s < n; ++s)
    if (!(seg[s].rank >= 0 && seg[s].rank > rq_hi)) c += (seg[s].len + kTileRows - 1) / kTileRows;
  return c;
}

}  // namespace rc
