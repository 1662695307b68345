// schedule.cuh -- the block-sparse tile scheduler.
//
// For query block qb the SSA window (QbitAI article on LongCat LoZA, paragraph
// on the 1024-token sparse window: one global block plus seven local blocks of
// 128 tokens) is the set of key blocks
//
//     W(qb) = {0 .. n_sink-1}  U  {max(n_sink, qb-n_local+1) .. qb},
//
// clipped to blocks <= qb (keys after the query are never visible).  The
// union is enumerated without duplicates: while the local run would reach
// into the sink blocks (qb < n_sink + n_local - 1) it simply starts after
// them.  Tiles come out in ascending block order, so the sink comes first and
// the diagonal block qb -- the only one that needs a per-token causal mask --
// is always the last tile.
#pragma once

#include <cstdint>

namespace loza {

struct TileRange {
  int n_sink_tiles;  // tiles 0 .. n_sink_tiles-1 are key blocks 0 .. n_sink_tiles-1
  int local_lo;      // remaining tiles are key blocks local_lo .. qb
  int count;         // total number of tiles
};

__host__ __device__ __forceinline__ TileRange tile_range(int qb, int n_sink, int n_local) {
  TileRange r;
  r.n_sink_tiles = n_sink < qb + 1 ? n_sink : qb + 1;
  int lo = qb - n_local + 1;
  r.local_lo = lo > n_sink ? lo : n_sink;
  int n_loc = qb - r.local_lo + 1;
  r.count = r.n_sink_tiles + (n_loc > 0 ? n_loc : 0);
  return r;
}

// Key block visited as the t-th tile (0 <= t < count).
__host__ __device__ __forceinline__ int tile_block(const TileRange& r, int t) {
  return t < r.n_sink_tiles ? t : r.local_lo + (t - r.n_sink_tiles);
}

}  // namespace loza
