// Persistent-grid tile order shared by the host planner and the kernels.
//
// Output tiles are numbered batch-major; inside a batch, tiles are visited in
// groups of `group_m` tile-rows swept one tile-column at a time, so the CTAs
// that run at the same moment share a few A row-panels and B column-panels in
// L2 (the grouped program-id reordering of mm_template in
// pytorch/torch/_inductor/kernel/mm.py, "re-order program ID for better L2
// performance").  A persistent CTA b handles tiles b, b + gridDim.x, ...
// (persistent_tma_mm_template, same file).
#pragma once

#if defined(__CUDACC__)
#define BSG_HD __host__ __device__ __forceinline__
#else
#define BSG_HD inline
#endif

namespace bsg {

struct TileCoord {
  int g;   // batch
  int pm;  // tile row (M direction)
  int pn;  // tile column (N direction)
};

BSG_HD TileCoord tile_coord(int t, int grid_m, int grid_n, int group_m) {
  const int per_batch = grid_m * grid_n;
  TileCoord c;
  c.g = t / per_batch;
  const int local = t - c.g * per_batch;
  const int width = group_m * grid_n;  // tiles in one full group
  const int group = local / width;
  const int first_m = group * group_m;
  const int rows = (grid_m - first_m) < group_m ? (grid_m - first_m) : group_m;
  const int in_group = local - group * width;
  c.pm = first_m + in_group % rows;
  c.pn = in_group / rows;
  return c;
}

// Stream-K split of the persistent loop (balances the last, partial wave of
// tiles over every unit -- a CTA pair or a single CTA).  Tiles
// [0, dp_tiles) are processed whole, unit u taking tiles u, u + units, ...
// (data-parallel rounds).  The K blocks of the remaining tiles form one
// sequence of sk_iters = (num_tiles - dp_tiles) * KB blocks, tile by tile,
// cut into `units` contiguous ranges: unit u takes indices
// [u * sk_iters / units, (u + 1) * sk_iters / units).  A tile whose K blocks
// fall into several ranges is finished by the unit holding its first block
// (the "head", which reaches it last: it is at the end of that unit's range);
// the others hand over their fp32 (int32) partial sums.
struct WorkItem {
  int tile;
  int kb0, kb1;  // K blocks [kb0, kb1) of the tile
};

BSG_HD long long sk_range_begin(long long sk_iters, int unit, int units) {
  return sk_iters * unit / units;
}

// The unit whose range holds stream-K block index i (the largest u with
// sk_range_begin(u) <= i).
BSG_HD int sk_unit_of(long long i, long long sk_iters, int units) {
  return static_cast<int>(((i + 1) * units - 1) / sk_iters);
}

// Only the position is state; the split's constants come with each call, so
// a kernel keeps three values live across its loops.
struct WorkIter {
  int next_dp;
  long long sk, sk_end;

  BSG_HD WorkIter(int unit, int units, long long sk_iters)
      : next_dp(unit),
        sk(sk_iters > 0 ? sk_range_begin(sk_iters, unit, units) : 0),
        sk_end(sk_iters > 0 ? sk_range_begin(sk_iters, unit + 1, units) : 0) {}

  // The next work item of this unit, in processing order; false when done.
  BSG_HD bool next(WorkItem& w, int units, int dp_tiles, int KB) {
    if (next_dp < dp_tiles) {
      w.tile = next_dp;
      w.kb0 = 0;
      w.kb1 = KB;
      next_dp += units;
      return true;
    }
    if (sk < sk_end) {
      const long long rel = sk / KB;
      const long long tile_end = (rel + 1) * KB;
      const long long stop = sk_end < tile_end ? sk_end : tile_end;
      w.tile = dp_tiles + static_cast<int>(rel);
      w.kb0 = static_cast<int>(sk - rel * KB);
      w.kb1 = w.kb0 + static_cast<int>(stop - sk);
      sk = stop;
      return true;
    }
    return false;
  }
};

}  // namespace bsg
