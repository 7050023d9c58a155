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

}  // namespace bsg
