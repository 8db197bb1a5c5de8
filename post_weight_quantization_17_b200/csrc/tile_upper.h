// Dense enumeration of the output tiles that touch the upper triangle (tile row <= tile column),
// in the grouped order of the CTA-pair GEMM: groups of `group` tile rows, each walked column by
// column starting at the group's own diagonal column, rows in order inside a column.  Every index
// below the count is a real tile, so tiles handed out in turn spread evenly over the CTA pairs
// (a walk over all tile slots that skipped the lower ones left some pairs with far more tiles).
#pragma once

namespace gptq {

// tiles of one group: `rows` tile rows, `cols` tile columns from the group's first row on;
// column c (relative) holds min(rows, c + 1) tiles
__host__ __device__ inline int upper_group_tiles(int rows, int cols) {
  if (cols <= 0 || rows <= 0) return 0;
  const int P = (rows - 1 < cols) ? rows - 1 : cols;  // columns with fewer than `rows` tiles
  return P * (P + 1) / 2 + (cols - P) * rows;
}

__host__ __device__ inline int upper_tiles(int tiles_m, int tiles_n, int group) {
  int n = 0;
  for (int first = 0; first < tiles_m; first += group) {
    const int rows = (tiles_m - first < group) ? tiles_m - first : group;
    n += upper_group_tiles(rows, tiles_n - first);
  }
  return n;
}

// tile t (0 <= t < upper_tiles(...)) -> (tm, tn)
__host__ __device__ inline void upper_tile(int tiles_m, int tiles_n, int group, int t, int& tm,
                                           int& tn) {
  int first = 0, rows = 0, cnt = 0;
  for (;; first += group) {
    rows = (tiles_m - first < group) ? tiles_m - first : group;
    cnt = upper_group_tiles(rows, tiles_n - first);
    if (t < cnt || first + group >= tiles_m) break;
    t -= cnt;
  }
  const int cols = tiles_n - first;
  const int P = (rows - 1 < cols) ? rows - 1 : cols;
  int c, r;
  if (t < P * (P + 1) / 2) {
    c = 0;
    while ((c + 1) * (c + 2) / 2 <= t) ++c;
    r = t - c * (c + 1) / 2;
  } else {
    const int t2 = t - P * (P + 1) / 2;
    c = P + t2 / rows;
    r = t2 % rows;
  }
  tm = first + r;
  tn = first + c;
}

}  // namespace gptq
