// Host check of the upper-triangle tile enumeration (tile_upper.h): every tile with tile row <=
// tile column exactly once, none other, groups in order.  Built and run by test_tile_order_cpu.py.
#define __host__
#define __device__
#include <cstdio>
#include <set>
#include <utility>
#include "tile_upper.h"
int main() {
  int bad = 0;
  for (int G : {8, 16})
  for (int tm = 1; tm <= 100; ++tm)
    for (int tnn = 1; tnn <= 100; ++tnn) {
      std::set<std::pair<int,int>> want, got;
      for (int a = 0; a < tm; ++a) for (int b = 0; b < tnn; ++b) if (a <= b) want.insert({a,b});
      int n = gptq::upper_tiles(tm, tnn, G);
      if (n != (int)want.size()) { printf("count %d %d: %d vs %zu\n", tm, tnn, n, want.size()); ++bad; continue; }
      int prev_first = -1;
      for (int t = 0; t < n; ++t) {
        int a, b; gptq::upper_tile(tm, tnn, G, t, a, b);
        if (a < 0 || a >= tm || b < 0 || b >= tnn || a > b || !got.insert({a,b}).second) { printf("bad tile %d %d t=%d -> %d %d\n", tm, tnn, t, a, b); ++bad; break; }
        int first = a / G * G;
        if (first < prev_first) { printf("group order %d %d t=%d\n", tm, tnn, t); ++bad; break; }
        prev_first = first;
      }
      if (got != want) { ++bad; }
    }
  printf("bad=%d\n", bad);
  return bad != 0;
}
