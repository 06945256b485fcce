// Host-only check of the stream-K schedule shared by the grouped GEMM's fp32 k-split mode and
// its summing kernel (common.cuh): CTA c of g owns k-blocks [c * work / g, (c + 1) * work / g)
// of work = tiles * nkb.  For many (tiles, nkb, slots, grid) the closed forms must agree with a
// brute-force owner table: streamk_owner(x) is the CTA holding k-block x, every tile meets at
// most `slots` CTA ranges, and every used range is non-empty.  Prints "ok" or the first failure.
#include <stdio.h>
#include <vector>

#include "common.cuh"

int main() {
  const int nkbs[] = {1, 2, 3, 4, 7, 16, 22, 32, 64, 112, 224};
  const int grids[] = {1, 2, 3, 37, 100, 147, 148};
  const int slot_counts[] = {2, 3, 8};
  long checked = 0;
  for (int tiles = 1; tiles <= 260; tiles += (tiles < 40 ? 1 : 23))
    for (int nkb : nkbs)
      for (int grid : grids)
        for (int slots : slot_counts) {
          const long long work = (long long)tiles * nkb;
          const int g = moe::streamk_ctas(work, nkb, slots, grid);
          if (g < 1 || g > grid) {
            printf("FAILED: %d CTAs for grid %d\n", g, grid);
            return 1;
          }
          std::vector<int> owner(work);
          for (int c = 0; c < g; ++c) {
            const long long lo = (long long)c * work / g, hi = (long long)(c + 1) * work / g;
            if (hi <= lo) {
              printf("FAILED: empty range of CTA %d (work %lld, g %d)\n", c, work, g);
              return 1;
            }
            for (long long x = lo; x < hi; ++x) owner[x] = c;
          }
          for (long long x = 0; x < work; ++x)
            if (moe::streamk_owner(x, work, g) != owner[x]) {
              printf("FAILED: owner of k-block %lld (work %lld, g %d)\n", x, work, g);
              return 1;
            }
          for (int t = 0; t < tiles; ++t) {
            const int segs = owner[(long long)(t + 1) * nkb - 1] - owner[(long long)t * nkb] + 1;
            if (segs > slots) {
              printf("FAILED: tile %d meets %d ranges, %d slots\n", t, segs, slots);
              return 1;
            }
          }
          ++checked;
        }
  printf("ok: %ld schedules\n", checked);
  return 0;
}
