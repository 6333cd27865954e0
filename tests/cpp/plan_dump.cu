// Host-only driver for the tile schedule in gla_common.cuh (no GPU needed):
// prints every CTA's tile sequence and the scan's per-unit slot ranges.
//   plan_dump <units> <tiles_per_unit> <ctas>
// Output lines:  T <cta> <unit> <tile> <first> <last> <slot>
//                U <unit> <first_cta> <last_cta> <slot_of(first_cta)>
#include <cstdio>
#include <cstdlib>

#include "gla_common.cuh"

int main(int argc, char** argv) {
  if (argc != 4) return 2;
  const long long units = atoll(argv[1]);
  const int tpu = atoi(argv[2]);
  const int G = atoi(argv[3]);
  const gla::WorkPlan wp = gla::WorkPlan::make(units, tpu, G);
  for (int c = 0; c < G; ++c) {
    gla::TileCursor cur;
    cur.init(wp, c);
    for (; cur.valid(); cur.advance())
      printf("T %d %d %d %d %d %lld\n", c, cur.u, cur.t, int(cur.first), int(cur.last),
             static_cast<long long>(cur.slot()));
  }
  for (long long u = 0; u < units; ++u) {
    int c0, c1;
    wp.slot_range(u, c0, c1);
    printf("U %lld %d %d %lld\n", u, c0, c1, static_cast<long long>(wp.slot(u, c0)));
  }
  return 0;
}
