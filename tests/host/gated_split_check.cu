// Host-side check of gated_cold_split (the cold split of gated decode calls,
// computed identically by the attention and merge kernels): over a grid of
// active-unit counts, blocks per unit and CTA limits it must give at most
// the limit's CTAs, cover every block exactly once, and let no unit span
// more CTAs than it has partial slots.  Prints "ok" or the first failure.
#include <cstdio>

#include "tq_internal.cuh"

int main() {
  using namespace tq;
  const int64_t blocks[] = {1, 2, 3, 63, 64, 65, 504, 2048, 9000};
  const int limits[] = {1, 7, 148, 296, 588, 592, 1184};
  long checked = 0;
  for (int64_t nb : blocks)
    for (int C : limits)
      for (int64_t na = 0; na <= 130; na += (na < 10 ? 1 : 13)) {
        int64_t bpc = 0;
        int ctas = -1;
        gated_cold_split(na, nb, C, &bpc, &ctas);
        const int64_t total = na * nb;
        if (bpc < 1 || ctas < 0 || ctas > C) {
          printf("limits: na=%lld nb=%lld C=%d -> bpc=%lld ctas=%d\n", (long long)na, (long long)nb, C,
                 (long long)bpc, ctas);
          return 1;
        }
        if ((int64_t)ctas * bpc < total || (ctas > 0 && (int64_t)(ctas - 1) * bpc >= total)) {
          printf("cover: na=%lld nb=%lld C=%d\n", (long long)na, (long long)nb, C);
          return 1;
        }
        for (int64_t p = 0; p < na; ++p) {
          const int64_t span = ((p + 1) * nb - 1) / bpc - (p * nb) / bpc + 1;
          if (span > kSlotsCold) {
            printf("slots: na=%lld nb=%lld C=%d unit %lld spans %lld\n", (long long)na, (long long)nb,
                   C, (long long)p, (long long)span);
            return 1;
          }
        }
        ++checked;
      }
  printf("ok %ld\n", checked);
  return 0;
}
