// Host check of the dK / dV kernel's inverse windows (inverse_range in
// na_stages.cuh): for every 1-D grid length up to 40, window, stride and
// window mode, and every key j, the queries whose window (window_range)
// holds j are exactly [i0, i1), and i0, i1 never decrease as j grows (the
// kernel takes a key block's query box from its first and last keys).
// Built and run by tests/test_inverse_window.py; exit status 0 when all hold.
#include <cstdint>
#include <cstdio>
#include "na_stages.cuh"
using namespace na;

int main() {
  long long checked = 0, bad = 0;
  for (int L = 1; L <= 40; ++L)
    for (int w = 1; w <= L; ++w)
      for (int s = 1; s <= w; ++s)
        for (int m = WIN_CLAMPED; m <= WIN_CAUSAL; ++m) {
          int p0 = 0, p1 = 0;
          for (int j = 0; j < L; ++j) {
            int i0, i1;
            inverse_range(L, w, s, m, j, i0, i1);
            if (j > 0 && (i0 < p0 || i1 < p1)) ++bad;
            p0 = i0;
            p1 = i1;
            for (int i = 0; i < L; ++i) {
              int lo, hi;
              window_range(L, w, s, m, i, lo, hi);
              const bool holds = lo <= j && j < hi;
              if (holds != (i0 <= i && i < i1)) ++bad;
              ++checked;
            }
          }
        }
  std::printf("inverse windows: %lld checked, %lld wrong\n", checked, bad);
  return bad == 0 ? 0 : 1;
}
