// Host check of the dK / dV kernel's inverse windows (inverse_range in
// na_stages.cuh), for every 1-D grid length up to 40, window, stride and
// window mode:
//  - both ends of the window (window_range) never decrease as the query
//    coordinate grows: the premise of the query-block key boxes, of the
//    window-gather kernel's staged key box and of the inverse windows;
//  - for every key j, the queries whose window (window_range) holds j are
//    exactly [i0, i1), and i0, i1 never decrease as j grows;
//  - for every key block [k0, k1] (grid lengths up to 24, all blocks), the
//    queries whose window meets the block are exactly [I0(k0), I1(k1)) and
//    the queries whose window holds the whole block are exactly
//    [I0(k1), I1(k0)) (empty when that is reversed): the kernel's query box
//    and the part of it where a chunk needs no key mask.
// Built and run by tests/test_inverse_window.py; exit status 0 when all hold.
#include <cstdint>
#include <cstdio>
#include <vector>
#include "na_stages.cuh"
using namespace na;

int main() {
  long long checked = 0, bad = 0, blocks = 0, bad_blocks = 0;
  for (int L = 1; L <= 40; ++L)
    for (int w = 1; w <= L; ++w)
      for (int s = 1; s <= w; ++s)
        for (int m = WIN_CLAMPED; m <= WIN_CAUSAL; ++m) {
          std::vector<int> lo(L), hi(L), i0(L), i1(L);
          for (int i = 0; i < L; ++i) {
            window_range(L, w, s, m, i, lo[i], hi[i]);
            if (i > 0 && (lo[i] < lo[i - 1] || hi[i] < hi[i - 1])) ++bad;
          }
          for (int j = 0; j < L; ++j) {
            inverse_range(L, w, s, m, j, i0[j], i1[j]);
            if (j > 0 && (i0[j] < i0[j - 1] || i1[j] < i1[j - 1])) ++bad;
            for (int i = 0; i < L; ++i) {
              const bool holds = lo[i] <= j && j < hi[i];
              if (holds != (i0[j] <= i && i < i1[j])) ++bad;
              ++checked;
            }
          }
          if (L > 24) continue;
          for (int k0 = 0; k0 < L; ++k0)
            for (int k1 = k0; k1 < L; ++k1) {
              for (int i = 0; i < L; ++i) {
                const bool meets = lo[i] <= k1 && hi[i] > k0;
                const bool covers = lo[i] <= k0 && hi[i] > k1;
                if (meets != (i0[k0] <= i && i < i1[k1])) ++bad_blocks;
                if (covers != (i0[k1] <= i && i < i1[k0])) ++bad_blocks;
              }
              ++blocks;
            }
        }
  std::printf("inverse windows: %lld checked, %lld wrong; key blocks: %lld checked, %lld wrong\n",
              checked, bad, blocks, bad_blocks);
  return bad == 0 && bad_blocks == 0 ? 0 : 1;
}
