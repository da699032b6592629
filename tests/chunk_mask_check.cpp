// Host check of the chunk key mask (chunk_key_mask and chunk_key_mask_compact
// in na_sched.cuh, used on the softmax's critical path of every partial
// chunk): for every chunk shape
// of 128 keys (powers of two per dimension) and pseudo-random chunk origins
// and windows, every bit against a direct per-key range test.  Built and run
// by tests/test_chunk_mask.py; exit status 0 when every bit matches.
#include <cstdint>
#include <cstdio>
#include "na_sched.cuh"
using namespace na;
int main() {
  long long checked = 0, bad = 0;
  for (int e0 = 0; e0 <= 7; ++e0) for (int e1 = 0; e0 + e1 <= 7; ++e1) {
    const int e2 = 7 - e0 - e1;
    const int kb[3] = {1 << e0, 1 << e1, 1 << e2}, kbl[3] = {e0, e1, e2};
    for (int trial = 0; trial < 4000; ++trial) {
      int a[3], wlo[3], whi[3];
      unsigned x = trial * 2654435761u + e0 * 97 + e1 * 13;
      for (int d = 0; d < 3; ++d) {
        x = x * 1103515245u + 12345u; a[d] = (x >> 8) % 300;
        x = x * 1103515245u + 12345u; wlo[d] = a[d] - kb[d] + (int)((x >> 8) % (3 * kb[d] + 2));
        x = x * 1103515245u + 12345u; whi[d] = wlo[d] + (int)((x >> 8) % (2 * kb[d] + 3));
      }
      uint32_t mk[4], mc[4];
      chunk_key_mask(a, wlo, whi, kb, kbl, mk);
      chunk_key_mask_compact(a, wlo, whi, kb, kbl, mc);
      for (int w = 0; w < 4; ++w)
        if (mk[w] != mc[w]) ++bad;   // the two forms agree word for word
      for (int j = 0; j < 128; ++j) {
        const int x0 = j >> (e1 + e2), x1 = (j >> e2) & (kb[1] - 1), x2 = j & (kb[2] - 1);
        const bool in = a[0] + x0 >= wlo[0] && a[0] + x0 < whi[0] && a[1] + x1 >= wlo[1] &&
                        a[1] + x1 < whi[1] && a[2] + x2 >= wlo[2] && a[2] + x2 < whi[2];
        const bool got = (mk[j >> 5] >> (j & 31)) & 1u;
        ++checked;
        if (in != got) ++bad;
      }
    }
  }
  printf("checked %lld bits, %lld wrong\n", checked, bad);
  return bad != 0;
}
