// Host check of the backward's two-tile stage slots (first_slot and
// second_slot in na_stages.cuh): for 2, 3 and 4 stages and the first 1000
// chunks, the two tiles of a chunk take the two slots of its stage; the
// first tile of chunk j + NST takes the slot the second tile of chunk j
// leaves and vice versa; and replaying the chunks in order, every slot is
// filled exactly once per round, by chunk round * NST + slot / 2, which is
// the fill number the producer's and issuer's barrier parities assume.
// Built and run by tests/test_slot_schedule.py; exit status 0 when all hold.
#include <cstdint>
#include <cstdio>
#include "na_stages.cuh"
using namespace na;

template <int NST>
static long long check() {
  long long bad = 0;
  int fills[2 * NST] = {};
  for (int j = 0; j < 1000; ++j) {
    const int a = first_slot<NST>(j), b = second_slot<NST>(j);
    if (a == b || a / 2 != j % NST || b / 2 != j % NST) ++bad;
    if (first_slot<NST>(j + NST) != b || second_slot<NST>(j + NST) != a) ++bad;
    const int used[2] = {a, b};
    for (int s : used) {
      if (fills[s] != j / NST) ++bad;   // fill number = round of the chunk
      ++fills[s];
    }
  }
  for (int s = 0; s < 2 * NST; ++s)
    if (fills[s] != 1000 / NST + (s / 2 < 1000 % NST ? 1 : 0)) ++bad;
  return bad;
}

int main() {
  const long long bad = check<2>() + check<3>() + check<4>();
  std::printf("slot schedule: %lld wrong\n", bad);
  return bad == 0 ? 0 : 1;
}
