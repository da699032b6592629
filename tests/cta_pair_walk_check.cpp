// Host check of the forward tensor-core kernel's key-chunk walk for one CTA,
// which owns two query blocks (2 p and 2 p + 1) that share one stream of K / V
// chunks: block_info for each block, chunk_grid_for over both, and a walk
// that streams every chunk non-EMPTY for at least one block, each block
// processing the chunks non-EMPTY for itself (chunk_status) and masking only
// the PARTIAL ones.  Random 1-D, 2-D and 3-D problems in every window mode;
// brute force over every query of each block and every key of the grid
// checks that:
//  - every key some query of the block attends lies in a chunk the block processes;
//  - every chunk a block processes holds a key one of its queries attends;
//  - a FULL chunk lies inside the grid and every query of the block attends
//    every key of it;
//  - the stream holds exactly the chunks some block processes.
// Built and run by tests/test_schedule_walks.py; exit status 0 when all hold.
#include <cstdint>
#include <cstdio>
#include <vector>
#include "na_sched.cuh"
using namespace na;

static uint64_t rng_state = 0xD1B54A32D192ED03ull;
static int rnd(int n) {
  rng_state = rng_state * 6364136223846793005ull + 1442695040888963407ull;
  return (int)((rng_state >> 33) % (uint64_t)n);
}

int main() {
  long long problems = 0, pairs = 0, streamed = 0, bad = 0;
  for (int trial = 0; trial < 3000; ++trial) {
    const int nd = 1 + trial % 3;
    Geom g;
    int qb[3], tl[3], kb[3];
    for (int d = 0; d < 3; ++d) {
      if (d < 3 - nd) {
        g.L[d] = g.w[d] = g.s[d] = 1;
        g.m[d] = WIN_CLAMPED;
        qb[d] = tl[d] = kb[d] = 1;
        continue;
      }
      const int Lmax = nd == 1 ? 96 : nd == 2 ? 24 : 12;
      g.L[d] = 1 + rnd(Lmax);
      g.w[d] = 1 + rnd(g.L[d]);
      g.s[d] = 1 + rnd(g.w[d]);
      g.m[d] = WIN_CLAMPED + rnd(3);
      qb[d] = 1 + rnd(nd == 1 ? 16 : 4);
      tl[d] = qb[d] * (1 + rnd(2));
      kb[d] = 1 + rnd(nd == 1 ? 16 : 4);
    }
    QTiling t;
    if (make_tiling(g, qb, tl, t) != 0) { ++bad; continue; }
    const int N = g.L[0] * g.L[1] * g.L[2];
    std::vector<int> wlo(3 * N), whi(3 * N);
    for (int q = 0; q < N; ++q) {
      const int c[3] = {q / (g.L[1] * g.L[2]), (q / g.L[2]) % g.L[1], q % g.L[2]};
      for (int d = 0; d < 3; ++d)
        window_range(g.L[d], g.w[d], g.s[d], g.m[d], c[d], wlo[3 * q + d], whi[3 * q + d]);
    }
    for (int p = 0; 2 * p < t.nblocks; ++p) {
      BlockInfo bi[2];
      block_info(g, t, 2 * p, bi[0]);
      block_info(g, t, 2 * p + 1, bi[1]);
      ChunkGrid cg;
      chunk_grid_for(bi, 2, kb, cg);
      // per block and key: attended by some / by every query of the block
      std::vector<char> some[2], all[2], done[2];
      for (int b = 0; b < 2; ++b) {
        some[b].assign(N, 0);
        all[b].assign(N, 1);
        done[b].assign(N, 0);
        if (!bi[b].exists) continue;
        for (int y0 = bi[b].o[0]; y0 < bi[b].o[0] + bi[b].n[0]; ++y0)
          for (int y1 = bi[b].o[1]; y1 < bi[b].o[1] + bi[b].n[1]; ++y1)
            for (int y2 = bi[b].o[2]; y2 < bi[b].o[2] + bi[b].n[2]; ++y2) {
              const int q = (y0 * g.L[1] + y1) * g.L[2] + y2;
              for (int k = 0; k < N; ++k) {
                const int x[3] = {k / (g.L[1] * g.L[2]), (k / g.L[2]) % g.L[1], k % g.L[2]};
                bool in = true;
                for (int d = 0; d < 3; ++d)
                  in = in && wlo[3 * q + d] <= x[d] && x[d] < whi[3 * q + d];
                if (in) some[b][k] = 1; else all[b][k] = 0;
              }
            }
      }
      ChunkIter it;
      iter_begin(cg, it);
      for (; it.idx < cg.total; iter_next(cg, kb, it)) {
        const int st[2] = {chunk_status(bi[0], it.a, kb), chunk_status(bi[1], it.a, kb)};
        if (st[0] == CHUNK_EMPTY && st[1] == CHUNK_EMPTY) continue;   // not streamed
        ++streamed;
        for (int b = 0; b < 2; ++b) {
          if (st[b] == CHUNK_EMPTY) continue;
          if (!bi[b].exists) { ++bad; continue; }
          bool inside = true;
          for (int d = 0; d < 3; ++d)
            inside = inside && it.a[d] >= 0 && it.a[d] + kb[d] <= g.L[d];
          if (st[b] == CHUNK_FULL && !inside) ++bad;
          bool holds_one = false;
          for (int x0 = it.a[0]; x0 < it.a[0] + kb[0] && x0 < g.L[0]; ++x0)
            for (int x1 = it.a[1]; x1 < it.a[1] + kb[1] && x1 < g.L[1]; ++x1)
              for (int x2 = it.a[2]; x2 < it.a[2] + kb[2] && x2 < g.L[2]; ++x2) {
                const int k = (x0 * g.L[1] + x1) * g.L[2] + x2;
                done[b][k] = 1;
                holds_one = holds_one || some[b][k];
                if (st[b] == CHUNK_FULL && !all[b][k]) ++bad;
              }
          if (!holds_one) ++bad;
        }
      }
      for (int b = 0; b < 2; ++b)
        for (int k = 0; k < N; ++k)
          if (some[b][k] && !done[b][k]) ++bad;
      ++pairs;
    }
    ++problems;
  }
  std::printf("CTA pair walks: %lld problems, %lld pairs, %lld chunks streamed, %lld wrong\n",
              problems, pairs, streamed, bad);
  return bad == 0 ? 0 : 1;
}
