// Host check of the dK / dV kernel's walk over query chunks, on 1-D, 2-D and
// 3-D grids with random window modes, windows, strides, key block shapes and
// query chunk shapes.  For every key block (block_info over the key tiling),
// the kernel takes its query box with key_block_query_box, lays a chunk grid
// over it (chunk_grid_for) and visits the chunks that chunk_status does not
// call EMPTY, masking only the PARTIAL ones.  Brute force over every key of
// the block and every query of the grid checks that:
//  - every query that attends some key of the block lies in a visited chunk;
//  - every visited chunk holds at least one such query;
//  - a FULL chunk lies inside the grid and every query of it attends every
//    key of the block.
// Built and run by tests/test_schedule_walks.py; exit status 0 when all hold.
#include <cstdint>
#include <cstdio>
#include <vector>
#include "na_stages.cuh"
using namespace na;

static uint64_t rng_state = 0x9E3779B97F4A7C15ull;
static int rnd(int n) {  // uniform-ish in [0, n)
  rng_state = rng_state * 6364136223846793005ull + 1442695040888963407ull;
  return (int)((rng_state >> 33) % (uint64_t)n);
}

int main() {
  long long problems = 0, blocks = 0, chunks = 0, bad = 0;
  for (int trial = 0; trial < 3000; ++trial) {
    const int nd = 1 + trial % 3;
    Geom g;
    int qb[3], tl[3], qc[3];
    for (int d = 0; d < 3; ++d) {
      if (d < 3 - nd) {  // leading unit dimensions, as the kernels see a lower-rank grid
        g.L[d] = g.w[d] = g.s[d] = 1;
        g.m[d] = WIN_CLAMPED;
        qb[d] = tl[d] = qc[d] = 1;
        continue;
      }
      const int Lmax = nd == 1 ? 96 : nd == 2 ? 24 : 12;
      g.L[d] = 1 + rnd(Lmax);
      g.w[d] = 1 + rnd(g.L[d]);
      g.s[d] = 1 + rnd(g.w[d]);
      g.m[d] = WIN_CLAMPED + rnd(3);
      qb[d] = 1 + rnd(nd == 1 ? 16 : 4);
      tl[d] = qb[d] * (1 + rnd(2));
      qc[d] = 1 + rnd(nd == 1 ? 16 : 4);
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
    for (int blk = 0; blk < t.nblocks; ++blk) {
      BlockInfo kb, ib;
      block_info(g, t, blk, kb);
      if (!kb.exists) continue;
      key_block_query_box(g, kb, ib);
      ChunkGrid cg;
      chunk_grid_for(&ib, 1, qc, cg);
      // per query: attends some key of the block / all keys of the block
      std::vector<char> some(N, 0), all(N, 1), visited(N, 0), full(N, 0);
      for (int q = 0; q < N; ++q)
        for (int x0 = kb.o[0]; x0 < kb.o[0] + kb.n[0]; ++x0)
          for (int x1 = kb.o[1]; x1 < kb.o[1] + kb.n[1]; ++x1)
            for (int x2 = kb.o[2]; x2 < kb.o[2] + kb.n[2]; ++x2) {
              const int x[3] = {x0, x1, x2};
              bool in = true;
              for (int d = 0; d < 3; ++d)
                in = in && wlo[3 * q + d] <= x[d] && x[d] < whi[3 * q + d];
              if (in) some[q] = 1; else all[q] = 0;
            }
      ChunkIter it;
      iter_begin(cg, it);
      for (; it.idx < cg.total; iter_next(cg, qc, it)) {
        const int st = chunk_status(ib, it.a, qc);
        if (st == CHUNK_EMPTY) continue;
        ++chunks;
        bool inside = true;
        for (int d = 0; d < 3; ++d) inside = inside && it.a[d] >= 0 && it.a[d] + qc[d] <= g.L[d];
        if (st == CHUNK_FULL && !inside) ++bad;
        bool holds_one = false;
        for (int y0 = it.a[0]; y0 < it.a[0] + qc[0] && y0 < g.L[0]; ++y0)
          for (int y1 = it.a[1]; y1 < it.a[1] + qc[1] && y1 < g.L[1]; ++y1)
            for (int y2 = it.a[2]; y2 < it.a[2] + qc[2] && y2 < g.L[2]; ++y2) {
              const int q = (y0 * g.L[1] + y1) * g.L[2] + y2;
              visited[q] = 1;
              holds_one = holds_one || some[q];
              if (st == CHUNK_FULL && !all[q]) ++bad;
            }
        if (!holds_one) ++bad;
      }
      for (int q = 0; q < N; ++q)
        if (some[q] && !visited[q]) ++bad;
      ++blocks;
    }
    ++problems;
  }
  std::printf("key-block walks: %lld problems, %lld key blocks, %lld chunks visited, %lld wrong\n",
              problems, blocks, chunks, bad);
  return bad == 0 ? 0 : 1;
}
