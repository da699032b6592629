// Schedule helpers of the backward kernels, shared by the device code and
// host checks (the same __host__ __device__ convention as na_sched.cuh): the
// inverse windows of the key-stationary dK / dV kernel and the tile-slot
// schedule of both gradient kernels' two-tile stages.
#pragma once

#include "na_sched.cuh"

namespace na {

// First i in [0, L) whose window satisfies pred (false then true as i grows).
template <class F>
NA_HD int first_query(int L, F pred) {
  int lo = 0, hi = L;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (pred(mid)) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// Queries whose window holds key j in one dimension: [i0, i1).  Both window
// ends are non-decreasing in the query coordinate (every mode), so the set is
// an interval, found by two binary searches.
NA_HD void inverse_range(int L, int w, int s, int m, int j, int& i0, int& i1) {
  i0 = first_query(L, [&](int i) { int lo, hi; window_range(L, w, s, m, i, lo, hi); return hi > j; });
  i1 = first_query(L, [&](int i) { int lo, hi; window_range(L, w, s, m, i, lo, hi); return lo > j; });
}

// Query side of one key block kb (the dK / dV kernel's work item), as a
// BlockInfo over the whole grid so that chunk_grid_for / chunk_status walk
// query chunks the way the forward walks key chunks.  Per dimension, with k0
// and k1 the block's first and last keys inside the grid: [lo, hi) =
// [I0(k0), I1(k1)), the queries whose window meets the block, and
// [ilo, ihi) = [I0(k1), I1(k0)), those whose window holds all of it.
NA_HD void key_block_query_box(const Geom& g, const BlockInfo& kb, BlockInfo& ib) {
  ib.exists = kb.exists;
  for (int d = 0; d < 3; ++d) {
    ib.o[d] = 0;
    ib.n[d] = g.L[d];
    if (!ib.exists) continue;
    const int L = g.L[d], w = g.w[d], s = g.s[d], m = g.m[d];
    const int k0 = kb.o[d], k1 = kb.o[d] + kb.n[d] - 1;
    int a0, a1, b0, b1;
    inverse_range(L, w, s, m, k0, a0, a1);
    inverse_range(L, w, s, m, k1, b0, b1);
    ib.lo[d] = a0;
    ib.hi[d] = b1;
    ib.ilo[d] = b0;
    ib.ihi[d] = a1;
  }
}

// Two-tile stages of the backward's pipelines: stage st = j % NST of chunk j
// owns tile slots 2 st and 2 st + 1; which of them holds the chunk's first
// tile and which its second alternates with the round j / NST, so that the
// first tile of chunk j + NST goes into the slot that the second tile of
// chunk j frees (dK / dV kernel: Q into dO's slot, freed by dV before dK
// reads Q; dQ kernel: K into V's slot, freed by dP before dQ reads K).  Each
// slot is filled once per round, so fill number j / NST.
template <int NST>
NA_HD int first_slot(int j) { return 2 * (j % NST) + ((j / NST) & 1); }
template <int NST>
NA_HD int second_slot(int j) { return 2 * (j % NST) + 1 - ((j / NST) & 1); }

}  // namespace na
