// Tile-slot schedule of the backward kernels' two-tile stages, shared by the
// device code and host checks (the same __host__ __device__ convention as
// na_sched.cuh).
#pragma once

#include "na_sched.cuh"

namespace na {

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
