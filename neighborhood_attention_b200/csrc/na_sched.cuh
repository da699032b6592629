// Window rule and tile scheduler of the CUDA path, usable on host and device.
//
// Geometry is always held in three dimensions (X1, X2, X3), X3 innermost in
// memory; a 1-D problem is (1, 1, L) and a 2-D problem (1, H, W).
//
// Window rule (per dimension; window w, stride s, length L): the query at
// coordinate i belongs to stride group g = i / s whose centre member is
// c = g*s + s/2; its window is [start, start + w) with
//   start = clamp(c - w/2, 0, L - w),
// so every query sees exactly prod(w) keys ("clamped" mode).  Stride 1 is neighborhood
// attention; stride equal to the tile with w an odd multiple of it is sliding
// tile attention ("Generalized Neighborhood Attention: Multi-dimensional
// Sparse Attention at the Speed of Light", abstract: sliding, strided sliding
// and blocked windows; "ENA: Efficient N-dimensional Attention", sliding tile
// attention: tokens of a tile share one window that shifts tile by tile).
//
// Schedule: queries are processed in blocks (boxes of the grid); a block's
// keys lie in the per-dimension union of its queries' windows, which is a box
// because the window start is monotone in the query coordinate and the N-d
// window is a product of 1-D windows.  That key box is walked in chunks
// (boxes of kb tokens).  A chunk is EMPTY for a block when it misses the
// block's key box, FULL when it lies inside the intersection of all the
// block's windows (no mask needed), else PARTIAL (element mask) -- the
// empty / partial / full block taxonomy of "Hilbert-Guided Sparse Local
// Attention" (Methodology in Plain English), with masks only on partial tiles.
#pragma once

#ifdef __CUDACC__
#define NA_HD __host__ __device__ __forceinline__
#else
#define NA_HD inline
#endif

namespace na {

enum ChunkStatus : int { CHUNK_EMPTY = 0, CHUNK_PARTIAL = 1, CHUNK_FULL = 2 };
enum WindowMode : int { WIN_CLAMPED = 0, WIN_TRUNCATED = 1, WIN_CAUSAL = 2 };

NA_HD int imin(int a, int b) { return a < b ? a : b; }
NA_HD int imax(int a, int b) { return a > b ? a : b; }
NA_HD int cdiv(int a, int b) { return (a + b - 1) / b; }

NA_HD int window_start(int L, int w, int s, int i) {
  int g = i / s;
  int c = g * s + s / 2;
  int start = c - w / 2;
  start = imax(start, 0);
  start = imin(start, L - w);
  return start;
}

// Window [lo, hi) of coordinate i in one dimension under `mode`.
NA_HD void window_range(int L, int w, int s, int mode, int i, int& lo, int& hi) {
  if (mode == WIN_CLAMPED) {
    lo = window_start(L, w, s, i);
    hi = lo + w;
    return;
  }
  const int g = i / s;
  const int a = (mode == WIN_TRUNCATED) ? g * s + s / 2 - w / 2 : (g + 1) * s - w;
  lo = imax(a, 0);
  hi = imin(a + w, L);
}

struct Geom {
  int L[3], w[3], s[3];
  int m[3];  // WindowMode per dimension
};

// A dilated problem runs as one grid per residue class: class (r0, r1, r2)
// holds the coordinates r + dil * x of the full grid (extents Lf), seen as a
// grid of its own with coordinates x.  full_token maps x back to the full
// grid's row-major token index.  Undilated: dil 1, res 0, Lf = the grid.
struct DilMap {
  int dil[3], res[3], Lf[3];
};

NA_HD long long full_token(const DilMap& m, int x0, int x1, int x2) {
  return ((long long)(m.res[0] + m.dil[0] * x0) * m.Lf[1] + (m.res[1] + m.dil[1] * x1)) *
             m.Lf[2] +
         (m.res[2] + m.dil[2] * x2);
}

NA_HD DilMap identity_map(const int L[3]) {
  DilMap m;
  for (int d = 0; d < 3; ++d) {
    m.dil[d] = 1;
    m.res[d] = 0;
    m.Lf[d] = L[d];
  }
  return m;
}

// Tiling of the queries: tiles of tl tokens per dim, each split into blocks
// of qb tokens (qb divides tl).  Blocks are numbered tile by tile, row-major
// over the tile grid and row-major over the blocks inside a tile, so that
// consecutive block ids stay inside one tile where possible.
struct QTiling {
  int qb[3];      // block shape
  int tl[3];      // tile shape (multiple of qb per dim)
  int nt[3];      // tiles per dim = ceil(L / tl)
  int bt[3];      // blocks per tile per dim = tl / qb
  int bpt;        // blocks per tile
  int nblocks;    // blocks per (batch, head)
};

// Per-dimension extents of one query block.
struct BlockInfo {
  int exists;      // 1 if the block holds at least one query inside the grid
  int o[3];        // origin (grid coordinates of row 0)
  int n[3];        // valid extent per dim (rows inside the grid)
  int lo[3], hi[3];    // union of the valid queries' windows: [lo, hi)
  int ilo[3], ihi[3];  // intersection of their windows: [ilo, ihi) (may be empty)
};

NA_HD void block_info(const Geom& g, const QTiling& t, int blk, BlockInfo& b) {
  b.exists = 0;
  if (blk < 0 || blk >= t.nblocks) return;
  int tile = blk / t.bpt, sub = blk % t.bpt;
  int tc[3], sc[3];
  tc[2] = tile % t.nt[2]; tile /= t.nt[2];
  tc[1] = tile % t.nt[1]; tc[0] = tile / t.nt[1];
  sc[2] = sub % t.bt[2]; sub /= t.bt[2];
  sc[1] = sub % t.bt[1]; sc[0] = sub / t.bt[1];
  b.exists = 1;
  for (int d = 0; d < 3; ++d) {
    b.o[d] = tc[d] * t.tl[d] + sc[d] * t.qb[d];
    b.n[d] = imin(t.qb[d], g.L[d] - b.o[d]);
    if (b.n[d] <= 0) { b.exists = 0; b.n[d] = 0; continue; }
    int flo, fhi, llo, lhi;  // windows of the first and last valid query
    window_range(g.L[d], g.w[d], g.s[d], g.m[d], b.o[d], flo, fhi);
    window_range(g.L[d], g.w[d], g.s[d], g.m[d], b.o[d] + b.n[d] - 1, llo, lhi);
    b.lo[d] = flo;
    b.hi[d] = lhi;
    b.ilo[d] = llo;
    b.ihi[d] = fhi;
  }
}

// Key box walked for a group of blocks (a CTA's blocks), in chunks of kb.
struct ChunkGrid {
  int org[3];     // origin of chunk (0,0,0)
  int nc[3];      // chunks per dim
  int total;
};

NA_HD void chunk_grid_for(const BlockInfo* bs, int nb, const int kb[3], ChunkGrid& cg) {
  int lo[3] = {0, 0, 0}, hi[3] = {0, 0, 0};
  int any = 0;
  for (int i = 0; i < nb; ++i) {
    if (!bs[i].exists) continue;
    for (int d = 0; d < 3; ++d) {
      lo[d] = any ? imin(lo[d], bs[i].lo[d]) : bs[i].lo[d];
      hi[d] = any ? imax(hi[d], bs[i].hi[d]) : bs[i].hi[d];
    }
    any = 1;
  }
  cg.total = any ? 1 : 0;
  for (int d = 0; d < 3; ++d) {
    cg.org[d] = lo[d];
    cg.nc[d] = any ? cdiv(hi[d] - lo[d], kb[d]) : 0;
    cg.total *= cg.nc[d];
  }
}

NA_HD void chunk_origin(const ChunkGrid& cg, const int kb[3], int c, int a[3]) {
  int c2 = c % cg.nc[2]; c /= cg.nc[2];
  int c1 = c % cg.nc[1]; int c0 = c / cg.nc[1];
  a[0] = cg.org[0] + c0 * kb[0];
  a[1] = cg.org[1] + c1 * kb[1];
  a[2] = cg.org[2] + c2 * kb[2];
}

// Row-major walk over a chunk grid without divisions.
struct ChunkIter {
  int idx;      // linear chunk index; == ChunkGrid::total when exhausted
  int c[3];     // chunk coordinates
  int a[3];     // chunk origin in grid coordinates
};

NA_HD void iter_begin(const ChunkGrid& cg, ChunkIter& it) {
  it.idx = 0;
  for (int d = 0; d < 3; ++d) {
    it.c[d] = 0;
    it.a[d] = cg.org[d];
  }
}

NA_HD void iter_next(const ChunkGrid& cg, const int kb[3], ChunkIter& it) {
  ++it.idx;
  if (++it.c[2] < cg.nc[2]) { it.a[2] += kb[2]; return; }
  it.c[2] = 0;
  it.a[2] = cg.org[2];
  if (++it.c[1] < cg.nc[1]) { it.a[1] += kb[1]; return; }
  it.c[1] = 0;
  it.a[1] = cg.org[1];
  ++it.c[0];
  it.a[0] += kb[0];
}

NA_HD int chunk_status(const BlockInfo& b, const int a[3], const int kb[3]) {
  if (!b.exists) return CHUNK_EMPTY;
  int full = 1;
  for (int d = 0; d < 3; ++d) {
    int c0 = a[d], c1 = a[d] + kb[d];
    if (c1 <= b.lo[d] || c0 >= b.hi[d]) return CHUNK_EMPTY;
    if (!(c0 >= b.ilo[d] && c1 <= b.ihi[d])) full = 0;
  }
  return full ? CHUNK_FULL : CHUNK_PARTIAL;
}

NA_HD int make_tiling(const Geom& g, const int qb[3], const int tl[3], QTiling& t) {
  t.bpt = 1;
  int ntiles = 1;
  for (int d = 0; d < 3; ++d) {
    t.qb[d] = qb[d];
    t.tl[d] = tl[d];
    if (qb[d] < 1 || tl[d] < qb[d] || tl[d] % qb[d]) return -1;
    t.nt[d] = cdiv(g.L[d], tl[d]);
    t.bt[d] = tl[d] / qb[d];
    t.bpt *= t.bt[d];
    ntiles *= t.nt[d];
  }
  t.nblocks = ntiles * t.bpt;
  return 0;
}

// Bits [a, b) of a 32-bit word (0 <= a <= b <= 32).
NA_HD uint32_t range_bits(int a, int b) {
  if (b - a >= 32) return 0xffffffffu;
  return ((1u << (b - a)) - 1u) << a;
}

// Bits i of 32-bit word w marking keys j = 32w + i whose coordinate along one
// dimension, (j >> sh) & (kb - 1) (kb a power of two), lies in [lo, hi).
// Along that dimension the key order repeats with period P = kb << sh: a
// period of at most 32 bits is one range of bits, copied across the word by
// at most five doubling shifts; a longer period puts one range of
// coordinates, or a single coordinate, in the word.  No division and no
// per-period loop: this runs on the softmax's critical path for every
// partial chunk.
NA_HD uint32_t dim_word_mask(int w, int sh, int kb, int lo, int hi) {
  if (lo >= hi) return 0u;
  const int P = kb << sh;
  if (P <= 32) {
    uint32_t v = range_bits(lo << sh, hi << sh);
    for (int step = P; step < 32; step <<= 1) v |= v << step;
    return v;
  }
  const int xs = ((32 * w) >> sh) & (kb - 1);   // first coordinate in this word
  if (sh >= 5) return (xs >= lo && xs < hi) ? 0xffffffffu : 0u;
  const int a = imax(lo, xs), b = imin(hi, xs + (32 >> sh));
  return a < b ? range_bits((a - xs) << sh, (b - xs) << sh) : 0u;
}

// Validity of the 128 keys of a chunk for one query: key j (chunk-local
// coordinates (j >> sh0, (j >> sh1) & (kb1-1), j & (kb2-1))) is inside the
// query's window [wlo_d, whi_d) in every dimension.
NA_HD void chunk_key_mask(const int a[3], const int wlo[3], const int whi[3],
                                               const int kb[3], const int kbl[3], uint32_t (&mk)[4]) {
  int lo[3], hi[3];
  const int sh[3] = {kbl[1] + kbl[2], kbl[2], 0};
  for (int d = 0; d < 3; ++d) {
    lo[d] = imin(imax(wlo[d] - a[d], 0), kb[d]);
    hi[d] = imin(imax(whi[d] - a[d], 0), kb[d]);
  }
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    uint32_t m = 0xffffffffu;
#pragma unroll
    for (int d = 0; d < 3; ++d) m &= dim_word_mask(wd, sh[d], kb[d], lo[d], hi[d]);
    mk[wd] = m;
  }
}

// The same mask from a loop over the periods of each dimension: slower on
// partial chunks, but its code is a fraction of the straight-line form's.
// The forward kernel at head_dim 128 uses it: there the straight-line form,
// inlined in the softmax loop, slowed the full-chunk path by about 5 %
// (measured on the sliding-tile workload, which has no partial chunks).
NA_HD uint32_t periodic_range_word(int w, int period, int a, int b) {
  uint32_t m = 0;
  const int base = 32 * w;
  for (int p0 = base - base % period; p0 < base + 32; p0 += period) {
    const int lo = imax(p0 + a, base) - base;
    const int hi = imin(p0 + b, base + 32) - base;
    if (lo < hi) m |= range_bits(lo, hi);
  }
  return m;
}

NA_HD void chunk_key_mask_compact(const int a[3], const int wlo[3], const int whi[3],
                                  const int kb[3], const int kbl[3], uint32_t (&mk)[4]) {
  int lo[3], hi[3], stride[3];
  stride[2] = 1;
  stride[1] = 1 << kbl[2];
  stride[0] = 1 << (kbl[1] + kbl[2]);
  for (int d = 0; d < 3; ++d) {
    lo[d] = imin(imax(wlo[d] - a[d], 0), kb[d]);
    hi[d] = imin(imax(whi[d] - a[d], 0), kb[d]);
  }
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    uint32_t m = 0xffffffffu;
    for (int d = 0; d < 3; ++d)
      m &= periodic_range_word(wd, kb[d] * stride[d], lo[d] * stride[d], hi[d] * stride[d]);
    mk[wd] = m;
  }
}

// Same for one block: the status of the chunk found (CHUNK_EMPTY at the end).
NA_HD int seek_block(const ChunkGrid& cg, const int* kb, const BlockInfo& b,
                                          ChunkIter& it) {
  for (; it.idx < cg.total; iter_next(cg, kb, it)) {
    const int st = chunk_status(b, it.a, kb);
    if (st != CHUNK_EMPTY) return st;
  }
  return CHUNK_EMPTY;
}

}  // namespace na
