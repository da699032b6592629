// Window-gather forward kernel (CUDA cores) for narrow windows: fp32, bf16 or
// f16 inputs, head_dim 32, 64 or 128, any grid, window, stride and window mode.
//
// With a handful of keys per query the forward is bound by HBM traffic (q, k,
// v read and out written once: a few FLOPs per byte), so this kernel moves
// bytes, not tiles of scores.  The work is cut into query tiles (boxes of the
// grid); a persistent grid of CTAs walks them.  A tile's query rows and the K
// and V rows of its key box -- the union of its queries' windows, itself a
// box -- arrive by bulk copies (one per run of rows adjacent in memory) into
// a shared-memory stage; with two stages the next tile streams in while the
// current one is computed.  Each query is served by a group of consecutive
// threads, each holding 32 elements of the head dimension: the group walks
// the query's own window key by key (the product of its per-dimension ranges,
// cut windows included) over the staged rows, reduces the partial dot
// products with shuffles and keeps an online softmax in the log2 domain.  The
// output goes out as 16-byte stores.  When even a one-query tile's key box
// would not fit in shared memory (a wide window), a direct form reads K and V
// straight from global memory instead.
//
// The arithmetic is the restricted softmax attention of "pi-Attention",
// section 3.1 eqs. (1)-(3) with the neighbourhood of section 3.2 (eq. (5) for
// cut windows); the lse output is the log of eq. (2)'s denominator.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "na_internal.h"
#include "na_ptx.cuh"

namespace na {
namespace {

constexpr int GATHER_THREADS = 256;
constexpr int KEYS_PER_STEP = 4;   // keys whose loads are in flight together

enum : int { G_F32 = 0, G_BF16 = 1, G_F16 = 2 };   // na_dtype numbering

// Elements per 16-byte slice.
template <int T>
__host__ __device__ constexpr int slice_elems() { return T == G_F32 ? 4 : 8; }

template <int T>
__device__ __forceinline__ void unpack(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  if constexpr (T == G_F32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = __uint_as_float(w[i]);
  } else if constexpr (T == G_BF16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      const float2 v = __half22float2(h);
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
  }
}

template <int T>
__device__ __forceinline__ uint4 pack(const float* f) {
  uint32_t w[4];
  if constexpr (T == G_F32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = __float_as_uint(f[i]);
  } else if constexpr (T == G_BF16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint4 load_slice(const void* base, size_t elem_off_bytes) {
  return __ldg(reinterpret_cast<const uint4*>(static_cast<const char*>(base) + elem_off_bytes));
}

// The per-query walk shared by both forms.  Row(j0, j1, j2) gives the K / V
// slice of the window's key (j0, j1, j2) (window-relative coordinates).
template <int D, int T, class KeyRow>
__device__ __forceinline__ void attend_row(const float (&qv)[slice_elems<T>()], int W, int Wmax,
                                           const int n[3], KeyRow row, float (&acc)[slice_elems<T>()],
                                           float& m, float& l) {
  constexpr int VE = slice_elems<T>();
  constexpr int G = D / VE;
#pragma unroll
  for (int e = 0; e < VE; ++e) acc[e] = 0.f;
  m = -INFINITY;
  l = 0.f;
  int j0 = 0, j1 = 0, j2 = 0;   // position in the window (odometer, innermost last)
  for (int base = 0; base < Wmax; base += KEYS_PER_STEP) {
    uint4 ku[KEYS_PER_STEP], vu[KEYS_PER_STEP];
    bool in[KEYS_PER_STEP];
#pragma unroll
    for (int u = 0; u < KEYS_PER_STEP; ++u) {
      in[u] = base + u < W;
      if (in[u]) {
        row(j0, j1, j2, ku[u], vu[u]);
        if (++j2 == n[2]) {
          j2 = 0;
          if (++j1 == n[1]) {
            j1 = 0;
            ++j0;
          }
        }
      } else {
        ku[u] = make_uint4(0, 0, 0, 0);
        vu[u] = ku[u];
      }
    }
    float s[KEYS_PER_STEP];
#pragma unroll
    for (int u = 0; u < KEYS_PER_STEP; ++u) {
      float kf[VE];
      unpack<T>(ku[u], kf);
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < VE; ++e) dot = fmaf(qv[e], kf[e], dot);
      s[u] = dot;
    }
#pragma unroll
    for (int off = G / 2; off > 0; off >>= 1) {
#pragma unroll
      for (int u = 0; u < KEYS_PER_STEP; ++u) s[u] += __shfl_xor_sync(0xffffffffu, s[u], off);
    }
    float mb = -INFINITY;
#pragma unroll
    for (int u = 0; u < KEYS_PER_STEP; ++u) {
      if (!in[u]) s[u] = -INFINITY;
      mb = fmaxf(mb, s[u]);
    }
    const float m_new = fmaxf(m, mb);
    if (m_new == -INFINITY) continue;   // no key of this row yet (uniform in the group)
    const float alpha = exp2f(m - m_new);
    l *= alpha;
#pragma unroll
    for (int e = 0; e < VE; ++e) acc[e] *= alpha;
#pragma unroll
    for (int u = 0; u < KEYS_PER_STEP; ++u) {
      const float p = exp2f(s[u] - m_new);
      l += p;
      float vf[VE];
      unpack<T>(vu[u], vf);
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] = fmaf(p, vf[e], acc[e]);
    }
    m = m_new;
  }
}

template <int D, int T>
__device__ __forceinline__ void finish_row(const GatherLaunch& P, size_t row_off_bytes,
                                           size_t lse_index, int part,
                                           float (&acc)[slice_elems<T>()], float m, float l) {
  constexpr int VE = slice_elems<T>();
  const float inv_l = 1.f / l;
#pragma unroll
  for (int e = 0; e < VE; ++e) acc[e] *= inv_l;
  *reinterpret_cast<uint4*>(static_cast<char*>(P.out) + row_off_bytes) = pack<T>(acc);
  if (part == 0) P.lse[lse_index] = (m + log2f(l)) * 0.69314718055994530942f;
}

template <int D, int T>
__device__ __forceinline__ void load_q(const GatherLaunch& P, size_t off, float (&qv)[slice_elems<T>()]) {
  unpack<T>(load_slice(P.q, off), qv);
#pragma unroll
  for (int e = 0; e < slice_elems<T>(); ++e) qv[e] *= P.scale_log2;   // log2-domain scores
}

// Staged form.  The grid is persistent: CTA b takes query tiles b, b + grid,
// ... (numbered head-major, then row-major over the tile grid), so the CTAs
// at work at any moment hold neighbouring tiles and share their halo rows
// in L2.  A tile's rows -- its queries, and the K and V rows of its key box
// (the union of its queries' windows, itself a box) -- arrive by bulk copies
// into a stage of shared memory: one copy per run of adjacent rows (a whole
// tile of a 1-D grid is one run per tensor), completion counted in bytes on
// the stage's mbarrier.  With two stages (where they fit) the next tile
// streams in while the CTA computes the current one from the other.
struct TileGeo {
  int bh;
  int o[3], nq[3];   // first query and extent of the tile per dimension
  int lo[3], kx[3];  // first key and extent of its key box
};

__device__ __forceinline__ TileGeo tile_geo(const GatherLaunch& P, int t) {
  TileGeo tg;
  const int tiles = P.nt[0] * P.nt[1] * P.nt[2];
  tg.bh = t / tiles;
  int tix = t % tiles;
  int tc[3];
  tc[2] = tix % P.nt[2];
  tix /= P.nt[2];
  tc[1] = tix % P.nt[1];
  tc[0] = tix / P.nt[1];
  for (int d = 0; d < 3; ++d) {
    tg.o[d] = tc[d] * P.qt[d];
    tg.nq[d] = imin(P.qt[d], P.g.L[d] - tg.o[d]);
    int a, b, c, e;
    window_range(P.g.L[d], P.g.w[d], P.g.s[d], P.g.m[d], tg.o[d], a, b);
    window_range(P.g.L[d], P.g.w[d], P.g.s[d], P.g.m[d], tg.o[d] + tg.nq[d] - 1, c, e);
    tg.lo[d] = a;   // both window ends are monotone in the query coordinate
    tg.kx[d] = e - a;
  }
  return tg;
}

// Bulk copies of one box of rows (extent n, origin a in grid coordinates)
// into consecutive shared-memory rows, row-major over the box; the lanes of
// one warp share the runs.
template <int RB>
__device__ __forceinline__ void copy_box(const GatherLaunch& P, size_t head, const int a[3],
                                         const int n[3], const void* src, unsigned char* dst,
                                         uint64_t* bar, int lane) {
  const int rows = n[0] * n[1] * n[2];
  const int len = P.map.dil[2] == 1 ? n[2] : 1;   // adjacent in memory along the innermost
  for (int r = lane * len; r < rows; r += 32 * len) {
    const int r2 = r % n[2], r1 = (r / n[2]) % n[1], r0 = r / (n[2] * n[1]);
    const size_t tok = (size_t)full_token(P.map, a[0] + r0, a[1] + r1, a[2] + r2);
    ptx::bulk_load(dst + (size_t)r * RB, static_cast<const char*>(src) + (head + tok) * RB,
                   (uint32_t)(len * RB), bar);
  }
}

template <int RB>
__device__ __forceinline__ void issue_tile(const GatherLaunch& P, int t, unsigned char* stage,
                                           uint64_t* bar, TileGeo* geo, int lane) {
  const TileGeo tg = tile_geo(P, t);
  if (lane == 0) *geo = tg;   // published to the consumers by the arrive below
  const int nqt = tg.nq[0] * tg.nq[1] * tg.nq[2];
  const int rows = tg.kx[0] * tg.kx[1] * tg.kx[2];
  if (lane == 0) ptx::mbar_expect_tx(bar, (uint32_t)((nqt + 2 * rows) * RB));
  __syncwarp();
  // Testing hook: CTA 0's first tile is announced but never copied, so the
  // waits on it run out and the timeout path unwinds.
  if ((P.debug_flags & 1) && t == 0) return;
  const size_t head = (size_t)tg.bh * (size_t)P.N;
  unsigned char* sK = stage + (size_t)P.qrows * RB;
  unsigned char* sV = sK + (size_t)P.krows * RB;
  copy_box<RB>(P, head, tg.o, tg.nq, P.q, stage, bar, lane);
  copy_box<RB>(P, head, tg.lo, tg.kx, P.k, sK, bar, lane);
  copy_box<RB>(P, head, tg.lo, tg.kx, P.v, sV, bar, lane);
}

// s += q . k over the 32 elements a thread holds, for 16-bit inputs: each
// product of two 16-bit values is formed exactly and added in fp32 by one
// mixed-precision FMA, so neither operand is widened first.
template <int T>
__device__ __forceinline__ void dot_words(uint32_t qw, uint32_t kw, float& a0, float& a1) {
  if constexpr (T == G_BF16)
    asm("{\n\t.reg .b16 ql, qh, kl, kh;\n\t"
        "mov.b32 {ql, qh}, %2;\n\t"
        "mov.b32 {kl, kh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, ql, kl, %0;\n\t"
        "fma.rn.f32.bf16 %1, qh, kh, %1;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "r"(qw), "r"(kw));
  else
    asm("{\n\t.reg .b16 ql, qh, kl, kh;\n\t"
        "mov.b32 {ql, qh}, %2;\n\t"
        "mov.b32 {kl, kh}, %3;\n\t"
        "fma.rn.f32.f16 %0, ql, kl, %0;\n\t"
        "fma.rn.f32.f16 %1, qh, kh, %1;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "r"(qw), "r"(kw));
}

__device__ __forceinline__ float ex2_approx(float x) {   // 2^x, 0 at -inf
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One tile from its stage.  Each query is served by G = D / 32 threads holding
// 32 elements each, so a key costs a thread four (16-bit) or eight (fp32)
// 16-byte shared-memory reads per operand and at most two shuffles.  Scores:
// for 16-bit inputs q stays in its 16-bit form and every product is one
// mixed-precision FMA (exact product, fp32 sum; the scale is applied to the
// sum); fp32 inputs use scaled fp32 q.  Values: the fp32 accumulator as
// packed pairs, one f32x2 FMA per two elements.  Register slot k of a thread
// holds one of its slices in an order rotated per lane: rows sit a whole
// number of 128-byte lines apart (head_dim >= 64 at 16 bits), so a 16-byte
// read's bank group is its slice's, and the rotation gives the eight lanes of
// each phase of a warp-wide read eight different bank groups.  ONED: a 1-D
// grid (the two outer extents 1), whose coordinates need no division.  KPS:
// keys per online-softmax step (3 or 5, whichever wastes fewer slots on the
// window; each step costs a rescale of the accumulator).
template <int D, int T, bool ONED, int KPS>
__device__ __forceinline__ void compute_tile(const GatherLaunch& P, const TileGeo tg,
                                             const unsigned char* stage) {
  constexpr int VE = slice_elems<T>();       // elements per 16-byte slice
  constexpr int ESZ = T == G_F32 ? 4 : 2;
  constexpr int RB = D * ESZ;                // bytes per row
  constexpr int SPR = RB / 16;               // slices per row (4 .. 32)
  constexpr int E = 32;                      // elements per thread
  constexpr int S = E / VE;                  // slices per thread (4 or 8)
  constexpr int G = D / E;                   // threads per query (1, 2 or 4)
  constexpr int QPC = GATHER_THREADS / G;    // queries per round
  constexpr bool MIX = T != G_F32;
  static_assert(SPR % S == 0 && (S & (S - 1)) == 0, "slices");
  const uint4* sQ = reinterpret_cast<const uint4*>(stage);
  const uint4* sK = sQ + (size_t)P.qrows * SPR;
  const uint4* sV = sK + (size_t)P.krows * SPR;
  const Geom& g = P.g;
  const int lane = threadIdx.x % 32;
  const int part = threadIdx.x % G;
  const int rot = S == 4 ? ((lane >> 1) & 3) : (lane & 7);
  auto sl = [&](int k) { return part * S + ((k + rot) & (S - 1)); };   // slice in slot k
  const size_t head = (size_t)tg.bh * (size_t)P.N;
  const int tile_q = tg.nq[0] * tg.nq[1] * tg.nq[2];

  for (int q0 = 0; q0 < tile_q; q0 += QPC) {
    const int qi = q0 + threadIdx.x / G;
    const bool valid = qi < tile_q;
    const int qq = valid ? qi : 0;
    int c[3], wl[3], n[3];
    if constexpr (ONED) {
      c[0] = c[1] = 0;
      c[2] = tg.o[2] + qq;
      int hi;
      if (g.s[2] == 1)   // no division by the stride
        window_range(g.L[2], g.w[2], 1, g.m[2], c[2], wl[2], hi);
      else
        window_range(g.L[2], g.w[2], g.s[2], g.m[2], c[2], wl[2], hi);
      n[2] = hi - wl[2];
      wl[2] -= tg.lo[2];
      n[0] = n[1] = 1;
      wl[0] = wl[1] = 0;
    } else {
      c[2] = tg.o[2] + qq % tg.nq[2];
      c[1] = tg.o[1] + (qq / tg.nq[2]) % tg.nq[1];
      c[0] = tg.o[0] + qq / (tg.nq[2] * tg.nq[1]);
      for (int d = 0; d < 3; ++d) {
        int hi;
        window_range(g.L[d], g.w[d], g.s[d], g.m[d], c[d], wl[d], hi);
        n[d] = hi - wl[d];
        wl[d] -= tg.lo[d];     // box-relative
      }
    }
    const int W = valid ? n[0] * n[1] * n[2] : 0;
    const int Wmax = __reduce_max_sync(0xffffffffu, W);   // uniform trip count for the shuffles
    const size_t token = (size_t)full_token(P.map, c[0], c[1], c[2]);
    const size_t row_off = (head + token) * RB;

    float acc[E];
    uint32_t qw[MIX ? E / 2 : 1];
    uint64_t q2[MIX ? 1 : E / 2];
#pragma unroll
    for (int k = 0; k < S; ++k) {
      const uint4 u = sQ[qq * SPR + sl(k)];
      if constexpr (MIX) {
        qw[k * 4 + 0] = u.x;
        qw[k * 4 + 1] = u.y;
        qw[k * 4 + 2] = u.z;
        qw[k * 4 + 3] = u.w;
      } else {
        float f[VE];
        unpack<T>(u, f);
#pragma unroll
        for (int i = 0; i < VE / 2; ++i)
          q2[k * VE / 2 + i] = ptx::f2(f[2 * i] * P.scale_log2, f[2 * i + 1] * P.scale_log2);
      }
    }
#pragma unroll
    for (int i = 0; i < E; ++i) acc[i] = 0.f;
    float m = -INFINITY, l = 0.f;

    int j0 = 0, j1 = 0, j2 = 0;   // odometer over the window, innermost last
    for (int base = 0; base < Wmax; base += KPS) {
      int r[KPS];
      bool in[KPS];
      float s[KPS];
#pragma unroll
      for (int u = 0; u < KPS; ++u) {
        in[u] = base + u < W;
        r[u] = 0;
        if (in[u]) {
          if constexpr (ONED) {
            r[u] = wl[2] + j2++;
          } else {
            r[u] = ((wl[0] + j0) * tg.kx[1] + (wl[1] + j1)) * tg.kx[2] + wl[2] + j2;
            if (++j2 == n[2]) {
              j2 = 0;
              if (++j1 == n[1]) {
                j1 = 0;
                ++j0;
              }
            }
          }
        }
        if constexpr (MIX) {
          float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int k = 0; k < S; ++k) {
            const uint4 kv = sK[r[u] * SPR + sl(k)];
            dot_words<T>(qw[k * 4 + 0], kv.x, a[0], a[1]);
            dot_words<T>(qw[k * 4 + 1], kv.y, a[2], a[3]);
            dot_words<T>(qw[k * 4 + 2], kv.z, a[0], a[1]);
            dot_words<T>(qw[k * 4 + 3], kv.w, a[2], a[3]);
          }
          s[u] = ((a[0] + a[1]) + (a[2] + a[3])) * P.scale_log2;   // log2-domain score
        } else {
          uint64_t a[2] = {ptx::f2(0.f, 0.f), ptx::f2(0.f, 0.f)};
#pragma unroll
          for (int k = 0; k < S; ++k) {
            const uint4 kv = sK[r[u] * SPR + sl(k)];
            a[0] = ptx::f2_fma(q2[2 * k], ptx::f2(__uint_as_float(kv.x), __uint_as_float(kv.y)), a[0]);
            a[1] = ptx::f2_fma(q2[2 * k + 1], ptx::f2(__uint_as_float(kv.z), __uint_as_float(kv.w)), a[1]);
          }
          float x0, x1;
          ptx::f2_split(ptx::f2_add(a[0], a[1]), x0, x1);
          s[u] = x0 + x1;
        }
      }
#pragma unroll
      for (int off = G / 2; off > 0; off >>= 1) {
#pragma unroll
        for (int u = 0; u < KPS; ++u) s[u] += __shfl_xor_sync(0xffffffffu, s[u], off);
      }
      float mb = -INFINITY;
#pragma unroll
      for (int u = 0; u < KPS; ++u) {
        if (!in[u]) s[u] = -INFINITY;
        mb = fmaxf(mb, s[u]);
      }
      const float m_new = fmaxf(m, mb);
      if (m_new == -INFINITY) continue;   // no key of this row yet (uniform in the group)
      const float alpha = ex2_approx(m - m_new);
      l *= alpha;
      const uint64_t alpha2 = ptx::f2(alpha, alpha);
#pragma unroll
      for (int i = 0; i < E / 2; ++i) {
        uint64_t t = ptx::f2(acc[2 * i], acc[2 * i + 1]);
        t = ptx::f2_mul(t, alpha2);
        ptx::f2_split(t, acc[2 * i], acc[2 * i + 1]);
      }
#pragma unroll
      for (int u = 0; u < KPS; ++u) {
        const float pu = ex2_approx(s[u] - m_new);   // 0 for a masked key
        l += pu;
        if (!in[u]) continue;
        const uint64_t p2 = ptx::f2(pu, pu);
#pragma unroll
        for (int k = 0; k < S; ++k) {
          float f[VE];
          unpack<T>(sV[r[u] * SPR + sl(k)], f);
#pragma unroll
          for (int i = 0; i < VE / 2; ++i) {
            float& x0 = acc[k * VE + 2 * i];
            float& x1 = acc[k * VE + 2 * i + 1];
            uint64_t t = ptx::f2(x0, x1);
            t = ptx::f2_fma(p2, ptx::f2(f[2 * i], f[2 * i + 1]), t);
            ptx::f2_split(t, x0, x1);
          }
        }
      }
      m = m_new;
    }

    if (valid) {
      float inv_l, lg;
      asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv_l) : "f"(l));
      asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(l));
#pragma unroll
      for (int k = 0; k < S; ++k) {
        float f[VE];
#pragma unroll
        for (int i = 0; i < VE; ++i) f[i] = acc[k * VE + i] * inv_l;
        *reinterpret_cast<uint4*>(static_cast<char*>(P.out) + row_off + (size_t)sl(k) * 16) =
            pack<T>(f);
      }
      if (part == 0) P.lse[head + token] = (m + lg) * 0.69314718055994530942f;
    }
  }
}

// The staged form's CTA loop.  There is no CTA-wide barrier per tile: every
// warp waits for a tile's stage to fill, computes its share of the tile and
// counts itself done with the stage; the warp that finishes the stage last
// refills it with the tile `nst` steps ahead.  With two stages a warp can run
// a whole tile ahead of the slowest one.
template <int D, int T, bool ONED, int KPS>
__global__ void __launch_bounds__(GATHER_THREADS, 2) gather_staged_kernel(const GatherLaunch P) {
  constexpr int RB = D * (T == G_F32 ? 4 : 2);
  constexpr int NWARPS = GATHER_THREADS / 32;
  extern __shared__ __align__(128) unsigned char smem[];
  // Header: a full barrier, a done count, an issue count and the geometry per stage.
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 16);
  int* done = reinterpret_cast<int*>(smem + 20);
  int* issued = reinterpret_cast<int*>(smem + 28);
  TileGeo* geo = reinterpret_cast<TileGeo*>(smem + 40);
  static_assert(40 + 2 * sizeof(TileGeo) <= GATHER_SMEM_HEADER, "header");
  unsigned char* stage0 = smem + GATHER_SMEM_HEADER;
  const int stage_bytes = (P.qrows + 2 * P.krows) * RB;
  const int nst = P.nstages;   // 1 or 2
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int total = P.BH * P.nt[0] * P.nt[1] * P.nt[2];   // the host keeps it below 2^30
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&full[s], 1);
      done[s] = 0;
      issued[s] = 0;
    }
    *abort_flag = *reinterpret_cast<volatile int*>(P.status) != 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  ptx::WaitCtl ctl;
  ctl.abort = abort_flag;
  ctl.status = P.status;
  ctl.timeout_ns = (uint64_t)P.timeout_ns;

  auto issue = [&](int tt, int s) {   // one warp, all lanes
    issue_tile<RB>(P, tt, stage0 + s * stage_bytes, &full[s], &geo[s], lane);
    if (lane == 0) ++issued[s];
  };
  if (warp == 0)
    for (int s = 0; s < nst; ++s)
      if (blockIdx.x + s * gridDim.x < (unsigned)total) issue(blockIdx.x + s * gridDim.x, s);

  int i = 0;
  for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
    const int st = nst == 2 ? (i & 1) : 0;
    const int par = (nst == 2 ? i >> 1 : i) & 1;
    if (!__all_sync(0xffffffffu, ptx::wait(&full[st], par, ctl))) break;
    compute_tile<D, T, ONED, KPS>(P, geo[st], stage0 + st * stage_bytes);
    // Release the stage; the last warp out refills it.
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      __threadfence_block();   // this warp's reads of the stage before its count
      last = atomicAdd(&done[st], 1) == NWARPS - 1;
    }
    if (__shfl_sync(0xffffffffu, last, 0)) {
      if (lane == 0) done[st] = 0;
      const int tn = t + nst * gridDim.x;
      if (tn < total) {
        __threadfence_block();
        // Generic-proxy reads of the stage are ordered before the bulk copies' writes.
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(tn, st);
      }
    }
  }
  // Every warp is out of its loop (a failed wait ends it early): copies still
  // in flight land before the CTA's shared memory goes away.
  __syncthreads();
  if (threadIdx.x == 0)
    for (int s = 0; s < nst; ++s)
      if (issued[s] > 0) ptx::wait_drain(&full[s], (issued[s] - 1) & 1, ctl);
}

// Direct form: no staging (a wide window); one query per thread group, every
// K / V slice read from global memory (L1 / L2 hits after the first touch).
template <int D, int T>
__global__ void __launch_bounds__(GATHER_THREADS) gather_direct_kernel(const GatherLaunch P) {
  constexpr int VE = slice_elems<T>();
  constexpr int G = D / VE;
  constexpr int QPC = GATHER_THREADS / G;
  constexpr int ESZ = T == G_F32 ? 4 : 2;
  static_assert(G >= 4 && G <= 32 && (G & (G - 1)) == 0, "group size");

  const Geom& g = P.g;
  const long long nsub = (long long)g.L[0] * g.L[1] * g.L[2];   // this grid's tokens per head
  const long long rows = (long long)P.BH * nsub;
  const long long row = (long long)blockIdx.x * QPC + threadIdx.x / G;
  const int part = threadIdx.x % G;
  const bool valid = row < rows;
  const long long r = valid ? row : 0;
  const size_t head = (size_t)(r / nsub) * (size_t)P.N;
  const int sub = (int)(r % nsub);
  int c[3];
  c[2] = sub % g.L[2];
  c[1] = (sub / g.L[2]) % g.L[1];
  c[0] = sub / (g.L[2] * g.L[1]);
  const size_t token = (size_t)full_token(P.map, c[0], c[1], c[2]);
  int lo[3], n[3];
  for (int d = 0; d < 3; ++d) {
    int hi;
    window_range(g.L[d], g.w[d], g.s[d], g.m[d], c[d], lo[d], hi);
    n[d] = hi - lo[d];
  }
  const int W = valid ? n[0] * n[1] * n[2] : 0;
  const int Wmax = __reduce_max_sync(0xffffffffu, W);   // all 32 lanes run the shuffles
  const size_t slice = (size_t)part * 16;
  const size_t row_off = (head + token) * D * ESZ + slice;
  float qv[VE], acc[VE], m, l;
  load_q<D, T>(P, row_off, qv);
  attend_row<D, T>(qv, W, Wmax, n,
                   [&](int j0, int j1, int j2, uint4& ku, uint4& vu) {
                     const size_t kt = (size_t)full_token(P.map, lo[0] + j0, lo[1] + j1, lo[2] + j2);
                     const size_t off = (head + kt) * D * ESZ + slice;
                     ku = load_slice(P.k, off);
                     vu = load_slice(P.v, off);
                   },
                   acc, m, l);
  if (valid) finish_row<D, T>(P, row_off, head + token, part, acc, m, l);
}

template <int D, int T>
cudaError_t launch_dt(const GatherLaunch& L, cudaStream_t stream) {
  if (L.qt[0] > 0) {
    const long long tiles = (long long)L.BH * L.nt[0] * L.nt[1] * L.nt[2];
    if (tiles <= 0 || tiles >= (1LL << 30)) return cudaErrorInvalidConfiguration;
    const int esz = T == G_F32 ? 4 : 2;
    if (L.qrows <= 0 || L.krows <= 0 || (L.nstages != 1 && L.nstages != 2) ||
        L.smem_bytes > GATHER_SMEM_MAX ||
        L.smem_bytes != gather_smem_bytes(L.qrows, L.krows, D, esz, L.nstages) || !L.status)
      return cudaErrorInvalidValue;
    const bool oned = L.g.L[0] == 1 && L.g.L[1] == 1;
    const int wk = L.g.w[0] * L.g.w[1] * L.g.w[2];   // keys of a whole window
    const bool k5 = (wk + 4) / 5 * 5 - wk < (wk + 2) / 3 * 3 - wk;   // fewer wasted slots
    using Kern = void (*)(GatherLaunch);
    const Kern kerns[4] = {gather_staged_kernel<D, T, false, 3>, gather_staged_kernel<D, T, false, 5>,
                           gather_staged_kernel<D, T, true, 3>, gather_staged_kernel<D, T, true, 5>};
    const Kern kern = kerns[(oned ? 2 : 0) + (k5 ? 1 : 0)];
    // Per device: the shared-memory opt-in, the SM count, and the resident
    // CTAs per SM at the last footprint launched.
    static int attr_done[64] = {0}, sms[64] = {0}, occ_smem[64] = {0}, occ[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
      for (const Kern f : kerns) {
        e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, GATHER_SMEM_MAX);
        if (e != cudaSuccess) return e;
      }
      e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
      attr_done[dev] = 1;
    }
    if (occ_smem[dev] != L.smem_bytes) {
      int nb = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kerns[0], GATHER_THREADS,
                                                        L.smem_bytes);
      if (e != cudaSuccess) return e;
      occ[dev] = nb > 0 ? nb : 1;
      occ_smem[dev] = L.smem_bytes;
    }
    const long long grid = std::min(tiles, (long long)sms[dev] * occ[dev]);
    kern<<<(unsigned)grid, GATHER_THREADS, L.smem_bytes, stream>>>(L);
  } else {
    const long long qpc = GATHER_THREADS / (D / slice_elems<T>());
    const long long rows = (long long)L.BH * L.g.L[0] * L.g.L[1] * L.g.L[2];
    const long long blocks = (rows + qpc - 1) / qpc;
    if (blocks <= 0 || blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    gather_direct_kernel<D, T><<<(unsigned)blocks, GATHER_THREADS, 0, stream>>>(L);
  }
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const GatherLaunch& L, cudaStream_t stream) {
  switch (L.dtype) {
    case G_F32: return launch_dt<D, G_F32>(L, stream);
    case G_BF16: return launch_dt<D, G_BF16>(L, stream);
    case G_F16: return launch_dt<D, G_F16>(L, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

cudaError_t launch_gather(const GatherLaunch& L, cudaStream_t stream) {
  switch (L.D) {
    case 32: return launch_d<32>(L, stream);
    case 64: return launch_d<64>(L, stream);
    case 128: return launch_d<128>(L, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace na
