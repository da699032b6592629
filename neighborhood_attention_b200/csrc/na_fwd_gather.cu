// Window-gather forward kernel (CUDA cores) for narrow windows: fp32, bf16 or
// f16 inputs, head_dim 32, 64 or 128, any grid, window, stride and window mode.
//
// With a handful of keys per query the forward is bound by HBM traffic (q, k,
// v read and out written once: a few FLOPs per byte), so this kernel moves
// bytes, not tiles of scores.  A CTA owns a box of queries (a tile of the
// grid).  It first stages the K and V rows of the tile's key box -- the union
// of its queries' windows, itself a box -- into shared memory with 16-byte
// asynchronous copies, coalesced along the grid's innermost dimension, each
// row fetched once per tile.  Then each query is served by a group of G
// consecutive threads, each holding one 16-byte slice of the head dimension:
// the group walks the query's own window key by key (the product of its
// per-dimension ranges, cut windows included) over the staged rows, reduces
// the partial dot products with shuffles and keeps an online softmax in the
// log2 domain.  The output slice goes out as one 16-byte store per thread,
// coalesced across the group and across consecutive queries.  When even a
// one-query tile's key box would not fit the shared-memory budget (a wide
// window), the same walk reads K and V straight from global memory instead.
//
// The arithmetic is the restricted softmax attention of "pi-Attention",
// section 3.1 eqs. (1)-(3) with the neighbourhood of section 3.2 (eq. (5) for
// cut windows); the lse output is the log of eq. (2)'s denominator.
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

// Staged form: one CTA per query tile, the tile's key box in shared memory.
// Each query is served by G = D / 32 threads holding 32 elements each (q and
// the output accumulator as packed f32x2 pairs), so a key costs a thread four
// (bf16 / f16) or eight (fp32) 16-byte shared-memory reads per operand and at
// most two shuffles.  Row r's 16-byte slice s sits at slot s ^ (r mod slots):
// the threads of a warp read different rows at the same logical slice, and
// the swizzle spreads them over all banks.
template <int D, int T>
__global__ void __launch_bounds__(GATHER_THREADS) gather_tile_kernel(const GatherLaunch P) {
  constexpr int VE = slice_elems<T>();       // elements per 16-byte slice
  constexpr int ESZ = T == G_F32 ? 4 : 2;
  constexpr int SPR = D * ESZ / 16;          // slices per row (4 .. 32)
  constexpr int E = 32;                      // elements per thread
  constexpr int S = E / VE;                  // slices per thread
  constexpr int G = D / E;                   // threads per query (1, 2 or 4)
  constexpr int QPC = GATHER_THREADS / G;    // queries per round
  constexpr int KPS = 2;                     // keys per online-softmax step
  static_assert(SPR % S == 0 && (SPR & (SPR - 1)) == 0, "slices");
  extern __shared__ uint4 smem[];

  const Geom& g = P.g;
  const int tiles = P.nt[0] * P.nt[1] * P.nt[2];
  const int bh = blockIdx.x / tiles;
  int tix = blockIdx.x % tiles;
  int o[3], nq[3], lo[3], kx[3];
  {
    int tc[3];
    tc[2] = tix % P.nt[2];
    tix /= P.nt[2];
    tc[1] = tix % P.nt[1];
    tc[0] = tix / P.nt[1];
    for (int d = 0; d < 3; ++d) {
      o[d] = tc[d] * P.qt[d];
      nq[d] = imin(P.qt[d], g.L[d] - o[d]);
      int a, b, c, e;
      window_range(g.L[d], g.w[d], g.s[d], g.m[d], o[d], a, b);
      window_range(g.L[d], g.w[d], g.s[d], g.m[d], o[d] + nq[d] - 1, c, e);
      lo[d] = a;          // both window ends are monotone in the query coordinate
      kx[d] = e - a;
    }
  }
  const int rows = kx[0] * kx[1] * kx[2];
  uint4* sK = smem;
  uint4* sV = smem + (size_t)rows * SPR;
  const size_t head = (size_t)bh * (size_t)P.N;

  // Stage the key box: slice sl of row r of K and V, 16 bytes per copy.
  for (int i = threadIdx.x; i < rows * SPR; i += GATHER_THREADS) {
    const int r = i / SPR, sl = i % SPR;
    const int r2 = r % kx[2], r1 = (r / kx[2]) % kx[1], r0 = r / (kx[2] * kx[1]);
    const size_t tok = (size_t)full_token(P.map, lo[0] + r0, lo[1] + r1, lo[2] + r2);
    const size_t off = (head + tok) * D * ESZ + (size_t)sl * 16;
    const int slot = r * SPR + (sl ^ (r & (SPR - 1)));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(sK + slot))),
                 "l"(static_cast<const char*>(P.k) + off)
                 : "memory");
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(sV + slot))),
                 "l"(static_cast<const char*>(P.v) + off)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  const int part = threadIdx.x % G;
  const int tile_q = nq[0] * nq[1] * nq[2];
  for (int q0 = 0; q0 < tile_q; q0 += QPC) {
    const int qi = q0 + threadIdx.x / G;
    const bool valid = qi < tile_q;
    const int qq = valid ? qi : 0;
    int c[3];
    c[2] = o[2] + qq % nq[2];
    c[1] = o[1] + (qq / nq[2]) % nq[1];
    c[0] = o[0] + qq / (nq[2] * nq[1]);
    int wl[3], n[3];
    for (int d = 0; d < 3; ++d) {
      int hi;
      window_range(g.L[d], g.w[d], g.s[d], g.m[d], c[d], wl[d], hi);
      n[d] = hi - wl[d];
      wl[d] -= lo[d];     // box-relative
    }
    const int W = valid ? n[0] * n[1] * n[2] : 0;
    const int Wmax = __reduce_max_sync(0xffffffffu, W);   // uniform trip count for the shuffles
    const size_t token = (size_t)full_token(P.map, c[0], c[1], c[2]);
    const size_t row_off = (head + token) * D * ESZ + (size_t)part * S * 16;

    uint64_t q2[E / 2], acc2[E / 2];
#pragma unroll
    for (int k = 0; k < S; ++k) {
      float f[VE];
      unpack<T>(load_slice(P.q, row_off + (size_t)k * 16), f);
#pragma unroll
      for (int i = 0; i < VE / 2; ++i)
        q2[k * VE / 2 + i] = ptx::f2(f[2 * i] * P.scale_log2, f[2 * i + 1] * P.scale_log2);
    }
#pragma unroll
    for (int i = 0; i < E / 2; ++i) acc2[i] = ptx::f2(0.f, 0.f);
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
          r[u] = ((wl[0] + j0) * kx[1] + (wl[1] + j1)) * kx[2] + wl[2] + j2;
          if (++j2 == n[2]) {
            j2 = 0;
            if (++j1 == n[1]) {
              j1 = 0;
              ++j0;
            }
          }
        }
        uint64_t a[4] = {ptx::f2(0.f, 0.f), ptx::f2(0.f, 0.f), ptx::f2(0.f, 0.f),
                         ptx::f2(0.f, 0.f)};
#pragma unroll
        for (int k = 0; k < S; ++k) {
          const int sl = part * S + k;
          float f[VE];
          unpack<T>(sK[r[u] * SPR + (sl ^ (r[u] & (SPR - 1)))], f);
#pragma unroll
          for (int i = 0; i < VE / 2; ++i) {
            const int j = k * VE / 2 + i;
            a[j & 3] = ptx::f2_fma(q2[j], ptx::f2(f[2 * i], f[2 * i + 1]), a[j & 3]);
          }
        }
        const uint64_t a01 = ptx::f2_add(a[0], a[1]), a23 = ptx::f2_add(a[2], a[3]);
        float x0, x1;
        ptx::f2_split(ptx::f2_add(a01, a23), x0, x1);
        s[u] = x0 + x1;
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
      const float alpha = exp2f(m - m_new);
      l *= alpha;
      const uint64_t alpha2 = ptx::f2(alpha, alpha);
#pragma unroll
      for (int i = 0; i < E / 2; ++i) acc2[i] = ptx::f2_mul(acc2[i], alpha2);
#pragma unroll
      for (int u = 0; u < KPS; ++u) {
        const float pu = exp2f(s[u] - m_new);   // 0 for a masked key
        l += pu;
        if (!in[u]) continue;
        const uint64_t p2 = ptx::f2(pu, pu);
#pragma unroll
        for (int k = 0; k < S; ++k) {
          const int sl = part * S + k;
          float f[VE];
          unpack<T>(sV[r[u] * SPR + (sl ^ (r[u] & (SPR - 1)))], f);
#pragma unroll
          for (int i = 0; i < VE / 2; ++i) {
            const int j = k * VE / 2 + i;
            acc2[j] = ptx::f2_fma(p2, ptx::f2(f[2 * i], f[2 * i + 1]), acc2[j]);
          }
        }
      }
      m = m_new;
    }

    if (valid) {
      const float inv_l = 1.f / l;
#pragma unroll
      for (int k = 0; k < S; ++k) {
        float f[VE];
#pragma unroll
        for (int i = 0; i < VE / 2; ++i) {
          ptx::f2_split(acc2[k * VE / 2 + i], f[2 * i], f[2 * i + 1]);
          f[2 * i] *= inv_l;
          f[2 * i + 1] *= inv_l;
        }
        *reinterpret_cast<uint4*>(static_cast<char*>(P.out) + row_off + (size_t)k * 16) =
            pack<T>(f);
      }
      if (part == 0) P.lse[head + token] = (m + log2f(l)) * 0.69314718055994530942f;
    }
  }
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
    const long long blocks = (long long)L.BH * L.nt[0] * L.nt[1] * L.nt[2];
    if (blocks <= 0 || blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (L.smem_bytes <= 0 || L.smem_bytes > GATHER_SMEM_BUDGET) return cudaErrorInvalidValue;
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
      const cudaError_t e = cudaFuncSetAttribute(
          gather_tile_kernel<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, GATHER_SMEM_BUDGET);
      if (e != cudaSuccess) return e;
      attr_done[dev] = 1;
    }
    gather_tile_kernel<D, T><<<(unsigned)blocks, GATHER_THREADS, L.smem_bytes, stream>>>(L);
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
