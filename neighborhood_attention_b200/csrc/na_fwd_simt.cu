// CUDA-core (SIMT) forward kernel: fp32, bf16 and f16 inputs, any window / stride /
// grid, head_dim 32, 64 or 128.  It serves the fp32 path (no exact fp32
// tensor-core contraction exists) and shapes the tensor-core kernel does not
// take.  Per query block it walks the key box of the block's windows in
// chunks of 32 keys staged in shared memory, skips EMPTY chunks, masks only
// PARTIAL ones, and keeps an online softmax per query row (the restricted
// softmax of "pi-Attention", section 3.1 eqs. (1)-(3) and section 3.2, with
// the tile-by-tile on-chip accumulation that page's section 3.4 describes).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "na_internal.h"

namespace na {
namespace {

constexpr int SIMT_THREADS = 128;
constexpr int SIMT_CHUNK = 32;

// Element types, numbered as na_dtype.
enum : int { ELEM_F32 = 0, ELEM_BF16 = 1, ELEM_F16 = 2 };

template <int T>
__device__ __forceinline__ float load_elem(const void* p, size_t i) {
  if constexpr (T == ELEM_BF16) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  } else if constexpr (T == ELEM_F16) {
    return __half2float(reinterpret_cast<const __half*>(p)[i]);
  } else {
    return reinterpret_cast<const float*>(p)[i];
  }
}

template <int D, int T>
__global__ void __launch_bounds__(SIMT_THREADS) simt_fwd_kernel(const SimtLaunch P) {
  constexpr int TPQ = D / 32;               // threads per query row
  constexpr int QPB = SIMT_THREADS / TPQ;   // queries per block
  __shared__ float Ks[SIMT_CHUNK * D];      // [key][c][g]: channel g*32 + c
  __shared__ float Vs[SIMT_CHUNK * D];

  const Geom& g = P.g;
  const QTiling& t = P.t;
  const int bh = blockIdx.x / t.nblocks;
  const int blk = blockIdx.x % t.nblocks;
  BlockInfo bi;
  block_info(g, t, blk, bi);
  if (!bi.exists) return;
  ChunkGrid cg;
  chunk_grid_for(&bi, 1, P.kb, cg);

  const int tid = threadIdx.x;
  const int qi = tid / TPQ, gg = tid % TPQ;
  int r[3];
  r[2] = qi % t.qb[2];
  r[1] = (qi / t.qb[2]) % t.qb[1];
  r[0] = qi / (t.qb[2] * t.qb[1]);
  int gc[3], wlo[3], wn[3];  // this query's window: [wlo, wlo + wn) per dimension
  bool valid = qi < QPB;
  for (int d = 0; d < 3; ++d) {
    gc[d] = bi.o[d] + r[d];
    if (gc[d] >= g.L[d]) valid = false;
    int whi;
    window_range(g.L[d], g.w[d], g.s[d], g.m[d], imin(gc[d], g.L[d] - 1), wlo[d], whi);
    wn[d] = whi - wlo[d];
  }
  const long long token = full_token(P.map, gc[0], gc[1], gc[2]);
  const size_t head_off = (size_t)bh * (size_t)P.N * D;

  float qr[32], acc[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    qr[c] = valid ? load_elem<T>(P.q, head_off + (size_t)token * D + gg * 32 + c) : 0.f;
    acc[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  for (int c = 0; c < cg.total; ++c) {
    int a[3];
    chunk_origin(cg, P.kb, c, a);
    const int st = chunk_status(bi, a, P.kb);
    if (st == CHUNK_EMPTY) continue;  // uniform across the block
    __syncthreads();
    for (int e = tid; e < SIMT_CHUNK * D; e += SIMT_THREADS) {
      const int key = e / D, ch = e % D;
      const int k2 = key % P.kb[2], k1 = (key / P.kb[2]) % P.kb[1], k0 = key / (P.kb[2] * P.kb[1]);
      const int x0 = a[0] + k0, x1 = a[1] + k1, x2 = a[2] + k2;
      float kv = 0.f, vv = 0.f;
      if (x0 < g.L[0] && x1 < g.L[1] && x2 < g.L[2]) {
        const size_t off = head_off + (size_t)full_token(P.map, x0, x1, x2) * D + ch;
        kv = load_elem<T>(P.k, off);
        vv = load_elem<T>(P.v, off);
      }
      const int si = key * D + (ch % 32) * TPQ + ch / 32;
      Ks[si] = kv;
      Vs[si] = vv;
    }
    __syncthreads();

    float s[SIMT_CHUNK];
    float mx = -INFINITY;
#pragma unroll
    for (int kk = 0; kk < SIMT_CHUNK; ++kk) {
      float dot = 0.f;
#pragma unroll
      for (int cc = 0; cc < 32; ++cc) dot = fmaf(qr[cc], Ks[kk * D + cc * TPQ + gg], dot);
#pragma unroll
      for (int off = 1; off < TPQ; off <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      float sv = dot * P.scale_log2;
      if (st == CHUNK_PARTIAL) {
        const int k2 = kk % P.kb[2], k1 = (kk / P.kb[2]) % P.kb[1], k0 = kk / (P.kb[2] * P.kb[1]);
        const bool in = (unsigned)(a[0] + k0 - wlo[0]) < (unsigned)wn[0] &&
                        (unsigned)(a[1] + k1 - wlo[1]) < (unsigned)wn[1] &&
                        (unsigned)(a[2] + k2 - wlo[2]) < (unsigned)wn[2];
        if (!in) sv = -INFINITY;
      }
      s[kk] = sv;
      mx = fmaxf(mx, sv);
    }
    const float m_new = fmaxf(m, mx);
    const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = exp2f(m - m_use);
    l *= alpha;
#pragma unroll
    for (int cc = 0; cc < 32; ++cc) acc[cc] *= alpha;
#pragma unroll
    for (int kk = 0; kk < SIMT_CHUNK; ++kk) {
      const float p = exp2f(s[kk] - m_use);
      l += p;
#pragma unroll
      for (int cc = 0; cc < 32; ++cc) acc[cc] = fmaf(p, Vs[kk * D + cc * TPQ + gg], acc[cc]);
    }
    m = m_new;
  }

  if (!valid) return;
  const float inv_l = 1.f / l;
  const size_t obase = head_off + (size_t)token * D + gg * 32;
  if constexpr (T == ELEM_BF16) {
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(P.out) + obase;
#pragma unroll
    for (int cc = 0; cc < 32; ++cc) o[cc] = __float2bfloat16_rn(acc[cc] * inv_l);
  } else if constexpr (T == ELEM_F16) {
    __half* o = reinterpret_cast<__half*>(P.out) + obase;
#pragma unroll
    for (int cc = 0; cc < 32; ++cc) o[cc] = __float2half_rn(acc[cc] * inv_l);
  } else {
    float* o = reinterpret_cast<float*>(P.out) + obase;
#pragma unroll
    for (int cc = 0; cc < 32; ++cc) o[cc] = acc[cc] * inv_l;
  }
  if (gg == 0) P.lse[(size_t)bh * P.N + token] = (m + log2f(l)) * 0.69314718055994530942f;
}

template <int D>
cudaError_t launch_d(const SimtLaunch& L, cudaStream_t stream) {
  const long long blocks = (long long)L.BH * L.t.nblocks;
  if (blocks <= 0 || blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  switch (L.dtype) {
    case ELEM_F32:
      simt_fwd_kernel<D, ELEM_F32><<<(unsigned)blocks, SIMT_THREADS, 0, stream>>>(L);
      break;
    case ELEM_BF16:
      simt_fwd_kernel<D, ELEM_BF16><<<(unsigned)blocks, SIMT_THREADS, 0, stream>>>(L);
      break;
    case ELEM_F16:
      simt_fwd_kernel<D, ELEM_F16><<<(unsigned)blocks, SIMT_THREADS, 0, stream>>>(L);
      break;
    default:
      return cudaErrorNotSupported;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_simt(const SimtLaunch& L, cudaStream_t stream) {
  switch (L.D) {
    case 32: return launch_d<32>(L, stream);
    case 64: return launch_d<64>(L, stream);
    case 128: return launch_d<128>(L, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace na
