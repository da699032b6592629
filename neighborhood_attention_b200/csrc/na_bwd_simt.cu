// CUDA-core (SIMT) backward kernels: the gradients dQ, dK, dV of the forward
// pass for an upstream gradient dO, with fp32 arithmetic on fp32, bf16 or f16
// inputs, any window / stride / mode / grid, head_dim 32, 64 or 128.
//
// The forward's softmax weights are recomputed from its per-row log-sum-exp:
//   P_ij  = exp(scale <q_i, k_j> - lse_i)          (j in the window W(i))
//   D_i   = <dO_i, out_i>                           (row_delta_kernel)
//   dZ_ij = P_ij (<dO_i, v_j> - D_i)
//   dQ_i  = scale sum_j dZ_ij k_j                   (bwd_dq_kernel, per query block)
//   dK_j  = scale sum_{i: j in W(i)} dZ_ij q_i,
//   dV_j  = sum_{i: j in W(i)} P_ij dO_i            (bwd_dkdv_kernel, per key block)
// -- the vector-Jacobian product of the restricted softmax of "pi-Attention",
// section 3.1 eqs. (1)-(3) with section 3.2's neighbourhood.  Every output row
// is written once by one CTA: no atomics, deterministic.
//
// A key j belongs to the windows of a box of queries: per dimension both
// window ends are non-decreasing in the query coordinate, so the queries whose
// window holds some key of a key block form the range [I0, I1) with
// I0 = the first query whose window ends after the block's first key and
// I1 = one past the last query whose window starts before the block's end.
// The dK/dV kernel walks that box in query chunks, skipping chunks whose
// windows miss the key block and masking only where some pair is outside.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "na_internal.h"

namespace na {
namespace {

constexpr int BWD_THREADS = 128;
constexpr int BWD_CHUNK = 32;   // keys (dQ) or queries (dK/dV) staged per step
enum : int { ELEM_F32 = 0, ELEM_BF16 = 1, ELEM_F16 = 2 };
constexpr float LOG2E = 1.4426950408889634f;

template <int T>
__device__ __forceinline__ float ld(const void* p, size_t i) {
  if constexpr (T == ELEM_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  else if constexpr (T == ELEM_F16) return __half2float(reinterpret_cast<const __half*>(p)[i]);
  else return reinterpret_cast<const float*>(p)[i];
}
template <int T>
__device__ __forceinline__ void st(void* p, size_t i, float x) {
  if constexpr (T == ELEM_BF16) reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
  else if constexpr (T == ELEM_F16) reinterpret_cast<__half*>(p)[i] = __float2half_rn(x);
  else reinterpret_cast<float*>(p)[i] = x;
}

// D_i = <dO_i, out_i>, one row per 32-thread group.
template <int T>
__global__ void row_delta_kernel(const BwdLaunch P) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= (long long)P.BH * P.N) return;
  float acc = 0.f;
  for (int c = lane; c < P.D; c += 32)
    acc = fmaf(ld<T>(P.dout, (size_t)row * P.D + c), ld<T>(P.out, (size_t)row * P.D + c), acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) P.delta[row] = acc;
}

// Block coordinates of row r (row-major over the block box).
__device__ __forceinline__ void box_coord(const int o[3], const int qb[3], int r, int g[3]) {
  g[2] = o[2] + r % qb[2];
  g[1] = o[1] + (r / qb[2]) % qb[1];
  g[0] = o[0] + r / (qb[2] * qb[1]);
}

// ------------------------------------------------------------------ dQ --
template <int D, int T>
__global__ void __launch_bounds__(BWD_THREADS) bwd_dq_kernel(const BwdLaunch P) {
  constexpr int TPQ = D / 32;                // threads per query row
  constexpr int QPB = BWD_THREADS / TPQ;     // queries per block
  __shared__ float Ks[BWD_CHUNK * D];        // [key][c][g]: channel g*32 + c
  __shared__ float Vs[BWD_CHUNK * D];
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
  box_coord(bi.o, t.qb, qi, r);
  int wlo[3], wn[3];
  bool valid = qi < QPB;
  for (int d = 0; d < 3; ++d) {
    if (r[d] >= g.L[d]) valid = false;
    int whi;
    window_range(g.L[d], g.w[d], g.s[d], g.m[d], imin(r[d], g.L[d] - 1), wlo[d], whi);
    wn[d] = whi - wlo[d];
  }
  const long long token = full_token(P.map, r[0], r[1], r[2]);
  const size_t head = (size_t)bh * (size_t)P.N * D;
  const size_t rowoff = head + (size_t)(valid ? token : 0) * D + gg * 32;
  float qr[32], dor[32], dq[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    qr[c] = valid ? ld<T>(P.q, rowoff + c) : 0.f;
    dor[c] = valid ? ld<T>(P.dout, rowoff + c) : 0.f;
    dq[c] = 0.f;
  }
  const float lse2 = valid ? P.lse[(size_t)bh * P.N + token] * LOG2E : 0.f;
  const float Di = valid ? P.delta[(size_t)bh * P.N + token] : 0.f;

  for (int c = 0; c < cg.total; ++c) {
    int a[3];
    chunk_origin(cg, P.kb, c, a);
    const int stc = chunk_status(bi, a, P.kb);
    if (stc == CHUNK_EMPTY) continue;  // uniform across the block
    __syncthreads();
    for (int e = tid; e < BWD_CHUNK * D; e += BWD_THREADS) {
      const int key = e / D, ch = e % D;
      const int k2 = key % P.kb[2], k1 = (key / P.kb[2]) % P.kb[1], k0 = key / (P.kb[2] * P.kb[1]);
      const int x0 = a[0] + k0, x1 = a[1] + k1, x2 = a[2] + k2;
      float kv = 0.f, vv = 0.f;
      if (x0 < g.L[0] && x1 < g.L[1] && x2 < g.L[2]) {
        const size_t off = head + (size_t)full_token(P.map, x0, x1, x2) * D + ch;
        kv = ld<T>(P.k, off);
        vv = ld<T>(P.v, off);
      }
      const int si = key * D + (ch % 32) * TPQ + ch / 32;
      Ks[si] = kv;
      Vs[si] = vv;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < BWD_CHUNK; ++kk) {
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int cc = 0; cc < 32; ++cc) {
        s = fmaf(qr[cc], Ks[kk * D + cc * TPQ + gg], s);
        dp = fmaf(dor[cc], Vs[kk * D + cc * TPQ + gg], dp);
      }
#pragma unroll
      for (int off = 1; off < TPQ; off <<= 1) {
        s += __shfl_xor_sync(0xffffffffu, s, off);
        dp += __shfl_xor_sync(0xffffffffu, dp, off);
      }
      bool in = valid;
      if (stc == CHUNK_PARTIAL) {
        const int k2 = kk % P.kb[2], k1 = (kk / P.kb[2]) % P.kb[1], k0 = kk / (P.kb[2] * P.kb[1]);
        in = in && (unsigned)(a[0] + k0 - wlo[0]) < (unsigned)wn[0] &&
             (unsigned)(a[1] + k1 - wlo[1]) < (unsigned)wn[1] &&
             (unsigned)(a[2] + k2 - wlo[2]) < (unsigned)wn[2];
      }
      const float p = in ? exp2f(s * P.scale_log2 - lse2) : 0.f;
      const float dz = p * (dp - Di);
#pragma unroll
      for (int cc = 0; cc < 32; ++cc) dq[cc] = fmaf(dz, Ks[kk * D + cc * TPQ + gg], dq[cc]);
    }
  }
  if (!valid) return;
  const size_t obase = head + (size_t)token * D + gg * 32;
#pragma unroll
  for (int cc = 0; cc < 32; ++cc) st<T>(P.dq, obase + cc, dq[cc] * P.scale);
}

// ---------------------------------------------------------------- dK dV --
// First index i in [0, L) with f(i) true for a predicate that is false then
// true as i grows (L if never true).
template <class F>
__device__ __forceinline__ int first_true(int L, F f) {
  int lo = 0, hi = L;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (f(mid)) hi = mid; else lo = mid + 1;
  }
  return lo;
}

template <int D, int T>
__global__ void __launch_bounds__(BWD_THREADS) bwd_dkdv_kernel(const BwdLaunch P) {
  constexpr int TPK = D / 32;                // threads per key row
  constexpr int KPB = BWD_THREADS / TPK;     // keys per block
  __shared__ float Qs[BWD_CHUNK * D];        // [query][c][g]
  __shared__ float Os[BWD_CHUNK * D];        // dO, same layout
  __shared__ float Ls[BWD_CHUNK], Dd[BWD_CHUNK];
  __shared__ int Wl[BWD_CHUNK][3], Wh[BWD_CHUNK][3];
  __shared__ int Qv[BWD_CHUNK];
  const Geom& g = P.g;
  const QTiling& t = P.t;          // key blocks use the query tiling's shapes
  const int bh = blockIdx.x / t.nblocks;
  const int blk = blockIdx.x % t.nblocks;
  BlockInfo kbk;                   // only origin / extent are used: the key block box
  block_info(g, t, blk, kbk);
  if (!kbk.exists) return;

  // Query box whose windows can hold keys of this block, per dimension.
  int I0[3], I1[3];
  for (int d = 0; d < 3; ++d) {
    const int L = g.L[d], w = g.w[d], s = g.s[d], m = g.m[d];
    const int k0 = kbk.o[d], k1 = kbk.o[d] + kbk.n[d];   // keys [k0, k1)
    I0[d] = first_true(L, [&](int i) { int lo, hi; window_range(L, w, s, m, i, lo, hi); return hi > k0; });
    I1[d] = first_true(L, [&](int i) { int lo, hi; window_range(L, w, s, m, i, lo, hi); return lo >= k1; });
  }
  const int* qc = P.kb;            // query chunk shape (BWD_CHUNK tokens)
  int nc[3], total = 1;
  for (int d = 0; d < 3; ++d) {
    nc[d] = I1[d] > I0[d] ? cdiv(I1[d] - I0[d], qc[d]) : 0;
    total *= nc[d];
  }

  const int tid = threadIdx.x;
  const int ki = tid / TPK, gg = tid % TPK;
  int kx[3];
  box_coord(kbk.o, t.qb, ki, kx);
  bool kvalid = ki < KPB;
  for (int d = 0; d < 3; ++d)
    if (kx[d] >= g.L[d]) kvalid = false;
  const long long ktok = full_token(P.map, kx[0], kx[1], kx[2]);
  const size_t head = (size_t)bh * (size_t)P.N * D;
  const size_t koff = head + (size_t)(kvalid ? ktok : 0) * D + gg * 32;
  float kr[32], vr[32], dk[32], dv[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    kr[c] = kvalid ? ld<T>(P.k, koff + c) : 0.f;
    vr[c] = kvalid ? ld<T>(P.v, koff + c) : 0.f;
    dk[c] = 0.f;
    dv[c] = 0.f;
  }
  // the key block's extent, for the full-chunk test
  int kbl[3], kbh[3];
  for (int d = 0; d < 3; ++d) {
    kbl[d] = kbk.o[d];
    kbh[d] = kbk.o[d] + kbk.n[d];
  }
  const bool kblock_whole = true;  // kbk.n already clips the block to the grid

  for (int c = 0; c < total; ++c) {
    int a[3];
    {
      int cc = c;
      const int c2 = cc % nc[2]; cc /= nc[2];
      const int c1 = cc % nc[1]; const int c0 = cc / nc[1];
      a[0] = I0[0] + c0 * qc[0];
      a[1] = I0[1] + c1 * qc[1];
      a[2] = I0[2] + c2 * qc[2];
    }
    // Chunk status against the key block from the windows of its first and
    // last in-grid query per dimension (window ends are monotone).
    int status = CHUNK_FULL;
    for (int d = 0; d < 3; ++d) {
      const int L = g.L[d];
      const int f = a[d], l = imin(a[d] + qc[d], L) - 1;
      if (a[d] + qc[d] > L) status = CHUNK_PARTIAL;        // padded positions
      int flo, fhi, llo, lhi;
      window_range(L, g.w[d], g.s[d], g.m[d], f, flo, fhi);
      window_range(L, g.w[d], g.s[d], g.m[d], l, llo, lhi);
      if (lhi <= kbl[d] || flo >= kbh[d]) { status = CHUNK_EMPTY; break; }
      if (!(llo <= kbl[d] && fhi >= kbh[d])) status = CHUNK_PARTIAL;
    }
    (void)kblock_whole;
    if (status == CHUNK_EMPTY) continue;  // uniform across the block
    __syncthreads();
    for (int e = tid; e < BWD_CHUNK * D; e += BWD_THREADS) {
      const int qq = e / D, ch = e % D;
      const int q2 = qq % qc[2], q1 = (qq / qc[2]) % qc[1], q0 = qq / (qc[2] * qc[1]);
      const int x0 = a[0] + q0, x1 = a[1] + q1, x2 = a[2] + q2;
      float qv = 0.f, ov = 0.f;
      const bool in = x0 < g.L[0] && x1 < g.L[1] && x2 < g.L[2];
      const long long qt = full_token(P.map, x0, x1, x2);
      if (in) {
        const size_t off = head + (size_t)qt * D + ch;
        qv = ld<T>(P.q, off);
        ov = ld<T>(P.dout, off);
      }
      const int si = qq * D + (ch % 32) * TPK + ch / 32;
      Qs[si] = qv;
      Os[si] = ov;
      if (ch == 0) {
        Qv[qq] = in;
        Ls[qq] = in ? P.lse[(size_t)bh * P.N + qt] * LOG2E : 0.f;
        Dd[qq] = in ? P.delta[(size_t)bh * P.N + qt] : 0.f;
        const int xs[3] = {x0, x1, x2};
        for (int d = 0; d < 3; ++d) {
          int lo, hi;
          window_range(g.L[d], g.w[d], g.s[d], g.m[d], imin(xs[d], g.L[d] - 1), lo, hi);
          Wl[qq][d] = lo;
          Wh[qq][d] = hi;
        }
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int qq = 0; qq < BWD_CHUNK; ++qq) {
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int cc = 0; cc < 32; ++cc) {
        s = fmaf(kr[cc], Qs[qq * D + cc * TPK + gg], s);
        dp = fmaf(vr[cc], Os[qq * D + cc * TPK + gg], dp);
      }
#pragma unroll
      for (int off = 1; off < TPK; off <<= 1) {
        s += __shfl_xor_sync(0xffffffffu, s, off);
        dp += __shfl_xor_sync(0xffffffffu, dp, off);
      }
      bool in = kvalid;
      if (status == CHUNK_PARTIAL) {
        in = in && Qv[qq] && kx[0] >= Wl[qq][0] && kx[0] < Wh[qq][0] && kx[1] >= Wl[qq][1] &&
             kx[1] < Wh[qq][1] && kx[2] >= Wl[qq][2] && kx[2] < Wh[qq][2];
      }
      const float p = in ? exp2f(s * P.scale_log2 - Ls[qq]) : 0.f;
      const float dz = p * (dp - Dd[qq]);
#pragma unroll
      for (int cc = 0; cc < 32; ++cc) {
        dv[cc] = fmaf(p, Os[qq * D + cc * TPK + gg], dv[cc]);
        dk[cc] = fmaf(dz, Qs[qq * D + cc * TPK + gg], dk[cc]);
      }
    }
  }
  if (!kvalid) return;
  const size_t obase = head + (size_t)ktok * D + gg * 32;
#pragma unroll
  for (int cc = 0; cc < 32; ++cc) {
    st<T>(P.dk, obase + cc, dk[cc] * P.scale);
    st<T>(P.dv, obase + cc, dv[cc]);
  }
}

// Which kernels a launch runs.
enum : int { RUN_DELTA = 1, RUN_DQ = 2, RUN_DKDV = 4 };

template <int D, int T>
cudaError_t launch_dt(const BwdLaunch& L, cudaStream_t stream, int which) {
  const long long rows = (long long)L.BH * L.N;
  const long long dblocks = (rows + 7) / 8;
  const long long blocks = (long long)L.BH * L.t.nblocks;
  if (blocks <= 0 || blocks > 0x7fffffffLL || dblocks > 0x7fffffffLL)
    return cudaErrorInvalidConfiguration;
  if (which & RUN_DELTA) row_delta_kernel<T><<<(unsigned)dblocks, 256, 0, stream>>>(L);
  if (which & RUN_DQ) bwd_dq_kernel<D, T><<<(unsigned)blocks, BWD_THREADS, 0, stream>>>(L);
  if (which & RUN_DKDV) bwd_dkdv_kernel<D, T><<<(unsigned)blocks, BWD_THREADS, 0, stream>>>(L);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const BwdLaunch& L, cudaStream_t stream, int which) {
  switch (L.dtype) {
    case ELEM_F32: return launch_dt<D, ELEM_F32>(L, stream, which);
    case ELEM_BF16: return launch_dt<D, ELEM_BF16>(L, stream, which);
    case ELEM_F16: return launch_dt<D, ELEM_F16>(L, stream, which);
    default: return cudaErrorNotSupported;
  }
}

cudaError_t launch_which(const BwdLaunch& L, cudaStream_t stream, int which) {
  switch (L.D) {
    case 32: return launch_d<32>(L, stream, which);
    case 64: return launch_d<64>(L, stream, which);
    case 128: return launch_d<128>(L, stream, which);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

cudaError_t launch_bwd_simt(const BwdLaunch& L, cudaStream_t stream) {
  return launch_which(L, stream, RUN_DELTA | RUN_DQ | RUN_DKDV);
}
cudaError_t launch_bwd_simt_delta(const BwdLaunch& L, cudaStream_t stream) {
  return launch_which(L, stream, RUN_DELTA);
}
cudaError_t launch_bwd_simt_dkdv(const BwdLaunch& L, cudaStream_t stream) {
  return launch_which(L, stream, RUN_DKDV);
}
cudaError_t launch_bwd_simt_grads(const BwdLaunch& L, cudaStream_t stream) {
  return launch_which(L, stream, RUN_DQ | RUN_DKDV);
}

}  // namespace na
