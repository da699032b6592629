// Tensor-core forward kernel for sm_100a (bf16 in, fp32 accumulate, bf16 out,
// fp32 log-sum-exp).
//
// One CTA owns a pair of 128-query blocks of one (batch, head).  It walks the
// key box of the pair's windows in chunks of 128 keys; every chunk is EMPTY,
// PARTIAL or FULL per block (na_sched.cuh), so masks are applied only on
// partial chunks and a block skips chunks it does not see.
//
// Roles (12 warps):
//   warp 0     TMA producer: Q blocks once, then K and V chunks through an
//              NS-slot shared-memory ring (128-byte swizzled, token-tile-major:
//              each tile is a multi-dimensional box of the grid);
//   warp 1     allocates tensor memory; lane 0 issues every tcgen05.mma:
//              S_b = Q_b K^T into TMEM, then O_b += P_b V with P_b read from TMEM;
//   warps 4-7  softmax for block 0, warps 8-11 softmax for block 1: one query
//              row per thread (tcgen05.ld 32x32b), online softmax in the log2
//              domain with a lazily moved reference max, P written back to
//              TMEM as bf16 over its S, O rescaled in TMEM when the max moves;
//              then the epilogue (O / l -> bf16, lse).
// Two blocks ping-pong: while one block's softmax runs, the tensor core works
// on the other block.
//
// The arithmetic is the restricted softmax attention of "pi-Attention",
// section 3.1 eqs. (1)-(3) and section 3.2 eq. (4), computed tile by tile
// on chip as that page's section 3.4 describes; the lse output is the log of
// eq. (2)'s denominator.
//
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <stdio.h>

#include <mutex>

#include "na_internal.h"
#include "na_ptx.cuh"

namespace na {
namespace {

constexpr int TC_THREADS = 384;
constexpr int BLOCK_M = 128;     // query rows per block
constexpr int CHUNK_N = 128;     // keys per chunk
constexpr int HALF_BYTES = 128 * 128;  // one 128-row x 64-element bf16 box (16 KB)

template <int D>
struct TcCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;             // Q block or K/V chunk
  static constexpr int NS = (D == 128) ? 5 : 8;              // ring slots
  static constexpr int HALVES = D / 64;                      // 64-element boxes per row
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL0 = 0;
  static constexpr int O_COL0 = 256;
  static constexpr uint32_t IDESC_QK = ptx::idesc_bf16_f32(BLOCK_M, CHUNK_N, false, false);
  static constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32(BLOCK_M, D, false, true);
};

template <int NS>
struct Bars {
  uint64_t q_full[2];
  uint64_t full[NS];
  uint64_t empty[NS];
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t o_done;
  uint32_t tmem_base;
  int abort;
};

template <int D>
constexpr size_t smem_bytes() {
  return 1024 /* alignment slack */ + (size_t)(2 + TcCfg<D>::NS) * TcCfg<D>::TILE_BYTES +
         sizeof(Bars<TcCfg<D>::NS>);
}

// Next chunk index >= c that is non-empty for at least one block.
__device__ __forceinline__ int next_chunk(const ChunkGrid& cg, const int* kb, const BlockInfo* bi,
                                          int c, int& st0, int& st1) {
  for (; c < cg.total; ++c) {
    int a[3];
    chunk_origin(cg, kb, c, a);
    st0 = chunk_status(bi[0], a, kb);
    st1 = chunk_status(bi[1], a, kb);
    if (st0 != CHUNK_EMPTY || st1 != CHUNK_EMPTY) return c;
  }
  st0 = st1 = CHUNK_EMPTY;
  return cg.total;
}

template <int D>
__global__ void __launch_bounds__(TC_THREADS, 1)
    tc_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const TcLaunch P) {
  using C = TcCfg<D>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = base;                                   // 2 tiles
  uint8_t* ring = base + 2 * C::TILE_BYTES;             // NS tiles
  Bars<NS>* bars = reinterpret_cast<Bars<NS>*>(ring + NS * C::TILE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (batch*head, pair of query blocks) ----
  const QTiling& t = P.t;
  const int npairs = (t.nblocks + 1) >> 1;
  const int bh = blockIdx.x / npairs;
  const int pair = blockIdx.x % npairs;
  BlockInfo bi[2];
  block_info(P.g, t, 2 * pair, bi[0]);
  block_info(P.g, t, 2 * pair + 1, bi[1]);
  ChunkGrid cg;
  chunk_grid_for(bi, 2, P.kb, cg);

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&bars->q_full[b], 1);
      ptx::mbar_init(&bars->s_full[b], 1);
      ptx::mbar_init(&bars->p_ready[b], BLOCK_M);
    }
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(&bars->full[s], 1);
      ptx::mbar_init(&bars->empty[s], 1);
    }
    ptx::mbar_init(&bars->o_done, 1);
    // A CTA that starts after some wait on this device already expired
    // unwinds at once instead of waiting out its own bounds.
    bars->abort = *reinterpret_cast<volatile int*>(P.status) != 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  ptx::WaitCtl ctl;
  ctl.abort = &bars->abort;
  ctl.status = P.status;
  ctl.timeout_ns = (uint64_t)P.timeout_ns;

  if (warp == 0) {
    // =========================== TMA producer ===========================
    if (lane == 0) {
      int seq = 0;
      int issued[NS];
#pragma unroll
      for (int s = 0; s < NS; ++s) issued[s] = 0;
      for (int b = 0; b < 2; ++b) {
        if (!bi[b].exists) continue;
        ptx::mbar_expect_tx(&bars->q_full[b], C::TILE_BYTES);
        for (int h = 0; h < C::HALVES; ++h)
          ptx::tma_load_5d(sQ + b * C::TILE_BYTES + h * HALF_BYTES, &tm_q, &bars->q_full[b],
                           h * 64, bi[b].o[2], bi[b].o[1], bi[b].o[0], bh);
      }
      int st0, st1;
      for (int c = next_chunk(cg, P.kb, bi, 0, st0, st1); c < cg.total;
           c = next_chunk(cg, P.kb, bi, c + 1, st0, st1)) {
        int a[3];
        chunk_origin(cg, P.kb, c, a);
        bool ok = true;
        for (int kv = 0; kv < 2 && ok; ++kv) {
          const int slot = seq % NS;
          if (seq >= NS) ok = ptx::wait(&bars->empty[slot], ((seq / NS) - 1) & 1, ctl);
          if (!ok) break;
          if (!((P.debug_flags & 1) && seq == 0)) {  // testing hook: withhold chunk 0's K
            ptx::mbar_expect_tx(&bars->full[slot], C::TILE_BYTES);
            for (int h = 0; h < C::HALVES; ++h)
              ptx::tma_load_5d(ring + slot * C::TILE_BYTES + h * HALF_BYTES, kv ? &tm_v : &tm_k,
                               &bars->full[slot], h * 64, a[2], a[1], a[0], bh);
            ++issued[slot];
          }
          ++seq;
        }
        if (!ok) break;
      }
      // Drain: every issued copy must land before the CTA can exit.
      for (int s = 0; s < NS; ++s)
        if (issued[s]) ptx::wait_drain(&bars->full[s], (issued[s] - 1) & 1, ctl);
      for (int b = 0; b < 2; ++b)
        if (bi[b].exists) ptx::wait_drain(&bars->q_full[b], 0, ctl);
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      const uint32_t sQa = ptx::smem_u32(sQ);
      const uint32_t ringa = ptx::smem_u32(ring);
      bool ok = true;
      for (int b = 0; b < 2 && ok; ++b)
        if (bi[b].exists) ok = ptx::wait(&bars->q_full[b], 0, ctl);
      int pcount[2] = {0, 0};
      bool have_pv[2] = {false, false};
      int seq = 0;
      int st0 = CHUNK_EMPTY, st1 = CHUNK_EMPTY;
      int cur = ok ? next_chunk(cg, P.kb, bi, 0, st0, st1) : cg.total;
      int cst[2] = {st0, st1};

      // S = Q K^T for one block into its S columns.
      auto issue_s = [&](int b, int kslot) {
        const uint32_t d_t = tmem + C::S_COL0 + b * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          const uint64_t ad = ptx::desc_sw128(sQa + b * C::TILE_BYTES + off, 16, 1024);
          const uint64_t bd = ptx::desc_sw128(ringa + kslot * C::TILE_BYTES + off, 16, 1024);
          ptx::mma_ss(d_t, ad, bd, C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
      };
      // O += P V for one block; P (bf16) sits in the block's S columns.
      auto issue_pv = [&](int b, int vslot, bool accumulate) {
        const uint32_t d_t = tmem + C::O_COL0 + b * D;
        const uint32_t a_t = tmem + C::S_COL0 + b * 128;
#pragma unroll
        for (int kk = 0; kk < CHUNK_N / 16; ++kk) {
          const uint64_t bd =
              ptx::desc_sw128(ringa + vslot * C::TILE_BYTES + kk * 2048, HALF_BYTES, 1024);
          ptx::mma_ts(d_t, a_t + kk * 8, bd, C::IDESC_PV, (accumulate || kk > 0) ? 1u : 0u);
        }
      };

      if (cur < cg.total) {
        const int kslot = seq % NS;
        ok = ptx::wait(&bars->full[kslot], (seq / NS) & 1, ctl);
        ++seq;
        if (ok) {
          ptx::tc_fence_after();
          for (int b = 0; b < 2; ++b)
            if (cst[b] != CHUNK_EMPTY) {
              issue_s(b, kslot);
              ptx::tc_commit(&bars->s_full[b]);
            }
          ptx::tc_commit(&bars->empty[kslot]);
        }
      }
      while (ok && cur < cg.total) {
        const int vslot = seq % NS;
        const int vseq = seq++;
        int nst0, nst1;
        const int nxt = next_chunk(cg, P.kb, bi, cur + 1, nst0, nst1);
        const int nst[2] = {nst0, nst1};
        int kslot = -1, kseq = -1;
        bool k_ready = false;
        if (nxt < cg.total) { kslot = seq % NS; kseq = seq++; }
        ok = ptx::wait(&bars->full[vslot], (vseq / NS) & 1, ctl);
        if (!ok) break;
        ptx::tc_fence_after();
        for (int b = 0; b < 2 && ok; ++b) {
          if (cst[b] != CHUNK_EMPTY) {
            ok = ptx::wait(&bars->p_ready[b], pcount[b] & 1, ctl);
            if (!ok) break;
            ++pcount[b];
            ptx::tc_fence_after();
            issue_pv(b, vslot, have_pv[b]);
            have_pv[b] = true;
          }
          if (nxt < cg.total && nst[b] != CHUNK_EMPTY) {
            if (!k_ready) {
              ok = ptx::wait(&bars->full[kslot], (kseq / NS) & 1, ctl);
              if (!ok) break;
              ptx::tc_fence_after();
              k_ready = true;
            }
            issue_s(b, kslot);
            ptx::tc_commit(&bars->s_full[b]);
          }
        }
        if (!ok) break;
        ptx::tc_commit(&bars->empty[vslot]);
        if (nxt < cg.total) {
          if (!k_ready) {
            ok = ptx::wait(&bars->full[kslot], (kseq / NS) & 1, ctl);
            if (!ok) break;
          }
          ptx::tc_commit(&bars->empty[kslot]);
        }
        cur = nxt;
        cst[0] = nst[0];
        cst[1] = nst[1];
      }
      // All MMAs done (normal or unwinding): release the epilogue, then make
      // sure nothing still writes tensor memory before it is freed.
      ptx::tc_commit(&bars->o_done);
      ptx::wait_drain(&bars->o_done, 0, ctl);
    }
  } else if (warp >= 4) {
    // ===================== softmax + epilogue (per block) =====================
    const int b = (warp - 4) >> 2;
    const BlockInfo& B = bi[b];
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::S_COL0 + b * 128;
    const uint32_t tO = tmem + lane_base + C::O_COL0 + b * D;

    // Query coordinates of this row (row-major over the block box).
    const int r2 = row % t.qb[2];
    const int r1 = (row / t.qb[2]) % t.qb[1];
    const int r0 = row / (t.qb[2] * t.qb[1]);
    const int g0 = B.o[0] + r0, g1 = B.o[1] + r1, g2 = B.o[2] + r2;
    const bool valid = B.exists && g0 < P.g.L[0] && g1 < P.g.L[1] && g2 < P.g.L[2];
    const int ws0 = window_start(P.g.L[0], P.g.w[0], P.g.s[0], imin(g0, P.g.L[0] - 1));
    const int ws1 = window_start(P.g.L[1], P.g.w[1], P.g.s[1], imin(g1, P.g.L[1] - 1));
    const int ws2 = window_start(P.g.L[2], P.g.w[2], P.g.s[2], imin(g2, P.g.L[2] - 1));
    const int kb2 = P.kb[2], kb12 = P.kb[1] * P.kb[2];
    const float sl2 = P.scale_log2;

    float m = -INFINITY;   // reference max, log2 domain
    float l = 0.f;
    int scount = 0;
    bool had_pv = false;
    bool ok = true;
    if (B.exists) {
      int st0, st1;
      for (int c = next_chunk(cg, P.kb, bi, 0, st0, st1); c < cg.total;
           c = next_chunk(cg, P.kb, bi, c + 1, st0, st1)) {
        const int st = b ? st1 : st0;
        if (st == CHUNK_EMPTY) continue;
        bool got = ptx::wait(&bars->s_full[b], scount & 1, ctl);
        got = __all_sync(0xffffffffu, got);
        if (!got) { ok = false; break; }
        ++scount;
        ptx::tc_fence_after();

        uint32_t s[128];
        {
          uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
          uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
          uint32_t (&s2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[64]);
          uint32_t (&s3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[96]);
          ptx::tmem_ld32(tS + 0, s0);
          ptx::tmem_ld32(tS + 32, s1);
          ptx::tmem_ld32(tS + 64, s2);
          ptx::tmem_ld32(tS + 96, s3);
          ptx::tmem_ld_wait();
          ptx::reg_fence(s0);
          ptx::reg_fence(s1);
          ptx::reg_fence(s2);
          ptx::reg_fence(s3);
        }
        if (st == CHUNK_PARTIAL) {
          int a[3];
          chunk_origin(cg, P.kb, c, a);
          const int d0 = a[0] - ws0, d1 = a[1] - ws1, d2 = a[2] - ws2;
#pragma unroll
          for (int j = 0; j < 128; ++j) {
            const int k2 = j % kb2, k1 = (j % kb12) / kb2, k0 = j / kb12;
            const bool in = (unsigned)(d0 + k0) < (unsigned)P.g.w[0] &&
                            (unsigned)(d1 + k1) < (unsigned)P.g.w[1] &&
                            (unsigned)(d2 + k2) < (unsigned)P.g.w[2];
            if (!in) s[j] = __float_as_uint(-INFINITY);
          }
        }
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 128; ++j) mx = fmaxf(mx, __uint_as_float(s[j]));
        const float mx2 = mx * sl2;
        // Move the reference max only when the new max exceeds it by more
        // than 2^8: P stays <= 256, exact after the final division by l.
        const bool need = mx2 > m + 8.f;
        const float m_new = need ? mx2 : m;
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = need ? ptx::ex2(m - m_use) : 1.f;
        const bool warp_need = __any_sync(0xffffffffu, need);

        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const float p0 = ptx::ex2(fmaf(__uint_as_float(s[2 * j]), sl2, -m_use));
          const float p1 = ptx::ex2(fmaf(__uint_as_float(s[2 * j + 1]), sl2, -m_use));
          sum += p0 + p1;
          s[j] = ptx::pack_bf16(p0, p1);
        }
        {
          uint32_t (&p0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
          uint32_t (&p1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
          ptx::tmem_st32(tS + 0, p0);
          ptx::tmem_st32(tS + 32, p1);
        }
        if (warp_need && had_pv) {
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            ptx::tmem_ld32(tO + cc * 32, o);
            ptx::tmem_ld_wait();
            ptx::reg_fence(o);
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
            ptx::tmem_st32(tO + cc * 32, o);
          }
        }
        l = l * alpha + sum;
        m = m_new;
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->p_ready[b]);
        had_pv = true;
      }
    }
    // ------------------------------ epilogue ------------------------------
    if (ok && had_pv) {
      bool got = ptx::wait(&bars->o_done, 0, ctl);
      got = __all_sync(0xffffffffu, got);
      if (got) {
        ptx::tc_fence_after();
        const long long token = ((long long)g0 * P.g.L[1] + g1) * P.g.L[2] + g2;
        const size_t rbase = ((size_t)bh * P.N + (size_t)(valid ? token : 0)) * D;
        const float inv_l = 1.f / l;
        uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(P.out) + rbase);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          ptx::tmem_ld32(tO + cc * 32, o);
          ptx::tmem_ld_wait();
          ptx::reg_fence(o);
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pk[j] = ptx::pack_bf16(__uint_as_float(o[2 * j]) * inv_l,
                                     __uint_as_float(o[2 * j + 1]) * inv_l);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              orow[cc * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
        if (valid)
          P.lse[(size_t)bh * P.N + token] = (m + __log2f(l)) * 0.69314718055994530942f;
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------ host side --
PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [BH, X1, X2, X3, D] bf16 as a 5-d tensor (D, X3, X2, X1, BH), 64-element
// inner box with 128-byte swizzle.
bool encode_map(CUtensorMap* m, const void* ptr, const TcLaunch& L, const int box[3]) {
  auto enc = get_encoder();
  if (!enc) return false;
  const cuuint64_t es = 2;
  cuuint64_t dims[5] = {(cuuint64_t)L.D, (cuuint64_t)L.g.L[2], (cuuint64_t)L.g.L[1],
                        (cuuint64_t)L.g.L[0], (cuuint64_t)L.BH};
  cuuint64_t strides[4] = {(cuuint64_t)L.D * es, (cuuint64_t)L.g.L[2] * L.D * es,
                           (cuuint64_t)L.g.L[1] * L.g.L[2] * L.D * es,
                           (cuuint64_t)L.N * L.D * es};
  cuuint32_t boxd[5] = {64, (cuuint32_t)box[2], (cuuint32_t)box[1], (cuuint32_t)box[0], 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides,
                   boxd, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(const TcLaunch& L, cudaStream_t stream, char* err, int errlen) {
  CUtensorMap mq, mk, mv;
  if (!encode_map(&mq, L.q, L, L.t.qb) || !encode_map(&mk, L.k, L, L.kb) ||
      !encode_map(&mv, L.v, L, L.kb)) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled failed (pointer alignment or shape)");
    return cudaErrorInvalidValue;
  }
  const size_t smem = smem_bytes<D>();
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(tc_fwd_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  const long long npairs = (L.t.nblocks + 1) / 2;
  const long long grid = npairs * L.BH;
  if (grid <= 0 || grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  tc_fwd_kernel<D><<<(unsigned)grid, TC_THREADS, smem, stream>>>(mq, mk, mv, L);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc(const TcLaunch& L, cudaStream_t stream, char* err, int errlen) {
  for (int d = 0; d < 3; ++d) {
    if (L.t.qb[d] > 256 || L.kb[d] > 256) return cudaErrorNotSupported;
  }
  if (L.t.qb[0] * L.t.qb[1] * L.t.qb[2] != BLOCK_M || L.kb[0] * L.kb[1] * L.kb[2] != CHUNK_N)
    return cudaErrorNotSupported;
  switch (L.D) {
    case 64: return launch_d<64>(L, stream, err, errlen);
    case 128: return launch_d<128>(L, stream, err, errlen);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace na
