// Tensor-core backward kernel for sm_100a, dQ part (bf16 or f16 in, fp32
// accumulate): for one 128-query block per CTA and every key chunk of the
// block's windows,
//   S  = Q K^T,  dP = dO V^T                  (tcgen05.mma, both operands in
//                                              shared memory, fp32 in TMEM)
//   P  = exp(scale S - lse),  dS = P (dP - delta)   (softmax warps, per row;
//                                              delta_i = <dO_i, out_i>)
//   dQ += dS K                                (tcgen05.mma, dS read from TMEM)
// and dq = scale dQ in the epilogue -- the dQ part of the vector-Jacobian
// product of the restricted softmax attention of "pi-Attention", section 3.1
// eqs. (1)-(3) with section 3.2's neighbourhood.  The backward needs no running
// maximum (lse is known), so each chunk's rows are split by keys between two
// warps per row quarter with no exchange between them.
//
// Roles (12 warps): warp 0 TMA producer (Q and dO once, then K / V chunks
// into two-tile stages whose slots swap roles every round, see first_slot
// in na_stages.cuh), warp 1 TMEM allocation and the MMA issuer (the whole
// warp, elect.sync choosing the issuing lane), warps 4-7 and 8-11 the
// element-wise part (warp 4+q keys 0-63, warp 8+q keys 64-127 of every
// chunk, rows 32q..32q+31), which exponentiates S as soon as it is in
// registers and waits for dP only to form dS.  Every wait is bounded (see
// na_ptx.cuh); the chunk stream ends with a marker in the next K slot.
// In both kernels S (S^T) of the next chunk is issued while the element-wise
// warps still work on the current one.
//
// The dK / dV part (tc_bwd_dkdv_kernel) is key-stationary: for one 128-key
// block per CTA (K and V resident in shared memory) and every chunk of the
// queries whose windows hold some of its keys,
//   S^T = K Q^T,  dP^T = V dO^T,  P^T = exp(scale S^T - lse),
//   dS^T = P^T (dP^T - delta),  dV += P^T dO,  dK += dS^T Q,
// with dk = scale dK.  The queries that see a key form a box per dimension
// (both window ends are monotone in the query coordinate), found by binary
// search, so the same chunk walk and full / partial / empty labels as the
// forward apply with the key block's inverse windows in place of windows.
// Its element-wise pass stores P^T (over S^T) before it forms dS^T (over
// dP^T), so dV of a chunk runs during the dS pass.
//
// TMEM columns (dQ kernel): S [0, 128), dP [128, 256) -- after the element-wise pass
// dS of keys 64h..64h+63 sits as packed 16-bit pairs in [128 + 64h, 160 + 64h),
// inside the half of dP that warp h itself read -- and dQ [256, 256 + D).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <stdio.h>

#include "na_internal.h"
#include "na_ptx.cuh"
#include "na_stages.cuh"

namespace na {
namespace {

constexpr int BT_THREADS = 384;
constexpr int BT_M = 128;                // query rows per block
constexpr int BT_N = 128;                // keys per chunk
constexpr int BT_HALF_BYTES = 128 * 128; // one 128-row x 64-element 16-bit box
constexpr int BT_REGS_LOADER = 64;
constexpr int BT_REGS_WORK = 208;
constexpr int BT_REGS_NEEDED = 128 * BT_REGS_LOADER + 256 * BT_REGS_WORK;
constexpr uint32_t BT_INFO_END = 0xFFFFu;
constexpr float BT_LOG2E = 1.4426950408889634f;

template <int D, bool F16>
struct BtCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int NS = (D == 128) ? 4 : 8;   // tile slots (K and V of NS / 2 chunks)
  static constexpr int HALVES = D / 64;
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL0 = 0;
  static constexpr int DP_COL0 = 128;
  static constexpr int DQ_COL0 = 256;
  static constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(BT_M, BT_N, false, false, F16);
  static constexpr uint32_t IDESC_DQ = ptx::idesc_bf16_f32(BT_M, D, false, true, F16);
};

template <int NS>
struct BtBars {
  uint64_t q_full;           // Q and dO tiles
  uint64_t full[NS];
  uint64_t empty[NS];
  uint64_t s_full;           // S of the current chunk
  uint64_t dp_full;          // dP of the current chunk
  uint64_t s_loaded;         // S read into registers (one arrival per element-wise warp)
  uint64_t p_ready;          // dS stored (256 arrivals)
  uint64_t o_done;
  uint32_t tmem_base;
  int abort;
  volatile uint32_t info[NS];
  BlockInfo bi;
  ChunkGrid cg;
};

template <int D>
constexpr size_t bt_smem_bytes() {
  return 1024 + (size_t)(2 + BtCfg<D, false>::NS) * BtCfg<D, false>::TILE_BYTES +
         sizeof(BtBars<BtCfg<D, false>::NS>);
}

template <int D, bool F16>
__global__ void __launch_bounds__(BT_THREADS, 1)
    tc_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const TcBwdLaunch P) {
  using C = BtCfg<D, F16>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = base;
  uint8_t* sDO = base + C::TILE_BYTES;
  uint8_t* ring = base + 2 * C::TILE_BYTES;
  BtBars<NS>* bars = reinterpret_cast<BtBars<NS>*>(ring + NS * C::TILE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const QTiling& t = P.t;
  const int bh = blockIdx.x / t.nblocks;
  const int blk = blockIdx.x % t.nblocks;
  const BlockInfo& B = bars->bi;
  const ChunkGrid& cg = bars->cg;

  if (threadIdx.x == 0) {
    block_info(P.g, t, blk, bars->bi);
    chunk_grid_for(&bars->bi, 1, P.kb, bars->cg);
    ptx::mbar_init(&bars->q_full, 1);
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(&bars->full[s], 1);
      ptx::mbar_init(&bars->empty[s], 1);
    }
    ptx::mbar_init(&bars->s_full, 1);
    ptx::mbar_init(&bars->dp_full, 1);
    ptx::mbar_init(&bars->s_loaded, 8);
    ptx::mbar_init(&bars->p_ready, 2 * BT_M);
    ptx::mbar_init(&bars->o_done, 1);
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

  if (warp < 4) {
    ptx::regs_dec<BT_REGS_LOADER>();
    if (warp == 0 && lane == 0 && B.exists) {
      // ========================= TMA producer =========================
      ptx::mbar_expect_tx(&bars->q_full, 2 * C::TILE_BYTES);
      for (int h = 0; h < C::HALVES; ++h) {
        ptx::tma_load_5d(sQ + h * BT_HALF_BYTES, &tm_q, &bars->q_full, h * 64, B.o[2], B.o[1],
                         B.o[0], bh);
        ptx::tma_load_5d(sDO + h * BT_HALF_BYTES, &tm_do, &bars->q_full, h * 64, B.o[2], B.o[1],
                         B.o[0], bh);
      }
      constexpr int NST = NS / 2;
      int c = 0;                 // chunk number
      int issued[NS];
#pragma unroll
      for (int s = 0; s < NS; ++s) issued[s] = 0;
      ChunkIter it;
      iter_begin(cg, it);
      bool ok = true;
      for (seek_block(cg, P.kb, B, it); ok && it.idx < cg.total;
           iter_next(cg, P.kb, it), seek_block(cg, P.kb, B, it), ++c) {
        for (int kv = 0; kv < 2 && ok; ++kv) {
          // K's slot was last read by dP, V's by dQ (fill number c / NST).
          const int slot = kv ? second_slot<NST>(c) : first_slot<NST>(c);
          if (c >= NST) ok = ptx::wait(&bars->empty[slot], ((c / NST) - 1) & 1, ctl);
          if (!ok) break;
          if (kv == 0) bars->info[slot] = 0;
          ptx::mbar_expect_tx(&bars->full[slot], C::TILE_BYTES);
          for (int h = 0; h < C::HALVES; ++h)
            ptx::tma_load_5d(ring + slot * C::TILE_BYTES + h * BT_HALF_BYTES, kv ? &tm_v : &tm_k,
                             &bars->full[slot], h * 64, it.a[2], it.a[1], it.a[0], bh);
          ++issued[slot];
        }
      }
      if (ok) {
        const int slot = first_slot<NST>(c);
        if (c >= NST) ok = ptx::wait(&bars->empty[slot], ((c / NST) - 1) & 1, ctl);
        if (ok) {
          bars->info[slot] = BT_INFO_END;
          ptx::mbar_arrive(&bars->full[slot]);
          ++issued[slot];
        }
      }
      for (int s = 0; s < NS; ++s)
        if (issued[s]) ptx::wait_drain(&bars->full[s], (issued[s] - 1) & 1, ctl);
      ptx::wait_drain(&bars->q_full, 0, ctl);
    } else if (warp == 1) {
      // =========================== MMA issuer ===========================
      // The whole warp issues: every lane sleeps in the hinted barrier wait
      // and elect.sync picks the lane that issues each MMA and commit.
      auto wait_i = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, ptx::wait_sleep(bar, parity, ctl));
      };
      auto commit_i = [&](uint64_t* bar) { ptx::tc_commit_warp(bar); };
      auto mma_ss_i = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
        ptx::mma_ss_warp(d, a, b, id, acc);
      };
      auto mma_ts_i = [&](uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
        ptx::mma_ts_warp(d, a, b, id, acc);
      };
      const uint32_t sQa = ptx::smem_u32(sQ), sDOa = ptx::smem_u32(sDO);
      const uint32_t ringa = ptx::smem_u32(ring);
      // S = Q K^T into [S_COL0, +128) and dP = dO V^T into [DP_COL0, +128):
      // both B operands are [keys x d] tiles read K-major.
      auto issue_s = [&](int kslot) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * BT_HALF_BYTES + (kk & 3) * 32;
          mma_ss_i(tmem + C::S_COL0, ptx::desc_sw128(sQa + off, 16, 1024),
                   ptx::desc_sw128(ringa + kslot * C::TILE_BYTES + off, 16, 1024), C::IDESC_S,
                   kk > 0 ? 1u : 0u);
        }
      };
      auto issue_dp = [&](int vslot) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * BT_HALF_BYTES + (kk & 3) * 32;
          mma_ss_i(tmem + C::DP_COL0, ptx::desc_sw128(sDOa + off, 16, 1024),
                   ptx::desc_sw128(ringa + vslot * C::TILE_BYTES + off, 16, 1024), C::IDESC_S,
                   kk > 0 ? 1u : 0u);
        }
      };
      // dQ += dS K: dS (16-bit pairs) of keys 64h.. in [DP_COL0 + 64h, +32),
      // K read MN-major (its rows are the reduction dimension here).
      auto issue_dq = [&](int kslot, bool accumulate) {
#pragma unroll
        for (int kk = 0; kk < BT_N / 16; ++kk) {
          const uint32_t a_t = tmem + C::DP_COL0 + (kk >> 2) * 64 + (kk & 3) * 8;
          const uint64_t bd =
              ptx::desc_sw128(ringa + kslot * C::TILE_BYTES + kk * 2048, BT_HALF_BYTES, 1024);
          mma_ts_i(tmem + C::DQ_COL0, a_t, bd, C::IDESC_DQ, (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      // Pipelined by one chunk: S of chunk j + 1 is issued as soon as the
      // element-wise warps have read S of chunk j into registers (S's
      // columns are then free; dS goes to dP's columns), so it runs during
      // their pass, and they exponentiate it while dQ of chunk j and dP of
      // chunk j + 1 run; dP of chunk j + 1 follows dQ of chunk j, which
      // reads dS from dP's columns (the tensor pipe executes in issue order).
      // K of chunk j sits in first_slot (j), V in second_slot (j); a slot is
      // released by the commit behind its last reader (dQ for K, dP for V).
      constexpr int NST = NS / 2;
      bool ok = B.exists;
      bool more = false;
      if (ok) ok = wait_i(&bars->q_full, 0);
      if (ok) ok = wait_i(&bars->full[first_slot<NST>(0)], 0);
      if (ok) {
        ptx::tc_fence_after();
        more = bars->info[first_slot<NST>(0)] != BT_INFO_END;
        if (more) {
          ok = wait_i(&bars->full[second_slot<NST>(0)], 0);
          if (ok) {
            ptx::tc_fence_after();
            issue_s(first_slot<NST>(0));
            commit_i(&bars->s_full);
            issue_dp(second_slot<NST>(0));
            commit_i(&bars->dp_full);
            commit_i(&bars->empty[second_slot<NST>(0)]);
          }
        }
      }
      for (int j = 0; ok && more; ++j) {
        const int ks = first_slot<NST>(j);
        const int nks = first_slot<NST>(j + 1), nvs = second_slot<NST>(j + 1);
        const uint32_t nph = ((j + 1) / NST) & 1;
        ok = wait_i(&bars->s_loaded, j & 1);
        if (!ok) break;
        ok = wait_i(&bars->full[nks], nph);
        if (!ok) break;
        ptx::tc_fence_after();
        more = bars->info[nks] != BT_INFO_END;
        if (more) {
          issue_s(nks);
          commit_i(&bars->s_full);
        }
        ok = wait_i(&bars->p_ready, j & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        issue_dq(ks, j > 0);
        commit_i(&bars->empty[ks]);
        if (!more) break;
        ok = wait_i(&bars->full[nvs], nph);
        if (!ok) break;
        ptx::tc_fence_after();
        issue_dp(nvs);
        commit_i(&bars->dp_full);
        commit_i(&bars->empty[nvs]);
      }
      commit_i(&bars->o_done);
      ptx::wait_drain(&bars->o_done, 0, ctl);
    }
  } else {
    // ======================= element-wise warps =======================
    ptx::regs_inc<BT_REGS_WORK>();
    const int quarter = warp & 3;
    const int h = (warp >> 3) & 1;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::S_COL0 + 64 * h;
    const uint32_t tDP = tmem + lane_base + C::DP_COL0 + 64 * h;
    const BlockInfo Bl = B;
    const ChunkGrid cgl = cg;
    const int kb[3] = {P.kb[0], P.kb[1], P.kb[2]};
    auto query_coord = [&](int rr, int gc[3]) {
      gc[2] = Bl.o[2] + rr % t.qb[2];
      gc[1] = Bl.o[1] + (rr / t.qb[2]) % t.qb[1];
      gc[0] = Bl.o[0] + rr / (t.qb[2] * t.qb[1]);
    };
    int wlo[3], whi[3];
    float lse2 = 0.f, Di = 0.f;
    {
      int gc[3];
      query_coord(row, gc);
      for (int d = 0; d < 3; ++d)
        window_range(P.g.L[d], P.g.w[d], P.g.s[d], P.g.m[d], imin(gc[d], P.g.L[d] - 1), wlo[d],
                     whi[d]);
      const bool valid = gc[0] < P.g.L[0] && gc[1] < P.g.L[1] && gc[2] < P.g.L[2];
      if (Bl.exists && valid) {
        const long long token = full_token(P.map, gc[0], gc[1], gc[2]);
        lse2 = P.lse[(size_t)bh * P.N + token] * BT_LOG2E;
        Di = P.delta[(size_t)bh * P.N + token];
      }
    }
    const float sl2 = P.scale_log2;
    bool ok = Bl.exists;
    int j = 0;
    if (ok) {
      ChunkIter it;
      iter_begin(cgl, it);
      for (int st = seek_block(cgl, kb, Bl, it); it.idx < cgl.total;
           iter_next(cgl, kb, it), st = seek_block(cgl, kb, Bl, it)) {
        bool got = ptx::wait(&bars->s_full, j & 1, ctl);
        got = __all_sync(0xffffffffu, got);
        if (!got) { ok = false; break; }
        ptx::tc_fence_after();
        uint32_t s[64];
        {
          uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
          uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
          ptx::tmem_ld32(tS, s0);
          ptx::tmem_ld32(tS + 32, s1);
          ptx::tmem_ld_wait();
          ptx::reg_fence(s0);
          ptx::reg_fence(s1);
        }
        // S's columns may now take the next chunk's scores.
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->s_loaded);
        if (st == CHUNK_PARTIAL) {
          uint32_t mk[4];
          chunk_key_mask(it.a, wlo, whi, kb, P.kb_log2, mk);
          const uint32_t w0 = h ? mk[2] : mk[0], w1 = h ? mk[3] : mk[1];
#pragma unroll
          for (int q = 0; q < 64; ++q)
            if (!(((q < 32 ? w0 : w1) >> (q & 31)) & 1u)) s[q] = __float_as_uint(-INFINITY);
        }
        // P = exp(scale S - lse) in fp32, while dQ of the previous chunk and
        // dP of this one run.
        const uint64_t scale2 = ptx::f2(sl2, sl2);
        const uint64_t neg2 = ptx::f2(-lse2, -lse2);
        const uint64_t negd2 = ptx::f2(-Di, -Di);
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const uint64_t x = ptx::f2_fma(
              ptx::f2(__uint_as_float(s[2 * q]), __uint_as_float(s[2 * q + 1])), scale2, neg2);
          float x0, x1;
          ptx::f2_split(x, x0, x1);
          s[2 * q] = __float_as_uint(ptx::ex2(x0));
          s[2 * q + 1] = __float_as_uint(ptx::ex2(x1));
        }
        got = ptx::wait(&bars->dp_full, j & 1, ctl);
        got = __all_sync(0xffffffffu, got);
        if (!got) { ok = false; break; }
        ptx::tc_fence_after();
        uint32_t dp[64];
        {
          uint32_t (&d0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dp[0]);
          uint32_t (&d1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dp[32]);
          ptx::tmem_ld32(tDP, d0);
          ptx::tmem_ld32(tDP + 32, d1);
          ptx::tmem_ld_wait();
          ptx::reg_fence(d0);
          ptx::reg_fence(d1);
        }
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const uint64_t g = ptx::f2_add(
              ptx::f2(__uint_as_float(dp[2 * q]), __uint_as_float(dp[2 * q + 1])), negd2);
          float z0, z1;
          ptx::f2_split(
              ptx::f2_mul(ptx::f2(__uint_as_float(s[2 * q]), __uint_as_float(s[2 * q + 1])), g),
              z0, z1);
          dp[q] = ptx::pack_half2<F16>(z0, z1);
        }
        {
          uint32_t (&ds)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dp[0]);
          ptx::tmem_st32(tDP, ds);
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->p_ready);
        ++j;
      }
    }
    // --------------------------- epilogue: dq ---------------------------
    if (ok && j > 0) {
      bool got = ptx::wait(&bars->o_done, 0, ctl);
      got = __all_sync(0xffffffffu, got);
      if (got) {
        ptx::tc_fence_after();
        int rr = row;
        asm volatile("" : "+r"(rr));
        int gc[3];
        query_coord(rr, gc);
        const bool valid = gc[0] < P.g.L[0] && gc[1] < P.g.L[1] && gc[2] < P.g.L[2];
        const long long token = full_token(P.map, gc[0], gc[1], gc[2]);
        const size_t rbase = ((size_t)bh * P.N + (size_t)(valid ? token : 0)) * D + h * (D / 2);
        uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(P.dq) + rbase);
        const float sc = P.scale;
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) {
          uint32_t o[32];
          ptx::tmem_ld32(tmem + lane_base + C::DQ_COL0 + h * (D / 2) + cc * 32, o);
          ptx::tmem_ld_wait();
          ptx::reg_fence(o);
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int q = 0; q < 16; ++q)
              pk[q] = ptx::pack_half2<F16>(__uint_as_float(o[2 * q]) * sc,
                                           __uint_as_float(o[2 * q + 1]) * sc);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              orow[cc * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      }
    } else if (ok && j == 0 && Bl.exists) {
      // a block with no chunk cannot occur (every query sees >= 1 key)
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ----------------------------------------------------------------- dK dV --
template <int D, bool F16>
struct BkCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int NQ = (D == 128) ? 2 : 4;   // query-chunk stages (Q and dO each)
  static constexpr int HALVES = D / 64;
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL0 = 0;                 // S^T, then P^T
  static constexpr int DP_COL0 = 128;              // dP^T, then dS^T
  static constexpr int DV_COL0 = 256;
  static constexpr int DK_COL0 = 256 + D;
  static constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(BT_M, BT_N, false, false, F16);
  static constexpr uint32_t IDESC_ACC = ptx::idesc_bf16_f32(BT_M, D, false, true, F16);
};

template <int NQ>
struct BkBars {
  uint64_t kv_full;          // K and V tiles of the key block
  uint64_t full[2 * NQ];     // tile slot loaded (TMA bytes + 32 producer lanes)
  uint64_t empty[2 * NQ];    // tile slot read by its last MMA
  uint64_t s_full;           // S^T of the current chunk
  uint64_t dp_full;          // dP^T of the current chunk
  uint64_t p_ready;          // P^T stored over S^T (256 arrivals)
  uint64_t ds_ready;         // dS^T stored over dP^T (256 arrivals)
  uint64_t o_done;
  uint32_t tmem_base;
  int abort;
  volatile uint32_t info[NQ];  // stage's chunk or end marker (with its Q slot)
  float lse2[NQ][BT_N];      // log2(e) * lse of the stage's queries
  float dlt[NQ][BT_N];       // delta of the stage's queries
  BlockInfo kb;              // the key block (origin, extent)
  BlockInfo ib;              // its inverse windows: lo/hi = union, ilo/ihi = intersection
  ChunkGrid cg;              // query chunks over ib
};

template <int NQ>
__device__ __forceinline__ int q_slot(int j) { return first_slot<NQ>(j); }
template <int NQ>
__device__ __forceinline__ int do_slot(int j) { return second_slot<NQ>(j); }

template <int D>
constexpr size_t bk_smem_bytes() {
  return 1024 + (size_t)(2 + 2 * BkCfg<D, false>::NQ) * BkCfg<D, false>::TILE_BYTES +
         sizeof(BkBars<BkCfg<D, false>::NQ>);
}

template <int D, bool F16>
__global__ void __launch_bounds__(BT_THREADS, 1)
    tc_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                       const TcBwdLaunch P) {
  using C = BkCfg<D, F16>;
  constexpr int NQ = C::NQ;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sK = base;
  uint8_t* sV = base + C::TILE_BYTES;
  uint8_t* stages = base + 2 * C::TILE_BYTES;      // tile slots (q_slot / do_slot)
  BkBars<NQ>* bars = reinterpret_cast<BkBars<NQ>*>(stages + 2 * NQ * C::TILE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const QTiling& t = P.t;                           // key blocks use the query tiling
  const int bh = blockIdx.x / t.nblocks;
  const int blk = blockIdx.x % t.nblocks;
  const BlockInfo& KB = bars->kb;
  const BlockInfo& IB = bars->ib;
  const ChunkGrid& cg = bars->cg;

  if (threadIdx.x == 0) {
    block_info(P.g, t, blk, bars->kb);
    key_block_query_box(P.g, bars->kb, bars->ib);
    chunk_grid_for(&bars->ib, 1, P.kb, bars->cg);
    ptx::mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < 2 * NQ; ++s) {
      ptx::mbar_init(&bars->full[s], 32);
      ptx::mbar_init(&bars->empty[s], 1);
    }
    ptx::mbar_init(&bars->s_full, 1);
    ptx::mbar_init(&bars->dp_full, 1);
    ptx::mbar_init(&bars->p_ready, 2 * BT_M);
    ptx::mbar_init(&bars->ds_ready, 2 * BT_M);
    ptx::mbar_init(&bars->o_done, 1);
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

  if (warp < 4) {
    ptx::regs_dec<BT_REGS_LOADER>();
    if (warp == 0 && KB.exists) {
      // ====================== producer (whole warp) ======================
      // Lane 0 issues the TMA copies; every lane stages lse / delta of four
      // of the chunk's queries and arrives on the stage's barrier.
      if (lane == 0) {
        ptx::mbar_expect_tx(&bars->kv_full, 2 * C::TILE_BYTES);
        for (int h = 0; h < C::HALVES; ++h) {
          ptx::tma_load_5d(sK + h * BT_HALF_BYTES, &tm_k, &bars->kv_full, h * 64, KB.o[2], KB.o[1],
                           KB.o[0], bh);
          ptx::tma_load_5d(sV + h * BT_HALF_BYTES, &tm_v, &bars->kv_full, h * 64, KB.o[2], KB.o[1],
                           KB.o[0], bh);
        }
      }
      int issued[2 * NQ];
#pragma unroll
      for (int s = 0; s < 2 * NQ; ++s) issued[s] = 0;
      int seq = 0;
      ChunkIter it;
      iter_begin(cg, it);
      bool ok = true;
      // Stage a chunk's per-query scalars, then load one of its tiles into
      // slot sl once the slot's previous tile has been read (fill number
      // seq / NQ of the slot).
      auto wait_slot = [&](int sl) {
        bool w = true;
        if (seq >= NQ) w = ptx::wait(&bars->empty[sl], ((seq / NQ) - 1) & 1, ctl);
        return __all_sync(0xffffffffu, w);
      };
      for (seek_block(cg, P.kb, IB, it); ok && it.idx < cg.total;
           iter_next(cg, P.kb, it), seek_block(cg, P.kb, IB, it), ++seq) {
        const int st = seq % NQ;
        const int qs = q_slot<NQ>(seq), ds = do_slot<NQ>(seq);
        float l2[BT_N / 32], dl[BT_N / 32];
#pragma unroll
        for (int r = 0; r < BT_N / 32; ++r) {
          const int e = lane + 32 * r;
          const int q2 = e % P.kb[2], q1 = (e / P.kb[2]) % P.kb[1], q0 = e / (P.kb[2] * P.kb[1]);
          const int x0 = it.a[0] + q0, x1 = it.a[1] + q1, x2 = it.a[2] + q2;
          l2[r] = 0.f;
          dl[r] = 0.f;
          if (x0 < P.g.L[0] && x1 < P.g.L[1] && x2 < P.g.L[2]) {
            const size_t tok = (size_t)full_token(P.map, x0, x1, x2);
            l2[r] = P.lse[(size_t)bh * P.N + tok] * BT_LOG2E;
            dl[r] = P.delta[(size_t)bh * P.N + tok];
          }
        }
        // Q (with lse and the chunk's marker): its slot was last read by dV.
        ok = wait_slot(qs);
        if (!ok) break;
#pragma unroll
        for (int r = 0; r < BT_N / 32; ++r) bars->lse2[st][lane + 32 * r] = l2[r];
        if (lane == 0) {
          bars->info[st] = 0;
          ptx::mbar_expect_tx(&bars->full[qs], C::TILE_BYTES);
          for (int h = 0; h < C::HALVES; ++h)
            ptx::tma_load_5d(stages + qs * C::TILE_BYTES + h * BT_HALF_BYTES, &tm_q,
                             &bars->full[qs], h * 64, it.a[2], it.a[1], it.a[0], bh);
        } else {
          ptx::mbar_arrive(&bars->full[qs]);
        }
        ++issued[qs];
        // dO (with delta): its slot was last read by dK.
        ok = wait_slot(ds);
        if (!ok) break;
#pragma unroll
        for (int r = 0; r < BT_N / 32; ++r) bars->dlt[st][lane + 32 * r] = dl[r];
        if (lane == 0) {
          ptx::mbar_expect_tx(&bars->full[ds], C::TILE_BYTES);
          for (int h = 0; h < C::HALVES; ++h)
            ptx::tma_load_5d(stages + ds * C::TILE_BYTES + h * BT_HALF_BYTES, &tm_do,
                             &bars->full[ds], h * 64, it.a[2], it.a[1], it.a[0], bh);
        } else {
          ptx::mbar_arrive(&bars->full[ds]);
        }
        ++issued[ds];
      }
      if (ok) {
        const int qs = q_slot<NQ>(seq);
        ok = wait_slot(qs);
        if (ok) {
          if (lane == 0) bars->info[seq % NQ] = BT_INFO_END;
          __syncwarp();
          ptx::mbar_arrive(&bars->full[qs]);
          ++issued[qs];
        }
      }
      if (lane == 0) {
        for (int s = 0; s < 2 * NQ; ++s)
          if (issued[s]) ptx::wait_drain(&bars->full[s], (issued[s] - 1) & 1, ctl);
        ptx::wait_drain(&bars->kv_full, 0, ctl);
      }
    } else if (warp == 1) {
      // =========================== MMA issuer ===========================
      // The whole warp issues: every lane sleeps in the hinted barrier wait
      // and elect.sync picks the lane that issues each MMA and commit.
      auto wait_i = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, ptx::wait_sleep(bar, parity, ctl));
      };
      auto commit_i = [&](uint64_t* bar) { ptx::tc_commit_warp(bar); };
      auto mma_ss_i = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
        ptx::mma_ss_warp(d, a, b, id, acc);
      };
      auto mma_ts_i = [&](uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
        ptx::mma_ts_warp(d, a, b, id, acc);
      };
      const uint32_t sKa = ptx::smem_u32(sK), sVa = ptx::smem_u32(sV);
      const uint32_t sta = ptx::smem_u32(stages);
      auto slot_addr = [&](int sl) { return sta + (uint32_t)(sl * C::TILE_BYTES); };
      auto issue_st = [&](int qs) {        // S^T = K Q^T
        const uint32_t qa = slot_addr(qs);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * BT_HALF_BYTES + (kk & 3) * 32;
          mma_ss_i(tmem + C::S_COL0, ptx::desc_sw128(sKa + off, 16, 1024),
                   ptx::desc_sw128(qa + off, 16, 1024), C::IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_dpt = [&](int ds) {       // dP^T = V dO^T
        const uint32_t da = slot_addr(ds);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * BT_HALF_BYTES + (kk & 3) * 32;
          mma_ss_i(tmem + C::DP_COL0, ptx::desc_sw128(sVa + off, 16, 1024),
                   ptx::desc_sw128(da + off, 16, 1024), C::IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      // dV += P^T dO and dK += dS^T Q: the chunk's tiles read MN-major (their
      // rows, the chunk's queries, are the reduction dimension).
      auto issue_dv = [&](int ds, bool accumulate) {   // dV += P^T dO
        const uint32_t da = slot_addr(ds);
#pragma unroll
        for (int kk = 0; kk < BT_N / 16; ++kk) {
          const uint32_t col = (kk >> 2) * 64 + (kk & 3) * 8;
          mma_ts_i(tmem + C::DV_COL0, tmem + C::S_COL0 + col,
                   ptx::desc_sw128(da + kk * 2048, BT_HALF_BYTES, 1024), C::IDESC_ACC,
                   (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      auto issue_dk = [&](int qs, bool accumulate) {   // dK += dS^T Q
        const uint32_t qa = slot_addr(qs);
#pragma unroll
        for (int kk = 0; kk < BT_N / 16; ++kk) {
          const uint32_t col = (kk >> 2) * 64 + (kk & 3) * 8;
          mma_ts_i(tmem + C::DK_COL0, tmem + C::DP_COL0 + col,
                   ptx::desc_sw128(qa + kk * 2048, BT_HALF_BYTES, 1024), C::IDESC_ACC,
                   (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      // The element-wise pass stores P^T first and dS^T second, so dV of
      // chunk j runs while dS^T is formed.  S^T of chunk j + 1 is issued
      // right behind that dV (into the columns dV just read), ahead of dK,
      // so the next chunk's exponentials overlap dK and dP^T; its Q sits in
      // the slot that dO of chunk j + 1 - NQ left when its dV completed.  The
      // tensor pipe runs in issue order, which keeps every overwrite of a
      // TMEM operand behind its reader.  A slot is released by the commit
      // behind its last reader: dV for dO, dK for Q.
      bool ok = KB.exists;
      bool more = false;
      if (ok) ok = wait_i(&bars->kv_full, 0);
      if (ok) ok = wait_i(&bars->full[q_slot<NQ>(0)], 0);
      if (ok) {
        ptx::tc_fence_after();
        more = bars->info[0] != BT_INFO_END;
        if (more) {
          issue_st(q_slot<NQ>(0));
          commit_i(&bars->s_full);
          ok = wait_i(&bars->full[do_slot<NQ>(0)], 0);
          if (ok) {
            ptx::tc_fence_after();
            issue_dpt(do_slot<NQ>(0));
            commit_i(&bars->dp_full);
          }
        }
      }
      for (int j = 0; ok && more; ++j) {
        const int qs = q_slot<NQ>(j), ds = do_slot<NQ>(j);
        const int nqs = q_slot<NQ>(j + 1), nds = do_slot<NQ>(j + 1);
        const uint32_t nph = ((j + 1) / NQ) & 1;
        ok = wait_i(&bars->p_ready, j & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        issue_dv(ds, j > 0);
        commit_i(&bars->empty[ds]);
        ok = wait_i(&bars->full[nqs], nph);
        if (!ok) break;
        ptx::tc_fence_after();
        more = bars->info[(j + 1) % NQ] != BT_INFO_END;
        if (more) {
          issue_st(nqs);
          commit_i(&bars->s_full);
        }
        ok = wait_i(&bars->ds_ready, j & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        issue_dk(qs, j > 0);
        commit_i(&bars->empty[qs]);
        if (!more) break;
        ok = wait_i(&bars->full[nds], nph);
        if (!ok) break;
        ptx::tc_fence_after();
        issue_dpt(nds);
        commit_i(&bars->dp_full);
      }
      commit_i(&bars->o_done);
      ptx::wait_drain(&bars->o_done, 0, ctl);
    }
  } else {
    // ======================= element-wise warps =======================
    ptx::regs_inc<BT_REGS_WORK>();
    const int quarter = warp & 3;
    const int h = (warp >> 3) & 1;              // query half of every chunk
    const int row = quarter * 32 + lane;        // key row of the block
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::S_COL0 + 64 * h;
    const uint32_t tDP = tmem + lane_base + C::DP_COL0 + 64 * h;
    const BlockInfo Kl = KB;
    const BlockInfo Il = IB;
    const ChunkGrid cgl = cg;
    const int qc[3] = {P.kb[0], P.kb[1], P.kb[2]};
    auto key_coord = [&](int rr, int gc[3]) {
      gc[2] = Kl.o[2] + rr % t.qb[2];
      gc[1] = Kl.o[1] + (rr / t.qb[2]) % t.qb[1];
      gc[0] = Kl.o[0] + rr / (t.qb[2] * t.qb[1]);
    };
    int ilo[3], ihi[3];    // queries whose window holds this key, per dimension
    {
      int gc[3];
      key_coord(row, gc);
      const bool kvalid = gc[0] < P.g.L[0] && gc[1] < P.g.L[1] && gc[2] < P.g.L[2];
      for (int d = 0; d < 3; ++d) {
        if (Kl.exists && kvalid) {
          inverse_range(P.g.L[d], P.g.w[d], P.g.s[d], P.g.m[d], gc[d], ilo[d], ihi[d]);
        } else {
          ilo[d] = 0;
          ihi[d] = 0;     // a key outside the grid is in no window
        }
      }
    }
    const float sl2 = P.scale_log2;
    bool ok = Kl.exists;
    int j = 0;
    if (ok) {
      ChunkIter it;
      iter_begin(cgl, it);
      for (int stc = seek_block(cgl, qc, Il, it); it.idx < cgl.total;
           iter_next(cgl, qc, it), stc = seek_block(cgl, qc, Il, it)) {
        const int st = j % NQ;
        bool got = ptx::wait(&bars->s_full, j & 1, ctl);
        got = __all_sync(0xffffffffu, got);
        if (!got) { ok = false; break; }
        ptx::tc_fence_after();
        // Phase 1: P^T = exp(scale S^T - lse) from S^T alone, stored over S^T
        // so that dV can start; P stays in registers (fp32) for phase 2.
        uint32_t s[64];
        {
          uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
          uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
          ptx::tmem_ld32(tS, s0);
          ptx::tmem_ld32(tS + 32, s1);
          ptx::tmem_ld_wait();
          ptx::reg_fence(s0);
          ptx::reg_fence(s1);
        }
        // Mask (partial chunks): query c of the chunk sees this key iff its
        // coordinates lie in the key's inverse ranges; padded keys see none.
        if (stc == CHUNK_PARTIAL || ihi[0] == 0) {
          uint32_t mk[4];
          chunk_key_mask(it.a, ilo, ihi, qc, P.kb_log2, mk);
          const uint32_t w0 = h ? mk[2] : mk[0], w1 = h ? mk[3] : mk[1];
#pragma unroll
          for (int q = 0; q < 64; ++q)
            if (!(((q < 32 ? w0 : w1) >> (q & 31)) & 1u)) s[q] = __float_as_uint(-INFINITY);
        }
        const uint64_t scale2 = ptx::f2(sl2, sl2);
        const float* l2p = &bars->lse2[st][64 * h];
        const float* dlp = &bars->dlt[st][64 * h];
        {
          uint32_t pw[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const float2 l2 = *reinterpret_cast<const float2*>(l2p + 2 * q);
            const uint64_t x = ptx::f2_fma(
                ptx::f2(__uint_as_float(s[2 * q]), __uint_as_float(s[2 * q + 1])), scale2,
                ptx::f2(-l2.x, -l2.y));
            float x0, x1;
            ptx::f2_split(x, x0, x1);
            const float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
            s[2 * q] = __float_as_uint(p0);       // P kept in fp32 for dS
            s[2 * q + 1] = __float_as_uint(p1);
            pw[q] = ptx::pack_half2<F16>(p0, p1);
          }
          ptx::tmem_st32(tS, pw);
          ptx::tmem_st_wait();
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->p_ready);
        // Phase 2: dS^T = P^T (dP^T - delta), stored over dP^T for dK.
        got = ptx::wait(&bars->dp_full, j & 1, ctl);
        got = __all_sync(0xffffffffu, got);
        if (!got) { ok = false; break; }
        ptx::tc_fence_after();
        uint32_t dp[64];
        {
          uint32_t (&d0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dp[0]);
          uint32_t (&d1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dp[32]);
          ptx::tmem_ld32(tDP, d0);
          ptx::tmem_ld32(tDP + 32, d1);
          ptx::tmem_ld_wait();
          ptx::reg_fence(d0);
          ptx::reg_fence(d1);
        }
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const float2 dl = *reinterpret_cast<const float2*>(dlp + 2 * q);
          const uint64_t g = ptx::f2_add(
              ptx::f2(__uint_as_float(dp[2 * q]), __uint_as_float(dp[2 * q + 1])),
              ptx::f2(-dl.x, -dl.y));
          float z0, z1;
          ptx::f2_split(ptx::f2_mul(ptx::f2(__uint_as_float(s[2 * q]), __uint_as_float(s[2 * q + 1])), g),
                        z0, z1);
          dp[q] = ptx::pack_half2<F16>(z0, z1);
        }
        {
          uint32_t (&dw)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dp[0]);
          ptx::tmem_st32(tDP, dw);
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->ds_ready);
        ++j;
      }
    }
    // ------------------------ epilogue: dk, dv ------------------------
    if (ok && j > 0) {
      bool got = ptx::wait(&bars->o_done, 0, ctl);
      got = __all_sync(0xffffffffu, got);
      if (got) {
        ptx::tc_fence_after();
        int rr = row;
        asm volatile("" : "+r"(rr));
        int gc[3];
        key_coord(rr, gc);
        const bool valid = gc[0] < P.g.L[0] && gc[1] < P.g.L[1] && gc[2] < P.g.L[2];
        const long long token = full_token(P.map, gc[0], gc[1], gc[2]);
        const size_t rbase = ((size_t)bh * P.N + (size_t)(valid ? token : 0)) * D + h * (D / 2);
        for (int which = 0; which < 2; ++which) {
          uint4* orow = reinterpret_cast<uint4*>(
              reinterpret_cast<uint16_t*>(which ? P.dk : P.dv) + rbase);
          const float sc = which ? P.scale : 1.f;
          const int col0 = (which ? C::DK_COL0 : C::DV_COL0) + h * (D / 2);
#pragma unroll
          for (int cc = 0; cc < D / 64; ++cc) {
            uint32_t o[32];
            ptx::tmem_ld32(tmem + lane_base + col0 + cc * 32, o);
            ptx::tmem_ld_wait();
            ptx::reg_fence(o);
            if (valid) {
              uint32_t pk[16];
#pragma unroll
              for (int q = 0; q < 16; ++q)
                pk[q] = ptx::pack_half2<F16>(__uint_as_float(o[2 * q]) * sc,
                                             __uint_as_float(o[2 * q + 1]) * sc);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                orow[cc * 4 + v] =
                    make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
          }
        }
      }
    } else if (ok && j == 0) {
      // No query sees any key of this block (possible: keys outside every
      // window, e.g. the last keys under causal windows with stride 1 never
      // are -- but a ragged grid can leave keys unseen): their gradients are
      // zero.
      int rr = row;
      int gc[3];
      key_coord(rr, gc);
      const bool valid = gc[0] < P.g.L[0] && gc[1] < P.g.L[1] && gc[2] < P.g.L[2];
      if (valid) {
        const long long token = full_token(P.map, gc[0], gc[1], gc[2]);
        const size_t rbase = ((size_t)bh * P.N + (size_t)token) * D + h * (D / 2);
        for (int which = 0; which < 2; ++which) {
          uint4* orow = reinterpret_cast<uint4*>(
              reinterpret_cast<uint16_t*>(which ? P.dk : P.dv) + rbase);
          for (int v = 0; v < D / 16; ++v) orow[v] = make_uint4(0u, 0u, 0u, 0u);
        }
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

template <int D, bool F16>
cudaError_t launch_dkdv_d(const TcBwdLaunch& L, cudaStream_t stream, char* err, int errlen) {
  CUtensorMap mk, mv, mq, mdo;
  if (!encode_grid_map_dil(&mk, L.k, L.f16, L.D, L.g.L, L.map, L.BH, L.N, L.t.qb) ||
      !encode_grid_map_dil(&mv, L.v, L.f16, L.D, L.g.L, L.map, L.BH, L.N, L.t.qb) ||
      !encode_grid_map_dil(&mq, L.q, L.f16, L.D, L.g.L, L.map, L.BH, L.N, L.kb) ||
      !encode_grid_map_dil(&mdo, L.dout, L.f16, L.D, L.g.L, L.map, L.BH, L.N, L.kb)) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled failed (pointer alignment or shape)");
    return cudaErrorInvalidValue;
  }
  const size_t smem = bk_smem_bytes<D>();
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, tc_bwd_dkdv_kernel<D, F16>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * BT_THREADS < BT_REGS_NEEDED) {
      snprintf(err, errlen, "kernel compiled with %d registers/thread; the register split needs %d",
               fa.numRegs, (BT_REGS_NEEDED + BT_THREADS - 1) / BT_THREADS);
      return cudaErrorInvalidConfiguration;
    }
    e = cudaFuncSetAttribute(tc_bwd_dkdv_kernel<D, F16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  const long long grid = (long long)L.t.nblocks * L.BH;
  if (grid <= 0 || grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  tc_bwd_dkdv_kernel<D, F16><<<(unsigned)grid, BT_THREADS, smem, stream>>>(mk, mv, mq, mdo, L);
  return cudaGetLastError();
}

template <int D, bool F16>
cudaError_t launch_dq_d(const TcBwdLaunch& L, cudaStream_t stream, char* err, int errlen) {
  CUtensorMap mq, mdo, mk, mv;
  if (!encode_grid_map_dil(&mq, L.q, L.f16, L.D, L.g.L, L.map, L.BH, L.N, L.t.qb) ||
      !encode_grid_map_dil(&mdo, L.dout, L.f16, L.D, L.g.L, L.map, L.BH, L.N, L.t.qb) ||
      !encode_grid_map_dil(&mk, L.k, L.f16, L.D, L.g.L, L.map, L.BH, L.N, L.kb) ||
      !encode_grid_map_dil(&mv, L.v, L.f16, L.D, L.g.L, L.map, L.BH, L.N, L.kb)) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled failed (pointer alignment or shape)");
    return cudaErrorInvalidValue;
  }
  const size_t smem = bt_smem_bytes<D>();
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, tc_bwd_dq_kernel<D, F16>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * BT_THREADS < BT_REGS_NEEDED) {
      snprintf(err, errlen, "kernel compiled with %d registers/thread; the register split needs %d",
               fa.numRegs, (BT_REGS_NEEDED + BT_THREADS - 1) / BT_THREADS);
      return cudaErrorInvalidConfiguration;
    }
    e = cudaFuncSetAttribute(tc_bwd_dq_kernel<D, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  const long long grid = (long long)L.t.nblocks * L.BH;
  if (grid <= 0 || grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  tc_bwd_dq_kernel<D, F16><<<(unsigned)grid, BT_THREADS, smem, stream>>>(mq, mdo, mk, mv, L);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_bwd_dkdv(const TcBwdLaunch& L0, cudaStream_t stream, char* err, int errlen) {
  TcBwdLaunch L = L0;
  for (int d = 0; d < 3; ++d) {
    if (L.t.qb[d] > 256 || L.kb[d] > 256) return cudaErrorNotSupported;
    if (L.kb[d] & (L.kb[d] - 1)) return cudaErrorNotSupported;
    int lg = 0;
    while ((1 << lg) < L.kb[d]) ++lg;
    L.kb_log2[d] = lg;
  }
  if (L.t.qb[0] * L.t.qb[1] * L.t.qb[2] != BT_M || L.kb[0] * L.kb[1] * L.kb[2] != BT_N)
    return cudaErrorNotSupported;
  switch (L.D) {
    case 64:
      return L.f16 ? launch_dkdv_d<64, true>(L, stream, err, errlen)
                   : launch_dkdv_d<64, false>(L, stream, err, errlen);
    case 128:
      return L.f16 ? launch_dkdv_d<128, true>(L, stream, err, errlen)
                   : launch_dkdv_d<128, false>(L, stream, err, errlen);
    default:
      return cudaErrorNotSupported;
  }
}

cudaError_t launch_tc_bwd_dq(const TcBwdLaunch& L0, cudaStream_t stream, char* err, int errlen) {
  TcBwdLaunch L = L0;
  for (int d = 0; d < 3; ++d) {
    if (L.t.qb[d] > 256 || L.kb[d] > 256) return cudaErrorNotSupported;
    if (L.kb[d] & (L.kb[d] - 1)) return cudaErrorNotSupported;
    int lg = 0;
    while ((1 << lg) < L.kb[d]) ++lg;
    L.kb_log2[d] = lg;
  }
  if (L.t.qb[0] * L.t.qb[1] * L.t.qb[2] != BT_M || L.kb[0] * L.kb[1] * L.kb[2] != BT_N)
    return cudaErrorNotSupported;
  switch (L.D) {
    case 64:
      return L.f16 ? launch_dq_d<64, true>(L, stream, err, errlen)
                   : launch_dq_d<64, false>(L, stream, err, errlen);
    case 128:
      return L.f16 ? launch_dq_d<128, true>(L, stream, err, errlen)
                   : launch_dq_d<128, false>(L, stream, err, errlen);
    default:
      return cudaErrorNotSupported;
  }
}

}  // namespace na
