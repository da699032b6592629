// Tensor-core forward kernel for sm_100a (bf16 or f16 in, fp32 accumulate,
// output in the input type, fp32 log-sum-exp).
//
// One CTA owns a pair of 128-query blocks of one (batch, head).  It walks the
// key box of the pair's windows in chunks of 128 keys; every chunk is EMPTY,
// PARTIAL or FULL per block (na_sched.cuh), so masks are applied only on
// partial chunks and a block skips chunks it does not see.
//
// Roles (12 warps, three warpgroups):
//   warp 0     TMA producer: Q blocks once, then K and V chunks through an
//              NS-slot shared-memory ring (128-byte swizzled, token-tile-major:
//              each tile is a multi-dimensional box of the grid);
//   warp 1     allocates tensor memory; lane 0 issues every tcgen05.mma:
//              S_b = Q_b K^T into TMEM, then O_b += P_b V with P_b read from TMEM;
//   warps 4-7  softmax for block 0, warps 8-11 softmax for block 1: one query
//              row per thread (tcgen05.ld 32x32b), online softmax in the log2
//              domain with a lazily moved reference max, P written back to
//              TMEM in the input type over its S, O rescaled in TMEM when the
//              max moves; then the epilogue (O / l -> input type, lse).
// Two blocks ping-pong: while one block's softmax runs, the tensor core works
// on the other block.  Warpgroup 0 hands most of its registers to the two
// softmax warpgroups (setmaxnreg).  The softmax can evaluate a fixed share of
// its exponentials on the FMA pipe (polynomial, EMU_NUM / EMU_DEN) instead of
// the MUFU unit.  The MMA issuer learns each chunk's per-block status from the
// producer (slot info written with the K tile), so its loop is straight-line.
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
constexpr int REGS_LOADER = 56;        // warpgroup 0 after setmaxnreg.dec
constexpr int REGS_SOFTMAX = 216;      // warpgroups 1 and 2 after setmaxnreg.inc
constexpr int REGS_NEEDED = 128 * REGS_LOADER + 256 * REGS_SOFTMAX;  // must fit the launch
// Exponentials of P pair j go to the FMA-pipe polynomial when
// (j * EMU_NUM) % EMU_DEN < EMU_NUM, i.e. EMU_NUM / EMU_DEN of them.  Measured
// on the sliding-tile workload: 0/5 978, 1/5 913, 2/5 890, 3/5 857 TFLOP/s --
// the softmax here is latency-bound in one warp per sub-partition, not
// MUFU-bound, so every exponential currently stays on the MUFU unit.
constexpr int EMU_NUM = 0;
constexpr int EMU_DEN = 5;

__host__ __device__ constexpr bool emulate_pair(int j) { return (j * EMU_NUM) % EMU_DEN < EMU_NUM; }
constexpr uint32_t INFO_END = 0xFFFFu;   // slot info: no more chunks
// Largest row sum of P accepted against a stale reference max: the sum bounds
// every P of the row, so P <= 2^14 -- inside bf16's and f16's range, and
// harmless to the fp32 accumulators -- while the reference rarely moves.
constexpr float P_LIMIT = 16384.f;

// Input types of the kernel (template argument DT).
constexpr int DT_BF16 = 0, DT_F16 = 1, DT_E4M3 = 2;
// E4M3 inputs: P is formed against a reference P8_OFFSET log2 units below the
// maximum it was set from, so typical weights land in the format's normal
// range (>= 2^-6) instead of its coarse subnormals; rows are redone once their
// sum (a bound of their largest P) exceeds P_LIMIT8, so P stays below the
// format's largest value, 448.
constexpr float P8_OFFSET = 4.f;
constexpr float P_LIMIT8 = 256.f;

template <int D, int DT = DT_BF16>
struct TcCfg {
  static constexpr bool F16 = DT == DT_F16;
  static constexpr bool E4M3 = DT == DT_E4M3;
  static constexpr int ESZ = E4M3 ? 1 : 2;                   // bytes per input element
  static constexpr int TILE_BYTES = 128 * D * ESZ;           // Q block or K/V chunk
  // TMA boxes: 128 rows of BOX_ELEMS elements, BOX_ROW bytes per row (the
  // swizzle span: 128 B, or 64 B for E4M3 at head_dim 64); NBOX boxes per row.
  static constexpr int BOX_ELEMS = E4M3 ? D : 64;
  static constexpr int BOX_ROW = BOX_ELEMS * ESZ;
  static constexpr int NBOX = D / BOX_ELEMS;
  static constexpr int BOX_BYTES = 128 * BOX_ROW;
  static constexpr uint32_t LAYOUT = BOX_ROW == 128 ? 2u : 4u;   // SWIZZLE_128B / SWIZZLE_64B
  static constexpr int SBO = 8 * BOX_ROW;                    // 8-row swizzle atom
  static constexpr int MMA_K = E4M3 ? 32 : 16;               // K elements per MMA (32 bytes)
  static constexpr int NS = E4M3 ? (D == 128 ? 10 : 16) : ((D == 128) ? 5 : 8);   // ring slots
  static constexpr float PLIM = E4M3 ? P_LIMIT8 : P_LIMIT;
  static constexpr float POFF = E4M3 ? P8_OFFSET : 0.f;
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL0 = 0;
  static constexpr int O_COL0 = 256;
  // Operand format code 0 is f16 for kind::f16 and E4M3 for kind::f8f6f4.
  static constexpr uint32_t IDESC_QK =
      ptx::idesc_bf16_f32(BLOCK_M, CHUNK_N, false, false, F16 || E4M3);
  static constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32(BLOCK_M, D, false, true, F16 || E4M3);
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
  volatile uint32_t info[NS];  // per K slot: chunk status of block 0 | block 1 << 2
  BlockInfo bi[2];   // this CTA's two query blocks
  ChunkGrid cg;      // and the chunk grid over their key box
};

template <int D, int DT>
constexpr size_t smem_bytes() {
  return 1024 /* alignment slack */ + (size_t)(2 + TcCfg<D, DT>::NS) * TcCfg<D, DT>::TILE_BYTES +
         sizeof(Bars<TcCfg<D, DT>::NS>);
}

// Advance `it` to the first chunk (at or after it) that is non-empty for at
// least one of the two blocks; it.idx == cg.total when there is none.
__device__ __forceinline__ void seek_pair(const ChunkGrid& cg, const int* kb, const BlockInfo* bi,
                                          ChunkIter& it, int& st0, int& st1) {
  for (; it.idx < cg.total; iter_next(cg, kb, it)) {
    st0 = chunk_status(bi[0], it.a, kb);
    st1 = chunk_status(bi[1], it.a, kb);
    if (st0 != CHUNK_EMPTY || st1 != CHUNK_EMPTY) return;
  }
  st0 = st1 = CHUNK_EMPTY;
}

template <int D, int DT>
__global__ void __launch_bounds__(TC_THREADS, 1)
    tc_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const TcLaunch P) {
  using C = TcCfg<D, DT>;
  constexpr int NS = C::NS;
  constexpr bool F16 = C::F16;
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
  // Block descriptors and chunk grid live in shared memory, so no role holds
  // them in registers across its main loop.
  BlockInfo* bi = bars->bi;
  const ChunkGrid& cg = bars->cg;

  if (threadIdx.x == 0) {
    block_info(P.g, t, 2 * pair, bars->bi[0]);
    block_info(P.g, t, 2 * pair + 1, bars->bi[1]);
    chunk_grid_for(bars->bi, 2, P.kb, bars->cg);
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

  if (warp < 4) {
  // Warpgroup 0: loader warps.  Each warpgroup rebalances registers at the top
  // of its own branch so the compiler can apply each limit to its code only.
  ptx::regs_dec<REGS_LOADER>();
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
        for (int h = 0; h < C::NBOX; ++h)
          ptx::tma_load_5d(sQ + b * C::TILE_BYTES + h * C::BOX_BYTES, &tm_q, &bars->q_full[b],
                           h * C::BOX_ELEMS, bi[b].o[2], bi[b].o[1], bi[b].o[0], bh);
      }
      ChunkIter it;
      iter_begin(cg, it);
      int st0, st1;
      bool ok = true;
      for (seek_pair(cg, P.kb, bi, it, st0, st1); ok && it.idx < cg.total;
           iter_next(cg, P.kb, it), seek_pair(cg, P.kb, bi, it, st0, st1)) {
        for (int kv = 0; kv < 2 && ok; ++kv) {
          const int slot = seq % NS;
          if (seq >= NS) ok = ptx::wait(&bars->empty[slot], ((seq / NS) - 1) & 1, ctl);
          if (!ok) break;
          // The K tile carries the chunk's per-block status to the MMA issuer
          // (published by the arrive below, read after its wait on `full`).
          if (kv == 0) bars->info[slot] = (uint32_t)st0 | ((uint32_t)st1 << 2);
          if (!((P.debug_flags & 1) && seq == 0)) {  // testing hook: withhold chunk 0's K
            ptx::mbar_expect_tx(&bars->full[slot], C::TILE_BYTES);
            for (int h = 0; h < C::NBOX; ++h)
              ptx::tma_load_5d(ring + slot * C::TILE_BYTES + h * C::BOX_BYTES, kv ? &tm_v : &tm_k,
                               &bars->full[slot], h * C::BOX_ELEMS, it.a[2], it.a[1], it.a[0], bh);
            ++issued[slot];
          }
          ++seq;
        }
      }
      if (ok) {
        // End-of-stream marker in the slot where the next K tile would go.
        const int slot = seq % NS;
        if (seq >= NS) ok = ptx::wait(&bars->empty[slot], ((seq / NS) - 1) & 1, ctl);
        if (ok) {
          bars->info[slot] = INFO_END;
          ptx::mbar_arrive(&bars->full[slot]);
          ++issued[slot];
          ++seq;
        }
      }
      // Drain: every issued copy must land before the CTA can exit.
      for (int s = 0; s < NS; ++s)
        if (issued[s]) ptx::wait_drain(&bars->full[s], (issued[s] - 1) & 1, ctl);
      for (int b = 0; b < 2; ++b)
        if (bi[b].exists) ptx::wait_drain(&bars->q_full[b], 0, ctl);
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    // At head_dim 64 the whole warp runs the issue loop (warp-uniform slot
    // descriptors; one elected lane issues, every lane sleeps in hinted
    // waits): 3-7 % faster on the head_dim 64 workloads.  At 128 lane 0
    // alone issues (the warp-wide form measured 1 % slower there).
    constexpr bool WARPWIDE = (D == 64);
    if (WARPWIDE || lane == 0) {
      const uint32_t sQa = ptx::smem_u32(sQ);
      const uint32_t ringa = ptx::smem_u32(ring);
      auto wait_i = [&](uint64_t* bar, uint32_t parity) {
        if constexpr (WARPWIDE)
          return __all_sync(0xffffffffu, ptx::wait_sleep(bar, parity, ctl));
        else
          return ptx::wait(bar, parity, ctl);
      };
      auto commit_i = [&](uint64_t* bar) {
        if constexpr (WARPWIDE) ptx::tc_commit_warp(bar); else ptx::tc_commit(bar);
      };
      auto mma_ss_i = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
        if constexpr (C::E4M3) {
          if constexpr (WARPWIDE) ptx::mma_ss_f8_warp(d, a, b, id, acc);
          else ptx::mma_ss_f8(d, a, b, id, acc);
        } else {
          if constexpr (WARPWIDE) ptx::mma_ss_warp(d, a, b, id, acc);
          else ptx::mma_ss(d, a, b, id, acc);
        }
      };
      auto mma_ts_i = [&](uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
        if constexpr (C::E4M3) {
          if constexpr (WARPWIDE) ptx::mma_ts_f8_warp(d, a, b, id, acc);
          else ptx::mma_ts_f8(d, a, b, id, acc);
        } else {
          if constexpr (WARPWIDE) ptx::mma_ts_warp(d, a, b, id, acc);
          else ptx::mma_ts(d, a, b, id, acc);
        }
      };
      bool ok = true;
      if (bi[0].exists) ok = wait_i(&bars->q_full[0], 0);
      if (ok && bi[1].exists) ok = wait_i(&bars->q_full[1], 0);

      // S = Q K^T for one block into its S columns.
      auto issue_s = [&](int b, int kslot) {
        const uint32_t d_t = tmem + C::S_COL0 + b * 128;
#pragma unroll
        for (int kk = 0; kk < D / C::MMA_K; ++kk) {
          // K slice kk: bytes [32 kk, 32 kk + 32) of each row, inside box
          // (32 kk) / BOX_ROW.
          const uint32_t off = ((kk * 32) / C::BOX_ROW) * C::BOX_BYTES + (kk * 32) % C::BOX_ROW;
          const uint64_t ad = ptx::desc_sw(sQa + b * C::TILE_BYTES + off, 16, C::SBO, C::LAYOUT);
          const uint64_t bd = ptx::desc_sw(ringa + kslot * C::TILE_BYTES + off, 16, C::SBO, C::LAYOUT);
          mma_ss_i(d_t, ad, bd, C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
      };
      // O += P V for one block; P (bf16) sits in the block's S columns.
      auto issue_pv = [&](int b, int vslot, bool accumulate) {
        const uint32_t d_t = tmem + C::O_COL0 + b * D;
        const uint32_t a_t = tmem + C::S_COL0 + b * 128;
#pragma unroll
        for (int kk = 0; kk < CHUNK_N / C::MMA_K; ++kk) {
          // keys [MMA_K kk, MMA_K (kk + 1)) of V (MN-major: boxes along the
          // head dimension BOX_BYTES apart); P's 32 bytes of them are 8 columns.
          const uint64_t bd = ptx::desc_sw(ringa + vslot * C::TILE_BYTES + kk * C::MMA_K * C::BOX_ROW,
                                           C::BOX_BYTES, C::SBO, C::LAYOUT);
          mma_ts_i(d_t, a_t + kk * 8, bd, C::IDESC_PV, (accumulate || kk > 0) ? 1u : 0u);
        }
      };

      // Straight-line issue loop: per-block state in scalars, chunk statuses
      // read from the slot info the producer wrote with each K tile.
      int seq = 0;
      uint32_t ph0 = 0, ph1 = 0;          // p_ready phases consumed per block
      bool acc0 = false, acc1 = false;    // O of the block already written once
      uint32_t cinfo = INFO_END;
      if (ok) {
        ok = wait_i(&bars->full[0], 0);  // first K tile (or the end marker)
        seq = 1;
        if (ok) {
          cinfo = bars->info[0];
          ptx::tc_fence_after();
          if (cinfo != INFO_END) {
            if (cinfo & 3u) { issue_s(0, 0); commit_i(&bars->s_full[0]); }
            if (cinfo >> 2) { issue_s(1, 0); commit_i(&bars->s_full[1]); }
          }
          commit_i(&bars->empty[0]);
        }
      }
      while (ok && cinfo != INFO_END) {
        const int vslot = seq % NS, vseq = seq++;
        const int kslot = seq % NS, kseq = seq++;   // next K tile or the end marker
        ok = wait_i(&bars->full[vslot], (vseq / NS) & 1);
        if (!ok) break;
        // The next K tile (loaded well ahead) is waited for here, before block
        // 0's P, so that no barrier check sits between block 0's two products.
        ok = wait_i(&bars->full[kslot], (kseq / NS) & 1);
        if (!ok) break;
        const uint32_t ninfo = bars->info[kslot];
        ptx::tc_fence_after();
        if (cinfo & 3u) {
          ok = wait_i(&bars->p_ready[0], ph0 & 1);
          if (!ok) break;
          ++ph0;
          ptx::tc_fence_after();
          issue_pv(0, vslot, acc0);
          acc0 = true;
        }
        const bool more = ninfo != INFO_END;
        if (more && (ninfo & 3u)) { issue_s(0, kslot); commit_i(&bars->s_full[0]); }
        if (cinfo >> 2) {
          ok = wait_i(&bars->p_ready[1], ph1 & 1);
          if (!ok) break;
          ++ph1;
          ptx::tc_fence_after();
          issue_pv(1, vslot, acc1);
          acc1 = true;
        }
        if (more && (ninfo >> 2)) { issue_s(1, kslot); commit_i(&bars->s_full[1]); }
        commit_i(&bars->empty[vslot]);
        commit_i(&bars->empty[kslot]);
        cinfo = ninfo;
      }
      // All MMAs done (normal or unwinding): release the epilogue, then make
      // sure nothing still writes tensor memory before it is freed.
      commit_i(&bars->o_done);
      ptx::wait_drain(&bars->o_done, 0, ctl);
    }
  }
  } else {
    // ===================== softmax + epilogue (per block) =====================
    ptx::regs_inc<REGS_SOFTMAX>();
    const int b = (warp - 4) >> 2;
    const BlockInfo& B = bi[b];
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::S_COL0 + b * 128;
    const uint32_t tO = tmem + lane_base + C::O_COL0 + b * D;

    // Grid coordinates of this thread's query (row-major over the block box);
    // recomputed in the epilogue rather than kept live across the main loop.
    auto query_coord = [&](int rr, int g[3]) {
      g[2] = B.o[2] + rr % t.qb[2];
      g[1] = B.o[1] + (rr / t.qb[2]) % t.qb[1];
      g[0] = B.o[0] + rr / (t.qb[2] * t.qb[1]);
    };
    int wlo[3], whi[3];   // this row's window [wlo, whi) per dimension
    {
      int g[3];
      query_coord(row, g);
      for (int d = 0; d < 3; ++d)
        window_range(P.g.L[d], P.g.w[d], P.g.s[d], P.g.m[d], imin(g[d], P.g.L[d] - 1), wlo[d],
                     whi[d]);
    }
    const float sl2 = P.scale_log2;

    float m = -INFINITY;   // reference max, log2 domain
    float l = 0.f;
    int scount = 0;
    bool had_pv = false;
    bool ok = true;
    if (B.exists) {
      ChunkIter it;
      iter_begin(cg, it);
      for (int st = seek_block(cg, P.kb, B, it); it.idx < cg.total;
           iter_next(cg, P.kb, it), st = seek_block(cg, P.kb, B, it)) {
        bool got = ptx::wait(&bars->s_full[b], scount & 1, ctl);
        got = __all_sync(0xffffffffu, got);
        if (!got) { ok = false; break; }
        ++scount;
        ptx::tc_fence_after();

        uint32_t s[128];
        uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
        uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
        uint32_t (&s2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[64]);
        uint32_t (&s3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[96]);
        // Scores of the chunk into registers (and -inf outside the row's
        // window on partial chunks).
        auto load_scores = [&]() {
          if (D == 64 && st == CHUNK_PARTIAL) {
            // Scores outside the row's window become -inf in TMEM, one
            // 32-key word at a time (a loop, not unrolled: the masked path
            // stays small in the instruction cache); words no lane of the
            // warp masks are skipped.
            int lo[3], hi[3];
            for (int d = 0; d < 3; ++d) {
              lo[d] = imin(imax(wlo[d] - it.a[d], 0), P.kb[d]);
              hi[d] = imin(imax(whi[d] - it.a[d], 0), P.kb[d]);
            }
            const int sh[3] = {P.kb_log2[1] + P.kb_log2[2], P.kb_log2[2], 0};
#pragma unroll 1
            for (int wd = 0; wd < 4; ++wd) {
              uint32_t mw = 0xffffffffu;
#pragma unroll
              for (int d = 0; d < 3; ++d) mw &= dim_word_mask(wd, sh[d], P.kb[d], lo[d], hi[d]);
              if (__any_sync(0xffffffffu, mw != 0xffffffffu)) {
                uint32_t r[32];
                ptx::tmem_ld32(tS + 32 * wd, r);
                ptx::tmem_ld_wait();
                ptx::reg_fence(r);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (!((mw >> j) & 1u)) r[j] = __float_as_uint(-INFINITY);
                ptx::tmem_st32(tS + 32 * wd, r);
              }
            }
            ptx::tmem_st_wait();
          }
          ptx::tmem_ld32(tS + 0, s0);
          ptx::tmem_ld32(tS + 32, s1);
          ptx::tmem_ld32(tS + 64, s2);
          ptx::tmem_ld32(tS + 96, s3);
          ptx::tmem_ld_wait();
          ptx::reg_fence(s0);
          ptx::reg_fence(s1);
          ptx::reg_fence(s2);
          ptx::reg_fence(s3);
          if (D == 128 && st == CHUNK_PARTIAL) {
            // At head_dim 128 the mask is applied in registers, built by
            // the loop form (see chunk_key_mask_compact).
            uint32_t mk[4];
            chunk_key_mask_compact(it.a, wlo, whi, P.kb, P.kb_log2, mk);
#pragma unroll
            for (int j = 0; j < 128; ++j)
              if (!((mk[j >> 5] >> (j & 31)) & 1u)) s[j] = __float_as_uint(-INFINITY);
          }
        };
        // Maximum of the row's scores, log2 domain.
        auto row_max = [&]() {
          float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
          for (int j = 0; j < 128; j += 8) {
            a0 = ptx::max3(a0, __uint_as_float(s[j]), __uint_as_float(s[j + 1]));
            a1 = ptx::max3(a1, __uint_as_float(s[j + 2]), __uint_as_float(s[j + 3]));
            a2 = ptx::max3(a2, __uint_as_float(s[j + 4]), __uint_as_float(s[j + 5]));
            a3 = ptx::max3(a3, __uint_as_float(s[j + 6]), __uint_as_float(s[j + 7]));
          }
          return ptx::max3(a0, a1, fmaxf(a2, a3)) * sl2;
        };
        // P = 2^(score * scale - m_ref), packed in place into s[0..63]; returns
        // the row sum of P.
        auto exp_pass = [&](float m_ref) {
          const uint64_t scale2 = ptx::f2(sl2, sl2);
          const uint64_t negm2 = ptx::f2(-m_ref, -m_ref);
          uint64_t acc0 = ptx::f2(0.f, 0.f), acc1 = acc0, acc2 = acc0, acc3 = acc0;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const uint64_t x = ptx::f2_fma(
                ptx::f2(__uint_as_float(s[2 * j]), __uint_as_float(s[2 * j + 1])), scale2, negm2);
            float x0, x1, p0, p1;
            ptx::f2_split(x, x0, x1);
            if (emulate_pair(j)) {
              ptx::exp2_poly_x2(x0, x1, p0, p1);
            } else {
              p0 = ptx::ex2(x0);
              p1 = ptx::ex2(x1);
            }
            const uint64_t p = ptx::f2(p0, p1);
            switch (j & 3) {
              case 0: acc0 = ptx::f2_add(acc0, p); break;
              case 1: acc1 = ptx::f2_add(acc1, p); break;
              case 2: acc2 = ptx::f2_add(acc2, p); break;
              default: acc3 = ptx::f2_add(acc3, p); break;
            }
            if constexpr (C::E4M3) {
              // four keys per 32-bit column: pair j - 1 in bytes 0-1, pair j in 2-3
              if (j & 1)
                s[j >> 1] = ptx::pack_e4m3x4(__uint_as_float(s[2 * j - 2]),
                                             __uint_as_float(s[2 * j - 1]), p0, p1);
              else {
                s[2 * j] = __float_as_uint(p0);   // kept until pair j + 1 is done
                s[2 * j + 1] = __float_as_uint(p1);
              }
            } else {
              s[j] = ptx::pack_half2<F16>(p0, p1);
            }
          }
          float q0, q1, q2, q3, q4, q5, q6, q7;
          ptx::f2_split(acc0, q0, q1);
          ptx::f2_split(acc1, q2, q3);
          ptx::f2_split(acc2, q4, q5);
          ptx::f2_split(acc3, q6, q7);
          return ((q0 + q1) + (q2 + q3)) + ((q4 + q5) + (q6 + q7));
        };
        // With a reference m from earlier chunks the exponentials start at
        // once; the reference is moved (and the chunk redone from the scores
        // still in TMEM) only when a row's sum -- an upper bound of its largest
        // P -- exceeds P_LIMIT.  Without a reference yet (first chunk, or rows
        // masked so far) the chunk's own maximum becomes the reference first.
        float m_new = m, alpha = 1.f, sum;
        bool need = false;
        if constexpr (D == 64) {
          // One copy of the score load, the row maximum and the exponential
          // pass serves every path (the loop runs a second time only for a
          // redo): at head_dim 64 the softmax loop's code then stays small
          // enough for the instruction cache.
          bool fresh = __any_sync(0xffffffffu, m == -INFINITY);
#pragma unroll 1
          for (;;) {
            load_scores();
            float m_use = m;
            if (fresh) {
              const float mx2 = row_max() - C::POFF;
              need = mx2 > m;
              m_new = need ? mx2 : m;
              m_use = (m_new == -INFINITY) ? 0.f : m_new;
              alpha = need ? ptx::ex2(m - m_use) : 1.f;
            }
            sum = exp_pass(m_use);
            if (fresh || !__any_sync(0xffffffffu, !(sum <= C::PLIM))) break;
            fresh = true;
          }
        } else {
          // At head_dim 128 the straight-line form (a copy of the pass per
          // path) schedules better and the loop's code fits either way.
          load_scores();
          if (__any_sync(0xffffffffu, m == -INFINITY)) {
            const float mx2 = row_max() - C::POFF;
            need = mx2 > m;
            m_new = need ? mx2 : m;
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            alpha = need ? ptx::ex2(m - m_use) : 1.f;
            sum = exp_pass(m_use);
          } else {
            sum = exp_pass(m);
            if (__any_sync(0xffffffffu, !(sum <= C::PLIM))) {
              load_scores();
              const float mx2 = row_max() - C::POFF;
              need = mx2 > m;
              m_new = need ? mx2 : m;
              alpha = need ? ptx::ex2(m - m_new) : 1.f;
              sum = exp_pass(m_new);
            }
          }
        }
        const bool warp_need = __any_sync(0xffffffffu, need);
        ptx::tmem_st32(tS + 0, s0);
        if constexpr (!C::E4M3) ptx::tmem_st32(tS + 32, s1);
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
        int rr = row;
        asm volatile("" : "+r"(rr));  // recompute, do not carry the coordinates
        int g[3];
        query_coord(rr, g);
        const bool valid = B.exists && g[0] < P.g.L[0] && g[1] < P.g.L[1] && g[2] < P.g.L[2];
        const long long token = full_token(P.map, g[0], g[1], g[2]);
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
              pk[j] = ptx::pack_half2<F16>(__uint_as_float(o[2 * j]) * inv_l,
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

__global__ void exp2_poly_selftest_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    ptx::exp2_poly_x2(x[i], x[i + 1], y[i], y[i + 1]);
  } else if (i < n) {
    float dummy;
    ptx::exp2_poly_x2(x[i], 0.f, y[i], dummy);
  }
}

// ------------------------------------------------------------ host side --
bool encode_map(CUtensorMap* m, const void* ptr, const TcLaunch& L, const int box[3]) {
  return encode_grid_map_dil(m, ptr, L.dt, L.D, L.g.L, L.map, L.BH, L.N, box);
}

template <int D, int DT>
cudaError_t launch_d(const TcLaunch& L, cudaStream_t stream, char* err, int errlen) {
  CUtensorMap mq, mk, mv;
  if (!encode_map(&mq, L.q, L, L.t.qb) || !encode_map(&mk, L.k, L, L.kb) ||
      !encode_map(&mv, L.v, L, L.kb)) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled failed (pointer alignment or shape)");
    return cudaErrorInvalidValue;
  }
  const size_t smem = smem_bytes<D, DT>();
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    // setmaxnreg.inc waits for registers that the .dec of warpgroup 0 frees;
    // refuse to launch if the compiled register count could not cover the split.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, tc_fwd_kernel<D, DT>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * TC_THREADS < REGS_NEEDED) {
      snprintf(err, errlen, "kernel compiled with %d registers/thread; the register split needs %d",
               fa.numRegs, (REGS_NEEDED + TC_THREADS - 1) / TC_THREADS);
      return cudaErrorInvalidConfiguration;
    }
    e = cudaFuncSetAttribute(tc_fwd_kernel<D, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  const long long npairs = (L.t.nblocks + 1) / 2;
  const long long grid = npairs * L.BH;
  if (grid <= 0 || grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  tc_fwd_kernel<D, DT><<<(unsigned)grid, TC_THREADS, smem, stream>>>(mq, mk, mv, L);
  return cudaGetLastError();
}

}  // namespace

// [BH, X1, X2, X3, D] bf16 / f16 / E4M3 as a 5-d tensor (D, X3, X2, X1, BH).
// Inner box: 64 elements of 16-bit types, D elements of E4M3 (one row), with
// the swizzle of its width in bytes (128 B, or 64 B for E4M3 at head_dim 64).
bool encode_grid_map(CUtensorMap* m, const void* ptr, int dt, int D, const int L[3], int BH,
                     int N, const int box[3]) {
  return encode_grid_map_dil(m, ptr, dt, D, L, identity_map(L), BH, N, box);
}

// Residue class of a dilated grid: coordinate x of dimension d steps map.dil[d]
// tokens of the full grid, and the class starts at token full_token(map, 0, 0, 0).
bool encode_grid_map_dil(CUtensorMap* m, const void* ptr, int dt, int D, const int L[3],
                         const DilMap& map, int BH, int N, const int box[3]) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (!enc) return false;
  const bool e4m3 = dt == 2;
  const cuuint64_t es = e4m3 ? 1 : 2;
  cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)L[2], (cuuint64_t)L[1], (cuuint64_t)L[0],
                        (cuuint64_t)BH};
  const cuuint64_t row = (cuuint64_t)D * es;
  cuuint64_t strides[4] = {(cuuint64_t)map.dil[2] * row,
                           (cuuint64_t)map.dil[1] * map.Lf[2] * row,
                           (cuuint64_t)map.dil[0] * map.Lf[1] * map.Lf[2] * row,
                           (cuuint64_t)N * row};
  ptr = static_cast<const char*>(ptr) + (size_t)full_token(map, 0, 0, 0) * row;
  const cuuint32_t inner = e4m3 ? (cuuint32_t)D : 64;
  cuuint32_t boxd[5] = {inner, (cuuint32_t)box[2], (cuuint32_t)box[1], (cuuint32_t)box[0], 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUtensorMapDataType ty = e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                      : (dt == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  const CUtensorMapSwizzle sw =
      inner * es == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = enc(m, ty, 5, const_cast<void*>(ptr), dims, strides, boxd, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t launch_exp2_selftest(const float* x, float* y, int n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int threads = 256;
  const int blocks = ((n + 1) / 2 + threads - 1) / threads;
  exp2_poly_selftest_kernel<<<blocks, threads, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_tc(const TcLaunch& L0, cudaStream_t stream, char* err, int errlen) {
  TcLaunch L = L0;
  for (int d = 0; d < 3; ++d) {
    if (L.t.qb[d] > 256 || L.kb[d] > 256) return cudaErrorNotSupported;
    if (L.kb[d] & (L.kb[d] - 1)) return cudaErrorNotSupported;  // powers of two only
    int lg = 0;
    while ((1 << lg) < L.kb[d]) ++lg;
    L.kb_log2[d] = lg;
  }
  if (L.t.qb[0] * L.t.qb[1] * L.t.qb[2] != BLOCK_M || L.kb[0] * L.kb[1] * L.kb[2] != CHUNK_N)
    return cudaErrorNotSupported;
  switch (L.D * 4 + L.dt) {
    case 64 * 4 + DT_BF16: return launch_d<64, DT_BF16>(L, stream, err, errlen);
    case 64 * 4 + DT_F16: return launch_d<64, DT_F16>(L, stream, err, errlen);
    case 64 * 4 + DT_E4M3: return launch_d<64, DT_E4M3>(L, stream, err, errlen);
    case 128 * 4 + DT_BF16: return launch_d<128, DT_BF16>(L, stream, err, errlen);
    case 128 * 4 + DT_F16: return launch_d<128, DT_F16>(L, stream, err, errlen);
    case 128 * 4 + DT_E4M3: return launch_d<128, DT_E4M3>(L, stream, err, errlen);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace na
