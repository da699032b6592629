// C-ABI layer: argument validation, schedule planning, kernel dispatch and
// the device status word.  Declarations and the contract are in include/na.h.
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <array>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "../../include/na.h"
#include "na_internal.h"

using namespace na;

namespace {

thread_local char g_err[512] = "";

na_status fail(na_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return s;
}

constexpr int MAX_DEVICES = 64;
std::mutex g_status_mu;
int* g_status[MAX_DEVICES] = {nullptr};

// ------------------------------------------------------------ problem --
struct Problem {
  int ndim = 0, D = 0;
  Geom g{};
  int dil[3] = {1, 1, 1};    // dilation per (padded) dimension
  int tile[3] = {0, 0, 0};   // 0 = none given
  int dtype = NA_BF16;
  na_options opt{};
};

struct Plan {
  int kernel = NA_KERNEL_SIMT;
  QTiling t{};
  int kb[3] = {1, 1, 1};
  // window-gather kernel: query tile staged per CTA (gq[0] == 0: direct reads),
  // its shared memory, and the K / V rows staged per head
  int gq[3] = {0, 0, 0};
  int gqrows = 0, gkrows = 0;   // rows of a stage's Q region and of its K / V regions
  int gnst = 0;                 // stages (1 or 2)
  int gsmem = 0;
  long long gstaged = 0;
};

// Key-box extents along one dimension for query tiles of extent t: the
// largest box (shared memory) and the sum over tile positions (rows staged).
void gather_box_extent(const Geom& g, int d, int t, int& kmax, long long& sum) {
  kmax = 0;
  sum = 0;
  for (int o = 0; o < g.L[d]; o += t) {
    const int n = imin(t, g.L[d] - o);
    int a, b, c, e;
    window_range(g.L[d], g.w[d], g.s[d], g.m[d], o, a, b);
    window_range(g.L[d], g.w[d], g.s[d], g.m[d], o + n - 1, c, e);
    kmax = imax(kmax, e - a);
    sum += e - a;
  }
}

// Query tile and stage count of the window-gather kernel's staged form,
// among boxes of 2^k queries (k <= 8) no wider than the grid needs.  A stage
// holds a tile's queries and the K and V rows of its key box.  Preference, in
// order: a tile that fills a round of the CTA's threads (or the whole grid)
// with two stages that leave room for two CTAs per SM; the same with one
// stage; any tile with two CTAs per SM; a full-round tile alone on its SM;
// any tile that fits at all.  Two stages wherever they fit the tier's
// budget.  Within the first tier that has one, the tile that stages the
// fewest K / V rows per head, counting each tile as 32 rows of fixed cost.
// No fitting tile (a wide window): gq stays 0 and the kernel reads K and V
// directly.
void choose_gather_tile(const Problem& P, Plan& plan) {
  const int esz = P.dtype == NA_F32 ? 4 : 2;
  const long long ntok = (long long)P.g.L[0] * P.g.L[1] * P.g.L[2];
  const long long fill = std::min<long long>(gather_tile_queries_per_round(P.D), ntok);
  constexpr int TIERS = 5;
  double best[TIERS] = {};
  bool found[TIERS] = {};
  Plan pick[TIERS];
  for (int lp = 8; lp >= 0; --lp) {
    for (int e0 = 0; e0 <= lp; ++e0)
      for (int e1 = 0; e0 + e1 <= lp; ++e1) {
        const int e[3] = {e0, e1, lp - e0 - e1};
        int t[3], km[3];
        long long sm[3];
        bool ok = true;
        long long box = 1, staged = 1, tiles = 1, tq = 1;
        for (int d = 0; d < 3 && ok; ++d) {
          t[d] = 1 << e[d];
          if (t[d] > 1 && t[d] / 2 >= P.g.L[d]) ok = false;   // no wider than needed
          if (!ok) break;
          gather_box_extent(P.g, d, t[d], km[d], sm[d]);
          box *= km[d];
          staged *= sm[d];
          tiles *= (P.g.L[d] + t[d] - 1) / t[d];
          tq *= std::min(t[d], P.g.L[d]);
        }
        if (!ok) continue;
        const long long one = gather_smem_bytes(tq, box, P.D, esz, 1);
        const long long two = gather_smem_bytes(tq, box, P.D, esz, 2);
        const bool full = tq >= fill;
        int tier, nst;
        if (full && two <= GATHER_SMEM_TWO_PER_SM) tier = 0, nst = 2;
        else if (full && one <= GATHER_SMEM_TWO_PER_SM) tier = 1, nst = 1;
        else if (one <= GATHER_SMEM_TWO_PER_SM) tier = 2, nst = two <= GATHER_SMEM_TWO_PER_SM ? 2 : 1;
        else if (full && one <= GATHER_SMEM_MAX) tier = 3, nst = two <= GATHER_SMEM_MAX ? 2 : 1;
        else if (one <= GATHER_SMEM_MAX) tier = 4, nst = two <= GATHER_SMEM_MAX ? 2 : 1;
        else continue;
        const double cost = (double)staged + 32.0 * (double)tiles;
        if (!found[tier] || cost < best[tier] - 1e-9) {
          found[tier] = true;
          best[tier] = cost;
          for (int d = 0; d < 3; ++d) pick[tier].gq[d] = t[d];
          pick[tier].gqrows = (int)tq;
          pick[tier].gkrows = (int)box;
          pick[tier].gnst = nst;
          pick[tier].gsmem = (int)(nst == 2 ? two : one);
          pick[tier].gstaged = staged;
        }
      }
  }
  for (int tier = 0; tier < TIERS; ++tier) {
    if (!found[tier]) continue;
    for (int d = 0; d < 3; ++d) plan.gq[d] = pick[tier].gq[d];
    plan.gqrows = pick[tier].gqrows;
    plan.gkrows = pick[tier].gkrows;
    plan.gnst = pick[tier].gnst;
    plan.gsmem = pick[tier].gsmem;
    plan.gstaged = pick[tier].gstaged;
    return;
  }
  plan.gq[0] = plan.gq[1] = plan.gq[2] = 0;
  plan.gqrows = plan.gkrows = plan.gnst = plan.gsmem = 0;
  plan.gstaged = 0;
}

na_status read_problem(const int dims[2], const int* grid, const int* window, const int* stride,
                       const int* tile, na_dtype dtype, const na_options* opt, Problem& P) {
  if (!dims) return fail(NA_ERR_INVALID_ARG, "dims is NULL");
  const int nd = dims[0], D = dims[1];
  if (nd < 1 || nd > 3) return fail(NA_ERR_INVALID_ARG, "ndim=%d not in 1..3", nd);
  if (D <= 0) return fail(NA_ERR_INVALID_ARG, "head_dim=%d must be positive", D);
  if (D != 32 && D != 64 && D != 128)
    return fail(NA_ERR_UNSUPPORTED, "head_dim=%d not in {32, 64, 128}", D);
  if (!grid || !window) return fail(NA_ERR_INVALID_ARG, "grid or window is NULL");
  if (dtype != NA_F32 && dtype != NA_BF16 && dtype != NA_F16 && dtype != NA_E4M3)
    return fail(NA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  P.ndim = nd;
  P.D = D;
  P.dtype = dtype;
  const int pad = 3 - nd;
  for (int d = 0; d < 3; ++d) {
    P.g.L[d] = P.g.w[d] = P.g.s[d] = 1;
    P.g.m[d] = WIN_CLAMPED;
    P.tile[d] = tile ? 1 : 0;
  }
  long long N = 1;
  for (int i = 0; i < nd; ++i) {
    const int L = grid[i], w = window[i], s = stride ? stride[i] : 1;
    if (L < 1) return fail(NA_ERR_INVALID_ARG, "grid[%d]=%d must be >= 1", i, L);
    if (w < 1 || w > L)
      return fail(NA_ERR_INVALID_ARG, "window[%d]=%d must be in 1..grid[%d]=%d", i, w, i, L);
    if (s < 1 || s > w)
      return fail(NA_ERR_INVALID_ARG, "stride[%d]=%d must be in 1..window[%d]=%d", i, s, i, w);
    if (tile && tile[i] < 1) return fail(NA_ERR_INVALID_ARG, "tile[%d]=%d must be >= 1", i, tile[i]);
    P.g.L[pad + i] = L;
    P.g.w[pad + i] = w;
    P.g.s[pad + i] = s;
    if (tile) P.tile[pad + i] = tile[i];
    N *= L;
    // Token counts travel to the kernels as int: 2^31 tokens or more are refused.
    if (N >= (1LL << 31)) return fail(NA_ERR_UNSUPPORTED, "grid has 2^31 tokens or more");
  }
  P.opt = opt ? *opt : na_default_options();
  if (P.opt.kernel < NA_KERNEL_AUTO || P.opt.kernel > NA_KERNEL_GATHER)
    return fail(NA_ERR_INVALID_ARG, "unknown kernel selector %d", P.opt.kernel);
  for (int i = 0; i < nd; ++i) {
    const int m = P.opt.window_mode[i];
    if (m < NA_WINDOW_CLAMPED || m > NA_WINDOW_CAUSAL)
      return fail(NA_ERR_INVALID_ARG, "window_mode[%d]=%d is not a na_window_mode", i, m);
    P.g.m[pad + i] = m;
    const int dl = P.opt.dilation[i] == 0 ? 1 : P.opt.dilation[i];
    if (dl < 1)
      return fail(NA_ERR_INVALID_ARG, "dilation[%d]=%d must be >= 1", i, P.opt.dilation[i]);
    if ((long long)P.g.w[pad + i] * dl > P.g.L[pad + i])
      return fail(NA_ERR_INVALID_ARG, "window[%d] * dilation[%d] = %lld exceeds grid[%d]=%d", i,
                  i, (long long)P.g.w[pad + i] * dl, i, P.g.L[pad + i]);
    P.dil[pad + i] = dl;
  }
  return NA_OK;
}

bool dilated(const Problem& P) { return P.dil[0] > 1 || P.dil[1] > 1 || P.dil[2] > 1; }

// Residue class (r0, r1, r2) of a dilated problem as a problem of its own:
// per dimension the ceil((L - r) / dil) coordinates r, r + dil, ...  The tile
// hint, which describes the full grid, is dropped.
Problem residue_problem(const Problem& P, const int r[3], DilMap& map) {
  Problem Q = P;
  for (int d = 0; d < 3; ++d) {
    Q.g.L[d] = (P.g.L[d] - r[d] + P.dil[d] - 1) / P.dil[d];
    Q.dil[d] = 1;
    Q.tile[d] = 0;
    map.dil[d] = P.dil[d];
    map.res[d] = r[d];
    map.Lf[d] = P.g.L[d];
  }
  return Q;
}

// Shapes of `prod` tokens (powers of two per dimension, <= 256 each), with
// extent 1 on dimensions the problem does not have.
std::vector<std::array<int, 3>> shape_candidates(const Problem& P, int prod) {
  std::vector<std::array<int, 3>> out;
  int lp = 0;
  while ((1 << lp) < prod) ++lp;
  for (int e0 = 0; e0 <= lp; ++e0)
    for (int e1 = 0; e0 + e1 <= lp; ++e1) {
      const int e2 = lp - e0 - e1;
      const int e[3] = {e0, e1, e2};
      bool okc = true;
      for (int d = 0; d < 3; ++d) {
        if (P.g.L[d] == 1 && e[d] != 0) okc = false;
        if (e[d] > 8) okc = false;
      }
      if (okc) out.push_back({1 << e0, 1 << e1, 1 << e2});
    }
  return out;
}

struct Cost {
  double cost = 0;
  long long loads = 0, full = 0, partial = 0;
};

// Walk the CTA work items exactly like the kernels do.  group = 2 for the
// tensor-core kernel (a CTA owns a pair of blocks), 1 for the CUDA-core one.
Cost walk(const Geom& g, const QTiling& t, const int kb[3], int group, int max_items) {
  Cost c;
  const int items = (t.nblocks + group - 1) / group;
  const int n = (max_items > 0 && items > max_items) ? max_items : items;
  for (int i = 0; i < n; ++i) {
    const int it = (n == items) ? i : (int)((long long)i * items / n);
    BlockInfo bi[2];
    for (int b = 0; b < group; ++b) block_info(g, t, it * group + b, bi[b]);
    ChunkGrid cg;
    chunk_grid_for(bi, group, kb, cg);
    for (int ch = 0; ch < cg.total; ++ch) {
      int a[3];
      chunk_origin(cg, kb, ch, a);
      int active = 0;
      for (int b = 0; b < group; ++b) {
        const int st = chunk_status(bi[b], a, kb);
        if (st == CHUNK_EMPTY) continue;
        ++active;
        if (st == CHUNK_FULL) ++c.full; else ++c.partial;
        c.cost += (st == CHUNK_FULL) ? 1.0 : 1.3;
      }
      if (active) {
        ++c.loads;
        c.cost += 0.2 + ((group == 2 && active == 1) ? 0.5 : 0.0);
      }
    }
  }
  if (n != items && n > 0) c.cost *= (double)items / n;
  return c;
}

bool build_tiling(const Problem& P, const int qb[3], int kernel, QTiling& t) {
  int tl[3] = {qb[0], qb[1], qb[2]};
  if (P.tile[0] && kernel == NA_KERNEL_TC) {
    const int tprod = P.tile[0] * P.tile[1] * P.tile[2];
    if (tprod >= qb[0] * qb[1] * qb[2]) {
      bool nest = true;
      for (int d = 0; d < 3; ++d)
        if (P.tile[d] % qb[d]) nest = false;
      if (nest)
        for (int d = 0; d < 3; ++d) tl[d] = P.tile[d];
      else
        return false;
    } else {
      for (int d = 0; d < 3; ++d)
        if (qb[d] % P.tile[d]) return false;
    }
  }
  return make_tiling(P.g, qb, tl, t) == 0;
}

std::mutex g_plan_mu;
std::map<std::vector<long long>, Plan> g_plans;

na_status make_plan(const Problem& P, Plan& out) {
  int kernel = P.opt.kernel;
  const bool half = P.dtype == NA_BF16 || P.dtype == NA_F16;
  const long long wkeys = (long long)P.g.w[0] * P.g.w[1] * P.g.w[2];
  if (P.dtype == NA_E4M3) {
    // 8-bit inputs run on the tensor cores only (kind::f8f6f4 products).
    if (kernel == NA_KERNEL_SIMT || kernel == NA_KERNEL_GATHER)
      return fail(NA_ERR_UNSUPPORTED, "E4M3 inputs run on the tensor-core kernel only");
    kernel = NA_KERNEL_TC;
    if (P.D != 64 && P.D != 128)
      return fail(NA_ERR_UNSUPPORTED, "E4M3 inputs need head_dim 64 or 128");
  }
  if (kernel == NA_KERNEL_AUTO && wkeys <= NA_GATHER_MAX_KEYS) kernel = NA_KERNEL_GATHER;
  if (kernel == NA_KERNEL_AUTO)
    kernel = (half && (P.D == 64 || P.D == 128)) ? NA_KERNEL_TC : NA_KERNEL_SIMT;
  if (kernel == NA_KERNEL_TC && !half && P.dtype != NA_E4M3)
    return fail(NA_ERR_UNSUPPORTED, "the tensor-core kernel takes bf16, f16 or E4M3 only");
  if (kernel == NA_KERNEL_TC && P.D != 64 && P.D != 128)
    return fail(NA_ERR_UNSUPPORTED, "the tensor-core kernel takes head_dim 64 or 128");

  std::vector<long long> key = {P.ndim, P.D, P.dtype, kernel};
  for (int d = 0; d < 3; ++d) {
    key.insert(key.end(), {P.g.L[d], P.g.w[d], P.g.s[d], P.g.m[d], P.tile[d], P.opt.qblock[d],
                           P.opt.kvchunk[d]});
  }
  {
    std::lock_guard<std::mutex> lk(g_plan_mu);
    auto it = g_plans.find(key);
    if (it != g_plans.end()) {
      out = it->second;
      return NA_OK;
    }
  }
  if (kernel == NA_KERNEL_GATHER) {
    // No blocks or chunks: each query on its own with exactly its window's
    // keys; the query tile staged per CTA is chosen here (and cached).
    const int one[3] = {1, 1, 1};
    Plan g;
    g.kernel = NA_KERNEL_GATHER;
    if (make_tiling(P.g, one, one, g.t) != 0)
      return fail(NA_ERR_UNSUPPORTED, "window-gather kernel: grid too large");
    choose_gather_tile(P, g);
    {
      std::lock_guard<std::mutex> lk(g_plan_mu);
      g_plans[key] = g;
    }
    out = g;
    return NA_OK;
  }
  const int qprod = kernel == NA_KERNEL_TC ? 128 : 128 / (P.D / 32);
  const int kprod = kernel == NA_KERNEL_TC ? 128 : 32;
  const int group = kernel == NA_KERNEL_TC ? 2 : 1;

  std::vector<std::array<int, 3>> qcands, kcands;
  if (P.opt.qblock[0] > 0) {
    const int* q = P.opt.qblock;
    if (q[0] * q[1] * q[2] != qprod)
      return fail(NA_ERR_UNSUPPORTED, "qblock product must be %d for this kernel", qprod);
    qcands.push_back({q[0], q[1], q[2]});
  } else {
    qcands = shape_candidates(P, qprod);
  }
  if (P.opt.kvchunk[0] > 0) {
    const int* k = P.opt.kvchunk;
    if (k[0] * k[1] * k[2] != kprod)
      return fail(NA_ERR_UNSUPPORTED, "kvchunk product must be %d for this kernel", kprod);
    for (int d = 0; d < 3; ++d)
      if (k[d] > 256) return fail(NA_ERR_UNSUPPORTED, "kvchunk extents must be <= 256");
    kcands.push_back({k[0], k[1], k[2]});
  } else {
    kcands = shape_candidates(P, kprod);
  }

  bool found = false;
  Plan best;
  double best_cost = 0;
  for (int pass = 0; pass < 2 && !found; ++pass) {
    // pass 0 honours the tile hint; pass 1 drops it (it only orders queries).
    Problem Q = P;
    if (pass == 1) Q.tile[0] = Q.tile[1] = Q.tile[2] = 0;
    for (const auto& qb : qcands) {
      QTiling t;
      if (!build_tiling(Q, qb.data(), kernel, t)) continue;
      for (const auto& kb : kcands) {
        const Cost c = walk(Q.g, t, kb.data(), group, 48);
        if (!found || c.cost < best_cost - 1e-9) {
          found = true;
          best_cost = c.cost;
          best.kernel = kernel;
          best.t = t;
          for (int d = 0; d < 3; ++d) best.kb[d] = kb[d];
        }
      }
    }
  }
  if (!found) return fail(NA_ERR_UNSUPPORTED, "no query block / key chunk shape fits this grid");
  {
    std::lock_guard<std::mutex> lk(g_plan_mu);
    g_plans[key] = best;
  }
  out = best;
  return NA_OK;
}

long long default_timeout_ns() {
  const char* e = getenv("NA_WAIT_TIMEOUT_MS");
  if (e) {
    const long long ms = atoll(e);
    if (ms > 0) return ms * 1000000LL;
  }
  return 4000LL * 1000000LL;
}

na_status status_word(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(NA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= MAX_DEVICES) return fail(NA_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status[dev]) {
    int* p = nullptr;
    e = cudaMalloc(&p, sizeof(int));
    if (e != cudaSuccess) return fail(NA_ERR_CUDA, "cudaMalloc(status): %s", cudaGetErrorString(e));
    e = cudaMemset(p, 0, sizeof(int));
    if (e != cudaSuccess) return fail(NA_ERR_CUDA, "cudaMemset(status): %s", cudaGetErrorString(e));
    g_status[dev] = p;
  }
  *out = g_status[dev];
  return NA_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The tensor-core kernel's input-type code of a na_dtype (0 bf16, 1 f16, 2 E4M3).
int tc_dtype(int d) { return d == NA_F16 ? 1 : (d == NA_E4M3 ? 2 : 0); }

// ---------------------------------------------- allocation-free variant --
// Device scratch of na_forward_noalloc: a fixed array in the library's own
// device image instead of memory from cudaMalloc.  Every GPU that loads the
// library holds these bytes until the process exits.  The tensor-core kernel
// needs one 4-byte status word of it.
constexpr size_t NOALLOC_SCRATCH_BYTES = 256;
constexpr size_t TC_SCRATCH_BYTES = sizeof(int);
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[MAX_DEVICES] = {nullptr};

// The device address of g_noalloc_scratch on the current device, looked up
// once per device.  On the host the array's name is only a stand-in for the
// device copy, so kernels must be given this address, never &g_noalloc_scratch.
na_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(NA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= MAX_DEVICES) return fail(NA_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(NA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return NA_OK;
}

// Plan and launch the forward kernel for one grid (the whole problem, or one
// residue class of a dilated one: `map` takes its coordinates to the full
// grid's tokens).
na_status launch_forward(const Problem& P, const DilMap& map, long long BH, const void* q,
                         const void* k, const void* v, void* out, float* lse, void* stream) {
  Plan plan;
  na_status st = make_plan(P, plan);
  if (st != NA_OK) return st;
  const long long N = (long long)map.Lf[0] * map.Lf[1] * map.Lf[2];   // tokens per head
  const float scale = P.opt.scale > 0.f ? P.opt.scale : 1.0f / sqrtf((float)P.D);
  const float log2e = 1.4426950408889634f;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  if (plan.kernel == NA_KERNEL_TC) {
    int* status = nullptr;
    st = status_word(&status);
    if (st != NA_OK) return st;
    TcLaunch L;
    L.g = P.g;
    L.t = plan.t;
    for (int d = 0; d < 3; ++d) L.kb[d] = plan.kb[d];
    L.map = map;
    L.BH = (int)BH;
    L.N = (int)N;
    L.D = P.D;
    L.dt = tc_dtype(P.dtype);
    L.scale_log2 = scale * log2e;
    L.q = q; L.k = k; L.v = v; L.out = out; L.lse = lse;
    L.status = status;
    L.timeout_ns = P.opt.wait_timeout_ns > 0 ? P.opt.wait_timeout_ns : default_timeout_ns();
    L.debug_flags = P.opt.debug_flags;
    char msg[256] = "";
    cudaError_t e = launch_tc(L, s, msg, sizeof msg);
    if (e == cudaErrorNotSupported)
      return fail(NA_ERR_UNSUPPORTED, "tensor-core kernel does not take this shape");
    if (e != cudaSuccess)
      return fail(NA_ERR_CUDA, "tensor-core launch: %s %s", cudaGetErrorString(e), msg);
    return NA_OK;
  }
  SimtLaunch L;
  L.g = P.g;
  L.t = plan.t;
  for (int d = 0; d < 3; ++d) L.kb[d] = plan.kb[d];
  L.map = map;
  L.BH = (int)BH;
  L.N = (int)N;
  L.D = P.D;
  L.dtype = P.dtype;
  L.scale_log2 = scale * log2e;
  L.q = q; L.k = k; L.v = v; L.out = out; L.lse = lse;
  if (plan.kernel == NA_KERNEL_GATHER) {
    GatherLaunch G;
    G.g = P.g;
    G.map = map;
    G.BH = (int)BH;
    G.N = (int)N;
    G.D = P.D;
    G.dtype = P.dtype;
    G.scale_log2 = scale * log2e;
    G.q = q; G.k = k; G.v = v; G.out = out; G.lse = lse;
    for (int d = 0; d < 3; ++d) {
      G.qt[d] = plan.gq[d];
      G.nt[d] = plan.gq[0] > 0 ? (P.g.L[d] + plan.gq[d] - 1) / plan.gq[d] : 0;
    }
    G.qrows = plan.gqrows;
    G.krows = plan.gkrows;
    G.nstages = plan.gnst;
    G.smem_bytes = plan.gsmem;
    G.status = nullptr;
    G.timeout_ns = P.opt.wait_timeout_ns > 0 ? P.opt.wait_timeout_ns : default_timeout_ns();
    G.debug_flags = P.opt.debug_flags;
    if (plan.gq[0] > 0) {
      st = status_word(&G.status);
      if (st != NA_OK) return st;
    }
    cudaError_t e = launch_gather(G, s);
    if (e == cudaErrorNotSupported) return fail(NA_ERR_UNSUPPORTED, "window-gather kernel: shape");
    if (e != cudaSuccess)
      return fail(NA_ERR_CUDA, "window-gather launch: %s", cudaGetErrorString(e));
    return NA_OK;
  }
  cudaError_t e = launch_simt(L, s);
  if (e == cudaErrorNotSupported) return fail(NA_ERR_UNSUPPORTED, "CUDA-core kernel: shape");
  if (e != cudaSuccess) return fail(NA_ERR_CUDA, "CUDA-core launch: %s", cudaGetErrorString(e));
  return NA_OK;
}

// Schedule statistics of one grid (see na_plan_info).
na_status plan_info(const Problem& P, na_plan_info* info) {
  na_status st;
  Plan plan;
  st = make_plan(P, plan);
  if (st != NA_OK) return st;
  // sum over queries of the window size = product over dimensions of the sum
  // over coordinates of the 1-D window length (the window is a product).
  long long useful = 1;
  for (int d = 0; d < 3; ++d) {
    long long sum = 0;
    for (int i = 0; i < P.g.L[d]; ++i) {
      int lo, hi;
      window_range(P.g.L[d], P.g.w[d], P.g.s[d], P.g.m[d], i, lo, hi);
      sum += hi - lo;
    }
    useful *= sum;
  }
  const long long N = (long long)P.g.L[0] * P.g.L[1] * P.g.L[2];
  const bool gather = plan.kernel == NA_KERNEL_GATHER;
  const int group = plan.kernel == NA_KERNEL_TC ? 2 : 1;
  Cost c{};
  if (gather) {
    // one (query, key) pair per unit, exactly the window's keys: no walk needed;
    // "chunks" loaded = K / V rows staged in shared memory (staged form) or
    // read per query (direct form)
    c.full = useful;
    c.partial = 0;
    c.loads = plan.gq[0] > 0 ? plan.gstaged : useful;
  } else {
    c = walk(P.g, plan.t, plan.kb, group, 0);
  }
  memset(info, 0, sizeof *info);
  info->kernel = plan.kernel;
  for (int d = 0; d < 3; ++d) {
    info->qblock[d] = plan.t.qb[d];
    info->kvchunk[d] = plan.kb[d];
    info->tile[d] = plan.t.tl[d];
  }
  const long long rows = (long long)plan.t.qb[0] * plan.t.qb[1] * plan.t.qb[2];
  const long long keys = (long long)plan.kb[0] * plan.kb[1] * plan.kb[2];
  info->query_blocks = plan.t.nblocks;
  info->ctas = (plan.t.nblocks + group - 1) / group;
  if (gather) {
    if (plan.gq[0] > 0) {
      info->ctas = 1;
      for (int d = 0; d < 3; ++d) {
        info->qblock[d] = plan.gq[d];
        info->tile[d] = plan.gq[d];
        info->ctas *= (P.g.L[d] + plan.gq[d] - 1) / plan.gq[d];
      }
    } else {
      const long long rpc = gather_rows_per_cta(P.D, P.dtype);
      info->ctas = (plan.t.nblocks + rpc - 1) / rpc;
    }
  }
  info->chunks_loaded = c.loads;
  info->units_full = c.full;
  info->units_partial = c.partial;
  info->computed_pairs = (c.full + c.partial) * rows * keys;
  info->useful_pairs = useful;
  // Speedup bound: dense attention (every window the whole grid) under the
  // same block / chunk shapes computes every (block, chunk) unit; this
  // schedule computes only the non-empty ones, each at full tile cost.
  info->dense_pairs = N * N;
  if (gather) {
    info->dense_units = N * N;
  } else {
    Geom dense = P.g;
    for (int d = 0; d < 3; ++d) {
      dense.w[d] = dense.L[d];
      dense.s[d] = 1;
      dense.m[d] = WIN_CLAMPED;
    }
    const Cost cd = walk(dense, plan.t, plan.kb, group, 0);
    info->dense_units = cd.full + cd.partial;
  }
  const long long units = c.full + c.partial;
  info->speedup_bound = units > 0 ? (double)info->dense_units / (double)units : 0.0;
  return NA_OK;
}

}  // namespace

extern "C" {

na_options na_default_options(void) {
  na_options o;
  memset(&o, 0, sizeof o);
  o.scale = 0.f;
  o.kernel = NA_KERNEL_AUTO;
  o.wait_timeout_ns = 0;
  return o;
}

const char* na_status_string(na_status s) {
  switch (s) {
    case NA_OK: return "NA_OK";
    case NA_ERR_INVALID_ARG: return "NA_ERR_INVALID_ARG";
    case NA_ERR_UNSUPPORTED: return "NA_ERR_UNSUPPORTED";
    case NA_ERR_CUDA: return "NA_ERR_CUDA";
    case NA_ERR_TIMEOUT: return "NA_ERR_TIMEOUT";
  }
  return "NA_ERR_UNKNOWN";
}

const char* na_last_error(void) { return g_err; }

int na_version(void) { return 100; }

na_status na_selftest_exp2(const float* x, float* y, int n, void* stream) {
  g_err[0] = 0;
  if (n < 0 || (n > 0 && (!x || !y))) return fail(NA_ERR_INVALID_ARG, "bad self-test arguments");
  cudaError_t e = launch_exp2_selftest(x, y, n, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(NA_ERR_CUDA, "exp2 self-test: %s", cudaGetErrorString(e));
  return NA_OK;
}

int na_window_start(int L, int w, int s, int i) {
  if (L < 1 || w < 1 || w > L || s < 1 || s > w || i < 0 || i >= L) return -1;
  return window_start(L, w, s, i);
}

int na_window_range(int L, int w, int s, int mode, int i, int* lo, int* hi) {
  if (L < 1 || w < 1 || w > L || s < 1 || s > w || i < 0 || i >= L || !lo || !hi) return -1;
  if (mode < NA_WINDOW_CLAMPED || mode > NA_WINDOW_CAUSAL) return -1;
  window_range(L, w, s, mode, i, *lo, *hi);
  return 0;
}

na_status na_forward_ex(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                        int heads, const int dims[2], const int* grid, const int* window,
                        const int* stride, const int* tile, na_dtype dtype,
                        const na_options* opt, void* stream) {
  g_err[0] = 0;
  if (!q || !k || !v || !out || !lse) return fail(NA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  if (B < 1 || heads < 1) return fail(NA_ERR_INVALID_ARG, "B=%d heads=%d must be >= 1", B, heads);
  Problem P;
  na_status st = read_problem(dims, grid, window, stride, tile, dtype, opt, P);
  if (st != NA_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(lse, 4))
    return fail(NA_ERR_INVALID_ARG, "q, k, v, out must be 16-byte aligned and lse 4-byte aligned");
  const long long BH = (long long)B * heads;
  if (BH > (1LL << 30)) return fail(NA_ERR_UNSUPPORTED, "B*heads too large");
  if (!dilated(P)) return launch_forward(P, identity_map(P.g.L), BH, q, k, v, out, lse, stream);
  // One launch per residue class, each a grid of its own (same stream, so
  // they run in order; each writes only its own class's rows).
  int r[3];
  for (r[0] = 0; r[0] < P.dil[0]; ++r[0])
    for (r[1] = 0; r[1] < P.dil[1]; ++r[1])
      for (r[2] = 0; r[2] < P.dil[2]; ++r[2]) {
        DilMap map;
        const Problem Q = residue_problem(P, r, map);
        st = launch_forward(Q, map, BH, q, k, v, out, lse, stream);
        if (st != NA_OK) return st;
      }
  return NA_OK;
}

na_status na_forward(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                     int heads, const int dims[2], const int* grid, const int* window,
                     const int* stride, const int* tile, na_dtype dtype, void* stream) {
  return na_forward_ex(q, k, v, out, lse, B, heads, dims, grid, window, stride, tile, dtype,
                       nullptr, stream);
}

na_status na_backward(const void* q, const void* k, const void* v, const void* out,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv,
                      float* delta, int B, int heads, const int dims[2], const int* grid,
                      const int* window, const int* stride, const int* tile, na_dtype dtype,
                      const na_options* opt, void* stream) {
  g_err[0] = 0;
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !delta)
    return fail(NA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  if (B < 1 || heads < 1) return fail(NA_ERR_INVALID_ARG, "B=%d heads=%d must be >= 1", B, heads);
  Problem P;
  na_status st = read_problem(dims, grid, window, stride, tile, dtype, opt, P);
  if (st != NA_OK) return st;
  const void* ptrs[] = {q, k, v, out, dout, dq, dk, dv};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return fail(NA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (!aligned(lse, 4) || !aligned(delta, 4))
    return fail(NA_ERR_INVALID_ARG, "lse and delta must be 4-byte aligned");
  const long long BH = (long long)B * heads;
  if (BH > (1LL << 30)) return fail(NA_ERR_UNSUPPORTED, "B*heads too large");
  if (P.dtype == NA_E4M3)
    return fail(NA_ERR_UNSUPPORTED, "the backward takes fp32, bf16 or f16 inputs (not E4M3)");
  const bool tc_ok = (P.dtype == NA_BF16 || P.dtype == NA_F16) && (P.D == 64 || P.D == 128);
  if (P.opt.kernel == NA_KERNEL_GATHER)
    return fail(NA_ERR_UNSUPPORTED, "the window-gather kernel is forward only");
  if (P.opt.kernel == NA_KERNEL_TC && !tc_ok)
    return fail(NA_ERR_UNSUPPORTED, "the tensor-core backward takes bf16 / f16, head_dim 64 or 128");
  const bool use_tc = tc_ok && P.opt.kernel != NA_KERNEL_SIMT;
  const float scale = P.opt.scale > 0.f ? P.opt.scale : 1.0f / sqrtf((float)P.D);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* status = nullptr;
  if (use_tc) {
    st = status_word(&status);
    if (st != NA_OK) return st;
  }
  // One grid (a dilated problem: each residue class as a grid of its own,
  // `map` taking its coordinates to full-grid tokens) -> its launch structs.
  auto simt_launch = [&](const Problem& Q, const DilMap& map, BwdLaunch& L) -> na_status {
    Problem Qs = Q;
    Qs.opt.kernel = NA_KERNEL_SIMT;
    Qs.opt.qblock[0] = Qs.opt.qblock[1] = Qs.opt.qblock[2] = 0;   // a TC plan's shapes do not fit
    Qs.opt.kvchunk[0] = Qs.opt.kvchunk[1] = Qs.opt.kvchunk[2] = 0;
    Plan plan;
    const na_status r = make_plan(Qs, plan);
    if (r != NA_OK) return r;
    L.g = Q.g;
    L.t = plan.t;
    for (int d = 0; d < 3; ++d) L.kb[d] = plan.kb[d];
    L.map = map;
    L.BH = (int)BH;
    L.N = map.Lf[0] * map.Lf[1] * map.Lf[2];
    L.D = Q.D;
    L.dtype = Q.dtype;
    L.scale = scale;
    L.scale_log2 = scale * 1.4426950408889634f;
    L.q = q; L.k = k; L.v = v; L.out = out; L.dout = dout; L.lse = lse; L.delta = delta;
    L.dq = dq; L.dk = dk; L.dv = dv;
    return NA_OK;
  };
  auto grads = [&](const Problem& Q, const DilMap& map) -> na_status {
    BwdLaunch L;
    na_status r = simt_launch(Q, map, L);
    if (r != NA_OK) return r;
    if (!use_tc) {
      const cudaError_t e = launch_bwd_simt_grads(L, s);
      if (e == cudaErrorNotSupported) return fail(NA_ERR_UNSUPPORTED, "backward: shape");
      if (e != cudaSuccess) return fail(NA_ERR_CUDA, "backward launch: %s", cudaGetErrorString(e));
      return NA_OK;
    }
    Problem Qt = Q;
    Qt.opt.kernel = NA_KERNEL_TC;
    Plan tc_plan;
    r = make_plan(Qt, tc_plan);
    if (r != NA_OK) return r;
    TcBwdLaunch T;
    T.g = Q.g;
    T.t = tc_plan.t;
    for (int d = 0; d < 3; ++d) T.kb[d] = tc_plan.kb[d];
    T.map = map;
    T.BH = (int)BH;
    T.N = L.N;
    T.D = Q.D;
    T.f16 = Q.dtype == NA_F16;
    T.scale = scale;
    T.scale_log2 = L.scale_log2;
    T.q = q; T.k = k; T.v = v; T.dout = dout; T.lse = lse; T.delta = delta;
    T.dq = dq; T.dk = dk; T.dv = dv;
    T.status = status;
    T.timeout_ns = Q.opt.wait_timeout_ns > 0 ? Q.opt.wait_timeout_ns : default_timeout_ns();
    char msg[256] = "";
    cudaError_t e = launch_tc_bwd_dq(T, s, msg, sizeof msg);
    if (e == cudaErrorNotSupported) return fail(NA_ERR_UNSUPPORTED, "tensor-core dq: shape");
    if (e != cudaSuccess)
      return fail(NA_ERR_CUDA, "tensor-core dq: %s %s", cudaGetErrorString(e), msg);
    e = launch_tc_bwd_dkdv(T, s, msg, sizeof msg);
    if (e == cudaErrorNotSupported) return fail(NA_ERR_UNSUPPORTED, "tensor-core dk/dv: shape");
    if (e != cudaSuccess)
      return fail(NA_ERR_CUDA, "tensor-core dk/dv: %s %s", cudaGetErrorString(e), msg);
    return NA_OK;
  };

  // D_i = <dout_i, out_i> for every row of the full grid, once.
  {
    Problem Pu = P;
    for (int d = 0; d < 3; ++d) {
      Pu.dil[d] = 1;
      Pu.tile[d] = dilated(P) ? 0 : P.tile[d];
    }
    BwdLaunch L;
    st = simt_launch(Pu, identity_map(P.g.L), L);
    if (st != NA_OK) return st;
    const cudaError_t e = launch_bwd_simt_delta(L, s);
    if (e != cudaSuccess) return fail(NA_ERR_CUDA, "backward delta: %s", cudaGetErrorString(e));
  }
  if (!dilated(P)) return grads(P, identity_map(P.g.L));
  int r[3];
  for (r[0] = 0; r[0] < P.dil[0]; ++r[0])
    for (r[1] = 0; r[1] < P.dil[1]; ++r[1])
      for (r[2] = 0; r[2] < P.dil[2]; ++r[2]) {
        DilMap map;
        const Problem Q = residue_problem(P, r, map);
        st = grads(Q, map);
        if (st != NA_OK) return st;
      }
  return NA_OK;
}

na_status na_sync_status(void* stream) {
  g_err[0] = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(NA_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return NA_OK;
  int* p = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_status_mu);
    p = g_status[dev];
  }
  if (!p) return NA_OK;
  int h = 0;
  e = cudaMemcpy(&h, p, sizeof h, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(NA_ERR_CUDA, "reading status word: %s", cudaGetErrorString(e));
  if (h != DEV_OK) {
    cudaMemset(p, 0, sizeof(int));
    return fail(NA_ERR_TIMEOUT, "a bounded in-kernel wait expired (code %d)", h);
  }
  return NA_OK;
}

na_status na_plan(const int dims[2], const int* grid, const int* window, const int* stride,
                  const int* tile, na_dtype dtype, const na_options* opt, na_plan_info* info) {
  g_err[0] = 0;
  if (!info) return fail(NA_ERR_INVALID_ARG, "info is NULL");
  Problem P;
  na_status st = read_problem(dims, grid, window, stride, tile, dtype, opt, P);
  if (st != NA_OK) return st;
  if (!dilated(P)) return plan_info(P, info);
  // Dilated: each residue class is scheduled as a grid of its own; the counts
  // are summed over the classes.
  na_plan_info sum;
  memset(&sum, 0, sizeof sum);
  bool first = true;
  int r[3];
  for (r[0] = 0; r[0] < P.dil[0]; ++r[0])
    for (r[1] = 0; r[1] < P.dil[1]; ++r[1])
      for (r[2] = 0; r[2] < P.dil[2]; ++r[2]) {
        DilMap map;
        const Problem Q = residue_problem(P, r, map);
        na_plan_info one;
        st = plan_info(Q, &one);
        if (st != NA_OK) return st;
        if (first) {
          sum = one;
          first = false;
        } else {
          sum.query_blocks += one.query_blocks;
          sum.ctas += one.ctas;
          sum.chunks_loaded += one.chunks_loaded;
          sum.units_full += one.units_full;
          sum.units_partial += one.units_partial;
          sum.computed_pairs += one.computed_pairs;
          sum.useful_pairs += one.useful_pairs;
        }
      }
  const long long N = (long long)P.g.L[0] * P.g.L[1] * P.g.L[2];
  sum.dense_pairs = N * N;
  sum.dense_units = 0;
  sum.speedup_bound = 0.0;
  *info = sum;
  return NA_OK;
}

na_status na_block_schedule(const int dims[2], const int* grid, const int* window,
                            const int* stride, const int* window_mode, const int qblock[3],
                            const int kvchunk[3], long long block, int origin[3], int extent[3],
                            int lo[3], int hi[3], int ilo[3], int ihi[3], int* status,
                            int max_chunks, int* nchunks) {
  g_err[0] = 0;
  na_options o = na_default_options();
  if (window_mode && dims && dims[0] >= 1 && dims[0] <= 3)
    for (int i = 0; i < dims[0]; ++i) o.window_mode[i] = window_mode[i];
  Problem P;
  na_status st = read_problem(dims, grid, window, stride, nullptr, NA_BF16, &o, P);
  if (st != NA_OK) return st;
  if (!qblock || !kvchunk || !nchunks) return fail(NA_ERR_INVALID_ARG, "NULL argument");
  for (int d = 0; d < 3; ++d)
    if (qblock[d] < 1 || kvchunk[d] < 1) return fail(NA_ERR_INVALID_ARG, "shapes must be >= 1");
  QTiling t;
  if (make_tiling(P.g, qblock, qblock, t)) return fail(NA_ERR_INVALID_ARG, "bad qblock");
  if (block < 0 || block >= t.nblocks) return fail(NA_ERR_INVALID_ARG, "block out of range");
  BlockInfo b;
  block_info(P.g, t, (int)block, b);
  ChunkGrid cg;
  chunk_grid_for(&b, 1, kvchunk, cg);
  for (int d = 0; d < 3; ++d) {
    if (origin) origin[d] = b.o[d];
    if (extent) extent[d] = b.n[d];
    if (lo) lo[d] = b.lo[d];
    if (hi) hi[d] = b.hi[d];
    if (ilo) ilo[d] = b.ilo[d];
    if (ihi) ihi[d] = b.ihi[d];
  }
  *nchunks = cg.total;
  for (int c = 0; c < cg.total && c < max_chunks && status; ++c) {
    int a[3];
    chunk_origin(cg, kvchunk, c, a);
    status[c] = chunk_status(b, a, kvchunk);
  }
  return NA_OK;
}

na_status na_noalloc_status(void* stream) {
  g_err[0] = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(NA_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return NA_OK;
  void* p = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    p = g_noalloc_ptr[dev];
  }
  if (!p) return NA_OK;   // no na_forward_noalloc call on this device yet
  // A plain host int as the destination: the copy needs no device memory.
  int h = 0;
  e = cudaMemcpyAsync(&h, p, sizeof h, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(NA_ERR_CUDA, "reading the scratch status: %s", cudaGetErrorString(e));
  if (h != DEV_OK) {
    e = cudaMemsetAsync(p, 0, sizeof(int), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail(NA_ERR_CUDA, "clearing the scratch status: %s", cudaGetErrorString(e));
    return fail(NA_ERR_TIMEOUT, "a bounded in-kernel wait expired (code %d)", h);
  }
  return NA_OK;
}

na_status na_forward_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                             int B, int heads, const int dims[2], const int* grid,
                             const int* window, const int* stride, const int* tile,
                             na_dtype dtype, const na_options* opt, void* stream) {
  g_err[0] = 0;
  if (!q || !k || !v || !out || !lse) return fail(NA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  if (B < 1 || heads < 1) return fail(NA_ERR_INVALID_ARG, "B=%d heads=%d must be >= 1", B, heads);
  Problem P;
  na_status st = read_problem(dims, grid, window, stride, tile, dtype, opt, P);
  if (st != NA_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(lse, 4))
    return fail(NA_ERR_INVALID_ARG, "q, k, v, out must be 16-byte aligned and lse 4-byte aligned");
  const long long BH = (long long)B * heads;
  if (BH > (1LL << 30)) return fail(NA_ERR_UNSUPPORTED, "B*heads too large");
  if (P.opt.kernel == NA_KERNEL_SIMT || P.opt.kernel == NA_KERNEL_GATHER)
    return fail(NA_ERR_UNSUPPORTED, "na_forward_noalloc runs the tensor-core kernel only");
  if (dilated(P))
    return fail(NA_ERR_UNSUPPORTED, "na_forward_noalloc takes no dilation (use na_forward_ex)");
  P.opt.kernel = NA_KERNEL_TC;
  Plan plan;
  st = make_plan(P, plan);
  if (st != NA_OK) return st;
  if (TC_SCRATCH_BYTES > NOALLOC_SCRATCH_BYTES)
    return fail(NA_ERR_UNSUPPORTED, "needs %zu bytes of scratch; the static array holds %zu",
                TC_SCRATCH_BYTES, NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != NA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: the status word must start at 0.
  cudaError_t e = cudaMemsetAsync(scratch, 0, TC_SCRATCH_BYTES, s);
  if (e != cudaSuccess) return fail(NA_ERR_CUDA, "clearing scratch: %s", cudaGetErrorString(e));
  const float scale = P.opt.scale > 0.f ? P.opt.scale : 1.0f / sqrtf((float)P.D);
  TcLaunch L;
  L.g = P.g;
  L.t = plan.t;
  for (int d = 0; d < 3; ++d) L.kb[d] = plan.kb[d];
  L.map = identity_map(P.g.L);
  L.BH = (int)BH;
  L.N = (int)((long long)P.g.L[0] * P.g.L[1] * P.g.L[2]);   // < 2^31 (read_problem)
  L.D = P.D;
  L.dt = tc_dtype(P.dtype);
  L.scale_log2 = scale * 1.4426950408889634f;
  L.q = q; L.k = k; L.v = v; L.out = out; L.lse = lse;
  L.status = static_cast<int*>(scratch);
  L.timeout_ns = P.opt.wait_timeout_ns > 0 ? P.opt.wait_timeout_ns : default_timeout_ns();
  L.debug_flags = P.opt.debug_flags;
  char msg[256] = "";
  e = launch_tc(L, s, msg, sizeof msg);
  if (e == cudaErrorNotSupported)
    return fail(NA_ERR_UNSUPPORTED, "tensor-core kernel does not take this shape");
  if (e != cudaSuccess)
    return fail(NA_ERR_CUDA, "tensor-core launch: %s %s", cudaGetErrorString(e), msg);
  return NA_OK;
}

}  // extern "C"
