// Internal interface between the C-ABI layer (na_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "na_sched.cuh"

namespace na {

// Device status word values (written by kernels, read by na_sync_status).
enum : int { DEV_OK = 0, DEV_TIMEOUT = 1, DEV_BAD_SCHEDULE = 2 };

struct SimtLaunch {
  Geom g;
  QTiling t;
  int kb[3];
  DilMap map;            // grid coordinates -> token of the full (undilated) grid
  int BH, N, D;          // N: tokens per head of the full grid
  int dtype;             // na_dtype of q, k, v and out (fp32, bf16 or f16)
  float scale_log2;      // scale * log2(e)
  const void *q, *k, *v;
  void* out;
  float* lse;
};

struct TcLaunch {
  Geom g;
  QTiling t;
  int kb[3];
  int kb_log2[3];        // filled by launch_tc (chunk extents are powers of two)
  DilMap map;            // grid coordinates -> token of the full (undilated) grid
  int BH, N, D;          // N: tokens per head of the full grid
  int dt;                // inputs: 0 bf16, 1 f16 (out in the input type), 2 E4M3 (out bf16)
  float scale_log2;
  const void *q, *k, *v;
  void* out;
  float* lse;
  int* status;           // device status word
  long long timeout_ns;  // bound on every in-kernel wait
  int debug_flags;       // 1: withhold the first key chunk (timeout-path test)
};

// Backward pass (CUDA-core kernels): dq, dk, dv of the forward for upstream dout.
struct BwdLaunch {
  Geom g;
  QTiling t;             // query blocks (dQ) and key blocks (dK, dV)
  int kb[3];             // key chunks (dQ) and query chunks (dK, dV), 32 tokens
  DilMap map;            // grid coordinates -> token of the full (undilated) grid
  int BH, N, D;          // N: tokens per head of the full grid
  int dtype;             // na_dtype of q, k, v, out, dout and the gradients
  float scale;           // softmax scale
  float scale_log2;      // scale * log2(e)
  const void *q, *k, *v, *out, *dout;
  const float* lse;      // forward log-sum-exp (natural log)
  float* delta;          // [BH, N] workspace: <dout_i, out_i>
  void *dq, *dk, *dv;
};

// Tensor-core backward, dQ part: per query block, S = Q K^T and dP = dO V^T
// into tensor memory, dS = P (dP - delta) written back as 16-bit, dQ += dS K.
struct TcBwdLaunch {
  Geom g;
  QTiling t;             // query blocks (128 tokens)
  int kb[3];             // key chunks (128 tokens)
  int kb_log2[3];        // filled by the launcher
  DilMap map;            // grid coordinates -> token of the full (undilated) grid
  int BH, N, D;          // N: tokens per head of the full grid
  int f16;               // 1: f16, 0: bf16
  float scale, scale_log2;
  const void *q, *k, *v, *dout;
  const float* lse;
  const float* delta;    // <dout_i, out_i>, written by the row-delta kernel first
  void *dq, *dk, *dv;
  int* status;           // device status word
  long long timeout_ns;  // bound on every in-kernel wait
};

// Window-gather kernel (CUDA cores): each query reads its own window's keys.
// 256 threads per CTA.  Direct form: one 16-byte slice of the head dimension
// per thread, so query rows served at once per CTA =
inline int gather_rows_per_cta(int D, int dtype) { return 256 / (D / (dtype == 0 ? 4 : 8)); }
// Staged form: 32 head-dim elements per thread, so queries served per round =
inline int gather_tile_queries_per_round(int D) { return 256 / (D / 32); }

struct GatherLaunch {
  Geom g;
  DilMap map;            // grid coordinates -> token of the full (undilated) grid
  int BH, N, D;          // N: tokens per head of the full grid
  int dtype;             // na_dtype of q, k, v and out
  float scale_log2;      // scale * log2(e)
  const void *q, *k, *v;
  void* out;
  float* lse;
  int qt[3];             // query tile (a box of the grid); qt[0] == 0: no staging,
                         // every key read straight from global memory
  int nt[3];             // tiles per dimension
  int qrows, krows;      // staged form: rows of a stage's Q region (the tile) and of
                         // its K and V regions (the largest key box of a tile)
  int nstages;           // staged form: 1 or 2 stages
  int smem_bytes;        // staged form: header + the stages
  int* status;           // device status word
  long long timeout_ns;  // bound on every in-kernel wait
  int debug_flags;       // testing hook: 1 = CTA 0's first tile gets no copies
};

// Staged form: a header (barriers, tile geometry), then one or two stages of
// (Q tile, K box, V box).
constexpr int GATHER_SMEM_HEADER = 256;
// Footprints that let two CTAs share an SM, and one CTA's limit.
constexpr int GATHER_SMEM_TWO_PER_SM = 110 * 1024;
constexpr int GATHER_SMEM_MAX = 220 * 1024;
inline long long gather_smem_bytes(long long qrows, long long krows, int D, int esz, int nst) {
  return GATHER_SMEM_HEADER + nst * (qrows + 2 * krows) * D * esz;
}
cudaError_t launch_gather(const GatherLaunch& L, cudaStream_t stream);

// 5-d TMA descriptor of a [BH, X1, X2, X3, D] tensor of input type dt (0 bf16,
// 1 f16: 64-element inner box, 128-byte swizzle; 2 E4M3: one row of D bytes,
// 128- or 64-byte swizzle), `box` tokens.
bool encode_grid_map(CUtensorMap* m, const void* ptr, int dt, int D, const int L[3], int BH,
                     int N, const int box[3]);
// The same for a residue class of a dilated grid: the class's coordinates x
// address token map.res + map.dil * x of the full grid (N tokens per head).
bool encode_grid_map_dil(CUtensorMap* m, const void* ptr, int dt, int D, const int L[3],
                         const DilMap& map, int BH, int N, const int box[3]);

cudaError_t launch_simt(const SimtLaunch& L, cudaStream_t stream);
cudaError_t launch_bwd_simt(const BwdLaunch& L, cudaStream_t stream);
// The row-delta and dK/dV CUDA-core kernels alone (the dQ kernel left out).
cudaError_t launch_bwd_simt_delta(const BwdLaunch& L, cudaStream_t stream);
cudaError_t launch_bwd_simt_dkdv(const BwdLaunch& L, cudaStream_t stream);
cudaError_t launch_bwd_simt_grads(const BwdLaunch& L, cudaStream_t stream);   // dq, dk, dv
cudaError_t launch_tc_bwd_dq(const TcBwdLaunch& L, cudaStream_t stream, char* err, int errlen);
cudaError_t launch_tc_bwd_dkdv(const TcBwdLaunch& L, cudaStream_t stream, char* err, int errlen);

// y[i] = the tensor-core kernel's FMA-pipe 2^x applied to x[i] (self-test).
cudaError_t launch_exp2_selftest(const float* x, float* y, int n, cudaStream_t stream);

// Returns cudaErrorNotSupported when the shape is outside the kernel's range.
cudaError_t launch_tc(const TcLaunch& L, cudaStream_t stream, char* err, int errlen);

}  // namespace na
