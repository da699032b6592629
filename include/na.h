/*
 * na.h -- C ABI of the B200 forward pass of multi-dimensional local attention
 * (generalized neighborhood attention / sliding tile attention).
 *
 * Operation.  For every (batch b, head h) and every query token i of a 1-, 2-
 * or 3-D token grid of extents L, the library computes
 *     out_i = sum_{j in W(i)} softmax_j( <q_i, k_j> * scale ) v_j
 *     lse_i = ln sum_{j in W(i)} exp( <q_i, k_j> * scale )
 * i.e. softmax(QK^T / sqrt(d)) V of "pi-Attention: Online Efficient Sparse
 * Transformers for Long-Context Modeling" (section 3.1, eqs. (1)-(3)) with the
 * sum restricted to a neighbourhood (section 3.2, eqs. (4)-(5)), plus the log
 * of eq. (2)'s denominator.  The neighbourhood W(i) is the product over grid
 * dimensions of the 1-D windows
 *     g = i / s,  c = g*s + s/2,  start = clamp(c - w/2, 0, L - w),
 *     window = [start, start + w)
 * (window w, stride s): centred on the query's stride group and clamped
 * inside the grid, so every query sees exactly prod(w) keys.  stride 1 is
 * neighborhood attention; stride = tile with an odd number of tiles per
 * window is the sliding tile attention of "ENA: Efficient N-dimensional
 * Attention"; stride = window dividing the grid is blocked attention -- the
 * family named in the abstract of "Generalized Neighborhood Attention:
 * Multi-dimensional Sparse Attention at the Speed of Light".
 *
 * Window modes (na_options.window_mode, per grid dimension) replace the
 * clamp by a cut at the grid border, after "pi-Attention" section 3.2
 * eq. (5):
 *     truncated  [c - w/2, c - w/2 + w) intersected with [0, L)
 *                (s = 1, w = 2k+1: the bidirectional |j - i| <= k)
 *     causal     [(g+1)*s - w, (g+1)*s) intersected with [0, L)
 *                (s = 1, w = k+1: the causal max(0, i-k) <= j <= i)
 * so queries near a border (or near the start, for causal) see fewer keys.
 * With s > 1 a causal window covers the query's whole stride group (block
 * causal).
 *
 * Layout.  q, k, v and out are dense row-major [B, heads, X1, .., Xn, d]
 * (n = ndim, last grid dimension fastest, then d); lse is [B, heads, X1..Xn].
 *
 * Ownership.  Every tensor is caller-owned device memory.  The library keeps
 * one 4-byte device status word per device, allocated on that device's first
 * call (so make the first call outside any stream capture), and nothing else.
 *
 * Asynchrony.  Calls enqueue work on `stream` (a cudaStream_t; NULL = legacy
 * default stream) and return once it is queued.  Argument errors are returned
 * at once.  Errors that only the device can see (a bounded in-kernel wait that
 * ran out) are reported by na_sync_status().
 *
 * Determinism.  Identical inputs give bit-identical outputs run to run (fixed
 * reduction order, no atomics on data).
 */
#ifndef NA_H_
#define NA_H_

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NA_OK = 0,
  NA_ERR_INVALID_ARG = 1,  /* a pointer, size or window/stride violates the contract */
  NA_ERR_UNSUPPORTED = 2,  /* valid, but outside what the kernels implement */
  NA_ERR_CUDA = 3,         /* a CUDA runtime call failed; na_last_error() has the text */
  NA_ERR_TIMEOUT = 4       /* a bounded in-kernel wait expired (reported by na_sync_status) */
} na_status;

/* Input types.  NA_E4M3: q, k and v in the OFP8 E4M3 format (one byte per
 * element; finite range +-448, no infinities); out is then written as bf16
 * (two bytes per element), lse as fp32.  E4M3 runs on the tensor-core kernel
 * only (head_dim 64 or 128, forward only); the softmax weights fed to the
 * second product are rounded to E4M3 as well (see na_forward). */
typedef enum { NA_F32 = 0, NA_BF16 = 1, NA_F16 = 2, NA_E4M3 = 3 } na_dtype;

/* Per-dimension window rule (see the top of this file). */
typedef enum {
  NA_WINDOW_CLAMPED = 0,    /* shifted inside the grid: always w keys (default) */
  NA_WINDOW_TRUNCATED = 1,  /* centred, cut at the grid border */
  NA_WINDOW_CAUSAL = 2      /* ending with the query's stride group, cut at 0 */
} na_window_mode;

typedef enum {
  NA_KERNEL_AUTO = 0,   /* the window-gather kernel for windows of at most
                           NA_GATHER_MAX_KEYS keys (product of the window sizes),
                           else the tensor-core kernel where it applies, else the
                           CUDA-core tile kernel */
  NA_KERNEL_SIMT = 1,   /* CUDA-core tile kernel (fp32, bf16 and f16, head_dim 32/64/128) */
  NA_KERNEL_TC = 2,     /* tcgen05 tensor-core kernel (bf16 or f16, head_dim 64/128) */
  NA_KERNEL_GATHER = 3  /* CUDA-core window-gather kernel (fp32, bf16 and f16, head_dim
                           32/64/128): each query reads only its own window's keys, for
                           narrow windows where the pass is bound by HBM traffic.
                           Forward only. */
} na_kernel;

/* Largest window (keys per query, the product of the window sizes) that
 * NA_KERNEL_AUTO sends to the window-gather kernel. */
#define NA_GATHER_MAX_KEYS 32

/*
 * na_forward -- enqueue one forward pass.
 *   q, k, v   device pointers, [B, heads, X1..Xn, d], dtype `dtype`, 16-byte aligned.
 *   out       device pointer, same shape and dtype as q (written).
 *   lse       device pointer, float32 [B, heads, X1..Xn] (written).
 *   B, heads  >= 1.
 *   dims      {ndim, head_dim}: ndim in 1..3; head_dim in {32, 64, 128}.
 *   grid      ndim extents X1..Xn (>= 1).
 *   window    ndim window sizes, 1 <= window[i] <= grid[i].
 *   stride    ndim strides, 1 <= stride[i] <= window[i]; NULL = all 1.
 *   tile      ndim query-tile shape, or NULL for the library's choice.  It only
 *             groups queries for scheduling (results do not depend on it): the
 *             tensor-core path splits a tile of >= 128 tokens into 128-query
 *             blocks, or joins tiles of < 128 tokens into such blocks.
 *   dtype     NA_F32 (CUDA-core kernel), NA_BF16 or NA_F16 (tensor-core kernel
 *             when head_dim is 64 or 128; out is written in the input type and
 *             P, the softmax weights fed to the second product, are rounded to
 *             it as well), or NA_E4M3 (tensor-core kernel, head_dim 64 or 128:
 *             both products take 8-bit operands with fp32 accumulation, P is
 *             rounded to E4M3 -- formed at up to 2^4 times the row's running
 *             maximum weight so that typical weights stay in the format's
 *             normal range, with the reference moved before any weight could
 *             pass 256 -- and out is bf16 [B, heads, X1..Xn, d]).
 *   stream    cudaStream_t.
 * Returns NA_OK once the work is queued, NA_ERR_INVALID_ARG / NA_ERR_UNSUPPORTED
 * without touching the device, or NA_ERR_CUDA.  Scale is 1/sqrt(head_dim).
 */
na_status na_forward(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                     int heads, const int dims[2], const int* grid, const int* window,
                     const int* stride, const int* tile, na_dtype dtype, void* stream);

typedef struct {
  float scale;              /* <= 0: 1/sqrt(head_dim) */
  int kernel;               /* na_kernel */
  int qblock[3];            /* 0s: automatic; else the query block shape, padded to 3 dims
                               (outermost first; product 128 for NA_KERNEL_TC) */
  int kvchunk[3];           /* 0s: automatic; else the key chunk shape (product 128 for TC,
                               32 for SIMT) */
  long long wait_timeout_ns;/* bound on each in-kernel wait; <= 0: 4 s (or env NA_WAIT_TIMEOUT_MS) */
  int debug_flags;          /* TESTING HOOK, not a supported option: leave it 0.  1: the
                               tensor-core forward kernel's loader withholds the first key
                               chunk (the window-gather kernel's staged form: the copies of
                               the first query tile), so the consumers' bounded waits expire
                               and the timeout path (NA_ERR_TIMEOUT from na_sync_status) is
                               exercised without any fault or hang; the outputs of such a
                               call are undefined. */
  int window_mode[3];       /* na_window_mode of grid dimension i (i < ndim, the order of
                               `window`); entries from ndim on are ignored.  0 = clamped. */
  int dilation[3];          /* dilation of grid dimension i (i < ndim); 0 or 1 = none.  The
                               pages define none; the reading: coordinates split into
                               `dilation` interleaved residue classes (i mod dilation), and
                               a query's window is taken inside its own class -- the window
                               rule above on the class's positions, stride counted in class
                               positions -- so it attends to keys r + dilation * t.
                               Needs window[i] * dilation[i] <= grid[i] (else
                               NA_ERR_INVALID_ARG).  na_forward_ex and na_backward run one
                               launch per residue class; na_forward_noalloc returns
                               NA_ERR_UNSUPPORTED when it is set. */
} na_options;

/* na_options with every field at its default (automatic) value. */
na_options na_default_options(void);

/* na_forward with explicit options (NULL = defaults).  Same contract otherwise. */
na_status na_forward_ex(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                        int heads, const int dims[2], const int* grid, const int* window,
                        const int* stride, const int* tile, na_dtype dtype,
                        const na_options* opt, void* stream);

/*
 * na_backward -- enqueue the backward pass: the gradients of the forward's
 * `out` with respect to q, k and v for an upstream gradient `dout`.  The pages
 * give only the forward pass; these are its vector-Jacobian product over the
 * same windows (softmax weights recomputed from the forward's lse):
 *     P_ij  = exp(scale <q_i, k_j> - lse_i),   D_i = <dout_i, out_i>
 *     dZ_ij = P_ij (<dout_i, v_j> - D_i)
 *     dq_i  = scale sum_j dZ_ij k_j
 *     dk_j  = scale sum_{i : j in W(i)} dZ_ij q_i
 *     dv_j  = sum_{i : j in W(i)} P_ij dout_i
 *   q, k, v, out, lse  the forward's inputs and outputs (out and lse as
 *                      na_forward wrote them for the same arguments and options).
 *   dout              device, same shape / dtype as q.
 *   dq, dk, dv        device, same shape / dtype as q (written; every row once,
 *                     no atomics, deterministic).
 *   delta             device float32 [B, heads, X1..Xn] workspace (written: D_i).
 * Other arguments, options (scale, window_mode) and errors as na_forward_ex;
 * dtype NA_E4M3 is NA_ERR_UNSUPPORTED (the backward is not built for 8-bit inputs).
 * Kernels: the row delta D_i on the CUDA cores (fp32 arithmetic); for bf16 /
 * f16 with head_dim 64 or 128, dq (one kernel per query block) and dk / dv
 * (one kernel per key block, over the queries whose windows hold it) on the
 * tensor cores (tcgen05, fp32 accumulation in tensor memory) unless
 * opt->kernel = NA_KERNEL_SIMT; every other input on the CUDA cores.
 * opt->kernel = NA_KERNEL_TC for other inputs, and NA_KERNEL_GATHER (a
 * forward-only kernel), are NA_ERR_UNSUPPORTED.  A bounded
 * in-kernel wait that expires is reported by na_sync_status.
 */
na_status na_backward(const void* q, const void* k, const void* v, const void* out,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv,
                      float* delta, int B, int heads, const int dims[2], const int* grid,
                      const int* window, const int* stride, const int* tile, na_dtype dtype,
                      const na_options* opt, void* stream);

/*
 * na_sync_status -- synchronise `stream`, then read and clear this device's
 * status word.  NA_ERR_TIMEOUT if a kernel since the last call gave up on a
 * bounded wait (its outputs are then undefined); NA_ERR_CUDA if the
 * synchronisation itself failed; else NA_OK.
 */
na_status na_sync_status(void* stream);

/* Static, human-readable name of a status code. */
const char* na_status_string(na_status s);

/* Detail of the last failure on the calling thread ("" if none).  Thread-local, static storage. */
const char* na_last_error(void);

/*
 * Schedule statistics for one (batch, head), computed on the host with the
 * same scheduler the kernels run: the chosen block / chunk shapes and how much
 * work they imply.  Units: (query, key) pairs unless noted.
 */
typedef struct {
  int kernel;               /* na_kernel actually chosen */
  int qblock[3];            /* query block shape (3-d padded, outermost first); for the
                               window-gather kernel its query tile (staged form) or
                               1 x 1 x 1 (direct form: each query on its own) */
  int kvchunk[3];           /* key chunk shape; 1 x 1 x 1 for the window-gather kernel
                               (it reads exactly the window's keys) */
  int tile[3];              /* query tile shape used to order blocks */
  long long query_blocks;   /* blocks per head */
  long long ctas;           /* CTAs per head (window-gather: its query tiles per head in
                               the staged form, walked by a persistent grid; in the
                               direct form the head's rows / rows per CTA, rounded up,
                               CTAs straddling heads) */
  long long chunks_loaded;  /* key chunks staged per head */
  long long units_full;     /* (block, chunk) products with no mask */
  long long units_partial;  /* (block, chunk) products with an element mask */
  long long computed_pairs; /* (units_full + units_partial) * block rows * chunk keys */
  long long useful_pairs;   /* sum over queries of the window size (N * prod(window) when
                               every dimension is clamped) */
  long long dense_pairs;    /* N * N: the pairs of full self attention */
  long long dense_units;    /* (block, chunk) products of full self attention under the
                               same block and chunk shapes */
  /* With dilation the counts above are sums over the residue classes (each
     scheduled as a grid of its own); dense_units and speedup_bound are 0. */
  double speedup_bound;     /* dense_units / (units_full + units_partial): the speedup over
                               the same kernel run densely that tile-granular skipping
                               allows at most, a partial tile costing as much as a full
                               one -- the "realistic speedup upper bound" of the simulator
                               in the abstract of "Generalized Neighborhood Attention" */
} na_plan_info;

/* Fill *info for the given problem without touching the device. */
na_status na_plan(const int dims[2], const int* grid, const int* window, const int* stride,
                  const int* tile, na_dtype dtype, const na_options* opt, na_plan_info* info);

/* The 1-D clamped window start used by the kernels (host copy), -1 on invalid input. */
int na_window_start(int L, int w, int s, int i);

/* The 1-D window [*lo, *hi) of coordinate i under na_window_mode `mode`, as the
 * kernels compute it (host copy).  Returns 0, or -1 on invalid input. */
int na_window_range(int L, int w, int s, int mode, int i, int* lo, int* hi);

/*
 * Key box and chunk classification of one query block, for tests: the
 * block's origin and valid extent, the union [lo, hi) and intersection
 * [ilo, ihi) of its queries' windows (3-d padded), and per key chunk of the
 * block's own key box (row-major over the chunk grid) its status 0 = empty,
 * 1 = partial, 2 = full.  window_mode: ndim na_window_mode values, or NULL
 * for all clamped.  `status` holds up to `max_chunks` entries; the number of
 * chunks is returned in *nchunks.
 */
na_status na_block_schedule(const int dims[2], const int* grid, const int* window,
                            const int* stride, const int* window_mode, const int qblock[3],
                            const int kvchunk[3], long long block, int origin[3], int extent[3],
                            int lo[3], int hi[3], int ilo[3], int ihi[3], int* status,
                            int max_chunks, int* nchunks);

/* Library version, major*10000 + minor*100 + patch. */
int na_version(void);

/*
 * na_selftest_exp2 -- TESTING HOOK, not part of the attention interface.
 * y[i] = 2^x[i] computed by the FMA-pipe polynomial that the tensor-core
 * kernels can use for a share of their softmax exponentials (degree-3 minimax
 * fit of 2^f on [-1/2, 1/2], relative error <= 1.02e-4 for -125 <= x <= 8).
 * x and y are device float arrays of n elements; enqueued on `stream`.  It
 * lets the tests check that device arithmetic against exact values.
 */
na_status na_selftest_exp2(const float* x, float* y, int n, void* stream);

/*
 * na_forward_noalloc -- na_forward_ex for callers that must not allocate
 * device memory.  The paper has no counterpart: this is a deployment entry
 * point, not part of the method.
 *
 * Who needs it: hosts that own all device memory themselves -- for example a
 * serving engine that reserves nearly all of HBM for its own pools up front,
 * where a stray cudaMalloc would fail or slip past its memory accounting, or a
 * latency-critical loop that cannot afford cudaMalloc's implicit device-wide
 * synchronisation.  na_forward allocates one 4-byte status word per device on
 * its first call; this entry point instead keeps that word in a fixed
 * 256-byte array compiled into the library (every GPU that loads the library
 * holds it until the process exits) and calls no cudaMalloc, cudaFree or other
 * device-allocating routine.  Host-side planning may still use the C++ heap.
 *
 * Same arguments and layouts as na_forward_ex; the caller still passes q, k,
 * v, out and lse.  It runs the tensor-core kernel only (bf16, f16 or E4M3,
 * head_dim 64 or 128; opt->kernel must be NA_KERNEL_AUTO or
 * NA_KERNEL_TC -- AUTO means the tensor-core kernel here, whatever the
 * window size), else returns
 * NA_ERR_UNSUPPORTED.  The kernel's scratch need (4 bytes) is checked against
 * the array's size and refused with NA_ERR_UNSUPPORTED if it ever exceeded it.
 *
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture.
 *
 * The looked-up address belongs to the device's current context: after a
 * cudaDeviceReset (or anything else that destroys the primary context) the
 * library's cached address is stale, so do not reset a device between calls.
 *
 * Sharing: all calls on a device use the same array, which keeps the last
 * call's contents.  Each call clears the status word on `stream` before its
 * kernel, so calls whose kernels overlap on the GPU (different streams, no
 * ordering between them) race on it.  A bounded in-kernel wait that expires
 * leaves out/lse undefined; na_noalloc_status reports it (na_sync_status
 * reads only na_forward's status word).
 */
na_status na_forward_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                             int B, int heads, const int dims[2], const int* grid,
                             const int* window, const int* stride, const int* tile,
                             na_dtype dtype, const na_options* opt, void* stream);

/*
 * na_noalloc_status -- na_sync_status for na_forward_noalloc: synchronise
 * `stream`, then read this device's status word in the static array (copied
 * into a host int, so no device memory is allocated) and clear it if set.
 * NA_ERR_TIMEOUT if a na_forward_noalloc kernel since the last clear gave up on
 * a bounded wait (its out / lse are then undefined); NA_ERR_CUDA if a copy or
 * the synchronisation failed; NA_OK otherwise, also when na_forward_noalloc was
 * never called on this device.  Like the calls it reports on, it shares the
 * array with every other caller on the device.
 */
na_status na_noalloc_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NA_H_ */
