// Tensor-core issue-rate microbenchmark for the MMA shapes of the forward
// kernel (not part of the library).  One CTA per SM, one thread issuing
// back-to-back tcgen05.mma with precomputed descriptors; reports SM clocks per
// 128x128x16 bf16 MMA.  Modes:
//   ss      S = Q K^T form: A and B in shared memory (K-major)
//   ts      O += P V form: A (P) in tensor memory, B (V) MN-major in shared memory
//   step    one forward-kernel step: 8 ss into S, then 8 ts reading P from S's columns
//   step+t  the same step while 4 other warps stream tcgen05.ld/st traffic
//   step+s  the same step while 4 other warps stream st.shared traffic
//   ss64    S = Q K^T with N = 64 (a 64-key half chunk), A and B in shared memory
//   step64  one step of a half-chunk pipeline: 8 ss64 into the first 64 columns,
//           4 ts (N = 128) reading P from them
//   step+b  the step while one thread streams 32 KB bulk copies (global -> shared,
//           L2-resident source) into a separate shared-memory region, back to back
//   step+b20  the same with one copy per 1600 clocks (~20 B/clk, the forward
//           kernel's K/V load rate)
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 \
//        -o microbench_mma neighborhood_attention_b200/csrc/microbench_mma.cu && ./microbench_mma
//
// Buffers: 128 KB of shared memory (A tile [0,32K), K-major B [32K,64K), MN-major
// B [64K,96K) including its second 64-column half at +16 KB, bulk-copy target
// [96K,128K)), TMEM 512 columns (S 0..127, P read from 0..63, O 256..383, side
// traffic 384..511); a 32 KB global source buffer for the bulk copies.
#include <cstdint>
#include <cstdio>

#include <cuda_runtime.h>

#include "na_ptx.cuh"

using namespace na;

namespace {

constexpr int kIters = 256;  // each iteration = 8 or 16 MMAs
constexpr int kSmem = 131072;
constexpr uint32_t kCopyBytes = 32768;

template <int MODE>
__global__ void __launch_bounds__(160, 1) rate_kernel(unsigned long long* out, int* status,
                                                       const uint8_t* src) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t done;
  __shared__ uint64_t copied;
  __shared__ uint32_t tbase;
  __shared__ int abort_flag;
  __shared__ volatile int stop;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int i = threadIdx.x; i < kSmem / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(base)[i] = 0;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&done, 1);
    ptx::mbar_init(&copied, 1);
    abort_flag = 0;
    stop = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(&tbase, 512);
    ptx::tmem_relinquish();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tm = tbase;
  if (warp == 0) {
    if (lane == 0) {
      const uint32_t sa = ptx::smem_u32(base);
      const uint64_t dq = ptx::desc_sw128(sa, 16, 1024);
      const uint64_t dk = ptx::desc_sw128(sa + 32768, 16, 1024);
      const uint64_t dv = ptx::desc_sw128(sa + 65536, 16384, 1024);
      constexpr uint32_t kQK = ptx::idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kPV = ptx::idesc_bf16_f32(128, 128, false, true);
      const long long t0 = clock64();
      for (int i = 0; i < kIters; ++i) {
        if (MODE == 5 || MODE == 6) {
          constexpr uint32_t kQK64 = ptx::idesc_bf16_f32(128, 64, false, false);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
            ptx::mma_ss(tm, dq + off, dk + off, kQK64, kk > 0);
          }
          if (MODE == 6) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              ptx::mma_ts(tm + 256, tm + kk * 8, dv + ((kk * 2048) >> 4), kPV, 1u);
          }
        } else {
          if (MODE != 1) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
              ptx::mma_ss(tm, dq + off, dk + off, kQK, kk > 0);
            }
          }
          if (MODE != 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              ptx::mma_ts(tm + 256, tm + kk * 8, dv + ((kk * 2048) >> 4), kPV, 1u);
          }
        }
      }
      ptx::tc_commit(&done);
      ptx::WaitCtl c;
      c.abort = &abort_flag;
      c.status = status;
      c.timeout_ns = 2000000000ull;
      ptx::wait_drain(&done, 0, c);
      const long long t1 = clock64();
      stop = 1;
      if (blockIdx.x == 0) out[0] = (unsigned long long)(t1 - t0);
    }
  } else {
    const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t acc = 0;
    for (int it = 0; MODE != 7 && MODE != 8 && it < 100000 && !stop; ++it) {
      if (MODE == 3) {
        uint32_t r[32];
        ptx::tmem_ld32(tm + lb + 384 + (it & 3) * 32, r);
        ptx::tmem_ld_wait();
        ptx::reg_fence(r);
        acc += r[it & 31];
        ptx::tmem_st32(tm + lb + 384 + ((it + 1) & 3) * 32, r);
        ptx::tmem_st_wait();
      } else if (MODE == 4) {
        uint4* p = reinterpret_cast<uint4*>(base + 81920) + (threadIdx.x - 32);
#pragma unroll
        for (int u = 0; u < 8; ++u) p[u * 128] = make_uint4(it, u, acc, 0);
      }
    }
    if ((MODE == 7 || MODE == 8) && warp == 2 && lane == 0) {
      // One thread streams bulk copies; each is waited for before the next, so
      // none is in flight when the loop ends.
      ptx::WaitCtl c;
      c.abort = &abort_flag;
      c.status = status;
      c.timeout_ns = 2000000000ull;
      for (int it = 0; it < 100000 && !stop; ++it) {
        const long long t_issue = clock64();
        ptx::mbar_expect_tx(&copied, kCopyBytes);
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
            ::"r"(ptx::smem_u32(base + 98304)), "l"(src), "r"(kCopyBytes),
            "r"(ptx::smem_u32(&copied)) : "memory");
        if (!ptx::wait_drain(&copied, it & 1, c)) break;
        if (MODE == 8)
          while (clock64() - t_issue < 1600) {
          }
      }
    }
    if (acc == 12345u) out[1] = acc;
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tm, 512);
  }
}

template <int MODE>
void run(const char* name, double mmas_per_iter, unsigned long long* d, int* st, int grid,
         const uint8_t* src) {
  cudaFuncSetAttribute(rate_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem + 1024);
  rate_kernel<MODE><<<grid, 160, kSmem + 1024>>>(d, st, src);
  const cudaError_t e = cudaDeviceSynchronize();
  unsigned long long h = 0;
  cudaMemcpy(&h, d, sizeof h, cudaMemcpyDeviceToHost);
  printf("%-8s %6.1f clk per 128x128x16-equivalent MMA (%s)\n", name,
         (double)h / ((double)kIters * mmas_per_iter), cudaGetErrorString(e));
}

}  // namespace

int main() {
  unsigned long long* d = nullptr;
  int* st = nullptr;
  cudaMalloc(&d, 16);
  cudaMalloc(&st, 4);
  cudaMemset(st, 0, 4);
  uint8_t* src = nullptr;
  cudaMalloc(&src, kCopyBytes);
  cudaMemset(src, 0, kCopyBytes);
  int nsm = 0;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, 0);
  run<0>("ss", 8, d, st, nsm, src);
  run<1>("ts", 8, d, st, nsm, src);
  run<2>("step", 16, d, st, nsm, src);
  run<3>("step+t", 16, d, st, nsm, src);
  run<4>("step+s", 16, d, st, nsm, src);
  run<5>("ss64", 4, d, st, nsm, src);      // 8 MMAs of half the work
  run<6>("step64", 8, d, st, nsm, src);    // 8 half MMAs + 4 full
  run<7>("step+b", 16, d, st, nsm, src);
  run<8>("step+b20", 16, d, st, nsm, src);
  return 0;
}
