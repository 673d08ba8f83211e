// Issue-rate probe for tcgen05.mma (kind::f16, bf16 operands, M = 128, K = 16): one thread per CTA
// issues 64 x 8 MMAs back to back into a TMEM accumulator, with A and B in 128-byte-swizzled shared
// memory ("A:smem") or A in TMEM ("A:tmem"), for N = 64, 128, 256; one CTA alone and one per SM.
// It reports clocks per MMA at issue and until the final commit, beside the clocks the MMA's math
// takes at 8192 FLOP per clock per SM (the dense bf16 rate). The operands are zeros: only the rate
// is measured. Every wait is bounded and TMEM is freed before the kernel exits.
//
// Build and run (one GPU), from the repository root:
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 -I include \
//        paged_kv_cache_385_b200/measure/tc05_mma_rate.cu -o tc05_mma_rate
//   ./tc05_mma_rate
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>

#include "../csrc/pa_device.cuh"
#include "../csrc/tc05.cuh"
using namespace pa;

template <int N, bool TS>
__global__ void __launch_bounds__(128, 1) probe(unsigned long long* out, int iters) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  for (int i = threadIdx.x; i < 65536 / 16; i += blockDim.x)
    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(base + i * 16), "r"(0u) : "memory");
  const uint32_t bar = base + 65536, slot = base + 65536 + 8;
  if (threadIdx.x == 0) { mbar_init(bar, 1); fence_barrier_init(); }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (threadIdx.x < 32) tc05::alloc(slot, 512);
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + 65536 + 8);
  if (threadIdx.x == 0) {
    constexpr uint32_t idesc = tc05::idesc_f16(true, 128, N, false, false);
    const long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t cb = (ks & 3) * 32;
        const uint64_t bd = tc05::smem_desc_sw128(base + 32768 + cb, 16, 1024);
        if constexpr (TS) {
          tc05::mma_f16_ts(tmem, tmem + 256 + ks * 8, bd, idesc, it > 0 || ks > 0);
        } else {
          tc05::mma_f16(tmem, tc05::smem_desc_sw128(base + (ks >> 2) * 16384 + cb, 16, 1024), bd, idesc, it > 0 || ks > 0);
        }
      }
    }
    const long long t1 = clock64();
    tc05::commit(bar);
    const bool ok = mbar_wait_bounded(bar, 0, globaltimer_ns() + 1000000000ull);
    const long long t2 = clock64();
    out[blockIdx.x * 4 + 0] = t1 - t0;
    out[blockIdx.x * 4 + 1] = t2 - t0;
    out[blockIdx.x * 4 + 2] = ok;
    out[blockIdx.x * 4 + 3] = 0;
  }
  tc05::fence_before_sync();
  __syncthreads();
  if (threadIdx.x < 32) { tc05::fence_after_sync(); tc05::dealloc(tmem, 512); }
}

template <int N, bool TS>
void run(int grid, int iters) {
  unsigned long long* d;
  cudaMalloc(&d, grid * 4 * 8);
  auto k = probe<N, TS>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 65536 + 1024);
  for (int rep = 0; rep < 2; ++rep) k<<<grid, 128, 65536 + 1024>>>(d, iters);
  cudaError_t e = cudaDeviceSynchronize();
  unsigned long long h[148 * 4];
  cudaMemcpy(h, d, grid * 4 * 8, cudaMemcpyDeviceToHost);
  double issue = 0, tot = 0; int ok = 1;
  for (int b = 0; b < grid; ++b) { issue += h[b * 4]; tot += h[b * 4 + 1]; ok &= (int)h[b * 4 + 2]; }
  const double n = 8.0 * iters;
  printf("N=%3d %s grid=%3d iters=%4d: issue %.1f clk/mma, total %.1f clk/mma (work at 8192 flop/clk: %d) ok=%d err=%s\n",
         N, TS ? "A:tmem" : "A:smem", grid, iters, issue / grid / n, tot / grid / n, 128 * N * 16 * 2 / 8192, ok,
         cudaGetErrorString(e));
  cudaFree(d);
}

int main() {
  run<64, false>(1, 64); run<64, false>(148, 64);
  run<128, false>(1, 64); run<128, false>(148, 64);
  run<256, false>(1, 64); run<256, false>(148, 64);
  run<128, true>(1, 64); run<128, true>(148, 64);
  run<256, true>(148, 64);
  return 0;
}
