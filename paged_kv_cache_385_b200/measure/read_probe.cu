// Read-only HBM bandwidth probe: the practical ceiling of a pure read stream on this GPU, reported
// beside the copy (read + write) peak that the decode roofline is measured against.
//
// Each thread streams 16-byte loads over a 4 GiB buffer (far larger than L2) with a grid-stride
// loop and XOR-accumulates them; a store that never happens in practice keeps the loads live. The
// grid is a multiple of the 148 SMs; every (CTAs per SM, threads per CTA) pair up to 2048 resident
// threads per SM is timed over 10 launches with CUDA events after one warm-up launch.
//
// Build and run (one GPU):
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 paged_kv_cache_385_b200/measure/read_probe.cu -o read_probe
//   ./read_probe
#include <cuda_runtime.h>

#include <cstdio>

__global__ void read_stream(const uint4* __restrict__ p, size_t n, uint4* out) {
  uint4 acc = make_uint4(0, 0, 0, 0);
  size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
#pragma unroll 8
  for (; i < n; i += stride) {
    const uint4 v = __ldg(p + i);
    acc.x ^= v.x;
    acc.y ^= v.y;
    acc.z ^= v.z;
    acc.w ^= v.w;
  }
  if ((acc.x ^ acc.y ^ acc.z ^ acc.w) == 0x12345678u) out[0] = acc;
}

int main() {
  const size_t bytes = 4ull << 30, n = bytes / 16;
  uint4 *p = nullptr, *o = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess || cudaMalloc(&o, 64) != cudaSuccess) {
    std::printf("cudaMalloc failed\n");
    return 1;
  }
  cudaMemset(p, 1, bytes);
  cudaEvent_t a, b;
  cudaEventCreate(&a);
  cudaEventCreate(&b);
  for (int blocks_per_sm : {2, 4, 8, 16}) {
    for (int threads : {256, 512, 1024}) {
      if (threads * blocks_per_sm > 2048) continue;
      const int grid = 148 * blocks_per_sm;
      read_stream<<<grid, threads>>>(p, n, o);
      cudaEventRecord(a);
      for (int r = 0; r < 10; ++r) read_stream<<<grid, threads>>>(p, n, o);
      cudaEventRecord(b);
      cudaEventSynchronize(b);
      float ms = 0.f;
      cudaEventElapsedTime(&ms, a, b);
      std::printf("read probe: grid %d x %d threads: %.1f GB/s\n", grid, threads, 10.0 * bytes / (ms * 1e-3) / 1e9);
    }
  }
  const cudaError_t e = cudaGetLastError();
  std::printf("status %s\n", cudaGetErrorString(e));
  cudaFree(p);
  cudaFree(o);
  return e != cudaSuccess;
}
