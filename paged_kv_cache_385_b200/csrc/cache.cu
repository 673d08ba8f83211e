// reshape_and_cache for sm_100a: scatter new tokens' K and V into their pool slots.
//
// Source: vLLM notes page, "PagedAttention / Cache Engine": the engine computes the page of a
// position and reads or writes that page's data. For token t with slot = slot_mapping[t], K row
// [Hkv, D] goes to k_cache[slot / 16, :, slot % 16, :] (V likewise). A 16-bit cache stores the
// bits unchanged; an e4m3 cache stores e4m3_rn_satfinite(float32(x) * float32(1 / scale)).
//
// Grid (tokens, chunk groups): each thread moves one 16-byte chunk (8 elements) of a token's K or V
// row, so every load of a token is in flight at once (the step writes only a few hundred KB, so
// latency, not bandwidth, sets its time): a 16-byte load from the [T, Hkv, D] input, a 16-byte (or
// 8-byte for e4m3) store into the pool. Slot -1 skips the token; a slot outside the pool is
// skipped and reported.
#include <algorithm>

#include "internal.h"
#include "pa_device.cuh"

namespace pa {
namespace {

template <bool kSrcBf16, KvType KV>
__global__ void __launch_bounds__(128) reshape_and_cache_kernel(const CacheParams p) {
  const int64_t t = blockIdx.x;
  const int64_t slot = p.slots[t];
  if (slot == -1) return;
  if (slot < -1 || slot >= p.num_slots) {
    if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(p.err, 2u);
    return;
  }
  const int64_t blk = slot >> 4, off = slot & 15;
  const int D = p.head_dim;
  const int chunks_per_head = D / 8;
  const int nchunks = p.num_kv_heads * chunks_per_head;
  for (int c = blockIdx.y * blockDim.x + threadIdx.x; c < 2 * nchunks; c += gridDim.y * blockDim.x) {
    const bool is_v = c >= nchunks;
    const int cc = is_v ? c - nchunks : c;
    const int h = cc / chunks_per_head, d0 = (cc % chunks_per_head) * 8;
    const uint16_t* src = static_cast<const uint16_t*>(is_v ? p.value : p.key) +
                          t * (is_v ? p.v_stride_t : p.k_stride_t) + h * (is_v ? p.v_stride_h : p.k_stride_h) + d0;
    const uint4 raw = *reinterpret_cast<const uint4*>(src);
    const int64_t dst_elem = ((blk * p.num_kv_heads + h) * 16 + off) * D + d0;
    if constexpr (KV == KvType::E4M3) {
      const float inv = is_v ? p.v_inv_scale : p.k_inv_scale;
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
      uint32_t codes[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = unpack2<kSrcBf16>(w[i]);
        const uint32_t two = f32x2_to_e4m3x2(__fmul_rn(f.x, inv), __fmul_rn(f.y, inv));
        codes[i >> 1] |= two << (16 * (i & 1));
      }
      uint8_t* dst = static_cast<uint8_t*>(is_v ? p.v_cache : p.k_cache) + dst_elem;
      *reinterpret_cast<uint2*>(dst) = make_uint2(codes[0], codes[1]);
    } else {
      uint16_t* dst = static_cast<uint16_t*>(is_v ? p.v_cache : p.k_cache) + dst_elem;
      *reinterpret_cast<uint4*>(dst) = raw;
    }
  }
}

// Copy whole blocks (every KV head, K and V) for copy-on-write: grid (pairs, chunk groups), one
// 16-byte chunk per thread per cache. Pairs with an id outside the pool are skipped and reported.
__global__ void __launch_bounds__(256) copy_blocks_kernel(const CopyParams p) {
  const int64_t pair = blockIdx.x;
  const int64_t src = p.mapping[2 * pair], dst = p.mapping[2 * pair + 1];
  if (src < 0 || src >= p.num_blocks || dst < 0 || dst >= p.num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(p.err, 1u);
    return;
  }
  if (src == dst) return;
  const int64_t chunks = p.block_bytes / 16;
  for (int64_t c = static_cast<int64_t>(blockIdx.y) * blockDim.x + threadIdx.x; c < chunks;
       c += static_cast<int64_t>(gridDim.y) * blockDim.x) {
    const uint4* ks = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.k_cache) + src * p.block_bytes) + c;
    const uint4* vs = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.v_cache) + src * p.block_bytes) + c;
    const uint4 kv = *ks, vv = *vs;
    *(reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.k_cache) + dst * p.block_bytes) + c) = kv;
    *(reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.v_cache) + dst * p.block_bytes) + c) = vv;
  }
}

}  // namespace

cudaError_t launch_copy_blocks(const CopyParams& p, cudaStream_t st) {
  if (p.num_pairs == 0) return cudaSuccess;
  const int64_t chunks = p.block_bytes / 16;
  const unsigned groups = static_cast<unsigned>(std::min<int64_t>(65535, (chunks + 255) / 256));
  copy_blocks_kernel<<<dim3(static_cast<unsigned>(p.num_pairs), groups), 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_reshape_and_cache(int src_bf16, KvType cache, const CacheParams& p, cudaStream_t st) {
  if (p.num_tokens == 0) return cudaSuccess;
  const int chunks = 2 * p.num_kv_heads * (p.head_dim / 8);
  const unsigned groups = static_cast<unsigned>(std::min(65535, (chunks + 127) / 128));
  const dim3 grid(static_cast<unsigned>(p.num_tokens), groups);
  if (cache == KvType::E4M3) {
    if (src_bf16) reshape_and_cache_kernel<true, KvType::E4M3><<<grid, 128, 0, st>>>(p);
    else reshape_and_cache_kernel<false, KvType::E4M3><<<grid, 128, 0, st>>>(p);
  } else if (cache == KvType::BF16) {
    reshape_and_cache_kernel<true, KvType::BF16><<<grid, 128, 0, st>>>(p);
  } else {
    reshape_and_cache_kernel<false, KvType::F16><<<grid, 128, 0, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace pa
