// Chunked prefill over paged KV with 5th-generation tensor cores (tcgen05 + tensor memory).
//
// What is computed: as pa_prefill (notes page, kernels section: FlashAttention adapted to paged KV;
// "vLLM 前世今生" §5.4 chunked prefill): row (new token i, group head g) of sequence s is position
// p = start + i and attends over positions 0 .. p of its KV head.
//
// CTA = 128 query rows (tokens x group heads of one sequence and KV head). Per block of 128 keys
// (8 pages), with the block's K and V staged by TMA in 128-byte-swizzled shared memory:
//   S[128 x 128] = Q . K^T      tcgen05.mma kind::f16, A = Q (K-major), B = K (K-major), D in TMEM
//   softmax                     4 warps, one row per thread, S read from TMEM (tcgen05.ld), running
//                               max / sum in registers, P written (bf16/f16) to shared memory, O
//                               rescaled in TMEM when a row's max moved
//   O[128 x 128] += P . V       A = P (K-major), B = V (MN-major: d contiguous), D in TMEM
// Warps: 0-3 softmax + epilogue, 4 TMA producer (Q once, then K/V blocks into a 2-stage ring),
// 5 MMA issuer (one thread) and TMEM owner. Every mbarrier wait is bounded.
#include "internal.h"
#include "pa_device.cuh"
#include "tc05.cuh"

namespace pa {
namespace {

constexpr int kD = 128;
constexpr int kRows = 128;   // query rows per CTA
constexpr int kKeys = 128;   // keys per block
constexpr int kThreads = 192;
constexpr uint32_t kHalf = 16384;  // one 64-element (128-byte) column half of a 128-row tile
constexpr uint32_t kTile = 2 * kHalf;
constexpr uint32_t kQOff = 0;
constexpr uint32_t kStageOff = kTile;                 // stage s: K at kStageOff + s*2*kTile, V after it
constexpr uint32_t kPOff = kStageOff + 4 * kTile;     // P tile
constexpr uint32_t kBarOff = kPOff + kTile;           // mbarriers
constexpr uint32_t kSmemBytes = 1024 + kBarOff + 128;
// barrier slots (8 bytes each)
enum { kQFull = 0, kKvFull0 = 1, kKvEmpty0 = 3, kSFull = 5, kPFull = 6, kODone = 7, kAllDone = 8, kTmemSlot = 9 };

template <bool kBf16>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                  const __grid_constant__ CUtensorMap kmap,
                                                                  const __grid_constant__ CUtensorMap vmap,
                                                                  const MqParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t base = smem_u32(smem);
  const uint32_t bar = base + kBarOff;
  auto B = [&](int i) { return bar + 8u * i; };

  const int tile = blockIdx.x, hk = blockIdx.y, s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group;
  pdl_wait();

  const int q_row0 = p.query_start[s];
  const int n_new = p.query_start[s + 1] - q_row0;
  const int num_rows = n_new * G;
  if (tile * kRows >= num_rows) return;
  const int ctx = p.context_lens[s];
  const int start = ctx - n_new;
  if (start < 0 || ctx > p.max_blocks * 16) {
    if (threadIdx.x == 0) atomicOr(p.err, 8u);
    return;
  }
  if (tile == 0 && threadIdx.x == 0 && num_rows > static_cast<int>(gridDim.x) * kRows) atomicOr(p.err, 8u);
  const int last_row = min((tile + 1) * kRows, num_rows) - 1;
  const int max_lim = start + last_row / G + 1;  // keys visible to the tile's last row
  const int npages = (max_lim + 15) / 16;
  const int nkb = (max_lim + kKeys - 1) / kKeys;

  if (threadIdx.x == 0) {
    mbar_init(B(kQFull), 1);
    mbar_init(B(kKvFull0), 1);
    mbar_init(B(kKvFull0 + 1), 1);
    mbar_init(B(kKvEmpty0), 1);
    mbar_init(B(kKvEmpty0 + 1), 1);
    mbar_init(B(kSFull), 1);
    mbar_init(B(kPFull), 4);
    mbar_init(B(kODone), 1);
    mbar_init(B(kAllDone), 1);
    fence_barrier_init();
  }
  if (warp == 5) tc05::alloc(B(kTmemSlot), 256);
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kBarOff + 8 * kTmemSlot);
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint64_t deadline = globaltimer_ns() + 2000000000ull;
  bool ok = true;

  if (warp == 4) {
    // ---- producer -------------------------------------------------------------------------------
    if (lane == 0) {
      prefetch_tensormap(&qmap);
      mbar_arrive_expect_tx(B(kQFull), kTile);
      const int tok0 = q_row0 + tile * (kRows / G);
      tc05::tma_load_3d(base + kQOff, &qmap, B(kQFull), 0, hk * G, tok0);
      tc05::tma_load_3d(base + kQOff + kHalf, &qmap, B(kQFull), 64, hk * G, tok0);
      const int32_t* bt = p.block_tables + static_cast<int64_t>(s) * p.bt_stride;
      const int oob_row = p.num_blocks * p.num_kv_heads * 16;  // a box starting here is all zero fill
      for (int j = 0; j < nkb && ok; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait_bounded(B(kKvEmpty0 + st), ((j >> 1) - 1) & 1, deadline)) {
          ok = false;
          atomicOr(p.err, 4u);
          break;
        }
        const uint32_t kdst = base + kStageOff + st * 2 * kTile, vdst = kdst + kTile;
        // The block's 8 page ids are loaded together, then its 32 tile copies issued.
        int ys[kKeys / 16];
#pragma unroll
        for (int i = 0; i < kKeys / 16; ++i) {
          const int page = j * (kKeys / 16) + i;
          ys[i] = page < npages ? bt[page] : -1;
        }
#pragma unroll
        for (int i = 0; i < kKeys / 16; ++i) {
          const int page = j * (kKeys / 16) + i;
          const int bid = ys[i];
          ys[i] = oob_row;
          if (page < npages) {
            if (bid >= 0 && bid < p.num_blocks) ys[i] = (bid * p.num_kv_heads + hk) * 16;
            else atomicOr(p.err, 1u);
          }
        }
        mbar_arrive_expect_tx(B(kKvFull0 + st), 2 * kTile);
#pragma unroll
        for (int i = 0; i < kKeys / 16; ++i) {
          const int y = ys[i];
          for (int u = 0; u < 2; ++u) {
            tma_load_2d(kdst + u * kHalf + i * 2048, &kmap, B(kKvFull0 + st), u * 64, y);
            tma_load_2d(vdst + u * kHalf + i * 2048, &vmap, B(kKvFull0 + st), u * 64, y);
          }
        }
      }
    }
  } else if (warp == 5) {
    // ---- MMA issuer ------------------------------------------------------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc05::idesc_f16(kBf16, kRows, kKeys, false, false);
      constexpr uint32_t idesc_pv = tc05::idesc_f16(kBf16, kRows, kD, false, true);
      if (!mbar_wait_bounded(B(kQFull), 0, deadline)) ok = false;
      for (int j = 0; j < nkb && ok; ++j) {
        const int st = j & 1;
        if (!mbar_wait_bounded(B(kKvFull0 + st), (j >> 1) & 1, deadline)) {
          ok = false;
          break;
        }
        tc05::fence_after_sync();
        const uint32_t kbase = base + kStageOff + st * 2 * kTile, vbase = kbase + kTile;
        // S = Q K^T: 8 k-steps of 16 along d (4 per 64-element half, 32 bytes apart).
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
          tc05::mma_f16(tS, tc05::smem_desc_sw128(base + kQOff + off, 16, 1024),
                        tc05::smem_desc_sw128(kbase + off, 16, 1024), idesc_qk, ks > 0);
        }
        tc05::commit(B(kSFull));
        if (!mbar_wait_bounded(B(kPFull), j & 1, deadline)) {
          ok = false;
          break;
        }
        tc05::fence_after_sync();
        // O += P V: 8 k-steps of 16 keys; P K-major (halves of 64 keys), V MN-major (16 keys = 2048 B).
#pragma unroll
        for (int kt = 0; kt < kKeys / 16; ++kt) {
          const uint32_t poff = (kt >> 2) * kHalf + (kt & 3) * 32;
          tc05::mma_f16(tO, tc05::smem_desc_sw128(base + kPOff + poff, 16, 1024),
                        tc05::smem_desc_sw128(vbase + kt * 2048, kHalf, 1024), idesc_pv, (j > 0 || kt > 0));
        }
        tc05::commit(B(kODone));
        tc05::commit(B(kKvEmpty0 + st));
      }
      tc05::commit(B(kAllDone));
      mbar_wait_bounded(B(kAllDone), 0, globaltimer_ns() + 1000000000ull);
      if (!ok) atomicOr(p.err, 4u);
    }
  } else {
    // ---- softmax warps: thread = row ---------------------------------------------------------------
    const int r = threadIdx.x;  // 0..127, TMEM lane r
    const int R = tile * kRows + r;
    const bool valid = R < num_rows;
    const int lim = valid ? start + R / G + 1 : 0;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = p.score_scale_log2;
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < nkb; ++j) {
      const bool got = mbar_wait_bounded(B(kSFull), j & 1, deadline);
      if (!__all_sync(kFull, got)) {
        ok = false;
        break;
      }
      tc05::fence_after_sync();
      const int t0 = j * kKeys;
      // Pass 1: the row's max over the block.
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kKeys / 32; ++c) {
        float v[32];
        tc05::ld32(tS + lane_off + c * 32, v);
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (t0 + c * 32 + k < lim) mx = fmaxf(mx, v[k] * sl2);
      }
      const float mn = fmaxf(m, mx);
      const float ref = mn == -INFINITY ? 0.f : mn;
      const float alpha = ex2(m - ref);
      m = mn;
      // P (and O's rescale) may only change once the previous P . V has finished.
      if (j > 0) {
        const bool done = mbar_wait_bounded(B(kODone), (j - 1) & 1, deadline);
        if (!__all_sync(kFull, done)) {
          ok = false;
          break;
        }
        tc05::fence_after_sync();
      }
      // Pass 2: P = 2^(s - ref) in 16-bit, row sums of the rounded values, into the swizzled P tile.
      float rowsum = 0.f;
#pragma unroll
      for (int c = 0; c < kKeys / 32; ++c) {
        float v[32];
        tc05::ld32(tS + lane_off + c * 32, v);
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int t = t0 + c * 32 + 2 * k;
          const float p0 = t < lim ? ex2(v[2 * k] * sl2 - ref) : 0.f;
          const float p1 = t + 1 < lim ? ex2(v[2 * k + 1] * sl2 - ref) : 0.f;
          w[k] = pack2<kBf16>(p0, p1);
          const float2 f = unpack2<kBf16>(w[k]);
          rowsum += f.x + f.y;
        }
        // 32 keys = 64 bytes = 4 chunks of the row, in key half (c >> 1), chunks (c & 1) * 4 + q.
        const uint32_t row = base + kPOff + (c >> 1) * kHalf + r * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t chunk = ((c & 1) * 4 + q) ^ (r & 7);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + chunk * 16), "r"(w[4 * q]),
                       "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                       : "memory");
        }
      }
      l = l * alpha + rowsum;
      // Rescale O in TMEM when any row of the warp moved its max (j == 0: O is overwritten).
      if (j > 0 && __any_sync(kFull, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          float v[32];
          tc05::ld32(tO + lane_off + c * 32, v);
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] *= alpha;
          tc05::st32(tO + lane_off + c * 32, v);
        }
      }
      // Keys past every row's limit may hold any bits; zero those V rows so 0 * NaN cannot occur.
      if (t0 + kKeys > max_lim) {
        const bool landed = mbar_wait_bounded(B(kKvFull0 + (j & 1)), (j >> 1) & 1, deadline);
        if (!__all_sync(kFull, landed)) {
          ok = false;
          break;
        }
        const uint32_t vbase = base + kStageOff + (j & 1) * 2 * kTile + kTile;
        const int first = max_lim - t0;  // rows [first, 128) of the V tile, both halves
        for (int idx = r; idx < (kKeys - first) * 16; idx += 128) {
          const int row = first + idx / 16, c16 = idx % 16;
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(vbase + (c16 >> 3) * kHalf + row * 128 +
                                                                         (c16 & 7) * 16),
                       "r"(0u)
                       : "memory");
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc05::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(B(kPFull));
    }
    // Epilogue: O / l -> out rows.
    if (ok) {
      const bool done = mbar_wait_bounded(B(kODone), (nkb - 1) & 1, deadline);
      if (__all_sync(kFull, done)) {
        tc05::fence_after_sync();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint16_t* dst = static_cast<uint16_t*>(p.out) + static_cast<int64_t>(q_row0 + (valid ? R / G : 0)) * p.o_stride_t +
                        static_cast<int64_t>(hk * G + R % G) * p.o_stride_h;
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          float v[32];
          tc05::ld32(tO + lane_off + c * 32, v);
          if (valid) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 o;
              o.x = pack2<kBf16>(v[8 * q] * inv, v[8 * q + 1] * inv);
              o.y = pack2<kBf16>(v[8 * q + 2] * inv, v[8 * q + 3] * inv);
              o.z = pack2<kBf16>(v[8 * q + 4] * inv, v[8 * q + 5] * inv);
              o.w = pack2<kBf16>(v[8 * q + 6] * inv, v[8 * q + 7] * inv);
              *reinterpret_cast<uint4*>(dst + c * 32 + 8 * q) = o;
            }
          }
        }
      } else {
        ok = false;
      }
    }
    if (!ok && lane == 0) atomicOr(p.err, 4u);
  }
  pdl_launch_dependents();
  tc05::fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc05::fence_after_sync();
    tc05::dealloc(tmem, 256);
  }
}

}  // namespace

bool prefill_tc_supported(int head_dim, int group) {
  return head_dim == kD && group >= 1 && group <= 16 && (kRows % group) == 0;
}

cudaError_t launch_prefill_tc(KvType kv, const CUtensorMap& qm, const CUtensorMap& km, const CUtensorMap& vm,
                              const MqParams& p, int max_query_len, cudaStream_t st) {
  if (kv != KvType::F16 && kv != KvType::BF16) return cudaErrorInvalidValue;
  auto kern = kv == KvType::BF16 ? prefill_tc_kernel<true> : prefill_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(max_query_len) * p.group;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((rows + kRows - 1) / kRows), p.num_kv_heads, p.num_seqs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, qm, km, vm, p);
}

}  // namespace pa
