// Multi-query paged attention for sm_100a: tiles of 16 query rows per warp against a stream of
// 16-token pages, the dense tensor-core part of the path. Two uses:
//
// * Shared prefix ("cascade", MODE 0). Source: "vLLM 前世今生" section 3.2 (several sequences point at
//   the same physical blocks, e.g. a shared prompt prefix) and the notes page's prefix-caching
//   section (a shared prompt prefix computed once). Per KV head, all B * G query rows (sequence s,
//   group member g) against the prefix pages every block table shares: partial softmax state
//   (m, l, acc) per row and prefix chunk, merged later with the sequence's own suffix. It equals the
//   plain definition over the whole context (the same softmax split at a token boundary).
// * Chunked prefill (MODE 1). Source: the notes page's kernels section (FlashAttention adapted to
//   paged KV) and "vLLM 前世今生" section 5.4 (chunked prefill). Per sequence and KV head, rows
//   (new token i, group member g) attend causally over the sequence's pages: position
//   start + i sees tokens 0 .. start + i. Output written directly.
//
// Kernel: four consumer warps own 16 rows each; a fifth warp produces: it streams the CTA's K and V
// pages with TMA into a ring of stages guarded by full/empty mbarriers. Per page a consumer warp
// does S[16 rows x 16 tok] = Q K^T (mma.sync m16n8k16, K^T fragments by ldmatrix), an online
// softmax per row (per-row token limits: context, prefix end, or the causal diagonal), and
// O[16 x D] += P V (P reused from the score fragments, V^T fragments by ldmatrix.trans).
#include "internal.h"
#include "pa_device.cuh"

namespace pa {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kRowsPerCta = 16 * kConsumerWarps;
constexpr int kPrefixStages = 4;

template <KvType KV, int D>
struct PCfg {
  static_assert(KV != KvType::E4M3, "shared-prefix kernel takes 16-bit pages");
  static constexpr int kRowBytes = D * 2;
  static constexpr int kSubPages = kRowBytes / 128;
  static constexpr int kSubElems = 64;
  static constexpr int kPageBytes = 16 * kRowBytes;
  static constexpr int kStageBytes = 2 * kPageBytes;
  static constexpr int kThreads = 32 * (kConsumerWarps + 1);
  static constexpr int kSmemBytes = 1024 + kPrefixStages * kStageBytes + 2 * kPrefixStages * 8;
  static constexpr bool kBf16 = KV == KvType::BF16;
};

__device__ __forceinline__ uint32_t swz128(int tok, int chunk) {
  return static_cast<uint32_t>(tok * 128 + ((chunk ^ (tok & 7)) << 4));
}

template <KvType KV, int D, int MODE>
__global__ void __launch_bounds__(PCfg<KV, D>::kThreads) mq_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                    const __grid_constant__ CUtensorMap vmap,
                                                                    const MqParams p) {
  using C = PCfg<KV, D>;
  constexpr bool kPrefill = MODE == 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t ring = smem_u32(smem);
  const uint32_t full0 = smem_u32(smem + kPrefixStages * C::kStageBytes);
  const uint32_t empty0 = full0 + 8 * kPrefixStages;

  const int tile = blockIdx.x, hk = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group;
  const int Hq = p.num_kv_heads * G;
  pdl_wait();
  // Shared-prefix mode: the suffix decode after this grid waits for it only at its merge, so it may
  // launch now and overlap its page loop with this kernel.
  if constexpr (!kPrefill) pdl_launch_dependents();

  // Rows and pages of this CTA.
  int chunk = 0, s_seq = 0, num_rows, j0, npages, q_row0 = 0, start = 0;
  const int32_t* bt_row;
  if constexpr (kPrefill) {
    s_seq = blockIdx.z;
    q_row0 = p.query_start[s_seq];
    const int n_new = p.query_start[s_seq + 1] - q_row0;
    num_rows = n_new * G;
    if (tile * kRowsPerCta >= num_rows) return;
    const int ctx = p.context_lens[s_seq];
    start = ctx - n_new;
    if (tile == 0 && threadIdx.x == 0 && num_rows > static_cast<int>(gridDim.x) * kRowsPerCta)
      atomicOr(p.err, 8u);  // more new tokens than max_query_len: the rows past the grid are not computed
    const int last_tok = min(tile * kRowsPerCta + kRowsPerCta, num_rows) - 1;
    const int last_key = start + last_tok / G;  // the CTA's last row sees keys 0 .. last_key
    if (start < 0 || ctx > p.max_blocks * 16) {
      if (threadIdx.x == 0) atomicOr(p.err, 8u);
      return;
    }
    j0 = 0;
    npages = last_key / 16 + 1;
    bt_row = p.block_tables + static_cast<int64_t>(s_seq) * p.bt_stride;
  } else {
    chunk = blockIdx.z;
    num_rows = p.num_seqs * G;
    j0 = chunk * (p.chunk_tokens / 16);
    npages = min(p.chunk_tokens / 16, p.prefix_tokens / 16 - j0);
    bt_row = p.block_tables;  // sequence 0's row: every row shares these blocks
  }

  if (threadIdx.x == 0) {
    for (int st = 0; st < kPrefixStages; ++st) {
      mbar_init(full0 + 8 * st, 1);
      mbar_init(empty0 + 8 * st, kConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  const uint64_t deadline = globaltimer_ns() + 2000000000ull;
  bool ok = true;
  if (warp == kConsumerWarps) {
    // ---- producer: block ids 32 at a time in lanes, lane 0 streams the pages ------------------
    int bid = -1;
    if (lane == 0) prefetch_tensormap(&kmap), prefetch_tensormap(&vmap);
    for (int i = 0; i < npages; ++i) {
      if ((i & 31) == 0) {
        bid = i + lane < npages ? bt_row[j0 + i + lane] : -1;
        const bool bad = i + lane < npages && (bid < 0 || bid >= p.num_blocks);
        if (__any_sync(kFull, bad) && lane == 0) atomicOr(p.err, 1u);
      }
      const int b = __shfl_sync(kFull, bid, i & 31);
      const int st = i % kPrefixStages;
      if (lane == 0 && ok) {
        if (i >= kPrefixStages && !mbar_wait_bounded(empty0 + 8 * st, ((i / kPrefixStages) - 1) & 1, deadline)) {
          ok = false;
          atomicOr(p.err, 4u);
        }
        if (ok) {
          const uint32_t bar = full0 + 8 * st;
          if (b < 0 || b >= p.num_blocks) {
            mbar_arrive(bar);
          } else {
            mbar_arrive_expect_tx(bar, 2 * C::kPageBytes);
            const uint32_t dst = ring + st * C::kStageBytes;
            const int y = (b * p.num_kv_heads + hk) * 16;
#pragma unroll
            for (int u = 0; u < C::kSubPages; ++u) {
              tma_load_2d(dst + u * 2048, &kmap, bar, u * C::kSubElems, y);
              tma_load_2d(dst + C::kPageBytes + u * 2048, &vmap, bar, u * C::kSubElems, y);
            }
          }
        }
      }
      __syncwarp();
    }
    return;
  }

  // ---- consumers: 16 query rows each ------------------------------------------------------------
  constexpr int KS = D / 16;  // k-steps of Q K^T
  constexpr int NT = D / 8;   // n-tiles of P V
  const int r = lane >> 2, q4 = lane & 3;
  const int row_lo = tile * kRowsPerCta + warp * 16 + r, row_hi = row_lo + 8;

  // A row's last visible token + 1: its context, the prefix end, or its causal diagonal.
  auto row_limit = [&](int row) {
    if (row >= num_rows) return 0;
    if constexpr (kPrefill) return start + row / G + 1;
    return min(p.context_lens[row / G], p.prefix_tokens);
  };
  const int lim_lo = row_limit(row_lo), lim_hi = row_limit(row_hi);
  int lim_max = max(lim_lo, lim_hi);
  for (int off = 4; off < 32; off <<= 1) lim_max = max(lim_max, __shfl_xor_sync(kFull, lim_max, off));


  uint32_t qa[KS][4];
  {
    auto qrow = [&](int row) -> const uint16_t* {
      const int rr = min(row, num_rows - 1);
      const int64_t qr = kPrefill ? static_cast<int64_t>(q_row0 + rr / G) : static_cast<int64_t>(rr / G);
      return static_cast<const uint16_t*>(p.q) + qr * p.q_stride_s + static_cast<int64_t>(hk * G + rr % G) * p.q_stride_h;
    };
    const uint16_t* ql = qrow(row_lo);
    const uint16_t* qh = qrow(row_hi);
    const bool vl = row_lo < num_rows, vh = row_hi < num_rows;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int d = 16 * ks + 2 * q4;
      qa[ks][0] = vl ? *reinterpret_cast<const uint32_t*>(ql + d) : 0u;
      qa[ks][1] = vh ? *reinterpret_cast<const uint32_t*>(qh + d) : 0u;
      qa[ks][2] = vl ? *reinterpret_cast<const uint32_t*>(ql + d + 8) : 0u;
      qa[ks][3] = vh ? *reinterpret_cast<const uint32_t*>(qh + d + 8) : 0u;
    }
  }
  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
  const float sl2 = p.score_scale_log2;

  const int x7 = lane & 7;
  const int t_tok = ((lane >> 4) << 3) | x7, t_co = (lane >> 3) & 1;          // K^T matrices
  const int a_tok = (((lane >> 3) & 1) << 3) | x7, a_co = lane >> 4;          // V^T matrices

  int fail_at = 0;
  for (int i = 0; i < npages; ++i) {
    const int st = i % kPrefixStages;
    const bool got = mbar_wait_bounded(full0 + 8 * st, (i / kPrefixStages) & 1, deadline);
    if (!__all_sync(kFull, got)) {
      ok = false;
      fail_at = i;
      if (lane == 0) atomicOr(p.err, 4u);
      break;
    }
    const uint32_t kb = ring + st * C::kStageBytes, vb = kb + C::kPageBytes;
    const int t0 = (j0 + i) * 16;
    if (t0 >= lim_max) {  // past every row of this warp (causal tail): release the stage only
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * st);
      continue;
    }

    // S = Q K^T for tokens t0 .. t0 + 15 (two n-tiles of 8 tokens).
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t b[4];
      ldmatrix_x4(b, kb + (ks >> 2) * 2048 + swz128(t_tok, ((ks & 3) << 1) + t_co));
      mma_16816<C::kBf16>(sc[0], qa[ks], b[0], b[1]);
      mma_16816<C::kBf16>(sc[1], qa[ks], b[2], b[3]);
    }
    // Mask per row, online softmax (log2 units).
    float s[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const int t = t0 + 8 * n + 2 * q4;
      s[n][0] = t < lim_lo ? sc[n][0] * sl2 : -INFINITY;
      s[n][1] = t + 1 < lim_lo ? sc[n][1] * sl2 : -INFINITY;
      s[n][2] = t < lim_hi ? sc[n][2] * sl2 : -INFINITY;
      s[n][3] = t + 1 < lim_hi ? sc[n][3] * sl2 : -INFINITY;
    }
    float mx_lo = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
    float mx_hi = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(kFull, mx_lo, 1));
    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(kFull, mx_lo, 2));
    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(kFull, mx_hi, 1));
    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(kFull, mx_hi, 2));
    const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
    // A row with no valid token so far keeps max -inf; use 0 as its reference so no NaN appears.
    const float ref_lo = mn_lo == -INFINITY ? 0.f : mn_lo, ref_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
    const float al_lo = ex2(m_lo - ref_lo), al_hi = ex2(m_hi - ref_hi);
    m_lo = mn_lo;
    m_hi = mn_hi;
    uint32_t pa[4];
    pa[0] = pack2<C::kBf16>(ex2(s[0][0] - ref_lo), ex2(s[0][1] - ref_lo));
    pa[1] = pack2<C::kBf16>(ex2(s[0][2] - ref_hi), ex2(s[0][3] - ref_hi));
    pa[2] = pack2<C::kBf16>(ex2(s[1][0] - ref_lo), ex2(s[1][1] - ref_lo));
    pa[3] = pack2<C::kBf16>(ex2(s[1][2] - ref_hi), ex2(s[1][3] - ref_hi));
    {
      const float2 a = unpack2<C::kBf16>(pa[0]), b = unpack2<C::kBf16>(pa[2]);
      const float2 c = unpack2<C::kBf16>(pa[1]), d = unpack2<C::kBf16>(pa[3]);
      l_lo = l_lo * al_lo + (a.x + a.y + b.x + b.y);
      l_hi = l_hi * al_hi + (c.x + c.y + d.x + d.y);
    }
    if (__any_sync(kFull, al_lo != 1.f || al_hi != 1.f)) {  // skipped once the running max settles
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        acc[n][0] *= al_lo;
        acc[n][1] *= al_lo;
        acc[n][2] *= al_hi;
        acc[n][3] *= al_hi;
      }
    }
    // Tokens no row of this warp may read can hold any bits: zero their V so 0 * NaN never happens.
    const int nvalid = min(16, lim_max - t0);
    uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
    if (nvalid < 16) {
      mlo = (2 * q4 < nvalid ? 0x0000ffffu : 0u) | (2 * q4 + 1 < nvalid ? 0xffff0000u : 0u);
      mhi = (2 * q4 + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * q4 + 9 < nvalid ? 0xffff0000u : 0u);
    }
    // O += P V (pairs of n-tiles of 8 d per ldmatrix.x4.trans).
#pragma unroll
    for (int c = 0; c < NT; c += 2) {
      uint32_t b[4];
      ldmatrix_x4_trans(b, vb + (c >> 3) * 2048 + swz128(a_tok, (c & 7) + a_co));
      if (nvalid < 16) {
        b[0] &= mlo;
        b[1] &= mhi;
        b[2] &= mlo;
        b[3] &= mhi;
      }
      mma_16816<C::kBf16>(acc[c], pa, b[0], b[1]);
      mma_16816<C::kBf16>(acc[c + 1], pa, b[2], b[3]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * st);
  }
  if constexpr (kPrefill) pdl_launch_dependents();
  if (!ok) {
    // Give the copies the producer may have issued for pages fail_at .. fail_at + stages - 1 a bounded
    // chance to land before the CTA's shared memory goes. It cannot have issued any later page: that
    // needs this warp's release of page fail_at's stage, and each earlier fill of those stages was
    // consumed here, so the parity waits are exact.
    const uint64_t drain_deadline = globaltimer_ns() + 100000000ull;
    for (int k = fail_at; k < min(fail_at + kPrefixStages, npages); ++k)
      mbar_wait_bounded(full0 + 8 * (k % kPrefixStages), (k / kPrefixStages) & 1, drain_deadline);
    return;
  }

  l_lo += __shfl_xor_sync(kFull, l_lo, 1);
  l_lo += __shfl_xor_sync(kFull, l_lo, 2);
  l_hi += __shfl_xor_sync(kFull, l_hi, 1);
  l_hi += __shfl_xor_sync(kFull, l_hi, 2);

  if constexpr (kPrefill) {
    // Normalised rows straight to the output.
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int row = half ? row_hi : row_lo;
      if (row >= num_rows) continue;
      const float inv = 1.f / (half ? l_hi : l_lo);
      uint16_t* dst = static_cast<uint16_t*>(p.out) + static_cast<int64_t>(q_row0 + row / G) * p.o_stride_t +
                      static_cast<int64_t>(hk * G + row % G) * p.o_stride_h;
#pragma unroll
      for (int n = 0; n < NT; ++n)
        *reinterpret_cast<uint32_t*>(dst + 8 * n + 2 * q4) =
            pack2<C::kBf16>(acc[n][2 * half] * inv, acc[n][2 * half + 1] * inv);
    }
  } else {
    // Partial state of each row -> workspace slot `chunk` of (sequence, query head).
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int row = half ? row_hi : row_lo;
      if (row >= num_rows) continue;
      const int sq = row / G, h = hk * G + row % G;
      const int64_t slot = (static_cast<int64_t>(sq) * Hq + h) * p.ws_parts + chunk;
      float* dst = p.ws_acc + slot * D;
#pragma unroll
      for (int n = 0; n < NT; ++n)
        *reinterpret_cast<float2*>(dst + 8 * n + 2 * q4) = make_float2(acc[n][2 * half], acc[n][2 * half + 1]);
      if (q4 == 0) {
        p.ws_ml[slot * 2] = half ? m_hi : m_lo;
        p.ws_ml[slot * 2 + 1] = half ? l_hi : l_lo;
      }
    }
  }
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_prefix(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <KvType KV, int D, int MODE>
cudaError_t launch_mq_t(const CUtensorMap& km, const CUtensorMap& vm, const MqParams& p, dim3 grid, cudaStream_t st) {
  using C = PCfg<KV, D>;
  auto kern = mq_kernel<KV, D, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  return launch_pdl_prefix(kern, grid, dim3(C::kThreads), C::kSmemBytes, st, km, vm, p);
}

template <int MODE>
cudaError_t launch_mq(KvType kv, int head_dim, const CUtensorMap& km, const CUtensorMap& vm, const MqParams& p,
                      dim3 grid, cudaStream_t st) {
  if (kv == KvType::F16) {
    return head_dim == 128 ? launch_mq_t<KvType::F16, 128, MODE>(km, vm, p, grid, st)
                           : launch_mq_t<KvType::F16, 64, MODE>(km, vm, p, grid, st);
  }
  if (kv == KvType::BF16) {
    return head_dim == 128 ? launch_mq_t<KvType::BF16, 128, MODE>(km, vm, p, grid, st)
                           : launch_mq_t<KvType::BF16, 64, MODE>(km, vm, p, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_prefix(KvType kv, int head_dim, const CUtensorMap& km, const CUtensorMap& vm, const MqParams& p,
                          cudaStream_t st) {
  const int rows = p.num_seqs * p.group;
  const dim3 grid((rows + kRowsPerCta - 1) / kRowsPerCta, p.num_kv_heads, p.num_chunks);
  return launch_mq<0>(kv, head_dim, km, vm, p, grid, st);
}

cudaError_t launch_prefill(KvType kv, int head_dim, const CUtensorMap& km, const CUtensorMap& vm, const MqParams& p,
                           int max_query_len, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(max_query_len) * p.group;
  const dim3 grid(static_cast<unsigned>((rows + kRowsPerCta - 1) / kRowsPerCta), p.num_kv_heads, p.num_seqs);
  return launch_mq<1>(kv, head_dim, km, vm, p, grid, st);
}

}  // namespace pa
