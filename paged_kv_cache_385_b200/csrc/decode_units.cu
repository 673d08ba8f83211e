// Split-context paged decode with one warp per partition, persistent (sm_100a).
//
// Same result as the per-partition CTAs of decode.cu (vLLM notes page, "PagedAttention" and
// "内核优化"; "vLLM 前世今生" section 3.2): for each (sequence s, KV head hk, partition p) of
// partition_tokens tokens, the G query heads of hk attend over the partition's pages; the partial
// softmax state (acc, m, l) goes to the workspace and reduce_kernel merges a sequence's partitions
// in a fixed order (a sequence with one partition is written directly).
//
// Why a second form: with short partitions (<= 512 tokens, e.g. the 70B-shaped long-context batch)
// a CTA per partition spends a large share of its life on fixed costs (launch, table and q reads,
// the first page's latency, the merge of its warps) while its ring is not streaming. Here each
// resident warp takes whole partitions (units) in turn, u = warp id, + number of warps, ..., over
// a compact list of the batch's non-empty units, and its TMA ring runs on from one unit into the
// next: the first pages of unit k + 1 are in flight while unit k finishes and writes its partial.
// Nothing is merged across warps, so no barrier stops the CTA.
//
// Units. Sequence s has nparts(s) = max(1, ceil(span_s / partition_tokens)) partitions (span = its
// context, capped like the CTA form). Each CTA builds the exclusive prefix sum of nparts over the
// batch in shared memory; unit c is (s, p, hk) with c = (start[s] + p) * Hkv + hk. A sequence with an
// empty context has one unit with no pages, which writes zeros.
//
// pa_decode_step: the warp that enters the last partition of (s, hk) first writes the new token's
// K/V row of head hk into its slot (fenced for the async proxy) and only then issues that unit's
// page copies, so the copy of the slot's page sees the new row.
#include <algorithm>

#include "decode_math.cuh"
#include "internal.h"
#include "pa_device.cuh"

namespace pa {
namespace {

struct Unit {
  int s, hk, part, nparts;
  int j0;       // first logical block of the partition
  int np;       // pages of the partition (0 for an empty context)
  int ctx_eff;  // tokens [0, ctx_eff) exist for this sequence's bookkeeping
};

template <KvType KV, QType QT, int D, int NT, int OCC>
struct UnitCfg {
  using C = Cfg<KV, QT, D, NT, 1, OCC>;
  static constexpr int kBarBytes = C::kWarps * C::kStages * 8;
  static constexpr int kMetaBytes = C::kWarps * C::kStages * 4;
  static constexpr int kTableInts = 2 * kUnitMaxSeqs + 1;  // starts [B + 1], spans [B]
  static constexpr int kSmemBytes = 1024 + C::kPipeBytes + kBarBytes + kMetaBytes + kTableInts * 4;
};

template <KvType KV, QType QT, int D, int NT, int OCC>
__global__ void __launch_bounds__(kDecodeWarps * 32, OCC)
    decode_units_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                        const DecodeParams p) {
  using U = UnitCfg<KV, QT, D, NT, OCC>;
  using C = typename U::C;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kPipeBytes);
  int* meta = reinterpret_cast<int*>(smem + C::kPipeBytes + U::kBarBytes);  // [warp][stage]: page valid
  int* starts = meta + C::kWarps * S;                                        // [B + 1]
  int* spans = starts + kUnitMaxSeqs + 1;                                    // [B]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();  // pages, tables, q and lengths may come from the previous kernel on the stream
  const int B = p.num_seqs, Hkv = p.num_kv_heads, PT = p.partition_tokens, ppp = PT / 16;
  const int start = p.start_tokens;

  // ---- the batch's units: spans, partitions per sequence, exclusive prefix sum -----------------
  {
    constexpr int T = C::kThreads;
    const int per = (B + T - 1) / T;
    const int i0 = threadIdx.x * per, i1 = min(i0 + per, B);
    int sum = 0;
    for (int i = i0; i < i1; ++i) {
      const int ctx = p.context_lens[i];
      const int ctx_cap = min(ctx, p.max_blocks * 16);
      const int span = min(max(ctx_cap - start, 0), p.num_partitions * PT);
      if ((ctx_cap < ctx || ctx < 0 || span < ctx_cap - start) && blockIdx.x == 0) atomicOr(p.err, 8u);
      spans[i] = span;
      sum += max(1, (span + PT - 1) / PT);
    }
    // Block-wide exclusive scan of the per-thread sums (warp shuffles, then the four warp totals).
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(kFull, incl, off);
      if (lane >= off) incl += v;
    }
    __shared__ int warp_tot[C::kWarps];
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    int run = base + incl - sum;
    for (int i = i0; i < i1; ++i) {
      starts[i] = run;
      run += max(1, (spans[i] + PT - 1) / PT);
    }
    if (threadIdx.x == T - 1) starts[B] = base + incl;
  }
  // Per-warp barriers of the page ring.
  const uint32_t bar0 = smem_u32(bars + warp * S);
  if (lane == 0) {
    for (int st = 0; st < S; ++st) mbar_init(bar0 + 8 * st, 1);
    fence_barrier_init();
    if (warp == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
    }
  }
  __syncthreads();
  const int total = starts[B] * Hkv;
  const int W = gridDim.x * C::kWarps;
  const int wg = blockIdx.x * C::kWarps + warp;

  auto unit_of = [&](int c, Unit& u) {
    const int qi = c / Hkv;
    u.hk = c - qi * Hkv;
    int lo = 0, hi = B - 1;  // the last s with starts[s] <= qi (starts strictly increase)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (starts[mid] <= qi) lo = mid;
      else hi = mid - 1;
    }
    u.s = lo;
    u.part = qi - starts[lo];
    u.nparts = starts[lo + 1] - starts[lo];
    const int span = spans[lo];
    u.ctx_eff = start + span;
    u.j0 = start / 16 + u.part * ppp;
    u.np = max(0, min(ppp, (u.ctx_eff + 15) / 16 - u.j0));
  };
  // Block id of page `lane` of unit u (lanes past its pages: -1).
  auto bids_of = [&](const Unit& u) -> int {
    return lane < u.np ? p.block_tables[static_cast<int64_t>(u.s) * p.bt_stride + u.j0 + lane] : -1;
  };

  // pa_decode_step: before the last partition of (s, hk) issues a page, write head hk's new K/V row.
  auto write_new_token = [&](const Unit& u) {
    if (p.new_k == nullptr || u.part != u.nparts - 1) return;
    const int64_t slot = p.new_slots[u.s];
    const bool do_write = slot >= 0 && slot < static_cast<int64_t>(p.num_blocks) * 16;
    if (!do_write) {
      if (slot != -1 && lane == 0) atomicOr(p.err, 2u);
      return;
    }
    constexpr int kChunks = D / 8;  // 16-byte input chunks per row
    for (int c = lane; c < 2 * kChunks; c += 32) {
      const bool is_v = c >= kChunks;
      const int d0 = (is_v ? c - kChunks : c) * 8;
      const uint16_t* src = static_cast<const uint16_t*>(is_v ? p.new_v : p.new_k) +
                            u.s * (is_v ? p.nv_stride_s : p.nk_stride_s) + u.hk * (is_v ? p.nv_stride_h : p.nk_stride_h) +
                            d0;
      const uint4 raw = *reinterpret_cast<const uint4*>(src);
      const int64_t dst = (((slot >> 4) * p.num_kv_heads + u.hk) * 16 + (slot & 15)) * D + d0;
      if constexpr (C::kFp8) {
        const float inv = is_v ? p.v_inv_scale : p.k_inv_scale;
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t codes[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = p.new_src_bf16 ? unpack2<true>(w[i]) : unpack2<false>(w[i]);
          codes[i >> 1] |= f32x2_to_e4m3x2(__fmul_rn(f.x, inv), __fmul_rn(f.y, inv)) << (16 * (i & 1));
        }
        *reinterpret_cast<uint2*>(static_cast<uint8_t*>(is_v ? p.v_cache : p.k_cache) + dst) =
            make_uint2(codes[0], codes[1]);
      } else {
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(is_v ? p.v_cache : p.k_cache) + dst) = raw;
      }
    }
    fence_proxy_async_global();
    __syncwarp();
  };

  // The pages stream through L2 once (read first when L2 needs room); the partials are read back by
  // the merge kernel right after this grid (kept), so they need not go to DRAM and back.
  const uint64_t stream_pol = l2_evict_first_policy(), keep_pol = l2_evict_last_policy();

  // ---- issue side: the next page of this warp's unit stream into its ring ----------------------
  const uint32_t wbuf_s = smem_u32(smem + warp * S * C::kStageBytes);
  int ic = wg, ij = 0, issued = 0;
  Unit iu{};
  int ibid = -1, nbid = -1;  // block ids of the unit being issued and of the next one (prefetched)
  if (ic < total) {
    unit_of(ic, iu);
    ibid = bids_of(iu);
    if (ic + W < total) {
      Unit nu;
      unit_of(ic + W, nu);
      nbid = bids_of(nu);
    }
    write_new_token(iu);
  }
  auto issue_next = [&]() {
    while (ic < total && ij >= iu.np) {  // on to the next unit (units without pages pass through)
      ic += W;
      if (ic >= total) return;
      unit_of(ic, iu);
      ij = 0;
      ibid = nbid;
      if (ic + W < total) {
        Unit nu;
        unit_of(ic + W, nu);
        nbid = bids_of(nu);
      }
      write_new_token(iu);
    }
    if (ic >= total) return;
    const int bid = __shfl_sync(kFull, ibid, ij);
    if (lane == 0) {
      const int st = issued % S;
      const uint32_t bar = bar0 + 8 * st;
      const bool valid = bid >= 0 && bid < p.num_blocks;
      meta[warp * S + st] = valid;
      if (!valid) {
        atomicOr(p.err, 1u);
        mbar_arrive(bar);  // skipped page: complete the phase without data
      } else {
        mbar_arrive_expect_tx(bar, 2 * C::kPageBytes);
        const uint32_t kdst = wbuf_s + st * C::kStageBytes;
        const int y = (bid * p.num_kv_heads + iu.hk) * 16;
#pragma unroll
        for (int u = 0; u < C::kSubPages; ++u) {
          tma_load_2d_hint(kdst + u * 2048, &kmap, bar, u * C::kSubElems, y, stream_pol);
          tma_load_2d_hint(kdst + C::kPageBytes + u * 2048, &vmap, bar, u * C::kSubElems, y, stream_pol);
        }
      }
    }
    ++ij;
    ++issued;
  };

  // ---- consume side -----------------------------------------------------------------------------
  TcMath<C, D, NT> tc;
  tc.lane = lane;
  for (int k = 0; k < S; ++k) issue_next();
  const uint64_t deadline = globaltimer_ns() + 2000000000ull;
  bool ok = true;
  int consumed = 0;
  int cs = -1, chk = -1;  // (sequence, KV head) whose query the fragments hold
  for (int cc = wg; cc < total && ok; cc += W) {
    Unit cu;
    unit_of(cc, cu);
    if (cu.s != cs || cu.hk != chk) {
      tc.init(p, cu.s, cu.hk, lane);
      cs = cu.s;
      chk = cu.hk;
    } else {
      tc.reset();
    }
    // Pages two at a time (one softmax step for both) while the unit has two left, else one.
    for (int j = 0; j < cu.np;) {
      const int st = consumed % S;
      const bool pair = j + 1 < cu.np;
      const int st2 = (consumed + 1) % S;
      const bool got = mbar_wait_bounded(bar0 + 8 * st, (consumed / S) & 1, deadline) &&
                       (!pair || mbar_wait_bounded(bar0 + 8 * st2, ((consumed + 1) / S) & 1, deadline));
      if (!__all_sync(kFull, got)) {
        ok = false;
        break;
      }
      const uint32_t ka = wbuf_s + st * C::kStageBytes, kb2 = wbuf_s + st2 * C::kStageBytes;
      const int nva = min(16, cu.ctx_eff - (cu.j0 + j) * 16);
      const bool va = meta[warp * S + st] != 0;
      if (pair) {
        const int nvb = min(16, cu.ctx_eff - (cu.j0 + j + 1) * 16);
        const bool vb = meta[warp * S + st2] != 0;
        if (va && vb) {
          tc.page2(ka, ka + C::kPageBytes, nva, kb2, kb2 + C::kPageBytes, nvb, p.score_scale_log2);
        } else {  // a page skipped for a bad block id (already reported)
          if (va) tc.page(ka, ka + C::kPageBytes, nva, p.score_scale_log2);
          if (vb) tc.page(kb2, kb2 + C::kPageBytes, nvb, p.score_scale_log2);
        }
      } else if (va) {
        tc.page(ka, ka + C::kPageBytes, nva, p.score_scale_log2);
      }
      __syncwarp();
      const int n = pair ? 2 : 1;
      for (int i = 0; i < n; ++i) {
        ++consumed;
        issue_next();
      }
      j += n;
    }
    if (!ok) break;
    tc.template write_global<C::kQBf16>(p, cu.s, cu.hk, cu.part, !p.always_partials && cu.nparts <= 1, keep_pol);
  }
  if (!ok) {
    // Give the copies still in flight a bounded chance to land before the shared memory goes.
    for (int k = consumed; k < issued; ++k)
      mbar_wait_bounded(bar0 + 8 * (k % S), (k / S) & 1, globaltimer_ns() + 100000000ull);
    if (lane == 0) atomicOr(p.err, 4u);
  }
  pdl_launch_dependents();
}

template <KvType KV, QType QT, int D, int NT, int OCC>
cudaError_t launch_units_one(const CUtensorMap& km, const CUtensorMap& vm, const DecodeParams& p, cudaStream_t st) {
  using U = UnitCfg<KV, QT, D, NT, OCC>;
  auto kern = decode_units_kernel<KV, QT, D, NT, OCC>;
  static int configured_devices = 0;  // bit per device
  static int sm_count[31] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int sms = dev < 31 ? __atomic_load_n(&sm_count[dev], __ATOMIC_ACQUIRE) : 0;
  if (dev >= 31 || !(__atomic_load_n(&configured_devices, __ATOMIC_ACQUIRE) & (1 << dev))) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, U::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (dev < 31) {
      __atomic_store_n(&sm_count[dev], sms, __ATOMIC_RELEASE);
      __atomic_fetch_or(&configured_devices, 1 << dev, __ATOMIC_ACQ_REL);
    }
  }
  // One wave of resident CTAs, or fewer when the batch has fewer units than warps.
  const int64_t units = static_cast<int64_t>(p.num_seqs) * p.num_kv_heads * p.num_partitions;
  const int64_t want = (units + kDecodeWarps - 1) / kDecodeWarps;
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(sms) * OCC));
  return launch_pdl(kern, dim3(grid), dim3(kDecodeWarps * 32), U::kSmemBytes, st, km, vm, p);
}

template <KvType KV, QType QT, int D>
cudaError_t launch_units_kv(int nt, int group, const CUtensorMap& km, const CUtensorMap& vm, const DecodeParams& p,
                            cudaStream_t st) {
  if (nt == 1) {
    if constexpr (KV == KvType::E4M3) {
      return launch_units_one<KV, QT, D, 1, 4>(km, vm, p, st);
    } else {
      if (group > 1) return launch_units_one<KV, QT, D, 1, 3>(km, vm, p, st);
      return launch_units_one<KV, QT, D, 1, 2>(km, vm, p, st);
    }
  }
  if (nt == 2) return launch_units_one<KV, QT, D, 2, 2>(km, vm, p, st);
  return cudaErrorInvalidValue;
}

}  // namespace

bool decode_units_supported(const DecodeConfig& c, const DecodeParams& p) {
  if (!decode_supported(c) || c.kernel != 1) return false;
  if (p.num_seqs > kUnitMaxSeqs || p.partition_tokens > kUnitMaxPartitionTokens) return false;
  if (p.start_tokens != 0 || p.always_partials || p.merge_prefix_inline) return false;  // not the cascade suffix
  return static_cast<int64_t>(p.num_seqs) * p.num_kv_heads * p.num_partitions <= 0x7fffffffLL;
}

cudaError_t launch_decode_units(const DecodeConfig& c, const CUtensorMap& km, const CUtensorMap& vm,
                                const DecodeParams& p, cudaStream_t st) {
  if (!decode_units_supported(c, p)) return cudaErrorInvalidValue;
  const int g = p.group;
  if (c.kv == KvType::F16) {
    return c.head_dim == 128 ? launch_units_kv<KvType::F16, QType::F16, 128>(c.ntiles, g, km, vm, p, st)
                             : launch_units_kv<KvType::F16, QType::F16, 64>(c.ntiles, g, km, vm, p, st);
  }
  if (c.kv == KvType::BF16) {
    return c.head_dim == 128 ? launch_units_kv<KvType::BF16, QType::BF16, 128>(c.ntiles, g, km, vm, p, st)
                             : launch_units_kv<KvType::BF16, QType::BF16, 64>(c.ntiles, g, km, vm, p, st);
  }
  return c.q == QType::BF16 ? launch_units_kv<KvType::E4M3, QType::BF16, 128>(c.ntiles, g, km, vm, p, st)
                            : launch_units_kv<KvType::E4M3, QType::F16, 128>(c.ntiles, g, km, vm, p, st);
}

}  // namespace pa
