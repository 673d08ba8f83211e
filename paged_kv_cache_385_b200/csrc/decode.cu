// Paged-attention decode kernels for sm_100a.
//
// What is computed (vLLM notes page, "PagedAttention" and "内核优化"; "vLLM 前世今生" section
// 3.2): for sequence s, query head h and its KV head hk = h / G,
//   out[s, h] = sum_t softmax_t(scale * q[s, h] . K[s, t]) V[s, t],
// K[s, t] being row t % 16 of the page (block_tables[s][t / 16], hk) of the pool.
//
// Work split. One CTA per (partition, KV head, sequence); a partition is a run of
// partition_tokens tokens (a multiple of 16). The CTA's 4 warps take the partition's 16-token pages
// round-robin, each with its own pipeline of S stages: lane 0 issues TMA tile loads of the K page
// and the V page of KV head hk (2-D tensor maps over the pool viewed as [NB * Hkv * 16 rows, D],
// 128-byte swizzle) onto a per-stage mbarrier, the warp waits on that barrier, computes, and
// refills the stage. Each warp keeps an online softmax (running max m, sum l, accumulator acc)
// for the G query heads of hk (GQA/MQA packing: every K/V byte is read once per KV head); the
// warps are merged in fixed order through shared memory. With one partition the CTA writes the
// output; otherwise it writes (acc, m, l) to the workspace and reduce_kernel merges the partitions
// of a (sequence, head) in a fixed order. No float atomics: the result depends only on logical
// positions, so permuting physical blocks leaves it bit-identical.
//
// Per-page math has two variants:
//  * tensor-core (kernel 1): scores S^T[16 tok x 8g] = K[16 x D] . Q^T with mma.sync m16n8k16
//    (tokens on M, the query group on N), P^T moved into B-fragment layout with movmatrix, then
//    O^T[D x 8g] += V^T[D x 16] . P^T. K/V fragments come from ldmatrix (V transposed by
//    ldmatrix.trans); e4m3 pages are widened to f16 in registers (exact).
//  * CUDA-core (kernel 0): float32 FMA dot products and axpys, kept for comparison (opts.kernel 0).
//
// Two modes ride on the same kernel:
//  * pa_decode_step: the CTA of a sequence's last partition writes the new token's K/V row into
//    its slot (the Cache Engine write) and fences it for the asynchronous proxy before any copy of
//    that block's page is issued; the copies of its other first pages go out before the write, so
//    the write overlaps them.
//  * pa_decode_cascade (suffix grid): the CTAs cover tokens [shared prefix, context) and, while
//    the prefix kernel before them on the stream still runs, wait for it only before reading its
//    partials, which they fold into their own merge (or leave to reduce_kernel when the suffix
//    itself is split). The CTA of KV head 0, partition 0 of each sequence checks that its table
//    maps the prefix to sequence 0's blocks.
#include <algorithm>
#include <cfloat>
#include <utility>

#include "decode_math.cuh"
#include "internal.h"
#include "pa_device.cuh"

namespace pa {

__device__ uint32_t g_error_word;

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------------------------
// CUDA-core per-page math (float32 FMA). Score phase: lane = (token t = lane & 15, half = lane >> 4),
// each lane dots its half of the row with q (held in shared memory as float32, pre-scaled) for all G
// heads, halves combined with one shuffle. PV phase: lane owns 8 consecutive d of D (16 lanes cover
// D = 128, 8 lanes D = 64) and a share of the tokens; weights go through shared memory.
// ---------------------------------------------------------------------------------------------
template <class C, int D, int GMAX>
struct FmaMath {
  static constexpr int kDL = D / 8;           // lanes per row in the PV phase
  static constexpr int kTokGroups = 32 / kDL;  // token groups in the PV phase
  static constexpr int kTokPer = 16 / kTokGroups;
  float acc[GMAX][8];
  float m[GMAX];
  float l[GMAX];
  const float* qs;  // [GMAX][D] scaled query (shared)
  float* ps;        // [16][GMAX] weights of the current page (per warp, shared)
  int lane, G;

  __device__ __forceinline__ void init(const float* q_smem, float* p_smem, int lane_, int G_) {
    qs = q_smem;
    ps = p_smem;
    lane = lane_;
    G = G_;
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[g][i] = 0.f;
    }
  }

  __device__ __forceinline__ static void widen16(const uint4& raw, float (&f)[8]) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = unpack2<C::kMmaBf16>(w[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }

  __device__ __forceinline__ static void widen8(uint32_t lo, uint32_t hi, float (&f)[8]) {
    uint32_t w[4];
    e4m3x4_to_f16x2x2(lo, w[0], w[1]);
    e4m3x4_to_f16x2x2(hi, w[2], w[3]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = unpack2<false>(w[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }

  // Eight consecutive elements [d0, d0 + 8) of token row t, widened to float.
  __device__ __forceinline__ void row8(const uint8_t* page, int t, int d0, float (&f)[8]) const {
    const int byte = d0 * C::kEsz;
    const int sub = byte >> 7, in = byte & 127;
    const uint8_t* p = page + sub * 2048 + swz(t, in >> 4) + (in & 15);
    if constexpr (C::kFp8) {
      const uint2 raw = *reinterpret_cast<const uint2*>(p);
      widen8(raw.x, raw.y, f);
    } else {
      widen16(*reinterpret_cast<const uint4*>(p), f);
    }
  }

  __device__ __forceinline__ void page(const uint8_t* kp, const uint8_t* vp, int nv) {
    // Scores: lane (t, half) covers d in [half * D/2, half * D/2 + D/2).
    const int t = lane & 15, half = lane >> 4;
    float s[GMAX];
#pragma unroll
    for (int g = 0; g < GMAX; ++g) s[g] = 0.f;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      const int d0 = half * (D / 2) + c * 8;
      float f[8];
      row8(kp, t, d0, f);
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        if (g < G) {
          const float4 qa = *reinterpret_cast<const float4*>(qs + g * D + d0);
          const float4 qb = *reinterpret_cast<const float4*>(qs + g * D + d0 + 4);
          s[g] = fmaf(f[0], qa.x, s[g]);
          s[g] = fmaf(f[1], qa.y, s[g]);
          s[g] = fmaf(f[2], qa.z, s[g]);
          s[g] = fmaf(f[3], qa.w, s[g]);
          s[g] = fmaf(f[4], qb.x, s[g]);
          s[g] = fmaf(f[5], qb.y, s[g]);
          s[g] = fmaf(f[6], qb.z, s[g]);
          s[g] = fmaf(f[7], qb.w, s[g]);
        }
      }
    }
    const bool valid = t < nv;
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      if (g < G) {
        float v = s[g] + __shfl_xor_sync(kFull, s[g], 16);
        v = valid ? v : -INFINITY;
        float mx = v;
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
        const float mn = fmaxf(m[g], mx);
        const float al = ex2(m[g] - mn);
        m[g] = mn;
        const float pw = ex2(v - mn);
        float ls = pw;
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) ls += __shfl_xor_sync(kFull, ls, off);
        l[g] = l[g] * al + ls;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[g][i] *= al;
        if (half == 0) ps[t * GMAX + g] = pw;
      }
    }
    __syncwarp();
    // PV: lane owns d in [dl * 8, dl * 8 + 8) and tokens tg * kTokPer .. + kTokPer.
    const int dl = lane % kDL, tg = lane / kDL;
#pragma unroll
    for (int k = 0; k < kTokPer; ++k) {
      const int tt = tg * kTokPer + k;
      if (tt < nv) {
        float f[8];
        row8(vp, tt, dl * 8, f);
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
          if (g < G) {
            const float w = ps[tt * GMAX + g];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[g][i] = fmaf(w, f[i], acc[g][i]);
          }
        }
      }
    }
    __syncwarp();
  }

  __device__ __forceinline__ void store(float* mg, float* lg, float* ag) {
    const int dl = lane % kDL;
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      if (g < G) {
        // Sum the token groups' partial accumulators (lanes dl, dl + kDL, ...).
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float v = acc[g][i];
#pragma unroll
          for (int off = kDL; off < 32; off <<= 1) v += __shfl_xor_sync(kFull, v, off);
          acc[g][i] = v;
        }
        if (lane < kDL) {
#pragma unroll
          for (int i = 0; i < 8; ++i) ag[g * D + dl * 8 + i] = acc[g][i];
        }
        if (lane == 0) {
          mg[g] = m[g];
          lg[g] = l[g];
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------------------------
// The decode kernel: pipeline, per-warp loop, merge, epilogue.
// ---------------------------------------------------------------------------------------------
template <KvType KV, QType QT, int D, int NT, int KIND, int OCC>
__global__ void __launch_bounds__(Cfg<KV, QT, D, NT, KIND, OCC>::kThreads, Cfg<KV, QT, D, NT, KIND, OCC>::kMinBlocks)
    decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                  const DecodeParams p) {
  using C = Cfg<KV, QT, D, NT, KIND, OCC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kPipeBytes);

  const int part = blockIdx.x, hk = blockIdx.y, s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Launched as a programmatic dependent: everything this grid reads may come from the previous
  // kernel on the stream, so wait for it first (cascade: only before the prefix partials are read).
  // The next kernel (partition merge, next step) is let in once every CTA has finished its page loop
  // (below), when SM slots start to free up.
  const bool late_wait = p.late_dependency_wait != 0;
  if (!late_wait) pdl_wait();
  const int G = p.group;
  const int Hq = p.num_kv_heads * G;
  const int PT = p.partition_tokens;

  // The block-table entry of this lane's page, read before the context length is known so that the
  // two loads overlap (entries past the context are masked below; the read stays inside the table).
  const int j_lane = p.start_tokens / 16 + part * (PT / 16) + warp + lane * C::kWarps;
  const int bid_lane = j_lane < p.max_blocks ? p.block_tables[s * p.bt_stride + j_lane] : -1;
  // Cascade: the CTA of KV head 0, partition 0 of each sequence checks that its table maps the
  // shared prefix pages to sequence 0's blocks (the prefix kernels read sequence 0's). The first
  // 2 * kThreads entries are read here and compared later, so the reads overlap the page loop.
  const bool chk = p.start_tokens > 0 && hk == 0 && part == 0;
  const int npre_pages = p.start_tokens / 16;
  int chk_a[2] = {0, 0}, chk_b[2] = {0, 0};
  if (chk) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int j = threadIdx.x + u * C::kThreads;
      if (j < npre_pages) {
        chk_a[u] = p.block_tables[s * p.bt_stride + j];
        chk_b[u] = p.block_tables[j];
      }
    }
  }
  auto prefix_check = [&]() {
    if (!chk) return;
    bool bad = chk_a[0] != chk_b[0] || chk_a[1] != chk_b[1];
    for (int j = threadIdx.x + 2 * C::kThreads; j < npre_pages; j += C::kThreads)
      bad |= p.block_tables[s * p.bt_stride + j] != p.block_tables[j];
    if (bad) atomicOr(p.err, 16u);
  };
  // This grid covers tokens [start, start + span) of the sequence: all of it for plain decode, the
  // part after the shared prefix for cascade decode.
  const int ctx = p.context_lens[s];
  const int start = p.start_tokens;
  const int ctx_cap = min(ctx, p.max_blocks * 16);
  int span = min(max(ctx_cap - start, 0), p.num_partitions * PT);
  if (ctx_cap < ctx || ctx < 0 || span < ctx_cap - start) {
    if (part == 0 && hk == 0 && threadIdx.x == 0) atomicOr(p.err, 8u);
  }
  const int ctx_eff = start + span;  // tokens [0, ctx_eff) exist for this grid's bookkeeping
  const int nparts = (span + PT - 1) / PT;
  if (part >= max(nparts, 1)) {
    if (late_wait) pdl_wait();
    return;
  }

  // pa_decode_step: the CTA holding the sequence's last partition writes head hk's new K/V row
  // (position ctx - 1) into its slot; the proxy fence + barrier order the writes before any TMA load
  // of that page. The copies of this CTA's first pages are issued before the write (all but a page
  // in the slot's block), so the write's latency overlaps theirs.
  const bool fused_here = p.new_k != nullptr && part == max(nparts, 1) - 1;
  int64_t new_slot = -1;
  bool do_write = false;
  if (fused_here) {
    new_slot = p.new_slots[s];
    // With a shared prefix the new token must lie past it (prefix blocks are read-only here).
    const bool writable = start == 0 || nparts > 0;
    do_write = writable && new_slot >= 0 && new_slot < static_cast<int64_t>(p.num_blocks) * 16;
    if (!do_write && new_slot != -1 && threadIdx.x == 0) atomicOr(p.err, 2u);
  }
  auto write_new_token = [&]() {
    const int64_t slot = new_slot;
    if (do_write) {
      constexpr int kChunks = D / 8;  // 16-byte input chunks per row
      for (int c = threadIdx.x; c < 2 * kChunks; c += C::kThreads) {
        const bool is_v = c >= kChunks;
        const int d0 = (is_v ? c - kChunks : c) * 8;
        const uint16_t* src = static_cast<const uint16_t*>(is_v ? p.new_v : p.new_k) +
                              s * (is_v ? p.nv_stride_s : p.nk_stride_s) + hk * (is_v ? p.nv_stride_h : p.nk_stride_h) +
                              d0;
        const uint4 raw = *reinterpret_cast<const uint4*>(src);
        const int64_t dst = (((slot >> 4) * p.num_kv_heads + hk) * 16 + (slot & 15)) * D + d0;
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
    }
    __syncthreads();
  };
  if (fused_here && span == 0) write_new_token();

  typedef uint16_t out_t;
  if (span == 0) prefix_check();
  if (span == 0 && late_wait) pdl_wait();
  if (span == 0 && p.merge_prefix_inline) {
    // Nothing past the shared prefix: the output is the merge of the prefix partials alone.
    for (int idx = threadIdx.x; idx < G * D; idx += C::kThreads) {
      const int g = idx / D, d = idx % D, h = hk * G + g;
      const int64_t row0 = (static_cast<int64_t>(s) * Hq + h) * p.ws_parts;
      float M = -INFINITY;
      for (int k = 0; k < p.part_offset; ++k) M = fmaxf(M, p.ws_ml[(row0 + k) * 2]);
      float num = 0.f, den = 0.f;
      if (M != -INFINITY) {
        for (int k = 0; k < p.part_offset; ++k) {
          const float f = ex2(p.ws_ml[(row0 + k) * 2] - M);
          num = fmaf(f, p.ws_acc[(row0 + k) * D + d], num);
          den = fmaf(f, p.ws_ml[(row0 + k) * 2 + 1], den);
        }
      }
      const float o = den > 0.f ? num / den * p.v_scale : 0.f;
      uint16_t bits;
      if constexpr (C::kQBf16) {
        bits = __bfloat16_as_ushort(__float2bfloat16_rn(o));
      } else {
        bits = __half_as_ushort(__float2half_rn(o));
      }
      static_cast<uint16_t*>(p.out)[s * p.o_stride_s + h * p.o_stride_h + d] = bits;
    }
    return;
  }
  if (span == 0) {
    if (p.always_partials) return;  // the merge kernel covers this sequence from its other partials
    // empty context: output 0
    for (int i = threadIdx.x; i < G * D; i += C::kThreads) {
      const int g = i / D, d = i % D;
      static_cast<out_t*>(p.out)[s * p.o_stride_s + (hk * G + g) * p.o_stride_h + d] = 0;
    }
    return;
  }

  const int pages_per_part = PT / 16;
  const int j0 = start / 16 + part * pages_per_part;
  const int j1 = min(j0 + pages_per_part, (ctx_eff + 15) / 16);
  const int n_w = max(0, (j1 - j0 - warp + C::kWarps - 1) / C::kWarps);  // pages of this warp (<= 32)

  // Physical block of this warp's i-th page sits in lane i.
  const int my_bid = lane < n_w ? bid_lane : -1;
  const bool my_bad = lane < n_w && (my_bid < 0 || my_bid >= p.num_blocks);
  if (__any_sync(kFull, my_bad) && lane == 0) atomicOr(p.err, 1u);

  uint8_t* wbuf = smem + warp * C::kStages * C::kStageBytes;
  const uint32_t wbuf_s = smem_u32(wbuf);
  const uint32_t bar0 = smem_u32(bars + warp * C::kStages);
  if (lane == 0) {
    for (int st = 0; st < C::kStages; ++st) mbar_init(bar0 + 8 * st, 1);
    fence_barrier_init();
    if (warp == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
    }
  }
  __syncwarp();

  auto issue = [&](int i) {
    const int bid = __shfl_sync(kFull, my_bid, i & 31);
    if (lane == 0) {
      const int st = i % C::kStages;
      const uint32_t bar = bar0 + 8 * st;
      if (bid < 0 || bid >= p.num_blocks) {
        mbar_arrive(bar);  // skipped page: complete the phase without data
      } else {
        mbar_arrive_expect_tx(bar, 2 * C::kPageBytes);
        const uint32_t kdst = wbuf_s + st * C::kStageBytes;
        const int y = (bid * p.num_kv_heads + hk) * 16;
#pragma unroll
        for (int u = 0; u < C::kSubPages; ++u) {
          tma_load_2d(kdst + u * 2048, &kmap, bar, u * C::kSubElems, y);
          tma_load_2d(kdst + C::kPageBytes + u * 2048, &vmap, bar, u * C::kSubElems, y);
        }
      }
    }
  };

  // Per-warp math state.
  float* merge = reinterpret_cast<float*>(smem);  // reused after the pipeline drains
  float* mg = merge;                               // [W][GPad]
  float* lg = merge + C::kWarps * C::kGPad;        // [W][GPad]
  float* ag = merge + 2 * C::kWarps * C::kGPad;    // [W][GPad][D]

  __shared__ __align__(16) float q_s[KIND == 0 ? C::kGPad * D : 1];
  __shared__ __align__(16) float p_s[KIND == 0 ? C::kWarps * 16 * C::kGPad : 1];

  TcMath<C, D, NT> tc;
  FmaMath<C, D, C::kGPad> fm;
  if constexpr (KIND == 1) {
    tc.init(p, s, hk, lane);
  } else {
    const float qscale = p.score_scale_log2;
    for (int i = threadIdx.x; i < C::kGPad * D; i += C::kThreads) {
      const int g = i / D, d = i % D;
      float v = 0.f;
      if (g < G) {
        const uint16_t bits = static_cast<const uint16_t*>(p.q)[s * p.q_stride_s + (hk * G + g) * p.q_stride_h + d];
        if constexpr (C::kQBf16) {
          v = __uint_as_float(static_cast<uint32_t>(bits) << 16);
        } else {
          v = __half2float(__ushort_as_half(bits));
        }
      }
      q_s[i] = v * qscale;
    }
    __syncthreads();
    fm.init(q_s, p_s + warp * 16 * C::kGPad, lane, G);
  }

  const uint64_t deadline = globaltimer_ns() + 2000000000ull;
  // First pages: a page in the new token's block waits until the token is written.
  const int wblk = do_write && span > 0 ? static_cast<int>(new_slot >> 4) : -1;
  uint32_t deferred = 0;
  for (int i = 0; i < min(C::kStages, n_w); ++i) {
    if (wblk >= 0 && __shfl_sync(kFull, my_bid, i & 31) == wblk) {
      deferred |= 1u << i;
    } else {
      issue(i);
    }
  }
  if (fused_here && span > 0) write_new_token();
  for (int i = 0; i < min(C::kStages, n_w); ++i)
    if (deferred & (1u << i)) issue(i);
  bool ok = true;
  int i = 0;
  for (; i < n_w; ++i) {
    const int st = i % C::kStages;
    const bool got = mbar_wait_bounded(bar0 + 8 * st, (i / C::kStages) & 1, deadline);
    if (!__all_sync(kFull, got)) {
      ok = false;
      break;
    }
    const int bid = __shfl_sync(kFull, my_bid, i & 31);
    if (bid >= 0 && bid < p.num_blocks) {
      const int j = j0 + warp + i * C::kWarps;
      const int nv = min(16, ctx_eff - j * 16);
      if constexpr (KIND == 1) {
        tc.page(wbuf_s + st * C::kStageBytes, wbuf_s + st * C::kStageBytes + C::kPageBytes, nv, p.score_scale_log2);
      } else {
        fm.page(wbuf + st * C::kStageBytes, wbuf + st * C::kStageBytes + C::kPageBytes, nv);
      }
    }
    __syncwarp();
    if (i + C::kStages < n_w) issue(i + C::kStages);
  }
  if (!ok) {
    // Give the copies this warp still has in flight a bounded chance to land before its shared
    // memory is reused, then report.
    for (int k = i; k < min(i + C::kStages, n_w); ++k)
      mbar_wait_bounded(bar0 + 8 * (k % C::kStages), (k / C::kStages) & 1, globaltimer_ns() + 100000000ull);
    if (lane == 0) atomicOr(p.err, 4u);
  }
  const int any_fail = __syncthreads_or(!ok);
  prefix_check();
  pdl_launch_dependents();
  if (late_wait) pdl_wait();  // the prefix partials (and the prefix grid's completion) from here on

  // ---- merge the warps in fixed order -----------------------------------------------------
  if constexpr (KIND == 1) {
    tc.store(mg + warp * C::kGPad, lg + warp * C::kGPad, ag + warp * C::kGPad * D);
  } else {
    fm.store(mg + warp * C::kGPad, lg + warp * C::kGPad, ag + warp * C::kGPad * D);
  }
  if (n_w == 0) {  // a warp without pages contributes nothing
    for (int g = lane; g < C::kGPad; g += 32) {
      mg[warp * C::kGPad + g] = -INFINITY;
      lg[warp * C::kGPad + g] = 0.f;
    }
    for (int k = lane; k < C::kGPad * D; k += 32) ag[warp * C::kGPad * D + k] = 0.f;
  }
  __syncthreads();
  if (any_fail) return;

  const bool inline_merge = p.merge_prefix_inline && nparts <= 1;
  const bool direct = (!p.always_partials && nparts <= 1) || inline_merge;
  // Each thread owns one d and four group members at a time (g = gb .. gb + 3; members past G are
  // computed on a clamped g and dropped).
  static_assert(C::kThreads % D == 0, "threads must cover whole rows of d");
  constexpr int kDPar = C::kThreads / D;
  const int d = threadIdx.x % D;
  const int npre = p.part_offset;
  for (int gb = (threadIdx.x / D) * 4; gb < G; gb += kDPar * 4) {
    float M[4], num[4], den[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int g = min(gb + u, G - 1);
      M[u] = -INFINITY;
#pragma unroll
      for (int w = 0; w < C::kWarps; ++w) M[u] = fmaxf(M[u], mg[w * C::kGPad + g]);
      num[u] = 0.f;
      den[u] = 0.f;
#pragma unroll
      for (int w = 0; w < C::kWarps; ++w) {
        const float f = ex2(mg[w * C::kGPad + g] - M[u]);
        num[u] = fmaf(f, ag[(w * C::kGPad + g) * D + d], num[u]);
        den[u] = fmaf(f, lg[w * C::kGPad + g], den[u]);
      }
    }
    if (inline_merge) {
      // Fold in the shared-prefix partials (workspace slots 0 .. npre - 1), four slots of four members
      // per round: every load of a round is issued before any of them is used.
      for (int k0 = 0; k0 < npre; k0 += 4) {
        float pm[4][4], pl[4][4], pa[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int g = min(gb + u, G - 1);
          const int64_t row0 = (static_cast<int64_t>(s) * Hq + hk * G + g) * p.ws_parts;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int k = min(k0 + v, npre - 1);
            const float2 ml = *reinterpret_cast<const float2*>(p.ws_ml + (row0 + k) * 2);
            pa[u][v] = p.ws_acc[(row0 + k) * D + d];
            pm[u][v] = k0 + v < npre ? ml.x : -INFINITY;
            pl[u][v] = ml.y;
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float Mn = M[u];
#pragma unroll
          for (int v = 0; v < 4; ++v) Mn = fmaxf(Mn, pm[u][v]);
          if (Mn == -INFINITY) continue;
          const float a = ex2(M[u] - Mn);
          num[u] *= a;
          den[u] *= a;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const float f = ex2(pm[u][v] - Mn);
            num[u] = fmaf(f, pa[u][v], num[u]);
            den[u] = fmaf(f, pl[u][v], den[u]);
          }
          M[u] = Mn;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int g = gb + u;
      if (g >= G) break;
      const int h = hk * G + g;
      if (direct) {
        const float o = num[u] / den[u] * p.v_scale;
        out_t bits;
        if constexpr (C::kQBf16) {
          bits = __bfloat16_as_ushort(__float2bfloat16_rn(o));
        } else {
          bits = __half_as_ushort(__float2half_rn(o));
        }
        static_cast<out_t*>(p.out)[s * p.o_stride_s + h * p.o_stride_h + d] = bits;
      } else {
        const int64_t row = (static_cast<int64_t>(s) * Hq + h) * p.ws_parts + p.part_offset + part;
        p.ws_acc[row * D + d] = num[u];
        if (d == 0) {
          p.ws_ml[row * 2] = M[u];
          p.ws_ml[row * 2 + 1] = den[u];
        }
      }
    }
  }
}

// Merge the partitions of each (sequence, query head): one CTA per row, W warps. A row's
// partials are contiguous in the workspace, so they stream into shared memory as 1-D bulk copies of
// kRedChunk partitions (acc rows, and the (m, l) pairs from the 16-byte boundary at or below their
// start); chunk c goes to warp c % W, each warp with S chunks in flight (fewer warps and stages for
// short rows, so that many rows fit on an SM at once). Lane k of a
// chunk takes partition k's (m, l): the chunk's maximum and weights come from warp shuffles, and each
// lane accumulates its D / 32 values of d over the chunk's partitions in order. The warps' states are
// then combined in warp order. Every order is fixed, so the result is deterministic.
constexpr int kRedChunk = 16;
constexpr int kRedMlBytes = kRedChunk * 8 + 16;
template <int D, int W, int S>
struct RedCfg {
  static constexpr int kRedWarps = W;
  static constexpr int kRedStages = S;
  static constexpr int kAccBytes = kRedChunk * D * 4;  // one chunk of acc rows
  static constexpr int kWarpBytes = kRedStages * (kAccBytes + kRedMlBytes + 8);
  static constexpr int kCombineBytes = kRedWarps * (D + 2) * 4;
  static constexpr int kSmemBytes = kRedWarps * kWarpBytes + kCombineBytes;
};
template <int D, bool kBf16, int W, int S>
__global__ void __launch_bounds__(W * 32) reduce_kernel(const DecodeParams p) {
  using R = RedCfg<D, W, S>;
  constexpr int kRedWarps = W, kRedStages = S;
  constexpr int V = D / 32;  // values of d per lane
  extern __shared__ __align__(128) uint8_t red_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wsm = red_smem + warp * R::kWarpBytes;
  float* acc_s = reinterpret_cast<float*>(wsm);                       // [stage][chunk][D]
  uint8_t* ml_s = wsm + kRedStages * R::kAccBytes;                     // [stage][kRedMlBytes]
  const uint32_t bar0 = smem_u32(ml_s + kRedStages * kRedMlBytes);     // [stage]
  float* comb = reinterpret_cast<float*>(red_smem + kRedWarps * R::kWarpBytes);  // [warp][D + 2]
  // The next kernel on the stream is let in only as this grid's CTAs finish: a persistent decode grid
  // after it should find the SMs free, not partly held by this merge.
  pdl_wait();  // the partials come from the decode grid just before this one
  const int Hq = p.num_kv_heads * p.group;
  const int h = blockIdx.x, s = blockIdx.y;
  const int PT = p.partition_tokens;
  const int ctx_cap = min(p.context_lens[s], p.max_blocks * 16);
  const int span = min(max(ctx_cap - p.start_tokens, 0), p.num_partitions * PT);
  const int np = p.part_offset + (span + PT - 1) / PT;
  if (!p.always_partials && np <= 1) return;  // the decode kernel wrote this row
  const int64_t row0 = (static_cast<int64_t>(s) * Hq + h) * p.ws_parts;
  const int nchunks = (np + kRedChunk - 1) / kRedChunk;
  const int mine_n = nchunks > warp ? (nchunks - warp + kRedWarps - 1) / kRedWarps : 0;  // this warp's chunks
  if (lane == 0) {
    for (int st = 0; st < kRedStages; ++st) mbar_init(bar0 + 8 * st, 1);
    fence_barrier_init();
  }
  __syncwarp();
  // The warp's j-th chunk (chunk warp + j * kRedWarps) -> stage j % kRedStages. The (m, l) copy may
  // take up to 8 bytes on either side of the chunk's pairs, still inside the workspace: its (m, l)
  // area is a whole number of 256-byte lines.
  auto ml_start = [&](int k0) { return (row0 + k0) * 8 & ~int64_t(15); };
  auto issue = [&](int j) {
    if (lane != 0) return;
    const int st = j % kRedStages, k0 = (warp + j * kRedWarps) * kRedChunk, n = min(kRedChunk, np - k0);
    const uint32_t acc_bytes = static_cast<uint32_t>(n) * D * 4;
    const int64_t b0 = ml_start(k0), b1 = ((row0 + k0 + n) * 8 + 15) & ~int64_t(15);
    const uint32_t ml_bytes = static_cast<uint32_t>(b1 - b0);
    mbar_arrive_expect_tx(bar0 + 8 * st, acc_bytes + ml_bytes);
    bulk_load_1d(smem_u32(acc_s + st * kRedChunk * D), p.ws_acc + (row0 + k0) * D, acc_bytes, bar0 + 8 * st);
    bulk_load_1d(smem_u32(ml_s + st * kRedMlBytes), reinterpret_cast<const uint8_t*>(p.ws_ml) + b0, ml_bytes,
                 bar0 + 8 * st);
  };
  for (int j = 0; j < min(kRedStages, mine_n); ++j) issue(j);
  const uint64_t deadline = globaltimer_ns() + 2000000000ull;
  float M = -INFINITY, den = 0.f, num[V];
#pragma unroll
  for (int v = 0; v < V; ++v) num[v] = 0.f;
  bool ok = true;
  int j = 0;
  for (; j < mine_n; ++j) {
    const int st = j % kRedStages, k0 = (warp + j * kRedWarps) * kRedChunk, n = min(kRedChunk, np - k0);
    if (!__all_sync(kFull, mbar_wait_bounded(bar0 + 8 * st, (j / kRedStages) & 1, deadline))) {
      ok = false;
      break;
    }
    const float2* ml = reinterpret_cast<const float2*>(ml_s + st * kRedMlBytes + ((row0 + k0) * 8 - ml_start(k0)));
    const float* a = acc_s + st * kRedChunk * D;
    const float2 mine = lane < n ? ml[lane] : make_float2(-INFINITY, 0.f);
    float cmax = mine.x;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(kFull, cmax, off));
    const float Mn = fmaxf(M, cmax);
    if (Mn != -INFINITY) {
      const float r = ex2(M - Mn);
      const float f = ex2(mine.x - Mn);  // a partition without tokens has m = -inf: weight 0
      float fl = f * mine.y;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) fl += __shfl_xor_sync(kFull, fl, off);
      den = den * r + fl;
#pragma unroll
      for (int v = 0; v < V; ++v) num[v] *= r;
#pragma unroll
      for (int k = 0; k < kRedChunk; ++k) {
        const float fk = __shfl_sync(kFull, f, k);
        if (k < n) {  // slots past n hold stale bytes
          if constexpr (V == 4) {
            const float4 x = *reinterpret_cast<const float4*>(a + k * D + 4 * lane);
            num[0] = fmaf(fk, x.x, num[0]);
            num[1] = fmaf(fk, x.y, num[1]);
            num[2] = fmaf(fk, x.z, num[2]);
            num[3] = fmaf(fk, x.w, num[3]);
          } else {
            const float2 x = *reinterpret_cast<const float2*>(a + k * D + 2 * lane);
            num[0] = fmaf(fk, x.x, num[0]);
            num[1] = fmaf(fk, x.y, num[1]);
          }
        }
      }
      M = Mn;
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
    if (j + kRedStages < mine_n) issue(j + kRedStages);
  }
  if (!ok) {
    // Let the copies still in flight land (bounded) before the CTA's shared memory goes.
    if (lane == 0) {
      for (int k = j; k < min(j + kRedStages, mine_n); ++k)
        mbar_wait_bounded(bar0 + 8 * (k % kRedStages), (k / kRedStages) & 1, globaltimer_ns() + 100000000ull);
      atomicOr(p.err, 4u);
    }
  }
  // Combine the warps in warp order.
  float* cw = comb + warp * (D + 2);
#pragma unroll
  for (int v = 0; v < V; ++v) cw[V * lane + v] = num[v];
  if (lane == 0) {
    cw[D] = M;
    cw[D + 1] = den;
  }
  if (__syncthreads_or(!ok) || warp != 0) return;
  float Mt = -INFINITY;
#pragma unroll
  for (int w = 0; w < kRedWarps; ++w) Mt = fmaxf(Mt, comb[w * (D + 2) + D]);
  uint32_t out_w[V / 2];
#pragma unroll
  for (int v = 0; v < V / 2; ++v) out_w[v] = 0u;  // no token at all (empty context): 0
  if (Mt != -INFINITY) {
    float nt[V], dt = 0.f;
#pragma unroll
    for (int v = 0; v < V; ++v) nt[v] = 0.f;
#pragma unroll
    for (int w = 0; w < kRedWarps; ++w) {
      const float* c = comb + w * (D + 2);
      const float f = ex2(c[D] - Mt);  // a warp without partitions has m = -inf: weight 0
      dt = fmaf(f, c[D + 1], dt);
#pragma unroll
      for (int v = 0; v < V; ++v) nt[v] = fmaf(f, c[V * lane + v], nt[v]);
    }
    const float sc = p.v_scale / dt;
#pragma unroll
    for (int v = 0; v < V / 2; ++v) out_w[v] = pack2<kBf16>(nt[2 * v] * sc, nt[2 * v + 1] * sc);
  }
  uint16_t* o = static_cast<uint16_t*>(p.out) + s * p.o_stride_s + h * p.o_stride_h + V * lane;
  if constexpr (V == 4) {
    *reinterpret_cast<uint2*>(o) = make_uint2(out_w[0], out_w[1]);
  } else {
    *reinterpret_cast<uint32_t*>(o) = out_w[0];
  }
  pdl_launch_dependents();
}

template <KvType KV, QType QT, int D, int NT, int KIND, int OCC>
cudaError_t launch_one(const CUtensorMap& km, const CUtensorMap& vm, const DecodeParams& p, cudaStream_t st) {
  using C = Cfg<KV, QT, D, NT, KIND, OCC>;
  auto kern = decode_kernel<KV, QT, D, NT, KIND, OCC>;
  static int configured_devices = 0;  // bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 31 || !(__atomic_load_n(&configured_devices, __ATOMIC_ACQUIRE) & (1 << dev))) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev < 31) __atomic_fetch_or(&configured_devices, 1 << dev, __ATOMIC_ACQ_REL);
  }
  return launch_pdl(kern, dim3(p.num_partitions, p.num_kv_heads, p.num_seqs), dim3(C::kThreads), C::kSmemBytes, st,
                    km, vm, p);
}

// Occupancy per variant (see Cfg): tensor-core e4m3 with one n-tile 4 CTAs/SM, tensor-core 16-bit
// grouped queries 3, everything else 2.
template <KvType KV, QType QT, int D, int KIND>
cudaError_t launch_nt(int nt, int group, const CUtensorMap& km, const CUtensorMap& vm, const DecodeParams& p,
                      cudaStream_t st) {
  if constexpr (KIND == 1) {
    if (nt == 1) {
      if constexpr (KV == KvType::E4M3) return launch_one<KV, QT, D, 1, 1, 4>(km, vm, p, st);
      if (group > 1) return launch_one<KV, QT, D, 1, 1, 3>(km, vm, p, st);
      return launch_one<KV, QT, D, 1, 1, 2>(km, vm, p, st);
    }
    if (nt == 2) return launch_one<KV, QT, D, 2, 1, 2>(km, vm, p, st);
  } else {
    if (nt == 1) return launch_one<KV, QT, D, 1, 0, 2>(km, vm, p, st);
  }
  return cudaErrorInvalidValue;
}

template <KvType KV, QType QT, int D>
cudaError_t launch_kind(const DecodeConfig& c, int group, const CUtensorMap& km, const CUtensorMap& vm,
                        const DecodeParams& p, cudaStream_t st) {
  if (c.kernel == 1) return launch_nt<KV, QT, D, 1>(c.ntiles, group, km, vm, p, st);
  return launch_nt<KV, QT, D, 0>(c.ntiles, group, km, vm, p, st);
}

}  // namespace

bool decode_supported(const DecodeConfig& c) {
  if (c.head_dim != 64 && c.head_dim != 128) return false;
  if (c.kv == KvType::E4M3 && c.head_dim != 128) return false;
  if (c.kv == KvType::F16 && c.q != QType::F16) return false;
  if (c.kv == KvType::BF16 && c.q != QType::BF16) return false;
  if (c.kernel == 1) return c.ntiles == 1 || c.ntiles == 2;
  if (c.kernel == 0) return c.ntiles == 1;
  return false;
}

cudaError_t launch_decode(const DecodeConfig& c, const CUtensorMap& km, const CUtensorMap& vm, const DecodeParams& p,
                          cudaStream_t st) {
  if (!decode_supported(c)) return cudaErrorInvalidValue;
  const int g = p.group;
  if (c.kv == KvType::F16) {
    return c.head_dim == 128 ? launch_kind<KvType::F16, QType::F16, 128>(c, g, km, vm, p, st)
                             : launch_kind<KvType::F16, QType::F16, 64>(c, g, km, vm, p, st);
  }
  if (c.kv == KvType::BF16) {
    return c.head_dim == 128 ? launch_kind<KvType::BF16, QType::BF16, 128>(c, g, km, vm, p, st)
                             : launch_kind<KvType::BF16, QType::BF16, 64>(c, g, km, vm, p, st);
  }
  return c.q == QType::BF16 ? launch_kind<KvType::E4M3, QType::BF16, 128>(c, g, km, vm, p, st)
                            : launch_kind<KvType::E4M3, QType::F16, 128>(c, g, km, vm, p, st);
}

template <int D, bool kBf16, int W, int S>
cudaError_t launch_reduce_one(const DecodeParams& p, cudaStream_t st) {
  auto kern = reduce_kernel<D, kBf16, W, S>;
  constexpr int smem = RedCfg<D, W, S>::kSmemBytes;
  static int configured_devices = 0;  // bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 31 || !(__atomic_load_n(&configured_devices, __ATOMIC_ACQUIRE) & (1 << dev))) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (dev < 31) __atomic_fetch_or(&configured_devices, 1 << dev, __ATOMIC_ACQ_REL);
  }
  const dim3 grid(p.num_kv_heads * p.group, p.num_seqs);
  return launch_pdl(kern, grid, dim3(W * 32), smem, st, p);
}

template <int D, bool kBf16>
cudaError_t launch_reduce_d(const DecodeParams& p, cudaStream_t st) {
  // Rows of at most one chunk: one warp, one stage (many rows per SM). Longer rows: two warps with
  // four chunks in flight each.
  if (p.ws_parts <= kRedChunk) return launch_reduce_one<D, kBf16, 1, 1>(p, st);
  return launch_reduce_one<D, kBf16, 2, 4>(p, st);
}

cudaError_t launch_reduce(const DecodeConfig& c, const DecodeParams& p, cudaStream_t st) {
  const bool bf = c.q == QType::BF16;
  if (c.head_dim == 128) return bf ? launch_reduce_d<128, true>(p, st) : launch_reduce_d<128, false>(p, st);
  return bf ? launch_reduce_d<64, true>(p, st) : launch_reduce_d<64, false>(p, st);
}

uint32_t* decode_error_word() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_error_word) != cudaSuccess) return nullptr;
  return static_cast<uint32_t*>(ptr);
}

cudaError_t read_and_clear_error_word(uint32_t* bits, int clear) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(bits, g_error_word, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  if (clear) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(uint32_t));
  }
  return e;
}

}  // namespace pa
