// Chunked prefill over paged KV with 5th-generation tensor cores, two query tiles per CTA taking
// turns (sm_100a). Same result as prefill_tc.cu (notes page, kernels section: FlashAttention adapted
// to paged KV; "vLLM 前世今生" §5.4 chunked prefill): row (new token i, group head g) of sequence s is
// position p = start + i and attends over positions 0 .. p of its KV head.
//
// Why a second form. Per key, the softmax needs one exponential and the two products need 4 * D
// FLOPs; on this part the SM's exponential rate (16 per clock) equals its bf16 tensor rate over 4 * D
// for D = 128, so the two units can both stay busy only if one tile's softmax runs while the other
// tile's MMAs do. Two CTAs per SM cannot arrange that (their phases drift together); here one CTA
// holds two 128-row tiles that share every K and V block, and each tile's chain
//   QK(j) -> softmax(j) -> P.V(j) -> QK(j+1)
// leaves the tensor pipe to the other tile while its softmax runs. The two chains start half a
// period apart (QK of tile 1 is issued right after tile 0's) and stay so.
//
// CTA: 2 x 128 query rows of one (sequence, KV head), 128-key blocks (8 pages), one CTA per SM.
// TMEM (512 columns): per tile S (128 f32 columns; P in bf16/f16 written back over its first 64)
// and O (128 columns). Shared memory: Q of both tiles (2 x 32 KB), two K stages and two V stages
// (32 KB each), all 128-byte swizzled and filled by TMA.
// Warps: 0-3 softmax of tile 0, 4-7 softmax of tile 1 (one row per thread), 8 producer of Q and K,
// 9 producer of V, 10 MMA issuer (one thread) and TMEM owner. Every mbarrier wait is bounded.
#include "internal.h"
#include "pa_device.cuh"
#include "tc05.cuh"

namespace pa {
namespace {

constexpr int kD = 128;
constexpr int kRows = 128;  // query rows per tile
constexpr int kTiles = 2;
constexpr int kKeys = 128;  // keys per block
constexpr int kWarps = 11;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kHalf = kRows * 128;   // one 64-element (128-byte) column half of a Q tile
constexpr uint32_t kTileQ = 2 * kHalf;
constexpr uint32_t kHalfKV = kKeys * 128;  // one column half of a K or V block
constexpr uint32_t kTileKV = 2 * kHalfKV;
constexpr int kStages = 2;
constexpr uint32_t kQOff = 0;
constexpr uint32_t kKOff = kTiles * kTileQ;
constexpr uint32_t kVOff = kKOff + kStages * kTileKV;
constexpr uint32_t kBarOff = kVOff + kStages * kTileKV;
constexpr uint32_t kSmemBytes = kBarOff + 256;
constexpr uint32_t kTmemCols = 512;  // per tile: S (kKeys) then O (kD)
static_assert(kTiles * (kKeys + kD) <= kTmemCols, "S and O of both tiles must fit the allocation");
// barrier slots (8 bytes each)
enum {
  kQFull0 = 0,    // kTiles
  kKFull0 = 2,    // kStages
  kKEmpty0 = 4,   // kStages
  kVFull0 = 6,    // kStages
  kVEmpty0 = 8,   // kStages
  kSFull0 = 10,   // kTiles: QK(j) of the tile completed
  kPFull0 = 12,   // kTiles: the tile's 4 softmax warps wrote P(j)
  kODone0 = 14,   // kTiles: P(j).V of the tile completed
  kVLast = 16,    // the last V block with its rows past every row's limit zeroed
  kAllDone = 17,
  kTmemSlot = 18,
};
static_assert(8 * (kTmemSlot + 1) <= 256, "barrier area");
constexpr float kLazyRescale = 8.f;  // log2 units, as in prefill_tc.cu

// Max (kMax) or min of n values in four independent chains.
template <bool kMax, int n>
__device__ __forceinline__ float extreme(const float (&v)[n]) {
  float e[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
  for (int k = 4; k < n; ++k) e[k & 3] = kMax ? fmaxf(e[k & 3], v[k]) : fminf(e[k & 3], v[k]);
  return kMax ? fmaxf(fmaxf(e[0], e[1]), fmaxf(e[2], e[3])) : fminf(fminf(e[0], e[1]), fminf(e[2], e[3]));
}

template <bool kBf16>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_pp_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const MqParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  if (base & 1023u) {  // the swizzled tiles need 1024-byte alignment; never seen, but do not guess
    if (threadIdx.x == 0) atomicOr(p.err, 4u);
    return;
  }
  const uint32_t bar = base + kBarOff;
  auto B = [&](int i) { return bar + 8u * i; };
  const int pair = blockIdx.x, hk = blockIdx.y, s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group;
  pdl_wait();

  // Rows of this CTA: tile t holds rows row0 + t * kRows .. + kRows - 1 of the sequence's
  // n_new * G (token, group head) rows; keys [0, lim) are visible to a row.
  const int q_row0 = p.query_start[s];
  const int n_new = p.query_start[s + 1] - q_row0;
  const int num_rows = n_new * G;
  const int row0 = pair * (kTiles * kRows);
  if (row0 >= num_rows) return;
  const int ctx = p.context_lens[s];
  const int start = ctx - n_new;
  if (start < 0 || ctx > p.max_blocks * 16) {
    if (threadIdx.x == 0) atomicOr(p.err, 8u);
    return;
  }
  if (pair == 0 && threadIdx.x == 0 && num_rows > static_cast<int>(gridDim.x) * kTiles * kRows) atomicOr(p.err, 8u);
  // Tile 0 always has rows; tile 1 may not. A later tile sees at least as many keys.
  const int lim0 = start + (min(row0 + kRows, num_rows) - 1) / G + 1;
  const bool has1 = row0 + kRows < num_rows;
  const int lim1 = has1 ? start + (min(row0 + 2 * kRows, num_rows) - 1) / G + 1 : 0;
  const int nkb0 = (lim0 + kKeys - 1) / kKeys;
  const int nkb1 = has1 ? (lim1 + kKeys - 1) / kKeys : 0;
  const int max_lim = has1 ? lim1 : lim0;
  const int nkb = max(nkb0, nkb1);
  const int npages = (max_lim + 15) / 16;
  const int32_t* bt = p.block_tables + static_cast<int64_t>(s) * p.bt_stride;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTiles; ++i) {
      mbar_init(B(kQFull0 + i), 1);
      mbar_init(B(kSFull0 + i), 1);
      mbar_init(B(kPFull0 + i), 4);
      mbar_init(B(kODone0 + i), 1);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(B(kKFull0 + i), 1);
      mbar_init(B(kKEmpty0 + i), 1);
      mbar_init(B(kVFull0 + i), 1);
      mbar_init(B(kVEmpty0 + i), 1);
    }
    mbar_init(B(kVLast), 1);
    mbar_init(B(kAllDone), 1);
    fence_barrier_init();
  }
  if (warp == 10) tc05::alloc(B(kTmemSlot), kTmemCols);
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kBarOff + 8 * kTmemSlot);
  auto tS = [&](int t) { return tmem + static_cast<uint32_t>(t) * (kKeys + kD); };
  auto tO = [&](int t) { return tmem + static_cast<uint32_t>(t) * (kKeys + kD) + kKeys; };
  const uint64_t deadline = globaltimer_ns() + 2000000000ull;
  bool ok = true;

  // Producer of one stream (K by warp 8, V by warp 9): block j's 8 page ids, then its 16 tile copies
  // into stage j % kStages once that stage's previous block has been consumed. Returns the number of
  // blocks whose copies it issued.
  auto produce = [&](const CUtensorMap* map, uint32_t off, int full0, int empty0) -> int {
    const int oob_row = p.num_blocks * p.num_kv_heads * 16;  // a box starting here is all zero fill
    for (int j = 0; j < nkb; ++j) {
      const int st = j % kStages;
      if (j >= kStages && !mbar_wait_bounded(B(empty0 + st), ((j / kStages) - 1) & 1, deadline)) {
        atomicOr(p.err, 4u);
        return j;
      }
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
      const uint32_t dst = base + off + st * kTileKV;
      mbar_arrive_expect_tx(B(full0 + st), kTileKV);
#pragma unroll
      for (int i = 0; i < kKeys / 16; ++i)
        for (int u = 0; u < 2; ++u) tma_load_2d(dst + u * kHalfKV + i * 2048, map, B(full0 + st), u * 64, ys[i]);
    }
    return nkb;
  };
  int issued = 0;  // producer lanes: blocks of their stream whose copies they issued

  if (warp == 8) {
    // ---- producer of Q (both tiles) and K ------------------------------------------------------
    if (lane == 0) {
      prefetch_tensormap(&qmap);
      for (int t = 0; t < kTiles; ++t) {
        if (t == 1 && !has1) break;
        mbar_arrive_expect_tx(B(kQFull0 + t), kTileQ);
        const int tok0 = q_row0 + (row0 + t * kRows) / G;
        tc05::tma_load_3d(base + kQOff + t * kTileQ, &qmap, B(kQFull0 + t), 0, hk * G, tok0);
        tc05::tma_load_3d(base + kQOff + t * kTileQ + kHalf, &qmap, B(kQFull0 + t), 64, hk * G, tok0);
      }
      issued = produce(&kmap, kKOff, kKFull0, kKEmpty0);
    }
  } else if (warp == 9) {
    // ---- producer of V; the last block's keys past every row's limit are zeroed -----------------
    // (those pool rows may hold any bits, and their weights are 0: 0 * NaN must not occur)
    if (lane == 0) issued = produce(&vmap, kVOff, kVFull0, kVEmpty0);
    issued = __shfl_sync(kFull, issued, 0);
    if (issued == nkb) {
      const int j = nkb - 1, st = j % kStages;
      const bool landed = __all_sync(kFull, mbar_wait_bounded(B(kVFull0 + st), (j / kStages) & 1, deadline));
      if (landed) {
        const uint32_t vbase = base + kVOff + st * kTileKV;
        const int first = max_lim - j * kKeys;  // rows [first, kKeys) of both halves
        for (int idx = lane; idx < (kKeys - first) * 16; idx += 32) {
          const int row = first + idx / 16, c16 = idx % 16;
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(vbase + (c16 >> 3) * kHalfKV + row * 128 +
                                                                         (c16 & 7) * 16),
                       "r"(0u)
                       : "memory");
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(B(kVLast));
      } else {
        ok = false;
        if (lane == 0) atomicOr(p.err, 4u);
      }
    } else {
      ok = false;  // the producer gave up (and flagged it)
    }
  } else if (warp == 10) {
    // ---- MMA issuer: per tile, P(j).V then QK(j+1) into the same S ---------------------------------
    // P(j) sits in S's first 64 columns until P(j).V has read it, so QK(j+1) goes in two halves: keys
    // 64..127 (columns 64..127, free once the softmax has read its scores) right away, keys 0..63 once
    // P(j).V has completed. The first half keeps the tensor pipe busy across that wait.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc05::idesc_f16(kBf16, kRows, kKeys, false, false);
      constexpr uint32_t idesc_qk_half = tc05::idesc_f16(kBf16, kRows, kKeys / 2, false, false);
      constexpr uint32_t idesc_pv = tc05::idesc_f16(kBf16, kRows, kD, false, true);
      // S(t)[:, c0 .. c0 + n) = Q(t) . K(j)[c0 .. c0 + n)^T; key c0 is row c0 of the K stage (128 bytes
      // per row in each half, so c0 = 64 is 8 whole 1024-byte swizzle atoms in).
      auto qk = [&](int t, int j, int c0, uint32_t idesc) {
        const uint32_t kbase = base + kKOff + (j % kStages) * kTileKV + c0 * 128;
        const uint32_t qbase = base + kQOff + t * kTileQ;
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {  // 8 k-steps of 16 along d, 32 bytes apart in a half
          const uint32_t cb = (ks & 3) * 32;
          tc05::mma_f16(tS(t) + c0, tc05::smem_desc_sw128(qbase + (ks >> 2) * kHalf + cb, 16, 1024),
                        tc05::smem_desc_sw128(kbase + (ks >> 2) * kHalfKV + cb, 16, 1024), idesc, ks > 0);
        }
      };
      auto pv = [&](int t, int j) {
        // P from TMEM (8 columns = 16 keys per step), V MN-major in shared memory (16 keys = 2048 B)
        const uint32_t vbase = base + kVOff + (j % kStages) * kTileKV;
#pragma unroll
        for (int kt = 0; kt < kKeys / 16; ++kt)
          tc05::mma_f16_ts(tO(t), tS(t) + kt * 8, tc05::smem_desc_sw128(vbase + kt * 2048, kHalfKV, 1024), idesc_pv,
                           (j > 0 || kt > 0));
        tc05::commit(B(kODone0 + t));
      };
      ok = mbar_wait_bounded(B(kQFull0), 0, deadline) && (!has1 || mbar_wait_bounded(B(kQFull0 + 1), 0, deadline)) &&
           mbar_wait_bounded(B(kKFull0), 0, deadline);
      if (ok) {
        tc05::fence_after_sync();
        for (int t = 0; t < kTiles; ++t) {
          if (t == 1 && !has1) break;
          qk(t, 0, 0, idesc_qk);
          tc05::commit(B(kSFull0 + t));
        }
        tc05::commit(B(kKEmpty0));
      }
      for (int j = 0; j < nkb && ok; ++j) {
        // V(j): the last block only once its rows past every limit are zeroed.
        ok = j == nkb - 1 ? mbar_wait_bounded(B(kVLast), 0, deadline)
                          : mbar_wait_bounded(B(kVFull0 + j % kStages), (j / kStages) & 1, deadline);
        bool k_next = false;  // K(j + 1) waited for
        for (int t = 0; t < kTiles && ok; ++t) {
          const int nkb_t = t == 0 ? nkb0 : nkb1;
          if (j >= nkb_t) continue;
          // The tile's P barrier next completes for P(j+1), which needs QK(j+1) from here: the parity
          // wait is exact. Likewise O_done below.
          if (!mbar_wait_bounded(B(kPFull0 + t), j & 1, deadline)) {
            ok = false;
            break;
          }
          tc05::fence_after_sync();
          pv(t, j);
          if (j + 1 < nkb_t) {
            if (!k_next && !mbar_wait_bounded(B(kKFull0 + (j + 1) % kStages), ((j + 1) / kStages) & 1, deadline)) {
              ok = false;
              break;
            }
            k_next = true;
            tc05::fence_after_sync();
            qk(t, j + 1, kKeys / 2, idesc_qk_half);
            if (!mbar_wait_bounded(B(kODone0 + t), j & 1, deadline)) {
              ok = false;
              break;
            }
            tc05::fence_after_sync();
            qk(t, j + 1, 0, idesc_qk_half);
            // Also tracks P(j).V: once S(j+1) is seen complete, O(t) holds every product through j.
            tc05::commit(B(kSFull0 + t));
          }
        }
        if (!ok) break;
        tc05::commit(B(kVEmpty0 + j % kStages));                    // V(j) read by both tiles' P.V
        if (k_next) tc05::commit(B(kKEmpty0 + (j + 1) % kStages));  // K(j+1) read by the QKs issued
      }
      // The final commit covers every MMA of the CTA.
      tc05::commit(B(kAllDone));
      mbar_wait_bounded(B(kAllDone), 0, globaltimer_ns() + 1000000000ull);
      if (!ok) atomicOr(p.err, 4u);
    }
  } else {
    // ---- softmax warps: tile t = warp / 4, thread = row (TMEM lane 32 * (warp % 4) + lane) ----------
    const int t = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const int R = row0 + t * kRows + r;
    const bool valid = R < num_rows;
    const int lim = valid ? start + R / G + 1 : 0;  // keys [0, lim) visible to the row
    const int nkb_t = t == 0 ? nkb0 : nkb1;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t sT = tS(t) + lane_off, oT = tO(t) + lane_off;
    const float sl2 = p.score_scale_log2;
    float m = -INFINITY, l = 0.f;  // m: the reference P and l are taken against (lazily raised)
    for (int j = 0; j < nkb_t; ++j) {
      const bool got = mbar_wait_bounded(B(kSFull0 + t), j & 1, deadline);
      if (!__all_sync(kFull, got)) {
        ok = false;
        break;
      }
      tc05::fence_after_sync();
      const int t0 = j * kKeys;
      // The block's scores and their max in log2 units. Blocks where no row of the warp reaches its
      // limit keep raw scores (the scale goes into the exponent's FMA; the max of the scaled scores is
      // the raw max times a positive scale, the raw min times a negative one); blocks that reach a
      // limit are scaled here and the keys past it set to -inf.
      float sv[kKeys];
      tc05::ld64(sT, *reinterpret_cast<float(*)[64]>(&sv[0]));
      tc05::ld64(sT + 64, *reinterpret_cast<float(*)[64]>(&sv[64]));
      float mul = sl2, mx;
      if (__any_sync(kFull, t0 + kKeys > lim)) {
#pragma unroll
        for (int k = 0; k < kKeys; ++k) sv[k] = t0 + k < lim ? sv[k] * sl2 : -INFINITY;
        mul = 1.f;
        mx = extreme<true, kKeys>(sv);
      } else if (sl2 >= 0.f) {
        mx = extreme<true, kKeys>(sv) * sl2;
      } else {
        mx = extreme<false, kKeys>(sv) * sl2;
      }
      // Raise the reference only when some row of the warp grew past it by more than 2^8.
      const bool raise = __any_sync(kFull, mx > m + kLazyRescale);
      float alpha = 1.f;
      if (raise) {
        const float mn = fmaxf(m, mx);
        alpha = (m == -INFINITY || mn == -INFINITY) ? (m == -INFINITY ? 0.f : 1.f) : ex2(m - mn);
        m = mn;
      }
      const float nref = m == -INFINITY ? 0.f : -m;
      // P = 2^(s * scale - ref) (ex2 of -inf is +0) in 16-bit, two keys per word, stored over S's first
      // 64 columns in two 32-column halves; the row sum adds the float values in four chains.
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t w[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float p0 = ex2(fmaf(sv[64 * h + 2 * k], mul, nref));
          const float p1 = ex2(fmaf(sv[64 * h + 2 * k + 1], mul, nref));
          w[k] = pack2<kBf16>(p0, p1);
          rs[(2 * k) & 3] += p0;
          rs[(2 * k + 1) & 3] += p1;
        }
        tc05::st32u(sT + 32 * h, w);
      }
      l = l * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
      // O's rescale: P(j-1).V has completed, since S(j) was committed after it (the issuer's commit
      // tracks every MMA it issued before).
      if (raise && j > 0) {
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          float v[32];
          tc05::ld32(oT + c * 32, v);
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] *= alpha;
          tc05::st32(oT + c * 32, v);
        }
      }
      tc05::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(B(kPFull0 + t));
    }
    // Epilogue: O / l -> the row's output.
    if (ok) {
      // All MMAs done: the issuer's final commit.
      const bool done = __all_sync(kFull, mbar_wait_bounded(B(kAllDone), 0, deadline));
      if (!done) {
        ok = false;
      } else {
        tc05::fence_after_sync();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint16_t* dst = static_cast<uint16_t*>(p.out) +
                        static_cast<int64_t>(q_row0 + (valid ? R / G : 0)) * p.o_stride_t +
                        static_cast<int64_t>(hk * G + R % G) * p.o_stride_h;
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          float v[32];
          tc05::ld32(oT + c * 32, v);
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
      }
    }
    if (!ok && lane == 0) atomicOr(p.err, 4u);
  }
  pdl_launch_dependents();
  tc05::fence_before_sync();
  const int any_fail = __syncthreads_or(!ok);
  if (warp == 10) {
    tc05::fence_after_sync();
    tc05::dealloc(tmem, kTmemCols);
  }
  if (any_fail && (warp == 8 || warp == 9) && lane == 0) {
    // A wait gave up somewhere, so copies this producer issued may not have been consumed: give them
    // a bounded chance to land before the CTA's shared memory goes. A stage is refilled only after its
    // previous fill was consumed, so only the last fill of each stage can be outstanding, and the
    // parity wait for that fill is exact.
    const int full0 = warp == 8 ? kKFull0 : kVFull0;
    const uint64_t drain_deadline = globaltimer_ns() + 100000000ull;
    for (int j = max(0, issued - kStages); j < issued; ++j)
      mbar_wait_bounded(B(full0 + j % kStages), (j / kStages) & 1, drain_deadline);
    if (warp == 8) {
      mbar_wait_bounded(B(kQFull0), 0, drain_deadline);
      if (has1) mbar_wait_bounded(B(kQFull0 + 1), 0, drain_deadline);
    }
  }
}

template <bool kBf16>
cudaError_t launch_pp(dim3 grid, const CUtensorMap& qm, const CUtensorMap& km, const CUtensorMap& vm, const MqParams& p,
                      cudaStream_t st) {
  auto kern = prefill_pp_kernel<kBf16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
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

}  // namespace

// Same support condition as the one-tile form: D = 128 and a group that divides the 128-row tile (the
// Q maps' boxes are shared).
cudaError_t launch_prefill_pp(KvType kv, const CUtensorMap& qm, const CUtensorMap& km, const CUtensorMap& vm,
                              const MqParams& p, int max_query_len, cudaStream_t st) {
  if (kv != KvType::F16 && kv != KvType::BF16) return cudaErrorInvalidValue;
  const int64_t rows = static_cast<int64_t>(max_query_len) * p.group;
  const dim3 grid(static_cast<unsigned>((rows + kTiles * kRows - 1) / (kTiles * kRows)), p.num_kv_heads, p.num_seqs);
  return kv == KvType::BF16 ? launch_pp<true>(grid, qm, km, vm, p, st) : launch_pp<false>(grid, qm, km, vm, p, st);
}

}  // namespace pa
