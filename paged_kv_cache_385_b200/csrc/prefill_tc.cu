// Multi-query attention over paged KV with 5th-generation tensor cores (tcgen05 + tensor memory),
// in two modes:
// * Chunked prefill (pa_prefill; notes page, kernels section: FlashAttention adapted to paged KV;
//   "vLLM 前世今生" §5.4 chunked prefill): row (new token i, group head g) of sequence s is position
//   p = start + i and attends over positions 0 .. p of its KV head.
// * Shared prefix (pa_decode_cascade; "vLLM 前世今生" §3.2, several sequences mapping the same
//   physical blocks): row (sequence s, group head g) holds that sequence's decode query; a CTA takes
//   one chunk of the prefix pages every block table shares and writes the rows' partial softmax
//   state (m, l, unnormalised acc) to the split workspace, merged later with the sequence's suffix.
//
// Work item = 128 query rows of one KV head; two CTAs per SM (one's softmax overlaps the other's
// MMAs). Prefill runs a persistent grid: each CTA takes one item per round of gridDim.x items (longest
// first), and its rings and buffers run on from one item to the next, so the next item's Q
// and first K/V blocks load while the current one finishes and a CTA's setup is paid once. Per block
// of 64 keys (4 pages), with the block's K and V staged by TMA in 128-byte-swizzled shared memory:
//   S[128 x 64] = Q . K^T       tcgen05.mma kind::f16, A = Q (K-major), B = K (K-major), D in TMEM;
//                               two S buffers, so QK of the next block runs during this softmax
//   softmax                     4 warps, one row per thread, S read from TMEM (tcgen05.ld), running
//                               max / sum in registers, P (bf16/f16) written back to TMEM over S,
//                               O rescaled in TMEM only when a row's max grew past the lazy bound
//   O[128 x 128] += P . V       A = P from TMEM, B = V (MN-major: d contiguous), D in TMEM
// Full output tiles are staged in the V stages and leave as tensor stores.
// Warps: 0-3 softmax + epilogue, 4 TMA producer of Q and K (3-stage ring), 5 QK issuer (one thread)
// and TMEM owner, 6 TMA producer of V (2-stage ring) and of the output stores, 7 PV issuer (one
// thread). Every mbarrier wait is bounded.
#include "internal.h"
#include "pa_device.cuh"
#include "tc05.cuh"

namespace pa {
namespace {

constexpr int kD = 128;
constexpr int kRows = 128;   // query rows per work item
constexpr int kThreads = 256;
constexpr uint32_t kHalf = 16384;  // one 64-element (128-byte) column half of a 128-row tile
constexpr uint32_t kTile = 2 * kHalf;

// Shared memory (112 KB + barriers): the Q tile, three stages of K tiles and two of V tiles, 64 keys
// each. K and V rings are separate: a K stage frees when its QK has run, long before the block's P.V,
// so the K copies of block j + 2 are in flight while block j is still being processed. The V stages
// (32 KB) also hold an item's output tile between its epilogue and its tensor stores.
constexpr int kKeys = 64;
constexpr int kKStages = 3, kVStages = 2;
constexpr uint32_t kHalfKV = kKeys * 128;  // a 64-element column half of a K or V tile
constexpr uint32_t kTileKV = 2 * kHalfKV;
constexpr uint32_t kQOff = 0;
constexpr uint32_t kKOff = kTile;
constexpr uint32_t kVOff = kKOff + kKStages * kTileKV;
constexpr uint32_t kBarOff = kVOff + kVStages * kTileKV;
constexpr uint32_t kSmemBytes = kBarOff + 256;
// TMEM: two S buffers of kKeys columns, then O's 128 columns.
constexpr uint32_t kTmemCols = 256;
static_assert(2 * kKeys + kD <= kTmemCols, "S buffers and O must fit the allocation");
// barrier slots (8 bytes each)
enum {
  kQFull = 0,
  kKFull0 = 1,   // kKStages
  kKEmpty0 = 4,  // kKStages
  kVFull0 = 7,   // kVStages
  kVEmpty0 = 9,  // kVStages
  kSFull0 = 11,  // 2
  kPFull0 = 13,  // 2: block gb arrives on kPFull0 + (gb & 1)
  kODone0 = 15,  // 2: P(gb).V commits to kODone0 + (gb & 1)
  kAllDone = 17,
  kTmemSlot = 18,
  kQEmpty = 19,  // the item's QKs have run: the Q tile may be refilled
  kOFree = 20,   // the item's epilogue has read O (4 softmax warps)
  kStaged = 21,  // the item's epilogue is done, its output tile staged in the V stages (4 softmax warps)
};
static_assert(8 * (kStaged + 1) <= 256, "barrier area");
// O is rescaled only when a row's running max grows by more than this (log2 units); until then P and
// the row sum keep the older reference, so the result is unchanged and P stays below 2^8.
constexpr float kLazyRescale = 8.f;

// Max (kMax) or min of n values in four independent chains.
template <bool kMax, int n>
__device__ __forceinline__ float extreme(const float (&v)[n]) {
  float e[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
  for (int k = 4; k < n; ++k) e[k & 3] = kMax ? fmaxf(e[k & 3], v[k]) : fminf(e[k & 3], v[k]);
  return kMax ? fmaxf(fmaxf(e[0], e[1]), fmaxf(e[2], e[3])) : fminf(fminf(e[0], e[1]), fminf(e[2], e[3]));
}

template <bool kBf16, bool kPrefix>
__global__ void __launch_bounds__(kThreads, 2)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap omap,
                      const MqParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  if (base & 1023u) {  // the swizzled tiles need 1024-byte alignment; never seen, but do not guess
    if (threadIdx.x == 0) atomicOr(p.err, 4u);
    return;
  }
  const uint32_t bar = base + kBarOff;
  auto B = [&](int i) { return bar + 8u * i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group;
  pdl_wait();
  // Prefix mode: the suffix decode after this grid reads nothing of it until its merge (where it
  // waits for this grid), so let it launch now and overlap its page loop with these MMAs.
  if constexpr (kPrefix) pdl_launch_dependents();

  if (threadIdx.x == 0) {
    mbar_init(B(kQFull), 1);
    mbar_init(B(kQEmpty), 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(B(kKFull0 + i), 1);
      mbar_init(B(kKEmpty0 + i), 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(B(kVFull0 + i), 1);
      mbar_init(B(kVEmpty0 + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(B(kSFull0 + i), 1);
      mbar_init(B(kPFull0 + i), 4);
      mbar_init(B(kODone0 + i), 1);
    }
    mbar_init(B(kOFree), 4);
    mbar_init(B(kStaged), 4);
    mbar_init(B(kAllDone), 1);
    fence_barrier_init();
  }
  if (warp == 5) tc05::alloc(B(kTmemSlot), kTmemCols);
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kBarOff + 8 * kTmemSlot);
  const uint32_t tS0 = tmem, tO = tmem + 2 * kKeys;
  bool ok = true;

  // Work item w: (row tile, KV head, z). Prefill: z is the sequence, and items are numbered longest
  // first (the last row tiles of every sequence before the earlier ones); CTA c takes items c,
  // c + gridDim.x, ..., so every CTA starts on long items and ends on short ones. Prefix: z is the
  // prefix chunk and row R of the grid is (sequence R / G, group head R % G); one item per CTA, taken
  // from the CTA's 3-D index.
  struct Item {
    int tile, hk, s;
    int q_row0, num_rows, start, key0, max_lim, npages, nkb;
    const int32_t* bt;
  };
  auto item = [&](int w) -> Item {
    Item I{};
    const int X = p.row_tiles;
    if constexpr (kPrefix) {
      I.tile = blockIdx.x;  // a 3-D grid of one item per CTA: (row tile, KV head, prefix chunk)
      I.hk = blockIdx.y;
      I.s = blockIdx.z;
      I.num_rows = p.num_seqs * G;
      if (I.tile * kRows >= I.num_rows) return I;
      I.key0 = I.s * p.chunk_tokens;
      I.max_lim = min(p.chunk_tokens, p.prefix_tokens - I.key0);
      if (I.max_lim <= 0) return I;
      I.bt = p.block_tables + I.key0 / 16;  // sequence 0's row; every sequence must map the same blocks
    } else {
      const int per = p.num_kv_heads * p.num_seqs;
      I.tile = X - 1 - w / per;
      I.s = (w % per) / p.num_kv_heads;
      I.hk = w % p.num_kv_heads;
      I.q_row0 = p.query_start[I.s];
      const int n_new = p.query_start[I.s + 1] - I.q_row0;
      const int ctx = p.context_lens[I.s];  // with the two above: one round trip
      I.num_rows = n_new * G;
      if (I.tile * kRows >= I.num_rows) return I;
      I.start = ctx - n_new;
      if (I.start < 0 || ctx > p.max_blocks * 16) {
        if (threadIdx.x == 0) atomicOr(p.err, 8u);
        return I;
      }
      if (I.tile == 0 && threadIdx.x == 0 && I.num_rows > X * kRows) atomicOr(p.err, 8u);
      I.max_lim = I.start + (min((I.tile + 1) * kRows, I.num_rows) - 1) / G + 1;  // the tile's last row
      I.bt = p.block_tables + static_cast<int64_t>(I.s) * p.bt_stride;
    }
    I.npages = (I.max_lim + 15) / 16;
    I.nkb = (I.max_lim + kKeys - 1) / kKeys;
    return I;
  };
  // Every role walks the same items and blocks: g counts the blocks of the CTA's earlier items (the
  // ring and buffer phases run on across items) and it counts its items with work.
  // Block j of an item (global block gb) from one stream (K by warp 4, V by warp 6): the block's 4 page
  // ids, then its 8 tile copies into stage gb % ns once that stage's previous fill has been consumed.
  auto produce = [&](const Item& I, int j, int gb, const CUtensorMap* map, uint32_t off, int ns, int full0,
                     int empty0, uint64_t deadline) -> bool {
    const int st = gb % ns;
    if (gb >= ns && !mbar_wait_bounded(B(empty0 + st), ((gb / ns) - 1) & 1, deadline)) return false;
    const int oob_row = p.num_blocks * p.num_kv_heads * 16;  // a box starting here is all zero fill
    int ys[kKeys / 16];
#pragma unroll
    for (int i = 0; i < kKeys / 16; ++i) {
      const int page = j * (kKeys / 16) + i;
      ys[i] = page < I.npages ? I.bt[page] : -1;
    }
#pragma unroll
    for (int i = 0; i < kKeys / 16; ++i) {
      const int page = j * (kKeys / 16) + i;
      const int bid = ys[i];
      ys[i] = oob_row;
      if (page < I.npages) {
        if (bid >= 0 && bid < p.num_blocks) ys[i] = (bid * p.num_kv_heads + I.hk) * 16;
        else atomicOr(p.err, 1u);
      }
    }
    const uint32_t dst = base + off + st * kTileKV;
    mbar_arrive_expect_tx(B(full0 + st), kTileKV);
#pragma unroll
    for (int i = 0; i < kKeys / 16; ++i)
      for (int u = 0; u < 2; ++u) tma_load_2d(dst + u * kHalfKV + i * 2048, map, B(full0 + st), u * 64, ys[i]);
    return true;
  };
  // A full prefill tile leaves through the output map from the V stages, where the softmax warps
  // staged it; partial tiles (their last rows would be the next sequence's) are stored row by row.
  auto full_tile = [&](const Item& I) { return !kPrefix && (I.tile + 1) * kRows <= I.num_rows; };
  int issued = 0, q_issued = 0;  // producer lanes: fills issued (for the drain after a failure)

  if (warp == 4) {
    // ---- producer of Q and K ----------------------------------------------------------------------
    if (lane == 0) {
      prefetch_tensormap(&qmap);
      int g = 0, it = 0;
      for (int k = 0; ok && (!kPrefix || k == 0); ++k) {  // (a prefix CTA takes one item)
        const int64_t w64 = static_cast<int64_t>(k) * gridDim.x + blockIdx.x;
        if (w64 >= p.num_items) break;
        const int w = static_cast<int>(w64);
        const Item I = item(w);
        if (I.nkb == 0) continue;
        const uint64_t deadline = globaltimer_ns() + 2000000000ull;
        // Q(it) once every QK of the previous item has run (the issuer commits Q_empty after them).
        if (it > 0 && !mbar_wait_bounded(B(kQEmpty), (it - 1) & 1, deadline)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(B(kQFull), kTile);
        const int tok0 = I.q_row0 + I.tile * (kRows / G);
        tc05::tma_load_3d(base + kQOff, &qmap, B(kQFull), 0, I.hk * G, tok0);
        tc05::tma_load_3d(base + kQOff + kHalf, &qmap, B(kQFull), 64, I.hk * G, tok0);
        ++q_issued;
        for (int j = 0; j < I.nkb && ok; ++j) {
          ok = produce(I, j, g + j, &kmap, kKOff, kKStages, kKFull0, kKEmpty0, deadline);
          issued += ok;
        }
        g += I.nkb;
        ++it;
      }
      if (!ok) atomicOr(p.err, 4u);
    }
  } else if (warp == 6) {
    // ---- producer of V, and the output tiles' tensor stores ----------------------------------------
    if (lane == 0) {
      prefetch_tensormap(&omap);
      // Before V(it, 0) may land in the V stages, item it-1's output tile staged there must have been
      // read out: wait for the softmax warps' Staged arrival, issue its stores, and wait for their reads.
      auto drain_staged = [&](const Item& I, int i, uint64_t deadline) -> bool {
        if (!mbar_wait_bounded(B(kStaged), i & 1, deadline)) return false;
        if constexpr (kPrefix) {
          // The partial tile, from the K/V stages: boxes of 32 columns x this chunk's partition x G
          // heads x 128 / G sequences (those past the batch are clipped by the map).
#pragma unroll
          for (int c = 0; c < kD / 32; ++c)
            tma_store_4d(&omap, base + kKOff + c * (kRows * 128), 32 * c, I.s, I.hk * G, I.tile * (kRows / G));
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        } else if (full_tile(I)) {
          const int tok0 = I.q_row0 + I.tile * (kRows / G);
          tma_store_3d(&omap, base + kVOff, 0, I.hk * G, tok0);
          tma_store_3d(&omap, base + kVOff + kHalf, 64, I.hk * G, tok0);
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
        return true;
      };
      int g = 0, it = 0;
      Item prev{};
      for (int k = 0; ok && (!kPrefix || k == 0); ++k) {  // (a prefix CTA takes one item)
        const int64_t w64 = static_cast<int64_t>(k) * gridDim.x + blockIdx.x;
        if (w64 >= p.num_items) break;
        const int w = static_cast<int>(w64);
        const Item I = item(w);
        if (I.nkb == 0) continue;
        const uint64_t deadline = globaltimer_ns() + 2000000000ull;
        if (it > 0 && !drain_staged(prev, it - 1, deadline)) {
          ok = false;
          break;
        }
        for (int j = 0; j < I.nkb && ok; ++j) {
          ok = produce(I, j, g + j, &vmap, kVOff, kVStages, kVFull0, kVEmpty0, deadline);
          issued += ok;
        }
        g += I.nkb;
        ++it;
        prev = I;
      }
      if (ok && it > 0) ok = drain_staged(prev, it - 1, globaltimer_ns() + 2000000000ull);
      // (Every store has read its shared-memory source by here; the global writes are the grid's
      // own memory operations, visible to a stream-ordered or dependent grid once this one completes.)
      if (!ok) atomicOr(p.err, 4u);
    }
  } else if (warp == 5) {
    // ---- QK issuer: S(gb) = Q K(gb)^T into S buffer gb & 1 ----------------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc05::idesc_f16(kBf16, kRows, kKeys, false, false);
      int g = 0, it = 0;
      for (int k = 0; ok && (!kPrefix || k == 0); ++k) {  // (a prefix CTA takes one item)
        const int64_t w64 = static_cast<int64_t>(k) * gridDim.x + blockIdx.x;
        if (w64 >= p.num_items) break;
        const int w = static_cast<int>(w64);
        const Item I = item(w);
        if (I.nkb == 0) continue;
        const uint64_t deadline = globaltimer_ns() + 2000000000ull;
        // Q_full next completes for Q(it+1), loaded only after this item's QKs: the wait is exact.
        ok = mbar_wait_bounded(B(kQFull), it & 1, deadline);
        for (int j = 0; j < I.nkb && ok; ++j) {
          const int gb = g + j;
          // Buffer gb & 1 holds P(gb-2) until P(gb-2).V has completed. O_done is two barriers by block
          // parity, so the one waited here next completes for P(gb).V, which needs S(gb) from the QK
          // this thread has yet to issue: never two phases ahead. Nor one behind: QK(gb-2) was issued
          // only after P(gb-4).V completed on it.
          const int ks_ = gb % kKStages;
          if ((gb >= 2 && !mbar_wait_bounded(B(kODone0 + (gb & 1)), ((gb - 2) >> 1) & 1, deadline)) ||
              !mbar_wait_bounded(B(kKFull0 + ks_), (gb / kKStages) & 1, deadline)) {
            ok = false;
            break;
          }
          tc05::fence_after_sync();
          const uint32_t kbase = base + kKOff + ks_ * kTileKV;
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {  // 8 k-steps of 16 along d, 32 bytes apart in a half
            const uint32_t cb = (ks & 3) * 32;
            tc05::mma_f16(tS0 + (gb & 1) * kKeys, tc05::smem_desc_sw128(base + kQOff + (ks >> 2) * kHalf + cb, 16, 1024),
                          tc05::smem_desc_sw128(kbase + (ks >> 2) * kHalfKV + cb, 16, 1024), idesc_qk, ks > 0);
          }
          tc05::commit(B(kSFull0 + (gb & 1)));
          tc05::commit(B(kKEmpty0 + ks_));  // K stage free again once this QK has run
        }
        if (!ok) break;
        tc05::commit(B(kQEmpty));  // the Q tile is free once this item's QKs have run
        g += I.nkb;
        ++it;
      }
      if (!ok) atomicOr(p.err, 4u);
    }
  } else if (warp == 7) {
    // ---- PV issuer: O += P(gb) V(gb) ---------------------------------------------------------------
    // A separate thread from the QK issuer, so that P.V is issued as soon as P is ready even while the
    // QK issue of a later block waits for room in the tensor pipe.
    if (lane == 0) {
      constexpr uint32_t idesc_pv = tc05::idesc_f16(kBf16, kRows, kD, false, true);
      int g = 0, it = 0;
      for (int k = 0; ok && (!kPrefix || k == 0); ++k) {  // (a prefix CTA takes one item)
        const int64_t w64 = static_cast<int64_t>(k) * gridDim.x + blockIdx.x;
        if (w64 >= p.num_items) break;
        const int w = static_cast<int>(w64);
        const Item I = item(w);
        if (I.nkb == 0) continue;
        const uint64_t deadline = globaltimer_ns() + 2000000000ull;
        // The item's first P.V overwrites O: the previous item's epilogue must have read it. O_free next
        // completes for this item's epilogue, which needs these products: the wait is exact.
        if (it > 0 && !mbar_wait_bounded(B(kOFree), (it - 1) & 1, deadline)) ok = false;
        for (int j = 0; j < I.nkb && ok; ++j) {
          const int gb = g + j;
          // P_full is two barriers by block parity: block gb + 2 cannot arrive before this wait has
          // seen block gb (its QK needs P(gb).V), so a parity wait never meets a barrier two phases ahead.
          if (!mbar_wait_bounded(B(kPFull0 + (gb & 1)), (gb >> 1) & 1, deadline) ||
              !mbar_wait_bounded(B(kVFull0 + gb % kVStages), (gb / kVStages) & 1, deadline)) {
            ok = false;
            break;
          }
          tc05::fence_after_sync();
          // kKeys / 16 k-steps; P from TMEM (written over S(gb), 8 columns = 16 keys per step), V
          // MN-major in shared memory (16 keys = 2048 B).
          const uint32_t vbase = base + kVOff + (gb % kVStages) * kTileKV;
#pragma unroll
          for (int kt = 0; kt < kKeys / 16; ++kt) {
            tc05::mma_f16_ts(tO, tS0 + (gb & 1) * kKeys + kt * 8,
                             tc05::smem_desc_sw128(vbase + kt * 2048, kHalfKV, 1024), idesc_pv, (j > 0 || kt > 0));
          }
          tc05::commit(B(kODone0 + (gb & 1)));
          tc05::commit(B(kVEmpty0 + gb % kVStages));
        }
        g += I.nkb;
        ++it;
      }
      // Every QK has completed before its softmax finished, so this covers all of the CTA's MMAs.
      tc05::commit(B(kAllDone));
      mbar_wait_bounded(B(kAllDone), 0, globaltimer_ns() + 1000000000ull);
      if (!ok) atomicOr(p.err, 4u);
    }
  } else {
    // ---- softmax warps: thread = row ---------------------------------------------------------------
    const int r = threadIdx.x;  // 0..127, TMEM lane r
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = p.score_scale_log2;
    int g = 0;
    for (int k = 0; ok && (!kPrefix || k == 0); ++k) {  // (a prefix CTA takes one item)
      const int64_t w64 = static_cast<int64_t>(k) * gridDim.x + blockIdx.x;
      if (w64 >= p.num_items) break;
      const int w = static_cast<int>(w64);
      const Item I = item(w);
      if (I.nkb == 0) continue;
      const uint64_t deadline = globaltimer_ns() + 2000000000ull;
      const int R = I.tile * kRows + r;
      const bool valid = R < I.num_rows;
      // The row's visible keys, counted from key0: the causal diagonal, or the sequence's context
      // clipped to the prefix (none of this chunk when it is shorter).
      int lim = 0;
      if (valid) {
        if constexpr (kPrefix) {
          lim = min(p.context_lens[R / G], p.prefix_tokens) - I.key0;
        } else {
          lim = I.start + R / G + 1;
        }
      }
      float m = -INFINITY, l = 0.f;  // m: the reference P and l are taken against (lazily raised)
      for (int j = 0; j < I.nkb; ++j) {
        const int gb = g + j;
        const bool got = mbar_wait_bounded(B(kSFull0 + (gb & 1)), (gb >> 1) & 1, deadline);
        if (!__all_sync(kFull, got)) {
          ok = false;
          break;
        }
        tc05::fence_after_sync();
        const int t0 = j * kKeys;
        // The block's scores and their max in log2 units. Blocks where no row of the warp reaches its
        // limit keep raw scores (the scale is applied in the exponent's FMA; the max of the scaled
        // scores is the raw max times a positive scale, the raw min times a negative one); blocks
        // that reach a limit are scaled here and the keys past it set to -inf.
        float sv[kKeys];
        tc05::ld64(tS0 + (gb & 1) * kKeys + lane_off, sv);
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
        // P = 2^(s * scale - ref) (ex2 of -inf is +0) in 16-bit, packed two keys per word, stored over
        // the first kKeys / 2 columns of S(gb) (whose scores are all in registers by now) 16 columns at
        // a time as they are made; the row sum adds the float values in four chains.
        static_assert(kKeys == 64, "P is stored as two 16-column TMEM stores");
        float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t wd[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float p0 = ex2(fmaf(sv[32 * h + 2 * k], mul, nref));
            const float p1 = ex2(fmaf(sv[32 * h + 2 * k + 1], mul, nref));
            wd[k] = pack2<kBf16>(p0, p1);
            rs[(2 * k) & 3] += p0;
            rs[(2 * k + 1) & 3] += p1;
          }
          tc05::st16u_nowait(tS0 + (gb & 1) * kKeys + lane_off + 16 * h, wd);
        }
        l = l * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
        // O's rescale waits for the previous P . V (only when the reference moved). Its barrier next
        // completes for P(gb+1).V, which needs this warp's P(gb+1): never two phases ahead. It is not
        // one behind either: S(gb-1) came from QK(gb-1), issued after P(gb-3).V completed.
        if (raise && j > 0) {
          const bool done = mbar_wait_bounded(B(kODone0 + ((gb - 1) & 1)), ((gb - 1) >> 1) & 1, deadline);
          if (!__all_sync(kFull, done)) {
            ok = false;
            break;
          }
          tc05::fence_after_sync();
#pragma unroll
          for (int c = 0; c < kD / 32; ++c) {
            float v[32];
            tc05::ld32(tO + lane_off + c * 32, v);
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] *= alpha;
            tc05::st32(tO + lane_off + c * 32, v);
          }
        }
        tc05::st_wait();  // P (and O) in tensor memory before the arrive below
        // Keys past every row's limit may hold any bits; zero those V rows so 0 * NaN cannot occur.
        if (t0 + kKeys > I.max_lim) {
          const bool landed = mbar_wait_bounded(B(kVFull0 + gb % kVStages), (gb / kVStages) & 1, deadline);
          if (!__all_sync(kFull, landed)) {
            ok = false;
            break;
          }
          const uint32_t vbase = base + kVOff + (gb % kVStages) * kTileKV;
          const int first = I.max_lim - t0;  // rows [first, kKeys) of the V tile, both halves
          for (int idx = r; idx < (kKeys - first) * 16; idx += 128) {
            const int row = first + idx / 16, c16 = idx % 16;
            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(vbase + (c16 >> 3) * kHalfKV + row * 128 +
                                                                           (c16 & 7) * 16),
                         "r"(0u)
                         : "memory");
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        tc05::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(B(kPFull0 + (gb & 1)));
      }
      if (!ok) break;
      // Epilogue once the item's last P.V has completed. Its O_done barrier next completes for
      // P(gl+2).V, which needs this warp's next P: never two phases ahead; nor one behind, since
      // QK(gl) was issued after P(gl-2).V completed and this warp has seen S(gl).
      const int gl = g + I.nkb - 1;
      if (!__all_sync(kFull, mbar_wait_bounded(B(kODone0 + (gl & 1)), (gl >> 1) & 1, deadline))) {
        ok = false;
        break;
      }
      tc05::fence_after_sync();
      if constexpr (kPrefix) {
        // The row's (m, l, O) -> its workspace slot. O goes through shared memory (the K/V stages: a
        // prefix CTA takes one item, so nothing is prefetched into them) as four 32-column boxes in
        // the 128-byte-swizzled layout the workspace map names (16-byte chunk c of row r at position
        // c ^ (r % 8), conflict-free), which the V producer lane stores as tensor stores; (m, l)
        // directly. (That every sequence maps the prefix pages to sequence 0's blocks is checked by
        // the suffix decode, off this kernel's critical path.)
        const uint32_t stg = base + kKOff;
        static_assert(kKOff + (kD / 32) * kRows * 128 <= kBarOff, "the partial tile fits the K/V stages");
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          float v[32];
          tc05::ld32(tO + lane_off + c * 32, v);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(stg + c * (kRows * 128) + r * 128 +
                                                                           ((q ^ (r & 7)) << 4)),
                         "f"(v[4 * q]), "f"(v[4 * q + 1]), "f"(v[4 * q + 2]), "f"(v[4 * q + 3])
                         : "memory");
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (valid) {
          const int Hq = p.num_kv_heads * G;
          const int64_t slot = (static_cast<int64_t>(R / G) * Hq + I.hk * G + R % G) * p.ws_parts + I.s;
          *reinterpret_cast<float2*>(p.ws_ml + slot * 2) = make_float2(m, l);
        }
      } else {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        if (full_tile(I)) {
          // Into the V stages (free: the item's last P.V has run, and the V producer loads the next
          // item's V only after it has stored this tile) in the 128-byte-swizzled layout the output
          // map names: 16-byte chunk c of row r at position c ^ (r % 8), so the rows leave coalesced.
          const uint32_t stg = base + kVOff;
          static_assert(kVStages * kTileKV == kTile, "the output tile fills the V stages");
#pragma unroll
          for (int c = 0; c < kD / 32; ++c) {
            float v[32];
            tc05::ld32(tO + lane_off + c * 32, v);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int chunk = (c & 1) * 4 + q;  // 8 columns each, within the half c / 2
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(stg + (c >> 1) * kHalf + r * 128 +
                                                                            ((chunk ^ (r & 7)) << 4)),
                           "r"(pack2<kBf16>(v[8 * q] * inv, v[8 * q + 1] * inv)),
                           "r"(pack2<kBf16>(v[8 * q + 2] * inv, v[8 * q + 3] * inv)),
                           "r"(pack2<kBf16>(v[8 * q + 4] * inv, v[8 * q + 5] * inv)),
                           "r"(pack2<kBf16>(v[8 * q + 6] * inv, v[8 * q + 7] * inv))
                           : "memory");
            }
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        } else {
          uint16_t* dst = static_cast<uint16_t*>(p.out) + static_cast<int64_t>(I.q_row0 + (valid ? R / G : 0)) * p.o_stride_t +
                          static_cast<int64_t>(I.hk * G + R % G) * p.o_stride_h;
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
        }
      }
      // O is read (the next item's first P.V may overwrite it) and this warp's rows are staged.
      tc05::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(B(kOFree));
        mbar_arrive(B(kStaged));
      }
      g += I.nkb;
    }
    if (!ok && lane == 0) atomicOr(p.err, 4u);
  }
  if constexpr (!kPrefix) pdl_launch_dependents();
  tc05::fence_before_sync();
  const int any_fail = __syncthreads_or(!ok);
  if (warp == 5) {
    tc05::fence_after_sync();
    tc05::dealloc(tmem, kTmemCols);
  }
  if (any_fail && (warp == 4 || warp == 6) && lane == 0) {
    // A wait gave up somewhere, so copies this producer issued may not have been consumed: give them
    // a bounded chance to land before the CTA's shared memory goes. A stage is refilled only after
    // its previous fill was consumed, so only the last fill of each stage can be outstanding, and
    // the parity wait for that fill is exact; likewise the last Q fill.
    const int ns = warp == 4 ? kKStages : kVStages;
    const int full0 = warp == 4 ? kKFull0 : kVFull0;
    const uint64_t drain_deadline = globaltimer_ns() + 100000000ull;
    for (int j = max(0, issued - ns); j < issued; ++j)
      mbar_wait_bounded(B(full0 + j % ns), (j / ns) & 1, drain_deadline);
    if (warp == 4 && q_issued > 0) mbar_wait_bounded(B(kQFull), (q_issued - 1) & 1, drain_deadline);
  }
}

template <bool kBf16, bool kPrefix>
cudaError_t launch_tc(dim3 grid, const CUtensorMap& qm, const CUtensorMap& km, const CUtensorMap& vm,
                      const CUtensorMap& om, const MqParams& p, cudaStream_t st) {
  auto kern = prefill_tc_kernel<kBf16, kPrefix>;
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
  return cudaLaunchKernelEx(&cfg, kern, qm, km, vm, om, p);
}

// SMs of the current device, looked up once per device.
cudaError_t device_sms(int* sms) {
  static int cached[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int n = dev < 64 ? __atomic_load_n(&cached[dev], __ATOMIC_ACQUIRE) : 0;
  if (n == 0) {
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (dev < 64) __atomic_store_n(&cached[dev], n, __ATOMIC_RELEASE);
  }
  *sms = n;
  return cudaSuccess;
}

}  // namespace

bool prefill_tc_supported(int head_dim, int group) {
  return head_dim == kD && group >= 1 && group <= 16 && (kRows % group) == 0;
}

cudaError_t launch_prefill_tc(KvType kv, const CUtensorMap& qm, const CUtensorMap& km, const CUtensorMap& vm,
                              const CUtensorMap& om, const MqParams& p, int max_query_len, cudaStream_t st) {
  if (kv != KvType::F16 && kv != KvType::BF16) return cudaErrorInvalidValue;
  // Persistent: two CTAs per SM, each taking one item per round of gridDim.x items.
  const int64_t tiles = (static_cast<int64_t>(max_query_len) * p.group + kRows - 1) / kRows;
  const int64_t items = tiles * p.num_kv_heads * p.num_seqs;
  if (items > 0x7fffffff) return cudaErrorInvalidValue;
  int sms = 0;
  cudaError_t e = device_sms(&sms);
  if (e != cudaSuccess) return e;
  MqParams q = p;
  q.row_tiles = static_cast<int32_t>(tiles);
  q.num_items = static_cast<int32_t>(items);
  const dim3 grid(static_cast<unsigned>(std::min<int64_t>(items, 2 * static_cast<int64_t>(sms))));
  return kv == KvType::BF16 ? launch_tc<true, false>(grid, qm, km, vm, om, q, st)
                            : launch_tc<false, false>(grid, qm, km, vm, om, q, st);
}

// Shared-prefix mode: one CTA per (row tile of num_seqs * G, KV head, prefix chunk); chunk_tokens must
// be a multiple of the key block. wm maps the workspace's partial rows.
cudaError_t launch_prefix_tc(KvType kv, const CUtensorMap& qm, const CUtensorMap& km, const CUtensorMap& vm,
                             const CUtensorMap& wm, const MqParams& p, cudaStream_t st) {
  if (kv != KvType::F16 && kv != KvType::BF16) return cudaErrorInvalidValue;
  if (p.chunk_tokens <= 0 || p.chunk_tokens % kKeys || p.prefix_tokens % 16) return cudaErrorInvalidValue;
  // One item per CTA: (row tile of num_seqs * G, KV head, prefix chunk).
  const int64_t tiles = (static_cast<int64_t>(p.num_seqs) * p.group + kRows - 1) / kRows;
  const int64_t items = tiles * p.num_kv_heads * p.num_chunks;
  if (items > 0x7fffffff || p.num_kv_heads > 65535 || p.num_chunks > 65535) return cudaErrorInvalidValue;
  MqParams q = p;
  q.row_tiles = static_cast<int32_t>(tiles);
  q.num_items = static_cast<int32_t>(items);
  const dim3 grid(static_cast<unsigned>(tiles), p.num_kv_heads, p.num_chunks);
  return kv == KvType::BF16 ? launch_tc<true, true>(grid, qm, km, vm, wm, q, st)
                            : launch_tc<false, true>(grid, qm, km, vm, wm, q, st);
}

}  // namespace pa
