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
#include <cfloat>
#include <utility>

#include "internal.h"
#include "pa_device.cuh"

namespace pa {

__device__ uint32_t g_error_word;

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// OCC is the number of CTAs per SM a kernel is compiled for: the page pipeline gets 192 KB / OCC of
// shared memory (96, 64 or 48 KB) and registers are capped to fit. 16-bit pages with one query per
// KV head are pure bandwidth: deep pipelines, 2 CTAs/SM. Grouped queries add math per byte and
// e4m3 pages even more (widening, 3x the pages per byte moved), so those trade stages for resident
// warps: 3 and 4 CTAs/SM.
template <KvType KV, QType QT, int D, int NT, int KIND, int OCC>
struct Cfg {
  static constexpr bool kFp8 = KV == KvType::E4M3;
  static constexpr int kEsz = kFp8 ? 1 : 2;
  static constexpr int kRowBytes = D * kEsz;         // one token row of a page
  static constexpr int kSubPages = kRowBytes / 128;  // 128-byte swizzled sub-pages per page
  static constexpr int kSubElems = 128 / kEsz;       // TMA box width in elements
  static constexpr int kPageBytes = 16 * kRowBytes;
  static constexpr int kWarps = kDecodeWarps;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kStageBytes = 2 * kPageBytes;  // K page + V page
  static constexpr int kMinBlocks = OCC;
  static constexpr int kPipeBudget = OCC == 2 ? 96 * 1024 : (OCC == 3 ? 64 * 1024 : 48 * 1024);
  static constexpr int kStages = kPipeBudget / (kWarps * kStageBytes);
  static constexpr int kPipeBytes = kWarps * kStages * kStageBytes;
  static constexpr bool kMmaBf16 = KV == KvType::BF16;  // e4m3 pages are widened to f16
  static constexpr bool kQBf16 = QT == QType::BF16;
  static constexpr int kGPad = 8 * NT;
  static constexpr int kMergeFloats = kWarps * kGPad * (D + 2);
  static constexpr int kSmemBytes = 1024 + kPipeBytes + kWarps * kStages * 8;
  static_assert(kSubPages >= 1 && kRowBytes % 128 == 0, "page rows must be whole 128-byte lines");
  static_assert(kStages >= 2, "need at least two stages per warp");
  static_assert(kMergeFloats * 4 <= kPipeBytes, "merge area must fit in the pipeline buffers");
};

// Byte offset of 16-byte chunk `chunk` of token row `tok` in a 128-byte-swizzled sub-page.
__device__ __forceinline__ uint32_t swz(int tok, int chunk) {
  return static_cast<uint32_t>(tok * 128 + ((chunk ^ (tok & 7)) << 4));
}

template <class C>
__device__ __forceinline__ uint32_t q_pair(const void* qrow, int d) {
  // Two consecutive query elements (d, d+1) as the mma operand type.
  const uint32_t raw = *reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(qrow) + d);
  if constexpr (C::kFp8 && C::kQBf16) {
    const float2 f = unpack2<true>(raw);
    return pack2<false>(f.x, f.y);
  } else {
    return raw;
  }
}

// ---------------------------------------------------------------------------------------------
// Tensor-core per-page math.
// ---------------------------------------------------------------------------------------------
template <class C, int D, int NT>
struct TcMath {
  static constexpr int KS = D / 16;  // k-steps of QK^T == m-tiles of PV
  uint32_t qf[NT][KS][2];
  float acc[NT][KS][4];
  float m[NT][2];
  float l[NT][2];
  int lane;

  __device__ __forceinline__ void init(const DecodeParams& p, int s, int hk, int lane_) {
    lane = lane_;
    const int r = lane >> 2, q4 = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int g = nt * 8 + r;
      const bool gv = g < p.group;
      const void* qrow = static_cast<const uint16_t*>(p.q) + s * p.q_stride_s + (hk * p.group + (gv ? g : 0)) * p.q_stride_h;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t b0 = 0, b1 = 0;
        if (gv) {
          if constexpr (C::kFp8) {
            // Logical k (2q, 2q+1) <-> d = 16ks + 4q + {0,1}; (2q+8, 2q+9) <-> 16ks + 4q + {2,3}.
            b0 = q_pair<C>(qrow, 16 * ks + 4 * q4);
            b1 = q_pair<C>(qrow, 16 * ks + 4 * q4 + 2);
          } else {
            b0 = q_pair<C>(qrow, 16 * ks + 2 * q4);
            b1 = q_pair<C>(qrow, 16 * ks + 2 * q4 + 8);
          }
        }
        qf[nt][ks][0] = b0;
        qf[nt][ks][1] = b1;
      }
#pragma unroll
      for (int mt = 0; mt < KS; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][mt][i] = 0.f;
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
    }
  }

  // One 16-token page; kb/vb are the shared addresses of its K and V pages; nv valid tokens.
  __device__ __forceinline__ void page(uint32_t kb, uint32_t vb, int nv, float sl2) {
    const int x7 = lane & 7;
    const int a_tok = (((lane >> 3) & 1) << 3) | x7;  // K (and e4m3 V) matrices: tok half = bit 3
    const int a_co = lane >> 4;
    const int t_tok = ((lane >> 4) << 3) | x7;        // 16-bit V^T matrices: tok half = bit 4
    const int t_co = (lane >> 3) & 1;
    const int r = lane >> 2, q4 = lane & 3;

    // ---- S^T = K . Q^T --------------------------------------------------------------------
    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    if constexpr (C::kFp8) {
#pragma unroll
      for (int kp = 0; kp < KS / 2; ++kp) {
        uint32_t raw[4];
        ldmatrix_x4(raw, kb + swz(a_tok, 2 * kp + a_co));
        // a0a1 / a2a3 take codes (d 4q, 4q+1) of tokens r / r+8; a4a5 / a6a7 take (d 4q+2, 4q+3).
        uint32_t a0[4], a1[4];
        e4m3x4_to_f16x2x2(raw[0], a0[0], a0[2]);
        e4m3x4_to_f16x2x2(raw[1], a0[1], a0[3]);
        e4m3x4_to_f16x2x2(raw[2], a1[0], a1[2]);
        e4m3x4_to_f16x2x2(raw[3], a1[1], a1[3]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_16816<false>(sc[nt], a0, qf[nt][2 * kp][0], qf[nt][2 * kp][1]);
          mma_16816<false>(sc[nt], a1, qf[nt][2 * kp + 1][0], qf[nt][2 * kp + 1][1]);
        }
      }
    } else {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t a[4];
        ldmatrix_x4(a, kb + (ks >> 2) * 2048 + swz(a_tok, ((ks & 3) << 1) + a_co));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816<C::kMmaBf16>(sc[nt], a, qf[nt][ks][0], qf[nt][ks][1]);
      }
    }

    // ---- online softmax over this page (log2 domain) -------------------------------------
    const bool v_lo = r < nv, v_hi = r + 8 < nv;
    uint32_t pf[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float s0 = v_lo ? sc[nt][0] * sl2 : -INFINITY;
      float s1 = v_lo ? sc[nt][1] * sl2 : -INFINITY;
      float s2 = v_hi ? sc[nt][2] * sl2 : -INFINITY;
      float s3 = v_hi ? sc[nt][3] * sl2 : -INFINITY;
      float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
      }
      const float mn0 = fmaxf(m[nt][0], mx0), mn1 = fmaxf(m[nt][1], mx1);
      const float al0 = ex2(m[nt][0] - mn0), al1 = ex2(m[nt][1] - mn1);
      m[nt][0] = mn0;
      m[nt][1] = mn1;
      const uint32_t x0 = pack2<C::kMmaBf16>(ex2(s0 - mn0), ex2(s1 - mn1));
      const uint32_t x1 = pack2<C::kMmaBf16>(ex2(s2 - mn0), ex2(s3 - mn1));
      // The denominator sums the same rounded weights the PV product uses.
      const float2 f0 = unpack2<C::kMmaBf16>(x0), f1 = unpack2<C::kMmaBf16>(x1);
      l[nt][0] = l[nt][0] * al0 + (f0.x + f1.x);
      l[nt][1] = l[nt][1] * al1 + (f0.y + f1.y);
      if (__any_sync(kFull, al0 != 1.f || al1 != 1.f)) {  // skipped once the running max settles
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          acc[nt][mt][0] *= al0;
          acc[nt][mt][1] *= al1;
          acc[nt][mt][2] *= al0;
          acc[nt][mt][3] *= al1;
        }
      }
      pf[nt][0] = movmatrix_trans(x0);  // (k = tok 2q, 2q+1 ; n = g = r)
      pf[nt][1] = movmatrix_trans(x1);  // (k = tok 2q+8, 2q+9)
    }

    // Tokens past the context may hold any bits (NaN included): zero them in V^T so 0 * NaN
    // never reaches the accumulator.
    uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
    if (nv < 16) {
      mlo = (2 * q4 < nv ? 0x0000ffffu : 0u) | (2 * q4 + 1 < nv ? 0xffff0000u : 0u);
      mhi = (2 * q4 + 8 < nv ? 0x0000ffffu : 0u) | (2 * q4 + 9 < nv ? 0xffff0000u : 0u);
    }

    // ---- O^T += V^T . P^T -----------------------------------------------------------------
    if constexpr (C::kFp8) {
#pragma unroll
      for (int mp = 0; mp < KS / 2; ++mp) {
        uint32_t raw[4];
        ldmatrix_x4_trans(raw, vb + swz(a_tok, 2 * mp + a_co));
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          // (tok 2q, d), (tok 2q, d+1), (tok 2q+1, d), (tok 2q+1, d+1) -> pairs of tokens per d.
          const uint32_t t0 = __byte_perm(raw[2 * half], 0, 0x3120);
          const uint32_t t1 = __byte_perm(raw[2 * half + 1], 0, 0x3120);
          uint32_t a[4];
          e4m3x4_to_f16x2x2(t0, a[0], a[1]);
          e4m3x4_to_f16x2x2(t1, a[2], a[3]);
          if (nv < 16) {
            a[0] &= mlo;
            a[1] &= mlo;
            a[2] &= mhi;
            a[3] &= mhi;
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_16816<false>(acc[nt][2 * mp + half], a, pf[nt][0], pf[nt][1]);
        }
      }
    } else {
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        uint32_t a[4];
        ldmatrix_x4_trans(a, vb + (mt >> 2) * 2048 + swz(t_tok, ((mt & 3) << 1) + t_co));
        if (nv < 16) {
          a[0] &= mlo;
          a[1] &= mlo;
          a[2] &= mhi;
          a[3] &= mhi;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816<C::kMmaBf16>(acc[nt][mt], a, pf[nt][0], pf[nt][1]);
      }
    }
  }

  // Write this warp's (m, l, acc) into the merge area: mg[g], lg[g], ag[g][D] (floats).
  __device__ __forceinline__ void store(float* mg, float* lg, float* ag) {
    const int r = lane >> 2, q4 = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float lv = l[nt][j];
        lv += __shfl_xor_sync(kFull, lv, 4);
        lv += __shfl_xor_sync(kFull, lv, 8);
        lv += __shfl_xor_sync(kFull, lv, 16);
        if (r == 0) {
          mg[nt * 8 + 2 * q4 + j] = m[nt][j];
          lg[nt * 8 + 2 * q4 + j] = lv;
        }
      }
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        int d_lo, d_hi;
        if constexpr (C::kFp8) {
          d_lo = 16 * mt + 2 * r;
          d_hi = d_lo + 1;
        } else {
          d_lo = 16 * mt + r;
          d_hi = d_lo + 8;
        }
        const int g = nt * 8 + 2 * q4;
        ag[g * D + d_lo] = acc[nt][mt][0];
        ag[(g + 1) * D + d_lo] = acc[nt][mt][1];
        ag[g * D + d_hi] = acc[nt][mt][2];
        ag[(g + 1) * D + d_hi] = acc[nt][mt][3];
      }
    }
  }
};

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

// Merge the partitions of each (sequence, query head). blockDim.x / D groups (1 .. kReduceSplit) of D
// threads take partitions k = w, w + groups, ... (eight per round, all of a round's loads in flight),
// each keeping a running (M, num, den); the groups are then combined in fixed order, so the result is
// deterministic. Many partitions get several groups; a handful get one.
constexpr int kReduceSplit = 4;
template <int D, bool kBf16>
__global__ void __launch_bounds__(kReduceSplit * D) reduce_kernel(const DecodeParams p) {
  const int h = blockIdx.x, s = blockIdx.y, d = threadIdx.x % D, w = threadIdx.x / D;
  const int groups = blockDim.x / D;
  __shared__ float sm_num[kReduceSplit][D];
  __shared__ float sm_m[kReduceSplit], sm_den[kReduceSplit];
  pdl_wait();  // the partials come from the decode grid just before this one
  pdl_launch_dependents();
  const int Hq = p.num_kv_heads * p.group;
  const int PT = p.partition_tokens;
  const int ctx_cap = min(p.context_lens[s], p.max_blocks * 16);
  const int span = min(max(ctx_cap - p.start_tokens, 0), p.num_partitions * PT);
  const int np = p.part_offset + (span + PT - 1) / PT;
  if (!p.always_partials && np <= 1) return;  // the decode kernel wrote this row
  const int64_t row0 = (static_cast<int64_t>(s) * Hq + h) * p.ws_parts;
  float M = -INFINITY, num = 0.f, den = 0.f;
  for (int k0 = w; k0 < np; k0 += 8 * groups) {
    float mk[8], lk[8], ak[8];
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int k = k0 + v * groups;
      const int64_t slot = row0 + min(k, np - 1);
      const float2 ml = *reinterpret_cast<const float2*>(p.ws_ml + slot * 2);
      mk[v] = k < np ? ml.x : -INFINITY;
      lk[v] = ml.y;
      ak[v] = p.ws_acc[slot * D + d];
    }
    float Mn = M;
#pragma unroll
    for (int v = 0; v < 8; ++v) Mn = fmaxf(Mn, mk[v]);
    if (Mn == -INFINITY) continue;
    const float a = ex2(M - Mn);
    num *= a;
    den *= a;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const float f = ex2(mk[v] - Mn);
      num = fmaf(f, ak[v], num);
      den = fmaf(f, lk[v], den);
    }
    M = Mn;
  }
  sm_num[w][d] = num;
  if (d == 0) {
    sm_m[w] = M;
    sm_den[w] = den;
  }
  __syncthreads();
  if (w != 0) return;
  float Mt = -INFINITY;
  for (int g = 0; g < groups; ++g) Mt = fmaxf(Mt, sm_m[g]);
  uint16_t bits = 0;  // no token at all (empty context): 0
  if (Mt != -INFINITY) {
    float nt = 0.f, dt = 0.f;
    for (int g = 0; g < groups; ++g) {
      const float f = ex2(sm_m[g] - Mt);  // a group without partitions has m = -inf: weight 0
      nt = fmaf(f, sm_num[g][d], nt);
      dt = fmaf(f, sm_den[g], dt);
    }
    const float o = nt / dt * p.v_scale;
    if constexpr (kBf16) {
      bits = __bfloat16_as_ushort(__float2bfloat16_rn(o));
    } else {
      bits = __half_as_ushort(__float2half_rn(o));
    }
  }
  static_cast<uint16_t*>(p.out)[s * p.o_stride_s + h * p.o_stride_h + d] = bits;
}

// Launch with programmatic stream serialisation: the kernel may begin while the previous kernel on
// the stream finishes; it waits for it in pdl_wait() before reading anything.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
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
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
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

cudaError_t launch_reduce(const DecodeConfig& c, const DecodeParams& p, cudaStream_t st) {
  const dim3 grid(p.num_kv_heads * p.group, p.num_seqs);
  const bool bf = c.q == QType::BF16;
  const unsigned groups = p.ws_parts > 8 ? kReduceSplit : 1;
  if (c.head_dim == 128)
    return bf ? launch_pdl(reduce_kernel<128, true>, grid, dim3(groups * 128), 0, st, p)
              : launch_pdl(reduce_kernel<128, false>, grid, dim3(groups * 128), 0, st, p);
  return bf ? launch_pdl(reduce_kernel<64, true>, grid, dim3(groups * 64), 0, st, p)
            : launch_pdl(reduce_kernel<64, false>, grid, dim3(groups * 64), 0, st, p);
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
