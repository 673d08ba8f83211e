// Per-page tensor-core math and launch helpers shared by the decode kernels (decode.cu: one CTA per
// (partition, KV head, sequence); decode_units.cu: one warp per partition, persistent).
#pragma once

#include <utility>

#include "internal.h"
#include "pa_device.cuh"

namespace pa {

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

  // Token held in row m of S^T (and in k-slot m of the P.V product). 16-bit pages: m itself. e4m3
  // pages: the order pi(m) = 4 (m' >> 1) + (m' & 1) + 2 (m >> 3), m' = m & 7, which puts tokens
  // 4 q .. 4 q + 3 in the k-slots (2q, 2q+1, 2q+8, 2q+9) that lane q of the P.V product covers: the
  // order a transposed byte ldmatrix delivers V in, so V needs no byte shuffles before widening.
  static __device__ __forceinline__ int tok_of_row(int m) {
    if constexpr (C::kFp8) {
      return 4 * ((m & 7) >> 1) + (m & 1) + 2 * (m >> 3);
    } else {
      return m;
    }
  }

  // S^T = K . Q^T of one 16-token page (K page at shared address kb) into sc.
  __device__ __forceinline__ void qk(uint32_t kb, float (&sc)[NT][4]) {
    const int x7 = lane & 7;
    const int a_tok = tok_of_row((((lane >> 3) & 1) << 3) | x7);  // K matrices: row half = bit 3
    const int a_co = lane >> 4;
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
  }

  // Online softmax (log2 domain) over NP consecutive pages' scores (nv[i] valid tokens each): one
  // cross-lane max, one raise of the running max and one rescale test for all of them. Returns the
  // pages' P^T fragments for the P.V products. With NP = 1 this is the per-page step.
  template <int NP>
  __device__ __forceinline__ void softmax(const float (&sc)[NP][NT][4], const int (&nv)[NP], float sl2,
                                          uint32_t (&pf)[NP][NT][2]) {
    const int r = lane >> 2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float sv[NP][4];
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const bool v_lo = tok_of_row(r) < nv[i], v_hi = tok_of_row(r + 8) < nv[i];
        sv[i][0] = v_lo ? sc[i][nt][0] * sl2 : -INFINITY;
        sv[i][1] = v_lo ? sc[i][nt][1] * sl2 : -INFINITY;
        sv[i][2] = v_hi ? sc[i][nt][2] * sl2 : -INFINITY;
        sv[i][3] = v_hi ? sc[i][nt][3] * sl2 : -INFINITY;
        if (i == 0) {
          mx0 = fmaxf(sv[0][0], sv[0][2]);
          mx1 = fmaxf(sv[0][1], sv[0][3]);
        } else {
          mx0 = fmaxf(mx0, fmaxf(sv[i][0], sv[i][2]));
          mx1 = fmaxf(mx1, fmaxf(sv[i][1], sv[i][3]));
        }
      }
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
      }
      const float mn0 = fmaxf(m[nt][0], mx0), mn1 = fmaxf(m[nt][1], mx1);
      const float al0 = ex2(m[nt][0] - mn0), al1 = ex2(m[nt][1] - mn1);
      m[nt][0] = mn0;
      m[nt][1] = mn1;
      // The denominator sums the same rounded weights the PV product uses.
      float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const uint32_t x0 = pack2<C::kMmaBf16>(ex2(sv[i][0] - mn0), ex2(sv[i][1] - mn1));
        const uint32_t x1 = pack2<C::kMmaBf16>(ex2(sv[i][2] - mn0), ex2(sv[i][3] - mn1));
        const float2 f0 = unpack2<C::kMmaBf16>(x0), f1 = unpack2<C::kMmaBf16>(x1);
        if (i == 0) {
          ls0 = f0.x + f1.x;
          ls1 = f0.y + f1.y;
        } else {
          ls0 += f0.x + f1.x;
          ls1 += f0.y + f1.y;
        }
        pf[i][nt][0] = movmatrix_trans(x0);  // (k = tok 2q, 2q+1 ; n = g = r)
        pf[i][nt][1] = movmatrix_trans(x1);  // (k = tok 2q+8, 2q+9)
      }
      l[nt][0] = l[nt][0] * al0 + ls0;
      l[nt][1] = l[nt][1] * al1 + ls1;
      if (__any_sync(kFull, al0 != 1.f || al1 != 1.f)) {  // skipped once the running max settles
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          acc[nt][mt][0] *= al0;
          acc[nt][mt][1] *= al1;
          acc[nt][mt][2] *= al0;
          acc[nt][mt][3] *= al1;
        }
      }
    }
  }

  // O^T += V^T . P^T of one page (V page at shared address vb, nv valid tokens).
  __device__ __forceinline__ void pv(uint32_t vb, int nv, const uint32_t (&pf)[NT][2]) {
    const int x7 = lane & 7;
    const int t_tok = ((lane >> 4) << 3) | x7;  // 16-bit V^T matrices: tok half = bit 4
    const int t_co = (lane >> 3) & 1;
    const int q4 = lane & 3;
    // Tokens past the context may hold any bits (NaN included): zero them in V^T so 0 * NaN
    // never reaches the accumulator. mlo covers k-slots 2q, 2q+1, mhi k-slots 2q+8, 2q+9.
    uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
    if (nv < 16) {
      const int t0 = tok_of_row(2 * q4), t8 = tok_of_row(2 * q4 + 8);
      mlo = (t0 < nv ? 0x0000ffffu : 0u) | (t0 + 1 < nv ? 0xffff0000u : 0u);
      mhi = (t8 < nv ? 0x0000ffffu : 0u) | (t8 + 1 < nv ? 0xffff0000u : 0u);
    }
    if constexpr (C::kFp8) {
      // Lanes 0-15 address token rows of chunk 2 mp, lanes 16-31 those of chunk 2 mp + 1 (16 d each);
      // each lane gets tokens 4 q .. 4 q + 3 of d = r and r + 8 of both chunks: k-slots (2q, 2q+1)
      // and (2q+8, 2q+9) of m-tiles 2 mp and 2 mp + 1 after widening.
#pragma unroll
      for (int mp = 0; mp < KS / 2; ++mp) {
        uint32_t raw[4];
        ldmatrix_b8_x2_trans(raw, vb + swz(lane & 15, 2 * mp + (lane >> 4)));
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t a[4];
          e4m3x4_to_f16x2x2(raw[2 * half], a[0], a[2]);
          e4m3x4_to_f16x2x2(raw[2 * half + 1], a[1], a[3]);
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

  // One 16-token page; kb/vb are the shared addresses of its K and V pages; nv valid tokens.
  __device__ __forceinline__ void page(uint32_t kb, uint32_t vb, int nv, float sl2) {
    float sc[1][NT][4];
    qk(kb, sc[0]);
    uint32_t pf[1][NT][2];
    const int nvs[1] = {nv};
    softmax<1>(sc, nvs, sl2, pf);
    pv(vb, nv, pf[0]);
  }

  // Two consecutive pages of one partition (A before B in token order) as one softmax step.
  __device__ __forceinline__ void page2(uint32_t kba, uint32_t vba, int nva, uint32_t kbb, uint32_t vbb, int nvb,
                                        float sl2) {
    float sc[2][NT][4];
    qk(kba, sc[0]);
    qk(kbb, sc[1]);
    uint32_t pf[2][NT][2];
    const int nvs[2] = {nva, nvb};
    softmax<2>(sc, nvs, sl2, pf);
    pv(vba, nva, pf[0]);
    pv(vbb, nvb, pf[1]);
  }

  // Zero the running state (a new partition, same query).
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int mt = 0; mt < KS; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][mt][i] = 0.f;
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
    }
  }

  // This warp's state written straight to global memory for query heads hk * G + g, g < G: with
  // `direct`, the normalised output (acc / l * v_scale, rounded to nearest even; 0 when l is 0)
  // into out; otherwise the partial (acc, m, l) into workspace slot `part` of each head's row, stored
  // with L2 policy `keep` (the merge kernel reads it back right after).
  template <bool kOutBf16>
  __device__ __forceinline__ void write_global(const DecodeParams& p, int s, int hk, int part, bool direct,
                                               uint64_t keep) {
    const int r = lane >> 2, q4 = lane & 3;
    const int G = p.group, Hq = p.num_kv_heads * G;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float lv = l[nt][j];
        lv += __shfl_xor_sync(kFull, lv, 4);
        lv += __shfl_xor_sync(kFull, lv, 8);
        lv += __shfl_xor_sync(kFull, lv, 16);
        const int g = nt * 8 + 2 * q4 + j;
        if (g >= G) continue;
        const int h = hk * G + g;
        if (direct) {
          const float inv = lv > 0.f ? p.v_scale / lv : 0.f;
          uint16_t* o = static_cast<uint16_t*>(p.out) + s * p.o_stride_s + h * p.o_stride_h;
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            const float lo = acc[nt][mt][j] * inv, hi = acc[nt][mt][j + 2] * inv;
            const uint32_t w = pack2<kOutBf16>(lo, hi);  // d = 16 mt + r and 16 mt + r + 8
            o[16 * mt + r] = static_cast<uint16_t>(w & 0xffffu);
            o[16 * mt + r + 8] = static_cast<uint16_t>(w >> 16);
          }
        } else {
          const int64_t row = (static_cast<int64_t>(s) * Hq + h) * p.ws_parts + p.part_offset + part;
          float* a = p.ws_acc + row * D;
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            st_global_hint(a + 16 * mt + r, acc[nt][mt][j], keep);
            st_global_hint(a + 16 * mt + r + 8, acc[nt][mt][j + 2], keep);
          }
          if (r == 0) st_global_hint(p.ws_ml + row * 2, make_float2(m[nt][j], lv), keep);
        }
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
        const int d_lo = 16 * mt + r, d_hi = d_lo + 8;
        const int g = nt * 8 + 2 * q4;
        ag[g * D + d_lo] = acc[nt][mt][0];
        ag[(g + 1) * D + d_lo] = acc[nt][mt][1];
        ag[g * D + d_hi] = acc[nt][mt][2];
        ag[(g + 1) * D + d_hi] = acc[nt][mt][3];
      }
    }
  }
};

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

}  // namespace pa
