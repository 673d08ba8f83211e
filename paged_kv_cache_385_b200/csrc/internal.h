// Internal launch interface between the C-ABI layer (api.cu) and the kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pa {

enum class KvType : int { F16 = 0, BF16 = 1, E4M3 = 2 };
enum class QType : int { F16 = 0, BF16 = 1 };

// Kernel-side view of one pa_decode call. Strides are in elements.
struct DecodeParams {
  void* out;
  const void* q;
  int64_t q_stride_s, q_stride_h;
  int64_t o_stride_s, o_stride_h;
  const int32_t* block_tables;
  int64_t bt_stride;
  const int32_t* context_lens;
  int32_t num_seqs;
  int32_t num_blocks;
  int32_t num_kv_heads;
  int32_t group;             // query heads per KV head
  int32_t max_blocks;        // block-table width
  int32_t partition_tokens;  // tokens per partition (multiple of 16)
  int32_t num_partitions;    // grid.x; 1 = no split (decode writes out directly)
  float score_scale_log2;    // scale * log2(e) * k_scale (e4m3) -- folded into the scores
  float v_scale;             // applied once to the normalised output (e4m3), 1 otherwise
  float* ws_acc;             // [B, Hq, P, D] un-normalised partial outputs (split only)
  float* ws_ml;              // [B, Hq, P, 2] partial (running max in log2 units, sum) (split only)
  uint32_t* err;             // error word (never null)
  // Cascade (shared-prefix) decode: this grid covers tokens [start_tokens, ctx) of each sequence and
  // always writes partials, at workspace slots part_offset + partition of rows ws_parts slots long.
  // Plain decode: start_tokens 0, part_offset 0, ws_parts = num_partitions, always_partials 0.
  int32_t start_tokens;
  int32_t part_offset;
  int32_t ws_parts;
  int32_t always_partials;
  // Cascade with an unsplit suffix: the decode CTA merges the prefix partials (slots [0, part_offset))
  // with its own result and writes the output; no merge kernel runs.
  int32_t merge_prefix_inline;
  // Cascade: the kernel before this grid on the stream is the prefix kernel, which lets it launch
  // only after its own wait on the kernel before that, so pages, q and tables are already final when
  // this grid starts. It therefore waits for the prefix grid (griddepcontrol.wait) only before it
  // reads the prefix partials and before every exit, and its page loop overlaps the prefix kernel.
  int32_t late_dependency_wait;
  // Fused new-token write (pa_decode_step); new_k == nullptr for plain pa_decode.
  const void* new_k;         // [B, Hkv, D] f16/bf16
  const void* new_v;
  int64_t nk_stride_s, nk_stride_h, nv_stride_s, nv_stride_h;
  const int64_t* new_slots;  // [B] slot of position ctx - 1, or -1
  void* k_cache;
  void* v_cache;
  int32_t new_src_bf16;
  float k_inv_scale, v_inv_scale;  // e4m3 caches
};

struct DecodeConfig {
  KvType kv;
  QType q;
  int head_dim;  // 64 or 128
  int ntiles;    // ceil(group / 8): 1 or 2
  int kernel;    // 0 = CUDA-core FMA, 1 = tensor-core mma.sync
};

// Number of warps per CTA of the decode kernels; a partition holds at most 32 pages per warp.
constexpr int kDecodeWarps = 4;
constexpr int kMaxPartitionTokens = 16 * 32 * kDecodeWarps;

cudaError_t launch_decode(const DecodeConfig& cfg, const CUtensorMap& k_map, const CUtensorMap& v_map,
                          const DecodeParams& p, cudaStream_t stream);
// Split decode with one persistent warp per partition (decode_units.cu): tensor-core kernel,
// partitions of at most kUnitMaxPartitionTokens tokens (one page per lane), at most kUnitMaxSeqs
// sequences (their unit counts live in shared memory), plain decode or pa_decode_step (not the
// cascade suffix). Followed by launch_reduce like the per-partition CTAs.
constexpr int kUnitMaxSeqs = 512;
constexpr int kUnitMaxPartitionTokens = 512;
bool decode_units_supported(const DecodeConfig& cfg, const DecodeParams& p);
cudaError_t launch_decode_units(const DecodeConfig& cfg, const CUtensorMap& k_map, const CUtensorMap& v_map,
                                const DecodeParams& p, cudaStream_t stream);
cudaError_t launch_reduce(const DecodeConfig& cfg, const DecodeParams& p, cudaStream_t stream);
bool decode_supported(const DecodeConfig& cfg);

struct CacheParams {
  const void* key;
  const void* value;
  int64_t k_stride_t, k_stride_h;
  int64_t v_stride_t, v_stride_h;
  const int64_t* slots;
  void* k_cache;
  void* v_cache;
  int64_t num_tokens;
  int32_t num_kv_heads;
  int32_t head_dim;
  int64_t num_slots;  // num_blocks * 16
  float k_inv_scale, v_inv_scale;
  uint32_t* err;
};

// src: 0 = f16, 1 = bf16 source; cache: KvType.
cudaError_t launch_reshape_and_cache(int src_bf16, KvType cache, const CacheParams& p, cudaStream_t stream);

// Multi-query attention (multiquery.cu). Shared prefix: query rows (sequence, query head) of every
// sequence against the first prefix_tokens tokens, which every block-table row maps to the same
// blocks -> partials. Chunked prefill: rows (new token, query head) of each sequence, causal over
// its pages -> out.
struct MqParams {
  const void* q;
  int64_t q_stride_s, q_stride_h;  // prefix: per sequence; prefill: per token row of q
  const int32_t* block_tables;
  int64_t bt_stride;
  const int32_t* context_lens;
  int32_t num_seqs, num_blocks, num_kv_heads, group, max_blocks;
  int32_t prefix_tokens;  // prefix: multiple of 16
  int32_t chunk_tokens;   // prefix: tokens per CTA (multiple of 16)
  int32_t num_chunks;
  float score_scale_log2;
  float* ws_acc;  // prefix partials
  float* ws_ml;
  int32_t ws_parts;
  const int32_t* query_start;  // prefill: [B + 1] rows of q per sequence
  void* out;                   // prefill: [T, Hq, D]
  int64_t o_stride_t, o_stride_h;
  uint32_t* err;
  int32_t row_tiles, num_items;  // tcgen05 kernels: 128-row tiles per sequence (or per prefix chunk), work items
};
constexpr int kPrefixChunkTokens = 256;
cudaError_t launch_prefix(KvType kv, int head_dim, const CUtensorMap& k_map, const CUtensorMap& v_map,
                          const MqParams& p, cudaStream_t stream);
cudaError_t launch_prefill(KvType kv, int head_dim, const CUtensorMap& k_map, const CUtensorMap& v_map,
                           const MqParams& p, int max_query_len, cudaStream_t stream);
// tcgen05 prefill (prefill_tc.cu): q_map is a 3-D map over q [T, Hq, D] with box {64, G, 128 / G},
// o_map the same over out (full 128-row tiles leave through it as tensor stores).
bool prefill_tc_supported(int head_dim, int group);
cudaError_t launch_prefill_tc(KvType kv, const CUtensorMap& q_map, const CUtensorMap& k_map, const CUtensorMap& v_map,
                              const CUtensorMap& o_map, const MqParams& p, int max_query_len, cudaStream_t stream);
// The same kernel in shared-prefix mode: q_map over q [B, Hq, D], partials to ws slots 0 .. num_chunks-1;
// ws_map is a 4-D map over ws_acc {D, P, Hq, B} (float32) with box {32, 1, G, 128 / G}, 128-byte swizzle.
cudaError_t launch_prefix_tc(KvType kv, const CUtensorMap& q_map, const CUtensorMap& k_map, const CUtensorMap& v_map,
                             const CUtensorMap& ws_map, const MqParams& p, cudaStream_t stream);

struct CopyParams {
  void* k_cache;
  void* v_cache;
  const int64_t* mapping;  // [N, 2] (src, dst) block ids
  int64_t num_pairs;
  int64_t block_bytes;     // bytes of one block of one cache (Hkv * 16 * D * elem)
  int64_t num_blocks;
  uint32_t* err;
};
cudaError_t launch_copy_blocks(const CopyParams& p, cudaStream_t stream);

uint32_t* decode_error_word();  // device address of the library's own error word

// Record the reason pa_last_error() reports for this thread; returns status.
int set_last_error(int status, const char* fmt, ...);
cudaError_t read_and_clear_error_word(uint32_t* bits, int clear);

}  // namespace pa
