/*
 * pa.h -- C ABI of the B200 paged-KV-cache decode library (libpagedattn.so).
 *
 * What it computes. vLLM's PagedAttention keeps each sequence's KV cache in
 * fixed 16-token blocks scattered through one physical pool; a per-sequence
 * block table maps logical block (position // block_size) to physical block,
 * and a Block Manager hands blocks out and takes them back in O(1) with a free
 * list (vLLM notes page, "PagedAttention": Block Manager and Cache Engine;
 * "vLLM 前世今生" section 3.2: 16-token blocks, non-contiguous physical blocks,
 * block table, blocks shared by several sequences). This library provides the
 * decode-step hot path of that design on one GPU:
 *   - pa_reshape_and_cache: scatter each new token's K and V into its slot
 *     (the Cache Engine's write side);
 *   - pa_decode: one query token per sequence attends over its whole paged
 *     context, out = softmax(scale * q K^T) V, reading K/V through the block
 *     table (the PagedAttention kernel);
 *   - a host-side free-list block allocator with reference counts, used to
 *     build block tables and to share prefix blocks between sequences.
 *
 * Conventions (all calls).
 *   - Device tensors are caller-owned (PyTorch or any allocator); the library
 *     never allocates, frees or synchronises on pa_reshape_and_cache/pa_decode.
 *     Work is enqueued on the caller's stream (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream). Calls return after enqueueing.
 *   - Host-side validation (shapes, dtypes, strides, alignment, options, the
 *     workspace size) runs before any CUDA call and returns a negative
 *     pa_status without touching device memory; pa_last_error() then gives a
 *     one-line reason (thread-local). A failed CUDA call or launch returns
 *     PA_ERR_CUDA.
 *   - Conditions only the device can see (a block id or slot outside the pool,
 *     a context longer than max_context_len, a pipeline wait that timed out)
 *     never fault: the offending page or token is skipped and a bit is OR-ed
 *     into an error word (PA_DEVERR_*), the caller's if given, else the
 *     library's own, read with pa_read_device_error().
 *   - Block size is fixed at 16 tokens.
 *
 * Pool layout. Each cache (K and V separately) is a contiguous tensor
 * [num_blocks, num_kv_heads, 16, head_dim]: one (block, head) page is one
 * contiguous run of 16 * head_dim elements. Slot s of the pool is token row
 * s % 16 of physical block s / 16.
 */
#ifndef PAGED_KV_CACHE_PA_H
#define PAGED_KV_CACHE_PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_BLOCK_SIZE 16

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = -1, /* shape, dtype, stride, alignment or value outside the contract  */
  PA_ERR_UNSUPPORTED = -2, /* valid but not built: head_dim, group size or dtype combination  */
  PA_ERR_WORKSPACE = -3,   /* split partitions need a workspace that was missing or too small */
  PA_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed                            */
  PA_ERR_EXHAUSTED = -5,   /* allocator: no free block                                        */
  PA_ERR_BAD_BLOCK = -6    /* allocator: block id out of range, or not allocated              */
} pa_status;

/* Element types of pa_tensor.dtype. PA_E4M3 is OCP FP8 E4M3 ("fn": no infinities, max 448). */
typedef enum pa_dtype { PA_F16 = 0, PA_BF16 = 1, PA_E4M3 = 2, PA_I32 = 3, PA_I64 = 4, PA_F32 = 5 } pa_dtype;

/* Device-side error bits (OR-ed into the error word). */
#define PA_DEVERR_BAD_BLOCK 1u   /* a block-table entry read for a valid position is outside [0, num_blocks) */
#define PA_DEVERR_BAD_SLOT 2u    /* a slot_mapping entry is < -1 or >= num_blocks * 16                       */
#define PA_DEVERR_TIMEOUT 4u     /* a wait for an asynchronous page copy exceeded its bound                  */
#define PA_DEVERR_CTX_RANGE 8u   /* context_lens[s] > max_context_len (or > 16 * block-table width)          */
#define PA_DEVERR_PREFIX 16u     /* pa_decode_cascade: a block table does not share the prefix blocks        */

/* A strided view of caller-owned memory. Strides are in elements, not bytes.
 * Only the first ndim entries of shape/stride are read. The pointer is a
 * device pointer for pa_reshape_and_cache/pa_decode. */
typedef struct pa_tensor {
  void* data;
  int32_t dtype; /* pa_dtype */
  int32_t ndim;
  int64_t shape[4];
  int64_t stride[4];
} pa_tensor;

/* Optional knobs of pa_decode. Pass NULL for all defaults; a zeroed struct is
 * NOT the default (scales would be 0): call pa_decode_opts_init first. */
typedef struct pa_decode_opts {
  float k_scale;            /* e4m3 caches: stored code * k_scale is the key value; 1 otherwise      */
  float v_scale;            /* same for values                                                          */
  int32_t max_context_len;  /* host-known bound on context_lens (sizes the grid without a device read);
                               0 = 16 * block_tables.shape[1]                                           */
  int32_t partition_tokens; /* split each context into partitions of this many tokens (multiple of 16,
                               <= 2048), merged by a second kernel; 0 = library's choice
                               (pa_decode_partition_tokens)                                            */
  void* workspace;          /* device scratch for split partitions, >= pa_decode_workspace_bytes, 256-B
                               aligned; may be NULL when no split happens                               */
  size_t workspace_bytes;
  int32_t kernel;           /* -1 = choose (1); 0 = CUDA-core FMA kernel; 1 = tensor-core (mma) kernel,
                               whose split form (partitions of <= 512 tokens, <= 512 sequences, not
                               the cascade suffix) runs one persistent warp per partition; 2 = the
                               tensor-core kernel with one CTA per partition always                    */
  int32_t* error_word;      /* device int32 that receives PA_DEVERR_* bits; NULL = library's own word  */
  int32_t prefix_kernel;    /* pa_decode_cascade's shared-prefix kernel: -1 = choose (tcgen05 when
                               head_dim is 128, the group divides 128 and q rows are 16-B aligned);
                               0 = warp-level mma kernel; 1 = tcgen05 kernel (PA_ERR_UNSUPPORTED
                               when those conditions fail)                                             */
} pa_decode_opts;

/* Fill opts with the defaults (scales 1, everything else automatic). */
void pa_decode_opts_init(pa_decode_opts* opts);

/*
 * pa_reshape_and_cache -- write new tokens' K and V into the paged pool.
 *   key, value    [T, Hkv, D] device, dtype F16 or BF16, last stride 1, 16-B aligned rows.
 *   slot_mapping  [T] device I64: slot of token t, or -1 to skip it.
 *   k_cache, v_cache  [num_blocks, Hkv, 16, D] contiguous, same dtype as key (16-bit caches: the
 *                 bits are copied unchanged) or E4M3 (code = e4m3_rn_satfinite(float32(x) *
 *                 float32(1 / scale)), 1/scale formed once in float32 on the host).
 *   k_scale, v_scale  dequantisation scales of an E4M3 cache (> 0, finite); ignored otherwise.
 *   Slots outside [-1, num_blocks * 16) are skipped and set PA_DEVERR_BAD_SLOT in the library's
 *   error word. Untouched slots keep their bytes. Two tokens with the same slot race.
 *   Limits (else PA_ERR_UNSUPPORTED / PA_ERR_INVALID_ARG): D a multiple of 8, T < 2^31, the pool's
 *   size in bytes below 2^63.
 * Source: vLLM notes page, "PagedAttention / Cache Engine" (the engine writes a position's data
 * into its page). T == 0 is a no-op.
 */
int pa_reshape_and_cache(const pa_tensor* key, const pa_tensor* value, const pa_tensor* slot_mapping,
                         pa_tensor* k_cache, pa_tensor* v_cache, float k_scale, float v_scale, void* stream);

/*
 * pa_decode -- one decode step of paged attention.
 *   out           [B, Hq, D] device, same dtype as q, last stride 1, 16-B aligned rows.
 *   q             [B, Hq, D] device F16 or BF16 (F16 with an F16 cache, BF16 with a BF16 cache,
 *                 either with an E4M3 cache; with E4M3 q must lie within the f16 range).
 *   k_cache, v_cache  [num_blocks, Hkv, 16, D] contiguous, dtype F16, BF16 or E4M3 (both the same).
 *   block_tables  [B, max_blocks] device I32 (last stride 1): physical block of logical block j of
 *                 sequence s. Entries at j >= ceil(context_lens[s] / 16) are never read.
 *   context_lens  [B] device I32: tokens of sequence s (already including the token written this
 *                 step by pa_reshape_and_cache). 0 gives an all-zero output row.
 *   scale         multiplies q.k before the softmax (typically 1/sqrt(D)).
 *   num_kv_heads  Hkv; must equal k_cache.shape[1] and divide Hq. Query head h reads KV head
 *                 h / (Hq / Hkv). Supported: D in {64, 128} (E4M3: 128), Hq / Hkv <= 16,
 *                 B and Hkv <= 65535, num_blocks * Hkv * 16 < 2^31 pool rows (else
 *                 PA_ERR_UNSUPPORTED). Block-table columns past 2^31 / 16 are never read.
 * out[s, h, :] = sum_t softmax_t(scale * q[s, h] . K[s, t]) V[s, t], K[s, t] being row t % 16 of
 * page (block_tables[s][t / 16], h / G); accumulation in float32, result rounded to nearest even.
 * The result depends only on logical positions, never on which physical blocks hold them.
 * Source: vLLM notes page, "PagedAttention" (page of a position = position // block_size) and
 * "内核优化" (kernels section: the PagedAttention kernel, GQA and MQA kernels); "vLLM 前世今生"
 * section 3.2.
 */
int pa_decode(pa_tensor* out, const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
              const pa_tensor* block_tables, const pa_tensor* context_lens, float scale, int32_t num_kv_heads,
              const pa_decode_opts* opts, void* stream);

/*
 * pa_decode_step -- pa_reshape_and_cache of one new token per sequence followed by pa_decode, in one
 * launch: the CTA that reads a sequence's last page writes the new token's K/V row (for its KV head)
 * into the slot first, then decodes. Same results, pool bytes and errors as the two calls in order.
 *   key, value    [B, Hkv, D] device F16/BF16 (last stride 1, 16-B aligned rows): the token at position
 *                 context_lens[s] - 1 of sequence s.
 *   slot_mapping  [B] device I64: its slot, which must lie in the page that block_tables[s] maps
 *                 position context_lens[s] - 1 to (the normal decode step), or -1 to skip.
 *   Other arguments as pa_decode; opts->k_scale/v_scale also quantise the e4m3 write.
 * Source: vLLM notes page, "PagedAttention / Cache Engine" (write a position's page) and "内核优化";
 * fusing the two calls is this library's choice.
 */
int pa_decode_step(pa_tensor* out, const pa_tensor* q, const pa_tensor* key, const pa_tensor* value,
                   const pa_tensor* slot_mapping, pa_tensor* k_cache, pa_tensor* v_cache,
                   const pa_tensor* block_tables, const pa_tensor* context_lens, float scale, int32_t num_kv_heads,
                   const pa_decode_opts* opts, void* stream);

/*
 * pa_copy_blocks -- copy whole physical blocks (every KV head, K and V caches) for copy-on-write.
 *   k_cache, v_cache  [num_blocks, Hkv, 16, D] contiguous, same dtype and shape.
 *   block_mapping     [N, 2] device I64: (src, dst) block ids. Destinations must be distinct and not
 *                     also sources in the same call (pairs run concurrently). src == dst is a no-op;
 *                     an id outside [0, num_blocks) skips the pair and sets PA_DEVERR_BAD_BLOCK.
 * Source: "vLLM 前世今生" section 3.2 (several sequences point at one physical block; copy-on-write
 * on write). Use with pa_block_cow. N == 0 is a no-op.
 */
int pa_copy_blocks(pa_tensor* k_cache, pa_tensor* v_cache, const pa_tensor* block_mapping, void* stream);

/*
 * pa_decode_cascade -- pa_decode for a batch whose sequences all share their first
 * shared_prefix_tokens tokens in the same physical blocks (block_tables[s][j] == block_tables[0][j]
 * for j < shared_prefix_tokens / 16): the shared pages are read once per KV head for all B * G query
 * rows (a dense tensor-core contraction), each sequence's remaining tokens by the decode kernel, and
 * the two softmax partials are merged. Same result as pa_decode up to float32 rounding order.
 *   shared_prefix_tokens  > 0, multiple of 16, <= 16 * block_tables.shape[1]. Sequences shorter than
 *                 the prefix are fine (their rows stop at their context).
 *   key, value, slot_mapping  all NULL, or as in pa_decode_step (the new token is written in the same
 *                 call); a new token must lie past the shared prefix (the prefix blocks are shared
 *                 and read-only here: copy-on-write them first), else it is skipped with
 *                 PA_DEVERR_BAD_SLOT.
 *   F16/BF16 caches only. A workspace is always needed: pa_decode_cascade_workspace_bytes.
 *   opts->prefix_kernel picks the kernel of the shared part (tcgen05 by default where it applies).
 *   A block table that does not share the prefix blocks sets PA_DEVERR_PREFIX (results undefined;
 *   every row's first shared_prefix_tokens / 16 entries are compared with row 0's).
 * Source: "vLLM 前世今生" section 3.2 (sequences pointing at the same physical blocks; prefix
 * sharing) and the notes page's prefix-caching section (a shared prompt prefix computed once).
 */
int pa_decode_cascade(pa_tensor* out, const pa_tensor* q, const pa_tensor* key, const pa_tensor* value,
                      const pa_tensor* slot_mapping, pa_tensor* k_cache, pa_tensor* v_cache,
                      const pa_tensor* block_tables, const pa_tensor* context_lens, int32_t shared_prefix_tokens,
                      float scale, int32_t num_kv_heads, const pa_decode_opts* opts, void* stream);

/* Workspace bytes pa_decode_cascade needs (partition_tokens 0 = the library's choice); SIZE_MAX when
 * the size does not fit in 64 bits. Host only. */
size_t pa_decode_cascade_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                         int32_t head_dim, int32_t max_context_len, int32_t shared_prefix_tokens,
                                         int32_t partition_tokens);

/*
 * pa_prefill -- causal attention of a chunk of new tokens per sequence over its paged context
 * (prompt prefill, or one chunk of a chunked prefill).
 *   out, q        [T, Hq, D] device F16/BF16 (the caches' dtype), last stride 1, 16-B aligned rows. Rows
 *                 query_start[s] .. query_start[s + 1] - 1 belong to sequence s: its last
 *                 n_s = query_start[s + 1] - query_start[s] tokens.
 *   k_cache, v_cache  [num_blocks, Hkv, 16, D] F16/BF16, holding every token of the context already
 *                 (write the chunk's K/V with pa_reshape_and_cache first).
 *   block_tables  [B, max_blocks] I32; query_start [B + 1] I32; context_lens [B] I32: tokens of
 *                 sequence s including the chunk (n_s <= context_lens[s] <= 16 * max_blocks).
 *   max_query_len host-known bound on n_s (sizes the grid without a device read).
 *   kernel        -1 = choose (tcgen05 when D = 128 and Hq / Hkv <= 16 divides 128), 0 = warp-level mma.sync
 *                 tiles, 1 = tcgen05 (5th-generation tensor cores, accumulators in tensor memory).
 * Row i of sequence s is position p = context_lens[s] - n_s + i and sees positions 0 .. p:
 * out = softmax(scale * q K[0..p]^T) V[0..p], float32 accumulation, rounded to nearest even.
 * Violations only the device can see (n_s > context_lens[s], n_s > max_query_len) set
 * PA_DEVERR_CTX_RANGE. D in {64, 128}.
 * Source: the notes page's kernels section (FlashAttention adapted to paged KV) and "vLLM 前世今生"
 * section 5.4 (chunked prefill).
 */
int pa_prefill(pa_tensor* out, const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
               const pa_tensor* block_tables, const pa_tensor* query_start, const pa_tensor* context_lens,
               int32_t max_query_len, float scale, int32_t num_kv_heads, int32_t kernel, void* stream);

/* Partition size pa_decode uses when opts->partition_tokens == 0 and a workspace is given
 * (0 = no split: the batch's B * Hkv (sequence, KV head) units already fill the GPU, B * Hkv >= 592,
 * and every context fits one CTA, <= 2048 tokens). Otherwise the largest of 2048, 1024 and 512
 * shorter than max_context_len that still gives about four CTAs per SM,
 * B * Hkv * ceil(max_context_len / size) >= 592; else 256, or 0 when max_context_len <= 256.
 * Host only. */
int32_t pa_decode_partition_tokens(int32_t num_seqs, int32_t num_kv_heads, int32_t max_context_len);

/* Workspace bytes pa_decode needs for these sizes (0 when no split happens; SIZE_MAX when the size
 * does not fit in 64 bits). partition_tokens 0 applies pa_decode_partition_tokens. Host only. */
size_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t max_context_len, int32_t partition_tokens);

/*
 * pa_decode_no_alloc -- pa_decode for callers that cannot allocate device memory.
 * (The vLLM pages have no counterpart to this call; it is a property of this library's interface.)
 * pa_decode needs a caller-provided workspace whenever it splits contexts into partitions. Some
 * callers cannot get one: a plugin whose host framework owns all device memory and passes it only
 * inputs and outputs, a process whose device-memory budget is fixed at start-up, or a serving loop
 * that cannot afford a cudaMalloc (which may synchronise the whole device) inside a step. This call
 * is pa_decode with the scratch taken from a static array of PA_NO_ALLOC_SCRATCH_BYTES that the
 * library keeps in device memory; it allocates nothing and takes no workspace (opts->workspace must
 * be NULL and workspace_bytes 0, else PA_ERR_INVALID_ARG). All other arguments, results and errors
 * are those of pa_decode.
 *   - A batch whose split needs more than PA_NO_ALLOC_SCRATCH_BYTES (see pa_decode_workspace_bytes)
 *     is rejected with PA_ERR_WORKSPACE before any CUDA call, like every other argument error;
 *     larger partition_tokens needs less.
 *   - The first call on a device that splits a context looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current), after its argument checks, and caches it;
 *     make such a call before any stream capture. The cached address (like that of the library's
 *     own error word) belongs to the device's context as it was then: a cudaDeviceReset of that
 *     device after the first call is not supported in the same process.
 *   - The array takes PA_NO_ALLOC_SCRATCH_BYTES (32 MiB) on every device where the library's device
 *     code is loaded (depending on CUDA's module-loading mode, at start-up or at the latest on the
 *     first call), until the process exits.
 *   - All calls on a device share the array and it keeps the last call's contents (nothing in it
 *     needs to start at zero). Calls whose kernels overlap on the GPU, e.g. on two unordered
 *     streams, race on it: order them on one stream.
 */
#define PA_NO_ALLOC_SCRATCH_BYTES ((size_t)32 << 20)
int pa_decode_no_alloc(pa_tensor* out, const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
                       const pa_tensor* block_tables, const pa_tensor* context_lens, float scale,
                       int32_t num_kv_heads, const pa_decode_opts* opts, void* stream);

/* Static string for a pa_status value. */
const char* pa_status_string(int status);

/* Reason for the last non-OK return on this thread ("" if none). */
const char* pa_last_error(void);

/* Synchronise the current device, copy the library's own device error word (PA_DEVERR_* bits)
 * into *bits and, if clear != 0, reset it to 0. Not for hot paths. */
int pa_read_device_error(uint32_t* bits, int clear);

/* Host-side fault injection for testing a caller's error handling: the next `count` calls of
 * pa_reshape_and_cache, pa_decode, pa_decode_step, pa_decode_cascade, pa_decode_no_alloc,
 * pa_prefill and pa_copy_blocks that reach their first device call (every argument check passed
 * and there is work to enqueue) return PA_ERR_CUDA without any device work, as a call whose launch failed does (nothing is enqueued, pa_last_error says it was
 * injected). count 0 disarms. Process-wide; thread-safe. Nothing reaches the GPU: no device-side
 * fault is ever made. Returns PA_OK, or PA_ERR_INVALID_ARG for count < 0. */
int pa_debug_fail_next_launches(int32_t count);

/* Library version, "major.minor.patch". */
const char* pa_version(void);

/* Self-test of the bounded waits every kernel uses on its asynchronous-copy and MMA barriers (no
 * counterpart on the pages): launches one CTA on `stream` that waits on a barrier nothing ever
 * arrives on, gives up after timeout_us microseconds (1 .. 1000000) of global time, and ORs
 * PA_DEVERR_TIMEOUT into error_word (a device int32; NULL = the library's own word, read with
 * pa_read_device_error). The kernel then returns normally: no fault, no hang, the context stays
 * usable. Returns PA_ERR_INVALID_ARG for a timeout out of range, PA_ERR_CUDA if the launch fails. */
int pa_selftest_bounded_wait(int32_t timeout_us, int32_t* error_word, void* stream);

/* ---------------------------------------------------------------------------------------------
 * Host block allocator: free list of physical block ids with reference counts.
 * Source: vLLM notes page, "PagedAttention / Block Manager" (O(1) allocation and release with a
 * free list); "vLLM 前世今生" section 3.2 (blocks allocated on demand, freed when a sequence
 * finishes, several sequences may point at one physical block).
 * alloc pops the top of a stack of free ids; the release of a block's last reference pushes it
 * back on top. Every call is O(1) (the _n variants O(n)). Not thread-safe: one allocator per
 * thread, or external locking. No GPU involved.
 * ------------------------------------------------------------------------------------------- */
typedef struct pa_allocator pa_allocator;

/* New allocator over block ids [0, num_blocks). initial_order (nullable, a permutation of
 * [0, num_blocks)) is the order the first allocations come out in; NULL means 0, 1, 2, ...
 * Returns NULL on a bad argument (pa_last_error says why) or out of host memory. */
pa_allocator* pa_allocator_create(int32_t num_blocks, const int32_t* initial_order);
void pa_allocator_destroy(pa_allocator* a);

/* A free block id with refcount 1, or PA_ERR_EXHAUSTED. */
int32_t pa_block_alloc(pa_allocator* a);
/* Add a reference to an allocated block (share it). PA_ERR_BAD_BLOCK if not allocated. */
int pa_block_incref(pa_allocator* a, int32_t block);
/* Drop a reference; at 0 the block returns to the free list. PA_ERR_BAD_BLOCK if not allocated. */
int pa_block_free(pa_allocator* a, int32_t block);
/* Copy-on-write before writing into `block`: with one reference, *out_block = block and 0 is
 * returned (write in place). Shared, a fresh block is allocated, the caller's reference moves to it
 * (block's count drops by one, the new block's is 1), *out_block = the new id and 1 is returned: copy
 * the page with pa_copy_blocks before writing. PA_ERR_EXHAUSTED (nothing changed) if no block is
 * free; PA_ERR_BAD_BLOCK if `block` is not allocated. Source: "vLLM 前世今生" section 3.2. */
int pa_block_cow(pa_allocator* a, int32_t block, int32_t* out_block);
/* Reference count of a block (0 = free), or PA_ERR_BAD_BLOCK for an id outside the pool. */
int32_t pa_block_refcount(const pa_allocator* a, int32_t block);
int32_t pa_allocator_num_free(const pa_allocator* a);
int32_t pa_allocator_num_blocks(const pa_allocator* a);

/* Allocate n blocks into out[0..n) all-or-nothing: PA_ERR_EXHAUSTED (nothing taken) if fewer
 * than n are free. */
int pa_blocks_alloc_n(pa_allocator* a, int32_t n, int32_t* out);
/* incref / free each of blocks[0..n) (an id may repeat: it is counted once per listing),
 * all-or-nothing: if any id is not allocated, would be freed more often than it is referenced
 * (PA_ERR_BAD_BLOCK) or would overflow its count (PA_ERR_INVALID_ARG), nothing changes. */
int pa_blocks_incref_n(pa_allocator* a, int32_t n, const int32_t* blocks);
int pa_blocks_free_n(pa_allocator* a, int32_t n, const int32_t* blocks);

/* Block tables of a batch, built with the allocator: out is host I32 [num_seqs, max_blocks] (row
 * stride max_blocks), entries past ceil(context_lens[s] / 16) set to -1. Sequences are served in
 * order and each logical block in order: logical block j of sequence s gets a block popped from the
 * free list, except that the first shared_prefix_tokens / 16 logical blocks are shared by every
 * sequence reaching them: each is allocated by the first sequence that reaches it, and every later
 * one takes a reference to it (a sequence shorter than the prefix shares only the blocks it covers).
 *   context_lens  host I32 [num_seqs], >= 0; shared_prefix_tokens a multiple of 16 (0 = none).
 * All-or-nothing: PA_ERR_EXHAUSTED (nothing allocated, out untouched) if the free list holds fewer
 * blocks than the tables need; PA_ERR_INVALID_ARG (nothing changed) for a negative length, a
 * sequence needing more than max_blocks blocks, or a bad prefix length.
 * Source: vLLM notes page, "PagedAttention / Block Manager" (blocks handed out from a free list as
 * a request needs them) and "vLLM 前世今生" section 3.2 (non-contiguous physical blocks mapped by a
 * block table; sequences sharing a prompt prefix point at the same physical blocks). */
int pa_build_block_tables(pa_allocator* a, const int32_t* context_lens, int32_t num_seqs, int32_t max_blocks,
                          int32_t shared_prefix_tokens, int32_t* out);

/* Host helper: slot of each (sequence, position) pair, slot = bt[seq][pos / 16] * 16 + pos % 16.
 *   block_tables  host I32, num_seqs rows of row_stride elements, max_blocks valid entries each.
 *   token_seq, token_pos, slots_out  host arrays of num_tokens entries.
 * PA_ERR_INVALID_ARG if a sequence or logical block is out of range or the entry is negative.
 * Source: vLLM notes page, "PagedAttention / Cache Engine" (page = position // block_size); the
 * in-block offset position % 16 is the plain reading of a 16-token page. */
int pa_slots_for_positions(const int32_t* block_tables, int64_t row_stride, int32_t num_seqs, int32_t max_blocks,
                           const int32_t* token_seq, const int32_t* token_pos, int64_t num_tokens,
                           int64_t* slots_out);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_CACHE_PA_H */
