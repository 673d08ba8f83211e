// C-ABI entry points of libpagedattn: argument validation, TMA descriptor encoding, dispatch.
// Host code only. Every argument error is found here before the first device call; the kernels
// live in decode.cu, decode_units.cu, multiquery.cu, prefill_tc.cu, cache.cu, no_alloc.cu and selftest.cu.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <string>

#include "../../include/pa.h"
#include "builtin_scratch.h"
#include "internal.h"

namespace {

thread_local std::string g_last_error;

int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}

int ok() {
  g_last_error.clear();
  return PA_OK;
}

int elem_bytes(int dtype) {
  switch (dtype) {
    case PA_F16:
    case PA_BF16:
      return 2;
    case PA_E4M3:
      return 1;
    case PA_I32:
    case PA_F32:
      return 4;
    case PA_I64:
      return 8;
    default:
      return 0;
  }
}

// Product of non-negative sizes, or -1 when it does not fit in int64 (a descriptor may claim any
// shape; the checks below must not overflow on it).
int64_t checked_product(std::initializer_list<int64_t> xs) {
  int64_t r = 1;
  for (const int64_t x : xs)
    if (x < 0 || __builtin_mul_overflow(r, x, &r)) return -1;
  return r;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool is_contiguous(const pa_tensor* t) {
  int64_t expect = 1;
  for (int i = t->ndim - 1; i >= 0; --i) {
    if (t->shape[i] != 1 && t->stride[i] != expect) return false;
    expect *= t->shape[i];
  }
  return true;
}

const char* dtype_name(int d) {
  switch (d) {
    case PA_F16: return "F16";
    case PA_BF16: return "BF16";
    case PA_E4M3: return "E4M3";
    case PA_I32: return "I32";
    case PA_I64: return "I64";
    case PA_F32: return "F32";
    default: return "?";
  }
}

// Checks common to every tensor argument.
int check_tensor(const pa_tensor* t, const char* name, int ndim) {
  if (!t) return fail(PA_ERR_INVALID_ARG, "%s is NULL", name);
  if (t->ndim != ndim) return fail(PA_ERR_INVALID_ARG, "%s: ndim %d, expected %d", name, t->ndim, ndim);
  if (elem_bytes(t->dtype) == 0) return fail(PA_ERR_INVALID_ARG, "%s: unknown dtype %d", name, t->dtype);
  for (int i = 0; i < ndim; ++i)
    if (t->shape[i] < 0) return fail(PA_ERR_INVALID_ARG, "%s: negative shape[%d]", name, i);
  return PA_OK;
}

// ---- TMA descriptor encoding -----------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// The pool [NB, Hkv, 16, D] viewed as a 2-D tensor [NB * Hkv * 16 rows, D], loaded in boxes of
// 16 rows x 128 bytes with the 128-byte swizzle.
int encode_pool_map(CUtensorMap* map, const pa_tensor* cache, int esz) {
  auto fn = encode_fn();
  if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int64_t D = cache->shape[3];
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D),
                              static_cast<cuuint64_t>(cache->shape[0] * cache->shape[1] * 16)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D * esz)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), 16};
  const cuuint32_t estr[2] = {1, 1};
  CUtensorMapDataType dt = esz == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                    : (cache->dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                               : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  CUresult r = fn(map, dt, 2, cache->data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return PA_OK;
}

// q [T, Hq, D] (16-bit) as a 3-D tensor {D, Hq, T}, boxes of 64 x G x (128 / G): 128 rows of 128
// bytes (tokens x group heads of one KV head), 128-byte swizzle.
int encode_q_map(CUtensorMap* map, const pa_tensor* q, int group) {
  auto fn = encode_fn();
  if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(q->shape[2]), static_cast<cuuint64_t>(q->shape[1]),
                              static_cast<cuuint64_t>(q->shape[0])};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(q->stride[1] * 2), static_cast<cuuint64_t>(q->stride[0] * 2)};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(128 / group)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, q->dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                  q->data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled (q or out) failed (%d)", static_cast<int>(r));
  return PA_OK;
}

// The split workspace's partial rows ws_acc [B, Hq, P, D] (float32) as a 4-D tensor {D, P, Hq, B},
// boxes of 32 x 1 x G x (128 / G): 128 rows (sequences x group heads of one KV head, one partition) of
// 32 columns, 128-byte swizzle. The workspace is 256-byte aligned and D * 4 is a multiple of 16.
int encode_ws_map(CUtensorMap* map, float* ws_acc, int64_t B, int64_t Hq, int64_t P, int64_t D, int group) {
  auto fn = encode_fn();
  if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(P), static_cast<cuuint64_t>(Hq),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D * 4), static_cast<cuuint64_t>(P * D * 4),
                                 static_cast<cuuint64_t>(Hq * P * D * 4)};
  const cuuint32_t box[4] = {32, 1, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(128 / group)};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ws_acc, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled (workspace) failed (%d)", static_cast<int>(r));
  return PA_OK;
}

// Host-side fault injection (pa_debug_fail_next_launches): calls left that fail as a launch would.
std::atomic<int32_t> g_injected_failures{0};

// True (and one fewer left) when this call is to fail as if its launch had failed.
bool take_injected_failure() {
  int32_t n = g_injected_failures.load(std::memory_order_relaxed);
  while (n > 0 && !g_injected_failures.compare_exchange_weak(n, n - 1, std::memory_order_relaxed)) {
  }
  return n > 0;
}

// The device address of the library's error word, looked up once per device. Threads may race on
// the first lookup; they all store the same address, and the slots are atomics so that is well defined.
uint32_t* library_error_word() {
  static std::atomic<uint32_t*> words[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
  if (dev >= 64) return pa::decode_error_word();
  uint32_t* w = words[dev].load(std::memory_order_acquire);
  if (!w) {
    w = pa::decode_error_word();
    if (w) words[dev].store(w, std::memory_order_release);
  }
  return w;
}

// Split only when the batch alone cannot fill the GPU: with B * Hkv work units of up to 2048 tokens
// there are enough CTAs once B * Hkv >= kFillUnits; otherwise take the largest partition (fewer,
// longer CTAs: less prologue and merge work) that still yields kFillUnits CTAs.
constexpr int64_t kFillUnits = 4 * 148;

int32_t auto_partition_tokens(int32_t num_seqs, int32_t num_kv_heads, int32_t max_ctx) {
  const int64_t units = static_cast<int64_t>(num_seqs) * num_kv_heads;
  if (max_ctx <= pa::kMaxPartitionTokens && units >= kFillUnits) return 0;
  for (int32_t pt = pa::kMaxPartitionTokens; pt > 256; pt /= 2)
    if (units * ((static_cast<int64_t>(max_ctx) + pt - 1) / pt) >= kFillUnits && max_ctx > pt) return pt;
  return max_ctx > 256 ? 256 : 0;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Layout of the split-partition workspace: acc [B, Hq, P, D] floats, then (m, l) [B, Hq, P, 2].
// SIZE_MAX when the size does not fit in int64 (no buffer can hold it).
size_t workspace_layout(int64_t B, int64_t Hq, int64_t D, int64_t P, size_t* ml_offset) {
  const int64_t acc_bytes = checked_product({B, Hq, P, D, static_cast<int64_t>(sizeof(float))});
  const int64_t ml_bytes = checked_product({B, Hq, P, 2, static_cast<int64_t>(sizeof(float))});
  if (acc_bytes < 0 || ml_bytes < 0 || acc_bytes > (INT64_MAX >> 2) || ml_bytes > (INT64_MAX >> 2)) {
    if (ml_offset) *ml_offset = 0;
    return SIZE_MAX;
  }
  const size_t acc = round_up(static_cast<size_t>(acc_bytes), 256);
  const size_t ml = round_up(static_cast<size_t>(ml_bytes), 256);
  if (ml_offset) *ml_offset = acc;
  return acc + ml;
}

}  // namespace

namespace pa {
int set_last_error(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}
}  // namespace pa

extern "C" {

const char* pa_version(void) { return "0.1.0"; }

const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported configuration";
    case PA_ERR_WORKSPACE: return "workspace missing or too small";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_EXHAUSTED: return "no free block";
    case PA_ERR_BAD_BLOCK: return "bad block id";
    default: return "unknown status";
  }
}

const char* pa_last_error(void) { return g_last_error.c_str(); }

void pa_decode_opts_init(pa_decode_opts* o) {
  if (!o) return;
  std::memset(o, 0, sizeof(*o));
  o->k_scale = 1.0f;
  o->v_scale = 1.0f;
  o->kernel = -1;
  o->prefix_kernel = -1;
}

int32_t pa_decode_partition_tokens(int32_t num_seqs, int32_t num_kv_heads, int32_t max_context_len) {
  if (num_seqs <= 0 || num_kv_heads <= 0 || max_context_len <= 0) return 0;
  return auto_partition_tokens(num_seqs, num_kv_heads, max_context_len);
}

size_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t max_context_len, int32_t partition_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_context_len <= 0) return 0;
  const int32_t pt =
      partition_tokens > 0 ? partition_tokens : auto_partition_tokens(num_seqs, num_kv_heads, max_context_len);
  if (pt <= 0) return 0;
  const int64_t P = (static_cast<int64_t>(max_context_len) + pt - 1) / pt;
  if (P <= 1) return 0;
  return workspace_layout(num_seqs, num_q_heads, head_dim, P, nullptr);
}

int pa_debug_fail_next_launches(int32_t count) {
  if (count < 0) return fail(PA_ERR_INVALID_ARG, "count must be >= 0");
  g_injected_failures.store(count, std::memory_order_relaxed);
  return ok();
}

int pa_read_device_error(uint32_t* bits, int clear) {
  if (!bits) return fail(PA_ERR_INVALID_ARG, "bits is NULL");
  cudaError_t e = pa::read_and_clear_error_word(bits, clear);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
  return ok();
}

int pa_reshape_and_cache(const pa_tensor* key, const pa_tensor* value, const pa_tensor* slot_mapping,
                         pa_tensor* k_cache, pa_tensor* v_cache, float k_scale, float v_scale, void* stream) {
  int st;
  if ((st = check_tensor(key, "key", 3)) || (st = check_tensor(value, "value", 3)) ||
      (st = check_tensor(slot_mapping, "slot_mapping", 1)) || (st = check_tensor(k_cache, "k_cache", 4)) ||
      (st = check_tensor(v_cache, "v_cache", 4)))
    return st;
  const int64_t T = key->shape[0], Hkv = key->shape[1], D = key->shape[2];
  if (key->dtype != PA_F16 && key->dtype != PA_BF16)
    return fail(PA_ERR_INVALID_ARG, "key dtype %s; expected F16 or BF16", dtype_name(key->dtype));
  if (value->dtype != key->dtype) return fail(PA_ERR_INVALID_ARG, "value dtype differs from key dtype");
  for (int i = 0; i < 3; ++i)
    if (value->shape[i] != key->shape[i]) return fail(PA_ERR_INVALID_ARG, "value shape differs from key shape");
  if (slot_mapping->dtype != PA_I64) return fail(PA_ERR_INVALID_ARG, "slot_mapping dtype must be I64");
  if (slot_mapping->shape[0] != T) return fail(PA_ERR_INVALID_ARG, "slot_mapping has %lld entries, key has %lld tokens",
                                               (long long)slot_mapping->shape[0], (long long)T);
  if (T > 0x7fffffff) return fail(PA_ERR_INVALID_ARG, "too many tokens (%lld)", (long long)T);
  if (k_cache->dtype != v_cache->dtype) return fail(PA_ERR_INVALID_ARG, "k_cache and v_cache dtypes differ");
  const int cd = k_cache->dtype;
  if (cd != key->dtype && cd != PA_E4M3)
    return fail(PA_ERR_INVALID_ARG, "cache dtype %s does not match key dtype %s (or E4M3)", dtype_name(cd),
                dtype_name(key->dtype));
  for (int i = 0; i < 4; ++i)
    if (v_cache->shape[i] != k_cache->shape[i]) return fail(PA_ERR_INVALID_ARG, "v_cache shape differs from k_cache");
  if (k_cache->shape[1] != Hkv || k_cache->shape[2] != PA_BLOCK_SIZE || k_cache->shape[3] != D)
    return fail(PA_ERR_INVALID_ARG, "cache shape must be [num_blocks, %lld, 16, %lld]", (long long)Hkv, (long long)D);
  if (!is_contiguous(k_cache) || !is_contiguous(v_cache)) return fail(PA_ERR_INVALID_ARG, "caches must be contiguous");
  if (D % 8 != 0 || D <= 0) return fail(PA_ERR_UNSUPPORTED, "head_dim %lld is not a multiple of 8", (long long)D);
  if (checked_product({k_cache->shape[0], Hkv, PA_BLOCK_SIZE, D, 2}) < 0)
    return fail(PA_ERR_UNSUPPORTED, "pool too large (its size does not fit in 64 bits)");
  if (T == 0) return ok();
  if (key->stride[2] != 1 || value->stride[2] != 1) return fail(PA_ERR_INVALID_ARG, "key/value last stride must be 1");
  if (!aligned(key->data, 16) || !aligned(value->data, 16) || key->stride[0] % 8 || key->stride[1] % 8 ||
      value->stride[0] % 8 || value->stride[1] % 8)
    return fail(PA_ERR_INVALID_ARG, "key/value rows must be 16-byte aligned");
  if (slot_mapping->stride[0] != 1) return fail(PA_ERR_INVALID_ARG, "slot_mapping must be contiguous");
  if (!aligned(k_cache->data, 16) || !aligned(v_cache->data, 16))
    return fail(PA_ERR_INVALID_ARG, "caches must be 16-byte aligned");
  if (!key->data || !value->data || !slot_mapping->data || !k_cache->data || !v_cache->data)
    return fail(PA_ERR_INVALID_ARG, "NULL data pointer");

  pa::CacheParams p{};
  p.key = key->data;
  p.value = value->data;
  p.k_stride_t = key->stride[0];
  p.k_stride_h = key->stride[1];
  p.v_stride_t = value->stride[0];
  p.v_stride_h = value->stride[1];
  p.slots = static_cast<const int64_t*>(slot_mapping->data);
  p.k_cache = k_cache->data;
  p.v_cache = v_cache->data;
  p.num_tokens = T;
  p.num_kv_heads = static_cast<int32_t>(Hkv);
  p.head_dim = static_cast<int32_t>(D);
  p.num_slots = k_cache->shape[0] * PA_BLOCK_SIZE;
  p.k_inv_scale = 1.0f;
  p.v_inv_scale = 1.0f;
  if (cd == PA_E4M3) {
    if (!(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f))
      return fail(PA_ERR_INVALID_ARG, "E4M3 cache scales must be finite and > 0");
    volatile float one = 1.0f;  // keep the reciprocal an IEEE float32 division
    p.k_inv_scale = one / k_scale;
    p.v_inv_scale = one / v_scale;
  }
  if (take_injected_failure()) return fail(PA_ERR_CUDA, "injected launch failure (pa_debug_fail_next_launches)");
  p.err = library_error_word();
  if (!p.err) return fail(PA_ERR_CUDA, "no device error word (no current CUDA device?)");
  const pa::KvType kv = cd == PA_E4M3 ? pa::KvType::E4M3 : (cd == PA_BF16 ? pa::KvType::BF16 : pa::KvType::F16);
  cudaError_t e = pa::launch_reshape_and_cache(key->dtype == PA_BF16, kv, p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "reshape_and_cache launch: %s", cudaGetErrorString(e));
  return ok();
}

// pa_decode, and pa_decode_step when new_key/new_value/new_slots are given (the decode kernel then
// writes each sequence's new token into the cache before reading its pages).
static int decode_impl(pa_tensor* out, const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
                       const pa_tensor* block_tables, const pa_tensor* context_lens, float scale, int32_t num_kv_heads,
                       const pa_decode_opts* opts_in, void* stream, const pa_tensor* new_key,
                       const pa_tensor* new_value, const pa_tensor* new_slots, int32_t prefix_tokens = 0,
                       const pa::BuiltinScratch* builtin = nullptr) {
  pa_decode_opts opts;
  pa_decode_opts_init(&opts);
  if (opts_in) opts = *opts_in;
  int st;
  if ((st = check_tensor(out, "out", 3)) || (st = check_tensor(q, "q", 3)) || (st = check_tensor(k_cache, "k_cache", 4)) ||
      (st = check_tensor(v_cache, "v_cache", 4)) || (st = check_tensor(block_tables, "block_tables", 2)) ||
      (st = check_tensor(context_lens, "context_lens", 1)))
    return st;
  const int64_t B = q->shape[0], Hq = q->shape[1], D = q->shape[2];
  if (q->dtype != PA_F16 && q->dtype != PA_BF16) return fail(PA_ERR_INVALID_ARG, "q dtype must be F16 or BF16");
  if (out->dtype != q->dtype) return fail(PA_ERR_INVALID_ARG, "out dtype differs from q dtype");
  for (int i = 0; i < 3; ++i)
    if (out->shape[i] != q->shape[i]) return fail(PA_ERR_INVALID_ARG, "out shape differs from q shape");
  if (k_cache->dtype != v_cache->dtype) return fail(PA_ERR_INVALID_ARG, "k_cache and v_cache dtypes differ");
  const int cd = k_cache->dtype;
  if (cd != PA_F16 && cd != PA_BF16 && cd != PA_E4M3) return fail(PA_ERR_INVALID_ARG, "cache dtype must be F16, BF16 or E4M3");
  if (cd != PA_E4M3 && cd != q->dtype)
    return fail(PA_ERR_INVALID_ARG, "a %s cache needs a %s query (got %s)", dtype_name(cd), dtype_name(cd),
                dtype_name(q->dtype));
  for (int i = 0; i < 4; ++i)
    if (v_cache->shape[i] != k_cache->shape[i]) return fail(PA_ERR_INVALID_ARG, "v_cache shape differs from k_cache");
  if (num_kv_heads <= 0 || k_cache->shape[1] != num_kv_heads)
    return fail(PA_ERR_INVALID_ARG, "num_kv_heads %d does not match k_cache.shape[1] = %lld", num_kv_heads,
                (long long)k_cache->shape[1]);
  if (k_cache->shape[2] != PA_BLOCK_SIZE || k_cache->shape[3] != D)
    return fail(PA_ERR_INVALID_ARG, "cache shape must be [num_blocks, Hkv, 16, %lld]", (long long)D);
  if (!is_contiguous(k_cache) || !is_contiguous(v_cache)) return fail(PA_ERR_INVALID_ARG, "caches must be contiguous");
  if (Hq % num_kv_heads != 0) return fail(PA_ERR_INVALID_ARG, "num_q_heads %lld is not a multiple of num_kv_heads %d",
                                          (long long)Hq, num_kv_heads);
  if (block_tables->dtype != PA_I32 || block_tables->shape[0] != B)
    return fail(PA_ERR_INVALID_ARG, "block_tables must be I32 [num_seqs, max_blocks]");
  if (context_lens->dtype != PA_I32 || context_lens->shape[0] != B)
    return fail(PA_ERR_INVALID_ARG, "context_lens must be I32 [num_seqs]");
  if (!(std::isfinite(scale))) return fail(PA_ERR_INVALID_ARG, "scale must be finite");
  const int64_t G = Hq / num_kv_heads;
  if (B == 0 || Hq == 0) return ok();
  const int64_t NB = k_cache->shape[0];
  if (NB <= 0) return fail(PA_ERR_INVALID_ARG, "empty pool");
  if (NB > 0x7fffffffLL / 16 / num_kv_heads) return fail(PA_ERR_UNSUPPORTED, "pool too large (rows exceed 2^31)");
  if (B > 65535 || num_kv_heads > 65535) return fail(PA_ERR_UNSUPPORTED, "num_seqs and num_kv_heads must be <= 65535");
  if (G > 16) return fail(PA_ERR_UNSUPPORTED, "query group %lld > 16", (long long)G);
  if (q->stride[2] != 1 || out->stride[2] != 1) return fail(PA_ERR_INVALID_ARG, "q/out last stride must be 1");
  if (!aligned(q->data, 16) || !aligned(out->data, 16) || q->stride[0] % 8 || q->stride[1] % 8 || out->stride[0] % 8 ||
      out->stride[1] % 8)
    return fail(PA_ERR_INVALID_ARG, "q/out rows must be 16-byte aligned");
  if (!aligned(k_cache->data, 128) || !aligned(v_cache->data, 128))
    return fail(PA_ERR_INVALID_ARG, "caches must be 128-byte aligned");
  if (block_tables->stride[1] != 1 && block_tables->shape[1] > 1)
    return fail(PA_ERR_INVALID_ARG, "block_tables last stride must be 1");
  if (context_lens->stride[0] != 1 && B > 1) return fail(PA_ERR_INVALID_ARG, "context_lens must be contiguous");
  if (!out->data || !q->data || !k_cache->data || !v_cache->data || !block_tables->data || !context_lens->data)
    return fail(PA_ERR_INVALID_ARG, "NULL data pointer");
  const int64_t max_blocks = block_tables->shape[1];
  if (max_blocks <= 0) return fail(PA_ERR_INVALID_ARG, "block_tables has no columns");
  // Tokens a table row can address; contexts are int32, so columns past 2^31 / 16 are never read.
  const int64_t table_tokens = std::min<int64_t>(max_blocks, 0x7fffffff / 16) * 16;

  pa::DecodeConfig cfg{};
  cfg.kv = cd == PA_E4M3 ? pa::KvType::E4M3 : (cd == PA_BF16 ? pa::KvType::BF16 : pa::KvType::F16);
  cfg.q = q->dtype == PA_BF16 ? pa::QType::BF16 : pa::QType::F16;
  cfg.head_dim = static_cast<int>(D);
  cfg.ntiles = static_cast<int>((G + 7) / 8);
  if (opts.kernel < -1 || opts.kernel > 2) return fail(PA_ERR_INVALID_ARG, "opts.kernel must be -1, 0, 1 or 2");
  // 2: the tensor-core kernel, always one CTA per partition (no persistent per-warp split form).
  const bool cta_per_partition = opts.kernel == 2;
  cfg.kernel = opts.kernel < 0 || opts.kernel == 2 ? 1 : opts.kernel;
  if (!pa::decode_supported(cfg))
    return fail(PA_ERR_UNSUPPORTED, "no kernel for head_dim %lld, cache %s, q %s, group %lld, kernel %d", (long long)D,
                dtype_name(cd), dtype_name(q->dtype), (long long)G, cfg.kernel);

  float k_scale = 1.f, v_scale = 1.f;
  if (cd == PA_E4M3) {
    k_scale = opts.k_scale;
    v_scale = opts.v_scale;
    if (!(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f))
      return fail(PA_ERR_INVALID_ARG, "E4M3 cache scales must be finite and > 0");
  }

  int64_t max_ctx = opts.max_context_len > 0 ? opts.max_context_len : table_tokens;
  if (opts.max_context_len < 0) return fail(PA_ERR_INVALID_ARG, "max_context_len < 0");
  max_ctx = std::min<int64_t>(max_ctx, table_tokens);
  int64_t pt = opts.partition_tokens;
  if (pt < 0 || pt % 16 || pt > pa::kMaxPartitionTokens)
    return fail(PA_ERR_INVALID_ARG, "partition_tokens %lld must be a multiple of 16 in [0, %d]", (long long)pt,
                pa::kMaxPartitionTokens);
  const bool have_ws = (opts.workspace != nullptr && opts.workspace_bytes > 0) || builtin != nullptr;
  // Cascade: the shared prefix goes to the prefix kernel (n_pre chunks); this grid covers the suffix.
  const bool cascade = prefix_tokens > 0;
  int64_t n_pre = 0;
  bool use_tc_prefix = false;
  if (cascade) {
    if (cd == PA_E4M3) return fail(PA_ERR_UNSUPPORTED, "shared-prefix decode takes F16 or BF16 caches");
    if (prefix_tokens % 16) return fail(PA_ERR_INVALID_ARG, "shared_prefix_tokens must be a multiple of 16");
    if (prefix_tokens > table_tokens)
      return fail(PA_ERR_INVALID_ARG, "shared_prefix_tokens %d exceeds the block-table width", prefix_tokens);
    n_pre = (prefix_tokens + pa::kPrefixChunkTokens - 1) / pa::kPrefixChunkTokens;
    if (opts.prefix_kernel < -1 || opts.prefix_kernel > 1)
      return fail(PA_ERR_INVALID_ARG, "opts.prefix_kernel must be -1, 0 or 1");
    const bool tc_ok = pa::prefill_tc_supported(static_cast<int>(D), static_cast<int>(G)) && q->stride[2] == 1 &&
                       q->stride[1] % 8 == 0 && q->stride[0] % 8 == 0 && aligned(q->data, 16);
    if (opts.prefix_kernel == 1 && !tc_ok)
      return fail(PA_ERR_UNSUPPORTED, "the tcgen05 prefix kernel needs head_dim 128, a group dividing 128 and 16-byte aligned q rows");
    use_tc_prefix = opts.prefix_kernel == 1 || (opts.prefix_kernel == -1 && tc_ok);
  }
  const int64_t span_max = std::max<int64_t>(max_ctx - (cascade ? prefix_tokens : 0), 0);
  if (pt == 0) {
    pt = auto_partition_tokens(static_cast<int32_t>(B), num_kv_heads, static_cast<int32_t>(std::max<int64_t>(span_max, 1)));
    if (pt == 0 || (!have_ws && span_max <= pa::kMaxPartitionTokens))
      pt = std::max<int64_t>(16, (std::min<int64_t>(std::max<int64_t>(span_max, 1), pa::kMaxPartitionTokens) + 15) / 16 * 16);
  }
  int64_t P = (span_max + pt - 1) / pt;
  if (P < 1) P = 1;
  if (P > 0x7fffffff) return fail(PA_ERR_UNSUPPORTED, "too many partitions");
  const int64_t ws_parts = n_pre + P;

  pa::DecodeParams p{};
  p.out = out->data;
  p.q = q->data;
  p.q_stride_s = q->stride[0];
  p.q_stride_h = q->stride[1];
  p.o_stride_s = out->stride[0];
  p.o_stride_h = out->stride[1];
  p.block_tables = static_cast<const int32_t*>(block_tables->data);
  p.bt_stride = block_tables->stride[0];
  p.context_lens = static_cast<const int32_t*>(context_lens->data);
  p.num_seqs = static_cast<int32_t>(B);
  p.num_blocks = static_cast<int32_t>(NB);
  p.num_kv_heads = num_kv_heads;
  p.group = static_cast<int32_t>(G);
  p.max_blocks = static_cast<int32_t>(std::min<int64_t>(max_blocks, 0x7fffffff / 16));
  p.partition_tokens = static_cast<int32_t>(pt);
  p.num_partitions = static_cast<int32_t>(P);
  p.score_scale_log2 = scale * 1.4426950408889634f * k_scale;
  p.v_scale = v_scale;
  p.start_tokens = cascade ? prefix_tokens : 0;
  p.part_offset = static_cast<int32_t>(n_pre);
  p.ws_parts = static_cast<int32_t>(ws_parts);
  p.always_partials = cascade ? 1 : 0;
  p.merge_prefix_inline = cascade && P == 1 ? 1 : 0;
  p.late_dependency_wait = cascade ? 1 : 0;
  // The persistent per-warp split form where it applies (not the cascade suffix: its short units
  // stream faster with a CTA's four warps on each); else one CTA per partition.
  const bool use_units = ws_parts > 1 && !cta_per_partition && pa::decode_units_supported(cfg, p);
  size_t ml_off = 0;
  if (ws_parts > 1) {
    const size_t need = workspace_layout(B, Hq, D, ws_parts, &ml_off);
    if (need == SIZE_MAX)
      return fail(PA_ERR_UNSUPPORTED, "split into %lld partitions: the workspace size overflows", (long long)ws_parts);
    if (builtin) {
      // The built-in array's address is looked up below, after the last argument check.
      if (need > builtin->bytes)
        return fail(PA_ERR_WORKSPACE,
                    "this batch needs %zu bytes of scratch; the built-in array holds %zu (use pa_decode with a "
                    "workspace, or larger partition_tokens)", need, builtin->bytes);
    } else {
      if (!have_ws || opts.workspace_bytes < need)
        return fail(PA_ERR_WORKSPACE, "split into %lld partitions needs a workspace of %zu bytes (got %zu)",
                    (long long)ws_parts, need, have_ws ? opts.workspace_bytes : size_t(0));
      if (!aligned(opts.workspace, 256)) return fail(PA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
      p.ws_acc = static_cast<float*>(opts.workspace);
      p.ws_ml = reinterpret_cast<float*>(static_cast<char*>(opts.workspace) + ml_off);
    }
  }

  if (new_key) {
    if ((st = check_tensor(new_key, "key", 3)) || (st = check_tensor(new_value, "value", 3)) ||
        (st = check_tensor(new_slots, "slot_mapping", 1)))
      return st;
    if (new_key->dtype != PA_F16 && new_key->dtype != PA_BF16)
      return fail(PA_ERR_INVALID_ARG, "key dtype %s; expected F16 or BF16", dtype_name(new_key->dtype));
    if (new_value->dtype != new_key->dtype) return fail(PA_ERR_INVALID_ARG, "value dtype differs from key dtype");
    if (cd != PA_E4M3 && cd != new_key->dtype)
      return fail(PA_ERR_INVALID_ARG, "cache dtype %s does not match key dtype %s", dtype_name(cd),
                  dtype_name(new_key->dtype));
    for (int i = 0; i < 3; ++i) {
      const int64_t want = i == 0 ? B : (i == 1 ? num_kv_heads : D);
      if (new_key->shape[i] != want || new_value->shape[i] != want)
        return fail(PA_ERR_INVALID_ARG, "key/value must be [num_seqs, num_kv_heads, head_dim] (one new token each)");
    }
    if (new_slots->dtype != PA_I64 || new_slots->shape[0] != B || (new_slots->stride[0] != 1 && B > 1))
      return fail(PA_ERR_INVALID_ARG, "slot_mapping must be contiguous I64 [num_seqs]");
    if (new_key->stride[2] != 1 || new_value->stride[2] != 1 || !aligned(new_key->data, 16) ||
        !aligned(new_value->data, 16) || new_key->stride[0] % 8 || new_key->stride[1] % 8 ||
        new_value->stride[0] % 8 || new_value->stride[1] % 8)
      return fail(PA_ERR_INVALID_ARG, "key/value rows must be contiguous and 16-byte aligned");
    if (!new_key->data || !new_value->data || !new_slots->data) return fail(PA_ERR_INVALID_ARG, "NULL data pointer");
    p.new_k = new_key->data;
    p.new_v = new_value->data;
    p.nk_stride_s = new_key->stride[0];
    p.nk_stride_h = new_key->stride[1];
    p.nv_stride_s = new_value->stride[0];
    p.nv_stride_h = new_value->stride[1];
    p.new_slots = static_cast<const int64_t*>(new_slots->data);
    p.k_cache = k_cache->data;
    p.v_cache = v_cache->data;
    p.new_src_bf16 = new_key->dtype == PA_BF16;
    volatile float one = 1.0f;  // IEEE float32 reciprocals, as pa_reshape_and_cache forms them
    p.k_inv_scale = cd == PA_E4M3 ? one / k_scale : 1.0f;
    p.v_inv_scale = cd == PA_E4M3 ? one / v_scale : 1.0f;
  }

  // Every argument check is above: the device calls start here.
  if (take_injected_failure()) return fail(PA_ERR_CUDA, "injected launch failure (pa_debug_fail_next_launches)");
  p.err = opts.error_word ? reinterpret_cast<uint32_t*>(opts.error_word) : library_error_word();
  if (!p.err) return fail(PA_ERR_CUDA, "no device error word (no current CUDA device?)");
  if (builtin && ws_parts > 1) {
    void* base = nullptr;
    const cudaError_t le = builtin->lookup(&base);
    if (le != cudaSuccess || !base)
      return fail(PA_ERR_CUDA, "address of the built-in scratch array: %s", cudaGetErrorString(le));
    p.ws_acc = static_cast<float*>(base);
    p.ws_ml = reinterpret_cast<float*>(static_cast<char*>(base) + ml_off);
  }
  CUtensorMap km, vm;
  const int esz = elem_bytes(cd);
  if ((st = encode_pool_map(&km, k_cache, esz)) || (st = encode_pool_map(&vm, v_cache, esz))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (cascade) {
    pa::MqParams pp{};
    pp.q = q->data;
    pp.q_stride_s = q->stride[0];
    pp.q_stride_h = q->stride[1];
    pp.block_tables = p.block_tables;
    pp.bt_stride = p.bt_stride;
    pp.context_lens = p.context_lens;
    pp.num_seqs = p.num_seqs;
    pp.num_blocks = p.num_blocks;
    pp.num_kv_heads = num_kv_heads;
    pp.group = p.group;
    pp.max_blocks = p.max_blocks;
    pp.prefix_tokens = prefix_tokens;
    pp.chunk_tokens = pa::kPrefixChunkTokens;
    pp.num_chunks = static_cast<int32_t>(n_pre);
    pp.score_scale_log2 = p.score_scale_log2;
    pp.ws_acc = p.ws_acc;
    pp.ws_ml = p.ws_ml;
    pp.ws_parts = p.ws_parts;
    pp.err = p.err;
    if (use_tc_prefix) {
      CUtensorMap qm, wm;
      if ((st = encode_q_map(&qm, q, static_cast<int>(G))) ||
          (st = encode_ws_map(&wm, pp.ws_acc, B, Hq, ws_parts, D, static_cast<int>(G))))
        return st;
      e = pa::launch_prefix_tc(cfg.kv, qm, km, vm, wm, pp, s);
    } else {
      e = pa::launch_prefix(cfg.kv, cfg.head_dim, km, vm, pp, s);
    }
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "prefix launch: %s", cudaGetErrorString(e));
  }
  if (use_units)
    e = pa::launch_decode_units(cfg, km, vm, p, s);
  else
    e = pa::launch_decode(cfg, km, vm, p, s);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
  if (ws_parts > 1 && !p.merge_prefix_inline) {
    e = pa::launch_reduce(cfg, p, s);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "reduce launch: %s", cudaGetErrorString(e));
  }
  return ok();
}

int pa_copy_blocks(pa_tensor* k_cache, pa_tensor* v_cache, const pa_tensor* block_mapping, void* stream) {
  int st;
  if ((st = check_tensor(k_cache, "k_cache", 4)) || (st = check_tensor(v_cache, "v_cache", 4)) ||
      (st = check_tensor(block_mapping, "block_mapping", 2)))
    return st;
  if (k_cache->dtype != v_cache->dtype) return fail(PA_ERR_INVALID_ARG, "k_cache and v_cache dtypes differ");
  for (int i = 0; i < 4; ++i)
    if (v_cache->shape[i] != k_cache->shape[i]) return fail(PA_ERR_INVALID_ARG, "v_cache shape differs from k_cache");
  if (k_cache->shape[2] != PA_BLOCK_SIZE) return fail(PA_ERR_INVALID_ARG, "cache shape must be [num_blocks, Hkv, 16, D]");
  if (!is_contiguous(k_cache) || !is_contiguous(v_cache)) return fail(PA_ERR_INVALID_ARG, "caches must be contiguous");
  if (block_mapping->dtype != PA_I64 || block_mapping->shape[1] != 2 || !is_contiguous(block_mapping))
    return fail(PA_ERR_INVALID_ARG, "block_mapping must be contiguous I64 [num_pairs, 2]");
  const int64_t N = block_mapping->shape[0];
  if (N == 0) return ok();
  if (N > 0x7fffffff) return fail(PA_ERR_INVALID_ARG, "too many pairs");
  const int64_t block_bytes = checked_product({k_cache->shape[1], 16, k_cache->shape[3], elem_bytes(k_cache->dtype)});
  if (block_bytes < 0 || checked_product({k_cache->shape[0], block_bytes}) < 0)
    return fail(PA_ERR_UNSUPPORTED, "pool too large (its size does not fit in 64 bits)");
  if (block_bytes % 16) return fail(PA_ERR_UNSUPPORTED, "block size in bytes must be a multiple of 16");
  if (!aligned(k_cache->data, 16) || !aligned(v_cache->data, 16)) return fail(PA_ERR_INVALID_ARG, "caches must be 16-byte aligned");
  if (!block_mapping->data) return fail(PA_ERR_INVALID_ARG, "NULL data pointer");
  pa::CopyParams p{};
  p.k_cache = k_cache->data;
  p.v_cache = v_cache->data;
  p.mapping = static_cast<const int64_t*>(block_mapping->data);
  p.num_pairs = N;
  p.block_bytes = block_bytes;
  p.num_blocks = k_cache->shape[0];
  if (take_injected_failure()) return fail(PA_ERR_CUDA, "injected launch failure (pa_debug_fail_next_launches)");
  p.err = library_error_word();
  if (!p.err) return fail(PA_ERR_CUDA, "no device error word (no current CUDA device?)");
  cudaError_t e = pa::launch_copy_blocks(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "copy_blocks launch: %s", cudaGetErrorString(e));
  return ok();
}

int pa_decode(pa_tensor* out, const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
              const pa_tensor* block_tables, const pa_tensor* context_lens, float scale, int32_t num_kv_heads,
              const pa_decode_opts* opts, void* stream) {
  return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, opts, stream, nullptr,
                     nullptr, nullptr);
}

}  // extern "C"

namespace pa {
int decode_with_builtin_scratch(pa_tensor* out, const pa_tensor* q, const pa_tensor* k_cache,
                                const pa_tensor* v_cache, const pa_tensor* block_tables,
                                const pa_tensor* context_lens, float scale, int32_t num_kv_heads,
                                const pa_decode_opts* opts, void* stream, const BuiltinScratch& scratch) {
  if (opts && (opts->workspace != nullptr || opts->workspace_bytes != 0))
    return fail(PA_ERR_INVALID_ARG, "no workspace may be given with the built-in scratch (opts.workspace must be "
                                    "NULL, size 0)");
  return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, opts, stream, nullptr,
                     nullptr, nullptr, 0, &scratch);
}
}  // namespace pa

extern "C" {

int pa_decode_cascade(pa_tensor* out, const pa_tensor* q, const pa_tensor* key, const pa_tensor* value,
                      const pa_tensor* slot_mapping, pa_tensor* k_cache, pa_tensor* v_cache,
                      const pa_tensor* block_tables, const pa_tensor* context_lens, int32_t shared_prefix_tokens,
                      float scale, int32_t num_kv_heads, const pa_decode_opts* opts, void* stream) {
  if (shared_prefix_tokens <= 0) return fail(PA_ERR_INVALID_ARG, "shared_prefix_tokens must be > 0");
  if ((key == nullptr) != (value == nullptr) || (key == nullptr) != (slot_mapping == nullptr))
    return fail(PA_ERR_INVALID_ARG, "key, value and slot_mapping are given together or not at all");
  return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, opts, stream, key,
                     value, slot_mapping, shared_prefix_tokens);
}

size_t pa_decode_cascade_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                         int32_t head_dim, int32_t max_context_len, int32_t shared_prefix_tokens,
                                         int32_t partition_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || shared_prefix_tokens <= 0)
    return 0;
  const int64_t n_pre = (shared_prefix_tokens + pa::kPrefixChunkTokens - 1) / pa::kPrefixChunkTokens;
  const int64_t span = std::max<int64_t>(static_cast<int64_t>(max_context_len) - shared_prefix_tokens, 0);
  int64_t pt = partition_tokens;
  if (pt <= 0) {
    pt = auto_partition_tokens(num_seqs, num_kv_heads, static_cast<int32_t>(std::max<int64_t>(span, 1)));
    if (pt == 0) pt = std::max<int64_t>(16, (std::min<int64_t>(std::max<int64_t>(span, 1), pa::kMaxPartitionTokens) + 15) / 16 * 16);
  }
  const int64_t P = std::max<int64_t>(1, (span + pt - 1) / pt);
  return workspace_layout(num_seqs, num_q_heads, head_dim, n_pre + P, nullptr);
}

int pa_prefill(pa_tensor* out, const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
               const pa_tensor* block_tables, const pa_tensor* query_start, const pa_tensor* context_lens,
               int32_t max_query_len, float scale, int32_t num_kv_heads, int32_t kernel, void* stream) {
  int st;
  if ((st = check_tensor(out, "out", 3)) || (st = check_tensor(q, "q", 3)) || (st = check_tensor(k_cache, "k_cache", 4)) ||
      (st = check_tensor(v_cache, "v_cache", 4)) || (st = check_tensor(block_tables, "block_tables", 2)) ||
      (st = check_tensor(query_start, "query_start", 1)) || (st = check_tensor(context_lens, "context_lens", 1)))
    return st;
  const int64_t T = q->shape[0], Hq = q->shape[1], D = q->shape[2], B = block_tables->shape[0];
  const int cd = k_cache->dtype;
  if (cd != PA_F16 && cd != PA_BF16) return fail(PA_ERR_UNSUPPORTED, "prefill takes F16 or BF16 caches");
  if (q->dtype != cd || out->dtype != cd || v_cache->dtype != cd)
    return fail(PA_ERR_INVALID_ARG, "q, out and both caches must have one dtype");
  for (int i = 0; i < 3; ++i)
    if (out->shape[i] != q->shape[i]) return fail(PA_ERR_INVALID_ARG, "out shape differs from q shape");
  for (int i = 0; i < 4; ++i)
    if (v_cache->shape[i] != k_cache->shape[i]) return fail(PA_ERR_INVALID_ARG, "v_cache shape differs from k_cache");
  if (num_kv_heads <= 0 || k_cache->shape[1] != num_kv_heads || Hq % num_kv_heads)
    return fail(PA_ERR_INVALID_ARG, "num_kv_heads must equal k_cache.shape[1] and divide num_q_heads");
  if (k_cache->shape[2] != PA_BLOCK_SIZE || k_cache->shape[3] != D)
    return fail(PA_ERR_INVALID_ARG, "cache shape must be [num_blocks, Hkv, 16, %lld]", (long long)D);
  if (D != 64 && D != 128) return fail(PA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (!is_contiguous(k_cache) || !is_contiguous(v_cache)) return fail(PA_ERR_INVALID_ARG, "caches must be contiguous");
  if (block_tables->dtype != PA_I32 || (block_tables->stride[1] != 1 && block_tables->shape[1] > 1))
    return fail(PA_ERR_INVALID_ARG, "block_tables must be I32 [num_seqs, max_blocks], last stride 1");
  if (query_start->dtype != PA_I32 || query_start->shape[0] != B + 1 || (query_start->stride[0] != 1 && B > 0))
    return fail(PA_ERR_INVALID_ARG, "query_start must be contiguous I32 [num_seqs + 1]");
  if (context_lens->dtype != PA_I32 || context_lens->shape[0] != B || (context_lens->stride[0] != 1 && B > 1))
    return fail(PA_ERR_INVALID_ARG, "context_lens must be contiguous I32 [num_seqs]");
  if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale must be finite");
  if (T == 0 || B == 0) return ok();
  if (max_query_len <= 0) return fail(PA_ERR_INVALID_ARG, "max_query_len must be > 0");
  if (B > 65535 || num_kv_heads > 65535) return fail(PA_ERR_UNSUPPORTED, "num_seqs and num_kv_heads must be <= 65535");
  if (k_cache->shape[0] > 0x7fffffffLL / 16 / num_kv_heads) return fail(PA_ERR_UNSUPPORTED, "pool too large");
  if (q->stride[2] != 1 || out->stride[2] != 1 || !aligned(q->data, 16) || !aligned(out->data, 16) ||
      q->stride[0] % 8 || q->stride[1] % 8 || out->stride[0] % 8 || out->stride[1] % 8)
    return fail(PA_ERR_INVALID_ARG, "q/out rows must be contiguous and 16-byte aligned");
  if (!aligned(k_cache->data, 128) || !aligned(v_cache->data, 128))
    return fail(PA_ERR_INVALID_ARG, "caches must be 128-byte aligned");
  if (!out->data || !q->data || !k_cache->data || !v_cache->data || !block_tables->data || !query_start->data ||
      !context_lens->data)
    return fail(PA_ERR_INVALID_ARG, "NULL data pointer");
  // The kernel choice is an argument error, reported before any device call.
  const int G = static_cast<int>(Hq / num_kv_heads);
  if (kernel < -1 || kernel > 1) return fail(PA_ERR_INVALID_ARG, "kernel must be -1, 0 or 1");
  const bool tc_ok = pa::prefill_tc_supported(static_cast<int>(D), G);
  if (kernel == 1 && !tc_ok) return fail(PA_ERR_UNSUPPORTED, "the tcgen05 prefill needs head_dim 128 and a group of at most 16 dividing 128");
  pa::MqParams p{};
  p.q = q->data;
  p.q_stride_s = q->stride[0];
  p.q_stride_h = q->stride[1];
  p.out = out->data;
  p.o_stride_t = out->stride[0];
  p.o_stride_h = out->stride[1];
  p.block_tables = static_cast<const int32_t*>(block_tables->data);
  p.bt_stride = block_tables->stride[0];
  p.context_lens = static_cast<const int32_t*>(context_lens->data);
  p.query_start = static_cast<const int32_t*>(query_start->data);
  p.num_seqs = static_cast<int32_t>(B);
  p.num_blocks = static_cast<int32_t>(k_cache->shape[0]);
  p.num_kv_heads = num_kv_heads;
  p.group = static_cast<int32_t>(Hq / num_kv_heads);
  p.max_blocks = static_cast<int32_t>(std::min<int64_t>(block_tables->shape[1], 0x7fffffff / 16));
  p.score_scale_log2 = scale * 1.4426950408889634f;
  if (take_injected_failure()) return fail(PA_ERR_CUDA, "injected launch failure (pa_debug_fail_next_launches)");
  p.err = library_error_word();
  if (!p.err) return fail(PA_ERR_CUDA, "no device error word (no current CUDA device?)");
  CUtensorMap km, vm;
  if ((st = encode_pool_map(&km, k_cache, 2)) || (st = encode_pool_map(&vm, v_cache, 2))) return st;
  const pa::KvType kv = cd == PA_BF16 ? pa::KvType::BF16 : pa::KvType::F16;
  cudaError_t e;
  if (kernel == 1 || (kernel == -1 && tc_ok)) {
    CUtensorMap qm, om;
    if ((st = encode_q_map(&qm, q, G)) || (st = encode_q_map(&om, out, G))) return st;
    e = pa::launch_prefill_tc(kv, qm, km, vm, om, p, max_query_len, static_cast<cudaStream_t>(stream));
  } else {
    e = pa::launch_prefill(kv, static_cast<int>(D), km, vm, p, max_query_len, static_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
  return ok();
}

int pa_decode_step(pa_tensor* out, const pa_tensor* q, const pa_tensor* key, const pa_tensor* value,
                   const pa_tensor* slot_mapping, pa_tensor* k_cache, pa_tensor* v_cache,
                   const pa_tensor* block_tables, const pa_tensor* context_lens, float scale, int32_t num_kv_heads,
                   const pa_decode_opts* opts, void* stream) {
  if (!key || !value || !slot_mapping) return fail(PA_ERR_INVALID_ARG, "key, value and slot_mapping are required");
  return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, opts, stream, key,
                     value, slot_mapping);
}

}  // extern "C"
