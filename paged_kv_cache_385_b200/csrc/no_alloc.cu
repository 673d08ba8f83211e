// pa_decode_no_alloc: pa_decode with its split-partition scratch taken from a fixed array that the
// library itself carries in device memory, so the caller never provides (or allocates) a workspace.
//
// Why it exists: pa_decode needs caller-provided scratch whenever a context is split into
// partitions. Some callers have no way to get that memory: a plugin whose host framework owns all
// device memory and hands the plugin only its inputs and outputs; a process whose device-memory
// budget is fixed at start-up; a serving loop where a cudaMalloc (which can synchronise the whole
// device) in the middle of a decode step is not acceptable. They call this entry point instead.
//
// The array (PA_NO_ALLOC_SCRATCH_BYTES) is a file-scope static __device__ object: every device where
// the library's device code is loaded holds it until the process exits. In host code the array's name is only a
// host-side stand-in, never a device address, so its address is looked up with
// cudaGetSymbolAddress once per device, with that device current, on the first call on that device
// that splits a context (after all of its argument checks), and cached. Every call on a device shares the one array, which keeps the last call's
// contents; nothing in it has to start at zero, because each call writes every partial result it
// later reads. Calls whose kernels overlap on the GPU (for example, issued on two streams with no
// ordering between them) race on the array.
#include <mutex>

#include "../../include/pa.h"
#include "builtin_scratch.h"
#include "internal.h"

namespace {

__device__ __align__(256) unsigned char g_no_alloc_scratch[PA_NO_ALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up on first use, then cached).
cudaError_t scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_no_alloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int pa_decode_no_alloc(pa_tensor* out, const pa_tensor* q, const pa_tensor* k_cache,
                                  const pa_tensor* v_cache, const pa_tensor* block_tables,
                                  const pa_tensor* context_lens, float scale, int32_t num_kv_heads,
                                  const pa_decode_opts* opts, void* stream) {
  // Every argument check, including whether the batch's split fits the array, runs before the
  // array's address is looked up (the first CUDA call).
  const pa::BuiltinScratch scratch{static_cast<size_t>(PA_NO_ALLOC_SCRATCH_BYTES), scratch_on_current_device};
  return pa::decode_with_builtin_scratch(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads,
                                         opts, stream, scratch);
}
