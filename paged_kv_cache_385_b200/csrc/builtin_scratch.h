// Host-side interface between api.cu and no_alloc.cu: pa_decode with split-partition scratch that
// the library owns instead of a caller workspace.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "../../include/pa.h"

namespace pa {

// The scratch's size, checked against the batch's need with the other arguments, and the lookup of
// its device address on the current device, made only after every argument check has passed.
struct BuiltinScratch {
  size_t bytes;
  cudaError_t (*lookup)(void** device_address);
};

// pa_decode with its split scratch taken from `scratch`; opts->workspace must be NULL (size 0).
int decode_with_builtin_scratch(pa_tensor* out, const pa_tensor* q, const pa_tensor* k_cache,
                                const pa_tensor* v_cache, const pa_tensor* block_tables,
                                const pa_tensor* context_lens, float scale, int32_t num_kv_heads,
                                const pa_decode_opts* opts, void* stream, const BuiltinScratch& scratch);

}  // namespace pa
