// pa_selftest_bounded_wait: runs the bounded mbarrier wait that every kernel of the library uses on
// its copy and MMA barriers against a barrier nothing ever arrives on, so that the give-up path
// (deadline on the global timer, PA_DEVERR_TIMEOUT OR-ed into the error word, kernel returns) can be
// checked on a GPU without any fault or hang: the wait is bounded by the caller's timeout.
#include "../../include/pa.h"
#include "internal.h"
#include "pa_device.cuh"

namespace {

__global__ void bounded_wait_selftest_kernel(uint32_t* err, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = pa::smem_u32(&bar);
  if (threadIdx.x == 0) {
    pa::mbar_init(b, 1);
    pa::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing arrives on this barrier: the wait must give up at its deadline.
    if (!pa::mbar_wait_bounded(b, 0, pa::globaltimer_ns() + timeout_ns)) atomicOr(err, PA_DEVERR_TIMEOUT);
  }
}

}  // namespace

extern "C" int pa_selftest_bounded_wait(int32_t timeout_us, int32_t* error_word, void* stream) {
  if (timeout_us < 1 || timeout_us > 1000000)
    return pa::set_last_error(PA_ERR_INVALID_ARG, "timeout_us %d outside [1, 1000000]", timeout_us);
  uint32_t* err = error_word ? reinterpret_cast<uint32_t*>(error_word) : pa::decode_error_word();
  if (!err) return pa::set_last_error(PA_ERR_CUDA, "no device error word (no current CUDA device?)");
  bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      err, static_cast<uint64_t>(timeout_us) * 1000ull);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pa::set_last_error(PA_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(e));
  return pa::set_last_error(PA_OK, "");
}
