// Capped device-side wait, and its self-test.
//
// Every spin-wait in this library is bounded: after a fixed time it records
// LMOE_ETIMEOUT in the workspace status word and returns, so a wait that can
// never be satisfied costs a bounded delay and leaves the context usable.
// The self-test waits on a flag that nothing sets.
#include "common.cuh"
#include "kernels.h"

namespace lmoe {
namespace {

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__global__ void capped_wait_kernel(const volatile int32_t* flag, int32_t* status, int cap_ms) {
  const uint64_t limit = (uint64_t)cap_ms * 1000000ull;
  const uint64_t t0 = global_ns();
  while (*flag == 0) {
    if (global_ns() - t0 > limit) {
      record_status(status, kStatusTimeout);
      return;
    }
    __nanosleep(1000);
  }
}

}  // namespace

cudaError_t launch_capped_wait(int32_t* flag, int32_t* status, int cap_ms, cudaStream_t st) {
  capped_wait_kernel<<<1, 1, 0, st>>>(flag, status, cap_ms);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lmoe
