// Self-test of the failure path of the bounded device waits.
//
// Every wait inside the library's kernels (on an mbarrier, or on a counter in
// global memory that other CTAs advance) gives up after a time limit, raises a
// bit in the caller's status word and lets the kernel return, so that a stuck
// pipeline ends as an error the host can read (qlora_ws_status) instead of a
// hung GPU.  This kernel runs one such wait that can only run out: on an
// mbarrier of its own that no thread arrives on, or on a workspace counter that
// no thread advances, with a short limit.  It has no asynchronous copies or
// tensor-core work in flight and holds no TMEM, so giving up leaves nothing
// behind; the context stays usable.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace qlora {

namespace {

__global__ void selftest_wait_kernel(uint32_t* status, const uint32_t* counter, int kind, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  if (kind == 0) {
    const uint32_t b = sm100::smem_addr(&bar);
    sm100::mbar_init(b, 1);   // one arrival completes phase 0; none comes
    sm100::fence_mbar_init();
    sm100::mbar_wait_limit(b, 0, status, kFlagTimeoutSelftest, limit_ns);
  } else {
    sm100::wait_counter_limit(counter, 1u, status, kFlagTimeoutSelftest, limit_ns);   // stays 0
  }
}

}  // namespace

cudaError_t launch_selftest_wait(uint32_t* status, const uint32_t* counter, int kind, uint64_t limit_ns,
                                 cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(status, counter, kind, limit_ns);
  count_launch();
  return cudaGetLastError();
}

}  // namespace qlora
