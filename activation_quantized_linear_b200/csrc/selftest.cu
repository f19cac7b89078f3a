// Failure-detection self-test: a kernel whose bounded wait can never be
// satisfied, so that the host side of timeout reporting (the device status
// word, convrot_check_status) can be exercised without hanging or faulting a
// GPU.  The wait is bounded twice: by %globaltimer and by an iteration count.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace convrot {
namespace {

// Non-blocking probe of an mbarrier phase.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(ptx::smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// One thread waits for an arrival on an mbarrier that expects one and gets
// none.  It gives up after `limit_ns` of %globaltimer, or after 2^21 polls
// about 1 us apart, and then reports the timeout like a stalled GEMM stage.
__global__ void bounded_wait_selftest(unsigned int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  ptx::mbar_init(&bar, 1);
  ptx::fence_mbarrier_init();
  const uint64_t deadline = ptx::globaltimer_ns() + limit_ns;
  bool done = false;
  for (uint32_t i = 0; i < (1u << 21) && !done; ++i) {
    done = mbar_test_wait(&bar, 0);
    if (!done) {
      if (ptx::globaltimer_ns() > deadline) break;
      __nanosleep(1000);
    }
  }
  if (!done) atomicOr(status, 1u);
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, cudaStream_t stream) {
  unsigned int* status = nullptr;
  cudaError_t e = status_word(&status);
  if (e != cudaSuccess) return e;
  bounded_wait_selftest<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace convrot
