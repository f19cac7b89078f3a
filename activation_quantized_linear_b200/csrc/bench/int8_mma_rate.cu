// Measured int8 tensor-core issue rate of this GPU: the cross-check for the
// int8 GEMM's roofline denominator (no counterpart on the pages, which
// measure on an RTX 4090; the denominator itself is the measured bf16 GEMM
// rate times the nominal int8 : bf16 ratio of 2).
//
// Measurement tooling, not part of the layer: this file builds into its own
// library (libconvrot_bench.so) that only the benchmark and its tests load;
// the layer's library (libconvrot.so, include/convrot.h) does not export it.
//
// C entry point (plain int status, the convrot_status numbering):
//   int convrot_bench_int8_mma_rate(int iters, double* tops, void* stream);
//   iters in [1, 200000] (32768 runs for about 10 ms), else 1 (invalid
//   argument, before any launch); 3 on a CUDA error; 5 if the kernel's
//   bounded wait ran out; 0 with `tops` (a HOST pointer) set.  Synchronizes
//   `stream` (a cudaStream_t, NULL for the legacy default stream).
//
// One CTA per SM issues back-to-back tcgen05.mma.kind::i8 instructions
// (M = 128, N = 256, K = 32; the single-CTA form of the GEMM's instruction)
// on operands that stay in shared memory, accumulating into one 256-column
// TMEM buffer; nothing is loaded or stored, so the rate is the tensor cores'
// alone, at whatever clock the power limit allows under that load.
#include <cuda_runtime.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace convrot {
namespace {

__device__ unsigned int g_probe_status;  // bit 0: the bounded wait ran out

constexpr int kPeakThreads = 64;
constexpr int kARows = 128, kBRows = 256, kRowBytes = 128;
constexpr int kOperandBytes = (kARows + kBRows) * kRowBytes;  // 48 KB
// more shared memory than two CTAs can share, so each SM runs one
constexpr size_t kPeakSmem = 1024 + 120 * 1024;
constexpr uint32_t kPeakTmemCols = 256;
constexpr uint64_t kPeakWaitNs = 2000000000ull;  // the loop is sized to a few ms

__global__ void __launch_bounds__(kPeakThreads, 1)
    int8_mma_issue_loop(int iters, unsigned int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t done;
  __shared__ uint32_t tmem_base;
  const int warp = threadIdx.x >> 5;

  // operands of pseudo-random bytes (a multiplicative hash of the offset):
  // zeros would toggle less logic and draw less power than real data, and
  // the rate under load is set by the power limit; then made visible to the
  // tensor cores' (async) proxy
  for (int i = threadIdx.x * 16; i < kOperandBytes; i += kPeakThreads * 16) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = (static_cast<uint32_t>(i / 4 + j) + 1u) * 2654435761u;
    *reinterpret_cast<uint4*>(smem + i) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  ptx::fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    ptx::mbar_init(&done, 1);
    ptx::fence_mbarrier_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(&tmem_base, kPeakTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (threadIdx.x == 32) {
    constexpr uint32_t kIdesc = ptx::idesc_i8(kARows, kBRows);
    const uint32_t a_addr = ptx::smem_u32(smem);
    const uint32_t b_addr = a_addr + kARows * kRowBytes;
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int k = 0; k < kRowBytes / 32; ++k) {
        ptx::mma_i8(tmem, ptx::smem_desc_k_sw128(a_addr + 32 * k),
                    ptx::smem_desc_k_sw128(b_addr + 32 * k), kIdesc, (i | k) != 0 ? 1u : 0u);
      }
    }
    ptx::mma_commit(&done);  // arrives once every MMA above has completed
  }
  __syncwarp();
  const bool ok = ptx::mbar_wait(&done, 0, ptx::globaltimer_ns() + kPeakWaitNs);
  if (!ok && threadIdx.x == 0) atomicOr(status, 1u);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(tmem, kPeakTmemCols);
}

cudaError_t measure(int iters, double* tops, cudaStream_t stream) {
  unsigned int* status = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_probe_status);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(status, 0, sizeof(unsigned int), stream);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(int8_mma_issue_loop, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kPeakSmem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  cudaEvent_t e0, e1;
  e = cudaEventCreate(&e0);
  if (e != cudaSuccess) return e;
  e = cudaEventCreate(&e1);
  if (e != cudaSuccess) {
    cudaEventDestroy(e0);
    return e;
  }
  // a short warm-up launch, then the timed one
  int8_mma_issue_loop<<<sms, kPeakThreads, kPeakSmem, stream>>>(iters / 8 + 1, status);
  cudaEventRecord(e0, stream);
  int8_mma_issue_loop<<<sms, kPeakThreads, kPeakSmem, stream>>>(iters, status);
  cudaEventRecord(e1, stream);
  e = cudaEventSynchronize(e1);
  float ms = 0.f;
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, e0, e1);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (e != cudaSuccess) return e;
  const double macs = static_cast<double>(sms) * iters * (kRowBytes / 32) * kARows * kBRows * 32.0;
  *tops = ms > 0.f ? 2.0 * macs / (ms * 1e-3) / 1e12 : 0.0;
  return cudaSuccess;
}

}  // namespace
}  // namespace convrot

extern "C" int convrot_bench_int8_mma_rate(int iters, double* tops, void* stream) {
  if (tops == nullptr || iters < 1 || iters > 200000) return 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (convrot::measure(iters, tops, st) != cudaSuccess) return 3;
  unsigned int status = 0;
  if (cudaMemcpyFromSymbol(&status, convrot::g_probe_status, sizeof(status)) != cudaSuccess) return 3;
  return (status & 1u) ? 5 : 0;
}
