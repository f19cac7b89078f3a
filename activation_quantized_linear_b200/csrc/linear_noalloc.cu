// convrot_linear_int8_noalloc: the int8-compute forward for callers that
// cannot allocate device memory.
//
// Some callers of this library are not allowed to call cudaMalloc and have no
// workspace to hand over: a plugin or custom operator running inside a host
// framework that owns every byte of device memory and gives its extensions no
// scratch allocator, or a latency-critical serving path where an allocation
// (which can synchronize the device and can fail with out-of-memory halfway
// through a request) is forbidden.  convrot_linear_int8 needs a caller-supplied
// workspace for the int8 codes and the per-token scales between its two
// kernels; this entry point keeps that intermediate in a fixed-size array of
// static device memory instead, so the caller passes only inputs and outputs.
//
// The array lives in every GPU that loads the library, until the process
// exits.  A batch whose codes do not fit it runs in row slices, as
// convrot_linear_int8 does with a small workspace.  All calls share it and it
// keeps the previous call's contents; the kernels overwrite every byte they
// read, so nothing needs clearing between calls, but two calls that run at the
// same time on the GPU (different streams or threads) race on it and must be
// serialized by the caller.  Its device address is looked up once per device
// and kept: after cudaDeviceReset the entry point must not be called again in
// that process (the old address would be stale).
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <vector>

#include "convrot.h"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = CONVROT_NOALLOC_SCRATCH_BYTES;

// The scratch: int8 codes [rows, K] at offset 0, per-token scales [rows] after
// them (256-byte aligned), rows = as many tokens as fit.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Device address of the scratch on the current device, looked up once per
// device.  In host code g_noalloc_scratch names a host-side shadow, not device
// memory, so the address must come from cudaGetSymbolAddress.
cudaError_t scratch_address(void** out) {
  static std::mutex mu;
  static std::vector<void*> addr;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(addr.size()) <= dev) addr.resize(dev + 1, nullptr);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" size_t convrot_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" convrot_status convrot_linear_int8_noalloc(const convrot_bf16* x, int64_t M, int64_t K,
                                                      int64_t N, convrot_rotation_t R,
                                                      const int8_t* Wq, const float* s_w,
                                                      int64_t s_w_len, const convrot_bf16* bias,
                                                      convrot_bf16* y, convrot_stream_t stream) {
  if (M <= 0 || K <= 0) {
    // M == 0 is a no-op; negative or empty sizes get the regular argument error.
    return convrot_linear_int8(x, M, K, N, R, Wq, s_w, s_w_len, bias, y, nullptr, 0, stream);
  }
  // one token's codes and scale must fit; more tokens run in row slices
  const size_t need = round256(static_cast<size_t>(K)) + round256(sizeof(float));
  if (need > kNoAllocScratchBytes) {
    return convrot::set_last_error(
        CONVROT_ERR_UNSUPPORTED,
        "linear_int8_noalloc: one token's codes and scale (%zu bytes) exceed the static "
        "scratch of %zu bytes; call convrot_linear_int8 with a workspace instead",
        need, kNoAllocScratchBytes);
  }
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    return convrot::set_last_error(CONVROT_ERR_CUDA,
                                   "linear_int8_noalloc: cudaGetSymbolAddress: %s",
                                   cudaGetErrorString(e));
  }
  return convrot_linear_int8(x, M, K, N, R, Wq, s_w, s_w_len, bias, y, scratch,
                             kNoAllocScratchBytes, stream);
}
