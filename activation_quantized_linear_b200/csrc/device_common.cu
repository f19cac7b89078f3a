// Host helpers shared by the kernels: TMA descriptor encoding, the SM count,
// and the per-device kernel status word that bounded waits report into.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

namespace convrot {

// bit 0: a bounded wait inside a kernel ran out
__device__ unsigned int g_kernel_status;

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
  });
  return fn;
}

}  // namespace

bool encode_tma_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                   uint64_t inner_elems, uint64_t rows, uint64_t row_stride_bytes,
                   uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner_elems, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  std::memset(map, 0, sizeof(*map));
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
std::atomic<int> g_debug_fault{0};  // only the debug library's test hook sets it
}  // namespace

int debug_fault() { return CONVROT_DEBUG ? g_debug_fault.load() : 0; }
void set_debug_fault(int code) { g_debug_fault.store(code); }

int sm_count() {
  static std::mutex mu;
  static std::vector<int> sms;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(sms.size()) <= dev) sms.resize(dev + 1, 0);
  if (sms[dev] <= 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    sms[dev] = n > 0 ? n : 148;
  }
  return sms[dev];
}

cudaError_t status_word(unsigned int** ptr) {
  static std::mutex mu;
  static std::vector<unsigned int*> addr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(addr.size()) <= dev) addr.resize(dev + 1, nullptr);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_kernel_status);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<unsigned int*>(p);
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

cudaError_t read_and_clear_status(unsigned int* status, cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_kernel_status, sizeof(v));
  if (e != cudaSuccess) return e;
  if (v) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_kernel_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return e;
  }
  *status = v;
  return cudaSuccess;
}

}  // namespace convrot
