// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "convrot.h"

struct convrot_rotation_s {
  int G;
  int is_sylvester;   // R == H_G / sqrt(G) bit for bit
  int device;         // device holding R_dev / Rt_dev
  float* R_dev;       // [G, G] row-major
  float* Rt_dev;      // R transposed
};

// CONVROT_DEBUG=1 builds the debug library (libconvrot_debug.so): every
// kernel checks the indices of its global stores and scale/bias reads
// against the tensors' sizes, records a violation in bit 1 of the device
// status word (convrot_check_status: CONVROT_ERR_BOUNDS) and skips the access
// instead of trapping; and the host can inject faults for the tests
// (convrot_debug_set_fault).  The release library compiles all of it out.
#ifndef CONVROT_DEBUG
#define CONVROT_DEBUG 0
#endif

namespace convrot {

// Device status word bits.
constexpr unsigned int kStatusTimeout = 1u;  // a bounded wait ran out
constexpr unsigned int kStatusBounds = 2u;   // debug build: an index was out of range

// Faults the debug library's tests inject from the host (0 = none).  The
// launchers pass the current code to their kernels; the release library never
// sets it.
enum DebugFault : int {
  kFaultNone = 0,
  kFaultSkipStage = 1,   // int8 GEMM producers skip their first ring stage
  kFaultShortRows = 2,   // kernels check stores against one token / row fewer
};
int debug_fault();
void set_debug_fault(int code);

// In the debug build: false (and bit 1 of the status word set) when `ok` is
// false; the caller skips the access.  In the release build always true.
__device__ __forceinline__ bool in_bounds(bool ok, unsigned int* status) {
#if CONVROT_DEBUG
  if (!ok) atomicOr(status, kStatusBounds);
  return ok;
#else
  (void)status;
  return true;
#endif
}

// ------------------------------------------------------------------ rotations
// Each launcher enqueues on `stream` and returns the launch error (cudaSuccess
// when the kernels were enqueued).  Arguments are validated by the caller.

// x [M, K] bf16 (f16 = false) or fp16 -> xq [M, K] int8, s_tok [M] f32
// (per-token scale).
cudaError_t launch_rotate_quant_act(const convrot_rotation_s* R, const uint16_t* x, bool f16,
                                    int64_t M, int64_t K, int8_t* xq, float* s_tok,
                                    cudaStream_t stream);

// Wq [N, K] int8 -> W_hat [N, K] bf16 (f16 = false) or fp16, scale s_w[0]
// (s_w_len == 1) or s_w[n].
cudaError_t launch_dequant_derotate(const convrot_rotation_s* R, const int8_t* Wq,
                                    const float* s_w, int64_t s_w_len, int64_t N, int64_t K,
                                    uint16_t* W_hat, bool f16, cudaStream_t stream);

// W [N, K] bf16 (f16 = false) or fp16 -> Wq [N, K] int8, s_w[0] (one
// per-tensor scale).
cudaError_t launch_quantize_weight(const convrot_rotation_s* R, const uint16_t* W, bool f16,
                                   int64_t N, int64_t K, int8_t* Wq, float* s_w,
                                   cudaStream_t stream);

// ------------------------------------------------------------------ GEMM
struct GemmArgs {
  const int8_t* A;       // xq [M, K]
  const int8_t* B;       // Wq [N, K]
  const float* s_tok;    // [M]          (16-bit float output only)
  const float* s_w;      // [1] or [N]   (16-bit float output only)
  int64_t s_w_len;
  const uint16_t* bias;  // [N] or null, in the output's format
  void* out;             // y [M, N] bf16 / fp16, or int32 acc [M, N]
  int64_t M, N, K;
  bool out_s32;
  bool out_f16;          // y and bias are fp16 (else bf16)
  // 16-bit operands (launch_gemm16): x [M, K] and W [N, K] in y's format
  bool ops16 = false;
  const uint16_t* A16 = nullptr;
  const uint16_t* B16 = nullptr;
};

// Encodes the TMA descriptors and launches the tcgen05 GEMM.  Returns
// cudaErrorInvalidValue if a tensor map cannot be encoded.
cudaError_t launch_int8_gemm(const GemmArgs& a, cudaStream_t stream);

// The few-token variant (M <= 128): swap-AB with the K split over a cluster;
// up to kGemvMaxTokens tokens it hands over to the dp4a product below.
cudaError_t launch_int8_gemm_skinny(const GemmArgs& a, cudaStream_t stream);

// One or two tokens, whose codes (rounded up to 1 or 2 token rows of K bytes)
// fit kGemvMaxCodeBytes of shared memory: warps streaming whole weight rows
// with dp4a (int8_gemv.cu).  Same results as the tensor-core GEMMs.  (At 4
// and 8 tokens the per-token dot products made it slower than the swap-AB
// kernel on every measured weight.)
constexpr int kGemvMaxTokens = 2;
constexpr int64_t kGemvMaxCodeBytes = 64 << 10;
bool int8_gemv_applies(const GemmArgs& a);
cudaError_t launch_int8_gemv(const GemmArgs& a, cudaStream_t stream);

// y = f16(x W^T + bias) with 16-bit operands (a.ops16, a.A16, a.B16; bf16 or
// fp16 as a.out_f16), fp32 accumulation on the same CTA-pair pipeline.
cudaError_t launch_gemm16(const GemmArgs& a, cudaStream_t stream);

// Enqueues the failure-detection self-test: a bounded wait that runs out
// after `limit_ns` and records a timeout in the status word.
cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, cudaStream_t stream);

// Reads and clears the current device's kernel status word (0 = fine).
cudaError_t read_and_clear_status(unsigned int* status, cudaStream_t stream);

// Device address of the current device's kernel status word (kernels that
// give up a bounded wait atomically OR bit 0 into it).
cudaError_t status_word(unsigned int** ptr);

// 2-D tiled TMA descriptor with 128-byte swizzle and zero fill outside the
// tensor: `rows` rows of `inner_elems` elements, rows `row_stride_bytes` apart,
// box of `box_rows` x `box_inner` elements.
bool encode_tma_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                   uint64_t inner_elems, uint64_t rows, uint64_t row_stride_bytes,
                   uint32_t box_inner, uint32_t box_rows);

// Number of SMs of the current device.
int sm_count();

// Records `fmt` as the calling thread's last error message and returns `s`.
convrot_status set_last_error(convrot_status s, const char* fmt, ...);

// Largest K the rotate+quantize kernel keeps on chip for one token.
constexpr int64_t kMaxRotateK = 32768;  // 32 warps x 32 lanes x 32 elements

}  // namespace convrot
