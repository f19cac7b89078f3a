// convrot_linear_checked: the int8-compute forward with the first-call check
// against the default path (Invoke docs "int8 Compute", "When something goes
// wrong": the first result for each layer shape and token-count bucket is
// compared with the default path's; on a mismatch or a failed kernel the GPU
// keeps the default path until restart, after one warning; "Memory": the check
// keeps 256 rows of the layer's output from each path).
//
// The pages give no match criterion.  Both paths share the int8 weight codes;
// they differ by the per-token activation quantization alone, which on the
// pages' layers keeps the output's cosine to an unquantized layer near
// 0.999.  The default threshold, cosine >= 0.99 on the checked rows, leaves
// that margin and still fails any broken kernel, whose output is uncorrelated
// with the default path's.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <set>
#include <tuple>
#include <vector>

#include "convrot.h"
#include "internal.h"

namespace {

// ---------------------------------------------------------------- comparison
// sums[0..2]: sum a*b, a*a, b*b over the outputs finite in both paths;
// sums[3]: outputs finite in the default path (b) but not in the int8 path (a).
constexpr int kCmpThreads = 256;

template <bool kF16>
__device__ __forceinline__ float widen(uint16_t v) {
  if constexpr (kF16) return __half2float(__ushort_as_half(v));
  return __uint_as_float(static_cast<uint32_t>(v) << 16);
}

template <bool kF16>
__global__ void __launch_bounds__(kCmpThreads)
    compare_outputs(const uint16_t* a, const uint16_t* b, int64_t n, double* sums) {
  double s[4] = {0.0, 0.0, 0.0, 0.0};
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kCmpThreads + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * kCmpThreads) {
    const float x = widen<kF16>(a[i]);
    const float y = widen<kF16>(b[i]);
    const bool fx = isfinite(x), fy = isfinite(y);
    if (fx && fy) {
      s[0] += static_cast<double>(x) * y;
      s[1] += static_cast<double>(x) * x;
      s[2] += static_cast<double>(y) * y;
    } else if (fy) {
      s[3] += 1.0;
    }
  }
  __shared__ double part[kCmpThreads / 32][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    for (int o = 16; o > 0; o >>= 1) s[j] += __shfl_down_sync(0xffffffffu, s[j], o);
  }
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
#pragma unroll
    for (int j = 0; j < 4; ++j) part[warp][j] = s[j];
  }
  __syncthreads();
  if (threadIdx.x < 4) {
    double t = 0.0;
    for (int w = 0; w < kCmpThreads / 32; ++w) t += part[w][threadIdx.x];
    atomicAdd(&sums[threadIdx.x], t);
  }
}

// ---------------------------------------------------------------- state
struct Key {
  int device;
  int64_t N, K;
  int G;
  int f16;
  int bucket;
  bool operator<(const Key& o) const {
    return std::tie(device, N, K, G, f16, bucket) < std::tie(o.device, o.N, o.K, o.G, o.f16, o.bucket);
  }
};

std::mutex g_mu;
std::set<Key> g_checked;
std::vector<int> g_latched;  // per device: 1 = default path until restart
double g_min_cosine = 0.99;

int bucket_of(int64_t M) {
  int b = 0;
  while ((int64_t(1) << b) < M) ++b;
  return b;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool is_latched(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  return dev < static_cast<int>(g_latched.size()) && g_latched[dev] != 0;
}

// Latches `dev` onto the default path; the first latch prints the one warning.
void latch(int dev, const char* reason) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (static_cast<int>(g_latched.size()) <= dev) g_latched.resize(dev + 1, 0);
  if (!g_latched[dev]) {
    g_latched[dev] = 1;
    std::fprintf(stderr,
                 "convrot: int8 compute disabled on CUDA device %d: %s; its ConvRot layers use the "
                 "default path (dequantize per forward) until the process restarts\n",
                 dev, reason);
  }
}

// ---------------------------------------------------------------- the two paths
struct Call {
  const uint16_t* x;
  bool f16;
  int64_t M, K, N;
  convrot_rotation_t R;
  const int8_t* Wq;
  const float* s_w;
  int64_t s_w_len;
  const uint16_t* bias;
  uint16_t* y;
  void* ws;
  size_t ws_bytes;
  convrot_stream_t stream;
};

convrot_status run_int8(const Call& c) {
  return c.f16 ? convrot_linear_int8_f16(c.x, c.M, c.K, c.N, c.R, c.Wq, c.s_w, c.s_w_len, c.bias,
                                         c.y, c.ws, c.ws_bytes, c.stream)
               : convrot_linear_int8(c.x, c.M, c.K, c.N, c.R, c.Wq, c.s_w, c.s_w_len, c.bias, c.y,
                                     c.ws, c.ws_bytes, c.stream);
}

// The default path for `rows` rows into `y`, decoding into `ws`.
convrot_status run_dequant(const Call& c, int64_t rows, uint16_t* y, void* ws, size_t ws_bytes) {
  return c.f16 ? convrot_linear_dequant_f16(c.x, rows, c.K, c.N, c.R, c.Wq, c.s_w, c.s_w_len,
                                            c.bias, y, ws, ws_bytes, c.stream)
               : convrot_linear_dequant(c.x, rows, c.K, c.N, c.R, c.Wq, c.s_w, c.s_w_len, c.bias, y,
                                        ws, ws_bytes, c.stream);
}

convrot_status fallback(const Call& c, int dev, const char* reason, int* path) {
  latch(dev, reason);
  const convrot_status s = run_dequant(c, c.M, c.y, c.ws, c.ws_bytes);
  if (s == CONVROT_OK && path) *path = CONVROT_PATH_DEQUANT;
  return s;
}

convrot_status cuda_error(cudaError_t e, const char* what) {
  return convrot::set_last_error(CONVROT_ERR_CUDA, "linear_checked: %s: %s", what,
                                 cudaGetErrorString(e));
}

// First call of a key: the int8 result is in c.y.  Runs the default path on
// the first rows and compares.  Sets *match; returns an error only when the
// comparison itself could not be made.
convrot_status check_against_default(const Call& c, bool* match, char* reason, size_t reason_len) {
  const int64_t rows = c.M < CONVROT_CHECK_ROWS ? c.M : CONVROT_CHECK_ROWS;
  const size_t w_bytes = round256(2 * static_cast<size_t>(c.N) * static_cast<size_t>(c.K));
  char* base = static_cast<char*>(c.ws);
  uint16_t* y_ref = reinterpret_cast<uint16_t*>(base + w_bytes);
  double* sums = reinterpret_cast<double*>(
      base + w_bytes + round256(2 * static_cast<size_t>(rows) * static_cast<size_t>(c.N)));
  convrot_status s = run_dequant(c, rows, y_ref, c.ws, w_bytes);
  if (s != CONVROT_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(c.stream);
  cudaError_t e = cudaMemsetAsync(sums, 0, 4 * sizeof(double), st);
  if (e != cudaSuccess) return cuda_error(e, "cudaMemsetAsync");
  const int64_t n = rows * c.N;
  const int64_t want = (n + kCmpThreads - 1) / kCmpThreads;
  const int blocks = static_cast<int>(want < 4 * convrot::sm_count() ? want : 4 * convrot::sm_count());
  if (c.f16) {
    compare_outputs<true><<<blocks, kCmpThreads, 0, st>>>(c.y, y_ref, n, sums);
  } else {
    compare_outputs<false><<<blocks, kCmpThreads, 0, st>>>(c.y, y_ref, n, sums);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "compare launch");
  double h[4] = {0.0, 0.0, 0.0, 0.0};
  e = cudaMemcpyAsync(h, sums, sizeof(h), cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_error(e, "cudaMemcpyAsync");
  // synchronizes; a timeout here belongs to the default path, which has no fallback
  s = convrot_check_status(c.stream);
  if (s != CONVROT_OK) return s;
  double cosine;
  if (h[1] == 0.0 || h[2] == 0.0) {
    cosine = (h[1] == 0.0 && h[2] == 0.0) ? 1.0 : 0.0;
  } else {
    cosine = h[0] / std::sqrt(h[1] * h[2]);
  }
  double threshold;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    threshold = g_min_cosine;
  }
  if (h[3] > 0.0) {
    *match = false;
    std::snprintf(reason, reason_len, "%.0f of the first %lld rows' outputs are not finite", h[3],
                  static_cast<long long>(rows));
  } else if (!(cosine >= threshold)) {
    *match = false;
    std::snprintf(reason, reason_len,
                  "on the first %lld rows of a [%lld, %lld] layer the cosine to the default path "
                  "is %.6f, below %.4f",
                  static_cast<long long>(rows), static_cast<long long>(c.N),
                  static_cast<long long>(c.K), cosine, threshold);
  } else {
    *match = true;
  }
  return CONVROT_OK;
}

convrot_status checked_impl(const Call& c, int* path) {
  if (path) *path = 0;
  if (c.M <= 0) {
    // M == 0 is a no-op; anything else gets the regular argument error
    const convrot_status s = run_int8(c);
    if (s == CONVROT_OK && path) *path = CONVROT_PATH_INT8;
    return s;
  }
  if (c.R == nullptr) {
    return convrot::set_last_error(CONVROT_ERR_INVALID_ARG, "rotation handle is NULL");
  }
  const size_t need = convrot_workspace_bytes(CONVROT_OP_LINEAR_CHECKED, c.M, c.N, c.K);
  if (c.ws == nullptr || c.ws_bytes < need) {
    return convrot::set_last_error(CONVROT_ERR_WORKSPACE,
                                   "linear_checked: workspace of %zu bytes given, %zu needed",
                                   c.ws_bytes, need);
  }
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (is_latched(dev)) {
    const convrot_status s = run_dequant(c, c.M, c.y, c.ws, c.ws_bytes);
    if (s == CONVROT_OK && path) *path = CONVROT_PATH_DEQUANT;
    return s;
  }
  const Key key{dev, c.N, c.K, c.R->G, c.f16 ? 1 : 0, bucket_of(c.M)};
  bool checked;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    checked = g_checked.count(key) != 0;
  }
  convrot_status s = run_int8(c);
  if (s == CONVROT_ERR_CUDA) {
    char reason[600];
    std::snprintf(reason, sizeof(reason), "an int8 kernel failed (%s)", convrot_last_error_string());
    return fallback(c, dev, reason, path);
  }
  if (s != CONVROT_OK) return s;  // argument errors latch nothing
  if (checked) {
    if (path) *path = CONVROT_PATH_INT8;
    return CONVROT_OK;
  }
  // first call of this key: did the int8 kernels finish, and do they agree?
  s = convrot_check_status(c.stream);
  if (s == CONVROT_ERR_TIMEOUT) {
    return fallback(c, dev, "an int8 kernel gave up a wait (timeout)", path);
  }
  if (s != CONVROT_OK) return s;  // the device itself reported an error: nothing to fall back on
  bool match = false;
  char reason[400] = "";
  s = check_against_default(c, &match, reason, sizeof(reason));
  if (s != CONVROT_OK) return s;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    g_checked.insert(key);
  }
  if (!match) return fallback(c, dev, reason, path);
  if (path) *path = CONVROT_PATH_INT8;
  return CONVROT_OK;
}

}  // namespace

extern "C" {

convrot_status convrot_linear_checked(const convrot_bf16* x, int64_t M, int64_t K, int64_t N,
                                      convrot_rotation_t R, const int8_t* Wq, const float* s_w,
                                      int64_t s_w_len, const convrot_bf16* bias, convrot_bf16* y,
                                      void* ws, size_t ws_bytes, int* path,
                                      convrot_stream_t stream) {
  return checked_impl(Call{x, false, M, K, N, R, Wq, s_w, s_w_len, bias, y, ws, ws_bytes, stream},
                      path);
}

convrot_status convrot_linear_checked_f16(const convrot_f16* x, int64_t M, int64_t K, int64_t N,
                                          convrot_rotation_t R, const int8_t* Wq, const float* s_w,
                                          int64_t s_w_len, const convrot_f16* bias, convrot_f16* y,
                                          void* ws, size_t ws_bytes, int* path,
                                          convrot_stream_t stream) {
  return checked_impl(Call{x, true, M, K, N, R, Wq, s_w, s_w_len, bias, y, ws, ws_bytes, stream},
                      path);
}

convrot_status convrot_check_state(int device, int* latched, int* checked_keys) {
  if (device < 0) {
    return convrot::set_last_error(CONVROT_ERR_INVALID_ARG, "device=%d is negative", device);
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (latched) *latched = device < static_cast<int>(g_latched.size()) ? g_latched[device] : 0;
  if (checked_keys) {
    int n = 0;
    for (const Key& k : g_checked) n += k.device == device ? 1 : 0;
    *checked_keys = n;
  }
  return CONVROT_OK;
}

void convrot_check_reset(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_checked.clear();
  g_latched.clear();
}

convrot_status convrot_check_set_min_cosine(double threshold) {
  if (!(threshold > 0.0 && threshold <= 1.5)) {
    return convrot::set_last_error(CONVROT_ERR_INVALID_ARG,
                                   "threshold=%g must be in (0, 1.5]", threshold);
  }
  std::lock_guard<std::mutex> lock(g_mu);
  g_min_cosine = threshold;
  return CONVROT_OK;
}

double convrot_check_min_cosine(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  return g_min_cosine;
}

}  // extern "C"
