// Host side of the C ABI declared in include/convrot.h: argument checks,
// rotation handles, dispatch to the kernels, status and error reporting.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "convrot.h"
#include "convrot_debug.h"
#include "internal.h"

namespace {

thread_local std::string g_last_error;

convrot_status fail(convrot_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

convrot_status cuda_fail(cudaError_t e, const char* what) {
  return fail(CONVROT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define CHECK_PTR(p)                                                                  \
  do {                                                                                \
    if ((p) == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "%s is NULL", #p);       \
    if (!aligned16(p)) return fail(CONVROT_ERR_ALIGNMENT, "%s is not 16-byte aligned", #p); \
  } while (0)

bool valid_group(int G) { return G == 4 || G == 16 || G == 64 || G == 256; }

// Current device, and whether it is an sm_100 part.
convrot_status current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  static std::mutex mu;
  static std::vector<int> ok;  // -1 unknown, 0 no, 1 yes
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(ok.size()) <= *dev) ok.resize(*dev + 1, -1);
  if (ok[*dev] < 0) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    ok[*dev] = (major == 10 && minor == 0) ? 1 : 0;
  }
  if (!ok[*dev]) {
    return fail(CONVROT_ERR_UNSUPPORTED, "device %d is not sm_100 (B200); the kernels are sm_100a",
                *dev);
  }
  return CONVROT_OK;
}

convrot_status check_rotation(convrot_rotation_t R) {
  if (R == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "rotation handle is NULL");
  int dev = -1;
  convrot_status s = current_device(&dev);
  if (s != CONVROT_OK) return s;
  if (dev != R->device) {
    return fail(CONVROT_ERR_INVALID_ARG, "rotation was created on device %d, current device is %d",
                R->device, dev);
  }
  return CONVROT_OK;
}

convrot_status check_rotation_shape(convrot_rotation_t R, int64_t K) {
  if (K <= 0 || K % R->G != 0 || K % 32 != 0) {
    return fail(CONVROT_ERR_INVALID_ARG, "K=%lld must be positive and a multiple of G=%d and of 32",
                static_cast<long long>(K), R->G);
  }
  return CONVROT_OK;
}

convrot_status launched(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return cuda_fail(e, what);
  return CONVROT_OK;
}

cudaStream_t as_stream(convrot_stream_t s) { return static_cast<cudaStream_t>(s); }

constexpr int64_t kMaxGemmK = 131072;
constexpr int64_t kMaxDim = int64_t(1) << 31;

convrot_status check_gemm_shape(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || M >= kMaxDim) return fail(CONVROT_ERR_INVALID_ARG, "M=%lld out of range", (long long)M);
  if (N <= 0 || N % 16 != 0 || N >= kMaxDim) {
    return fail(CONVROT_ERR_INVALID_ARG, "N=%lld must be a positive multiple of 16", (long long)N);
  }
  if (K <= 0 || K % 16 != 0) {
    return fail(CONVROT_ERR_INVALID_ARG, "K=%lld must be a positive multiple of 16", (long long)K);
  }
  if (K > kMaxGemmK) {
    return fail(CONVROT_ERR_UNSUPPORTED, "K=%lld exceeds %lld", (long long)K, (long long)kMaxGemmK);
  }
  return CONVROT_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

namespace convrot {
convrot_status set_last_error(convrot_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}
}  // namespace convrot

extern "C" {

int convrot_version(void) { return 100; }

int convrot_device_supported(int device) {
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return major == 10 && minor == 0;
}

const char* convrot_last_error_string(void) { return g_last_error.c_str(); }

convrot_status convrot_rotation_create(const float* R_host, int G, convrot_rotation_t* out) {
  if (out == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (R_host == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "R_host is NULL");
  if (!valid_group(G)) {
    return fail(CONVROT_ERR_UNSUPPORTED, "group size G=%d is not one of 4, 16, 64, 256", G);
  }
  // Orthogonality, in double precision on the host.
  double worst = 0.0;
  for (int i = 0; i < G; ++i) {
    for (int j = 0; j < G; ++j) {
      double d = 0.0;
      for (int k = 0; k < G; ++k) d += double(R_host[i * G + k]) * double(R_host[j * G + k]);
      worst = std::fmax(worst, std::fabs(d - (i == j ? 1.0 : 0.0)));
    }
  }
  if (!(worst <= 1e-5)) {
    return fail(CONVROT_ERR_INVALID_ARG, "R is not orthogonal: max |R R^T - I| = %g", worst);
  }
  // Sylvester-Hadamard H_G / sqrt(G): entry (i, j) = (-1)^popcount(i & j) / sqrt(G).
  const float mag = 1.0f / std::sqrt(static_cast<float>(G));  // exact for powers of 4
  bool sylvester = true;
  for (int i = 0; i < G && sylvester; ++i) {
    for (int j = 0; j < G; ++j) {
      const float h = (__builtin_popcount(static_cast<unsigned>(i & j)) & 1) ? -mag : mag;
      if (std::memcmp(&h, &R_host[i * G + j], sizeof(float)) != 0) {
        sylvester = false;
        break;
      }
    }
  }
  int dev = -1;
  convrot_status s = current_device(&dev);
  if (s != CONVROT_OK) return s;

  std::vector<float> Rt(static_cast<size_t>(G) * G);
  for (int i = 0; i < G; ++i)
    for (int j = 0; j < G; ++j) Rt[j * G + i] = R_host[i * G + j];

  auto* h = new (std::nothrow) convrot_rotation_s();
  if (!h) return fail(CONVROT_ERR_INVALID_ARG, "out of host memory");
  h->G = G;
  h->is_sylvester = sylvester ? 1 : 0;
  h->device = dev;
  const size_t bytes = sizeof(float) * G * G;
  cudaError_t e = cudaMalloc(&h->R_dev, 2 * bytes);
  if (e != cudaSuccess) {
    delete h;
    return cuda_fail(e, "cudaMalloc(R)");
  }
  h->Rt_dev = h->R_dev + G * G;
  e = cudaMemcpy(h->R_dev, R_host, bytes, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->Rt_dev, Rt.data(), bytes, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(h->R_dev);
    delete h;
    return cuda_fail(e, "cudaMemcpy(R)");
  }
  *out = h;
  return CONVROT_OK;
}

convrot_status convrot_rotation_destroy(convrot_rotation_t R) {
  if (R == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "rotation handle is NULL");
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(R->device);
  cudaDeviceSynchronize();
  cudaError_t e = cudaFree(R->R_dev);
  if (prev >= 0) cudaSetDevice(prev);
  delete R;
  if (e != cudaSuccess) return cuda_fail(e, "cudaFree(R)");
  return CONVROT_OK;
}

convrot_status convrot_rotation_info(convrot_rotation_t R, int* G, int* is_sylvester) {
  if (R == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "rotation handle is NULL");
  if (G) *G = R->G;
  if (is_sylvester) *is_sylvester = R->is_sylvester;
  return CONVROT_OK;
}

static convrot_status quantize_weight_impl(const uint16_t* W, bool f16, int64_t N, int64_t K,
                                           convrot_rotation_t R, int8_t* Wq, float* s_w,
                                           convrot_stream_t stream) {
  CHECK_PTR(W);
  CHECK_PTR(Wq);
  if (s_w == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "s_w is NULL");
  if (reinterpret_cast<uintptr_t>(s_w) & 3u) return fail(CONVROT_ERR_ALIGNMENT, "s_w misaligned");
  if (N <= 0 || N >= kMaxDim) return fail(CONVROT_ERR_INVALID_ARG, "N=%lld out of range", (long long)N);
  if (R == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "rotation handle is NULL");
  convrot_status s = check_rotation_shape(R, K);
  if (s != CONVROT_OK) return s;
  s = check_rotation(R);
  if (s != CONVROT_OK) return s;
  return launched(convrot::launch_quantize_weight(R, W, f16, N, K, Wq, s_w, as_stream(stream)),
                  "quantize_weight launch");
}

convrot_status convrot_quantize_weight(const convrot_bf16* W, int64_t N, int64_t K,
                                       convrot_rotation_t R, int8_t* Wq, float* s_w,
                                       convrot_stream_t stream) {
  return quantize_weight_impl(W, false, N, K, R, Wq, s_w, stream);
}

convrot_status convrot_quantize_weight_f16(const convrot_f16* W, int64_t N, int64_t K,
                                           convrot_rotation_t R, int8_t* Wq, float* s_w,
                                           convrot_stream_t stream) {
  return quantize_weight_impl(W, true, N, K, R, Wq, s_w, stream);
}

static convrot_status dequant_derotate_impl(const int8_t* Wq, const float* s_w, int64_t s_w_len,
                                            int64_t N, int64_t K, convrot_rotation_t R,
                                            uint16_t* W_hat, bool f16, convrot_stream_t stream) {
  CHECK_PTR(Wq);
  CHECK_PTR(W_hat);
  if (s_w == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "s_w is NULL");
  if (N <= 0 || N >= kMaxDim) return fail(CONVROT_ERR_INVALID_ARG, "N=%lld out of range", (long long)N);
  if (s_w_len != 1 && s_w_len != N) {
    return fail(CONVROT_ERR_INVALID_ARG, "s_w_len=%lld must be 1 or N=%lld", (long long)s_w_len,
                (long long)N);
  }
  if (R == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "rotation handle is NULL");
  convrot_status s = check_rotation_shape(R, K);
  if (s != CONVROT_OK) return s;
  s = check_rotation(R);
  if (s != CONVROT_OK) return s;
  return launched(
      convrot::launch_dequant_derotate(R, Wq, s_w, s_w_len, N, K, W_hat, f16, as_stream(stream)),
      "dequant_derotate launch");
}

convrot_status convrot_dequant_derotate(const int8_t* Wq, const float* s_w, int64_t s_w_len,
                                        int64_t N, int64_t K, convrot_rotation_t R,
                                        convrot_bf16* W_hat, convrot_stream_t stream) {
  return dequant_derotate_impl(Wq, s_w, s_w_len, N, K, R, W_hat, false, stream);
}

convrot_status convrot_dequant_derotate_f16(const int8_t* Wq, const float* s_w, int64_t s_w_len,
                                            int64_t N, int64_t K, convrot_rotation_t R,
                                            convrot_f16* W_hat, convrot_stream_t stream) {
  return dequant_derotate_impl(Wq, s_w, s_w_len, N, K, R, W_hat, true, stream);
}

static convrot_status rotate_quant_act_impl(const uint16_t* x, bool f16, int64_t M, int64_t K,
                                            convrot_rotation_t R, int8_t* xq, float* s_tok,
                                            convrot_stream_t stream) {
  if (M < 0 || M >= kMaxDim) return fail(CONVROT_ERR_INVALID_ARG, "M=%lld out of range", (long long)M);
  if (R == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "rotation handle is NULL");
  convrot_status s = check_rotation_shape(R, K);
  if (s != CONVROT_OK) return s;
  if (K > convrot::kMaxRotateK) {
    return fail(CONVROT_ERR_UNSUPPORTED, "K=%lld exceeds %lld", (long long)K,
                (long long)convrot::kMaxRotateK);
  }
  if (M == 0) return CONVROT_OK;
  CHECK_PTR(x);
  CHECK_PTR(xq);
  if (s_tok == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "s_tok is NULL");
  s = check_rotation(R);
  if (s != CONVROT_OK) return s;
  return launched(convrot::launch_rotate_quant_act(R, x, f16, M, K, xq, s_tok, as_stream(stream)),
                  "rotate_quant_act launch");
}

convrot_status convrot_rotate_quant_act(const convrot_bf16* x, int64_t M, int64_t K,
                                        convrot_rotation_t R, int8_t* xq, float* s_tok,
                                        convrot_stream_t stream) {
  return rotate_quant_act_impl(x, false, M, K, R, xq, s_tok, stream);
}

convrot_status convrot_rotate_quant_act_f16(const convrot_f16* x, int64_t M, int64_t K,
                                            convrot_rotation_t R, int8_t* xq, float* s_tok,
                                            convrot_stream_t stream) {
  return rotate_quant_act_impl(x, true, M, K, R, xq, s_tok, stream);
}

static convrot_status gemm_common(const int8_t* xq, const float* s_tok, const int8_t* Wq,
                                  const float* s_w, int64_t s_w_len, const uint16_t* bias,
                                  int64_t M, int64_t N, int64_t K, void* out, bool s32, bool f16,
                                  convrot_stream_t stream) {
  convrot_status s = check_gemm_shape(M, N, K);
  if (s != CONVROT_OK) return s;
  if (M == 0) return CONVROT_OK;
  CHECK_PTR(xq);
  CHECK_PTR(Wq);
  CHECK_PTR(out);
  if (!s32) {
    if (s_tok == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "s_tok is NULL");
    if (s_w == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "s_w is NULL");
    if (s_w_len != 1 && s_w_len != N) {
      return fail(CONVROT_ERR_INVALID_ARG, "s_w_len=%lld must be 1 or N=%lld",
                  (long long)s_w_len, (long long)N);
    }
    if (s_w_len == N && !aligned16(s_w)) {
      return fail(CONVROT_ERR_ALIGNMENT, "per-channel s_w is not 16-byte aligned");
    }
    if (bias != nullptr && !aligned16(bias)) {
      return fail(CONVROT_ERR_ALIGNMENT, "bias is not 16-byte aligned");
    }
  }
  int dev = -1;
  s = current_device(&dev);
  if (s != CONVROT_OK) return s;
  convrot::GemmArgs a;
  a.A = xq;
  a.B = Wq;
  a.s_tok = s_tok;
  a.s_w = s_w;
  a.s_w_len = s32 ? 1 : s_w_len;
  a.bias = s32 ? nullptr : bias;
  a.out = out;
  a.M = M;
  a.N = N;
  a.K = K;
  a.out_s32 = s32;
  a.out_f16 = f16 && !s32;
  cudaError_t e = convrot::launch_int8_gemm(a, as_stream(stream));
  if (e == cudaErrorInvalidValue) {
    return fail(CONVROT_ERR_CUDA, "int8_gemm: TMA descriptor encoding failed");
  }
  return launched(e, "int8_gemm launch");
}

convrot_status convrot_int8_gemm(const int8_t* xq, const float* s_tok, const int8_t* Wq,
                                 const float* s_w, int64_t s_w_len, const convrot_bf16* bias,
                                 int64_t M, int64_t N, int64_t K, convrot_bf16* y,
                                 convrot_stream_t stream) {
  return gemm_common(xq, s_tok, Wq, s_w, s_w_len, bias, M, N, K, y, false, false, stream);
}

convrot_status convrot_int8_gemm_f16(const int8_t* xq, const float* s_tok, const int8_t* Wq,
                                     const float* s_w, int64_t s_w_len, const convrot_f16* bias,
                                     int64_t M, int64_t N, int64_t K, convrot_f16* y,
                                     convrot_stream_t stream) {
  return gemm_common(xq, s_tok, Wq, s_w, s_w_len, bias, M, N, K, y, false, true, stream);
}

convrot_status convrot_int8_gemm_s32(const int8_t* xq, const int8_t* Wq, int64_t M, int64_t N,
                                     int64_t K, int32_t* acc, convrot_stream_t stream) {
  return gemm_common(xq, nullptr, Wq, nullptr, 1, nullptr, M, N, K, acc, true, false, stream);
}

static convrot_status dense_linear_impl(const uint16_t* x, bool f16, int64_t M, int64_t K,
                                        int64_t N, const uint16_t* W, const uint16_t* bias,
                                        uint16_t* y, convrot_stream_t stream) {
  convrot_status s = check_gemm_shape(M, N, K);
  if (s != CONVROT_OK) return s;
  if (M == 0) return CONVROT_OK;
  CHECK_PTR(x);
  CHECK_PTR(W);
  CHECK_PTR(y);
  if (bias != nullptr && !aligned16(bias)) {
    return fail(CONVROT_ERR_ALIGNMENT, "bias is not 16-byte aligned");
  }
  int dev = -1;
  s = current_device(&dev);
  if (s != CONVROT_OK) return s;
  convrot::GemmArgs a;
  a.A = nullptr;
  a.B = nullptr;
  a.s_tok = nullptr;
  a.s_w = nullptr;
  a.s_w_len = 1;
  a.bias = bias;
  a.out = y;
  a.M = M;
  a.N = N;
  a.K = K;
  a.out_s32 = false;
  a.out_f16 = f16;
  a.ops16 = true;
  a.A16 = x;
  a.B16 = W;
  cudaError_t e = convrot::launch_gemm16(a, as_stream(stream));
  if (e == cudaErrorInvalidValue) {
    return fail(CONVROT_ERR_CUDA, "dense_linear: TMA descriptor encoding failed");
  }
  return launched(e, "dense_linear launch");
}

convrot_status convrot_dense_linear(const convrot_bf16* x, int64_t M, int64_t K, int64_t N,
                                    const convrot_bf16* W, const convrot_bf16* bias,
                                    convrot_bf16* y, convrot_stream_t stream) {
  return dense_linear_impl(x, false, M, K, N, W, bias, y, stream);
}

convrot_status convrot_dense_linear_f16(const convrot_f16* x, int64_t M, int64_t K, int64_t N,
                                        const convrot_f16* W, const convrot_f16* bias,
                                        convrot_f16* y, convrot_stream_t stream) {
  return dense_linear_impl(x, true, M, K, N, W, bias, y, stream);
}

// Workspace of a slice of `rows` tokens: the int8 codes, then (256-byte
// aligned) the per-token scales.
static size_t slice_bytes(int64_t rows, int64_t K) {
  return align256(static_cast<size_t>(rows) * static_cast<size_t>(K)) +
         align256(sizeof(float) * static_cast<size_t>(rows));
}

// The decoded weight of the default path.
static size_t decoded_weight_bytes(int64_t N, int64_t K) {
  return align256(2 * static_cast<size_t>(N) * static_cast<size_t>(K));
}

size_t convrot_workspace_bytes(int op, int64_t M, int64_t N, int64_t K) {
  if (M < 0 || K < 0 || N < 0) return 0;
  if (op == CONVROT_OP_LINEAR_INT8) return slice_bytes(M, K);
  if (op == CONVROT_OP_LINEAR_INT8_SLICED) {
    const int64_t rows = M < 2 * N ? M : 2 * N;
    return slice_bytes(rows, K);
  }
  if (op == CONVROT_OP_LINEAR_DEQUANT) return decoded_weight_bytes(N, K);
  if (op == CONVROT_OP_LINEAR_CHECKED) {
    // the int8 forward's codes, or (reusing the same bytes once it is done)
    // the decoded weight, the default path's rows under check and the sums
    const int64_t rows = M < CONVROT_CHECK_ROWS ? M : CONVROT_CHECK_ROWS;
    const size_t check = decoded_weight_bytes(N, K) +
                         align256(2 * static_cast<size_t>(rows) * static_cast<size_t>(N)) + 256;
    const size_t fwd = slice_bytes(M, K);
    return fwd > check ? fwd : check;
  }
  return 0;
}

static convrot_status linear_dequant_impl(const uint16_t* x, bool f16, int64_t M, int64_t K,
                                          int64_t N, convrot_rotation_t R, const int8_t* Wq,
                                          const float* s_w, int64_t s_w_len, const uint16_t* bias,
                                          uint16_t* y, void* ws, size_t ws_bytes,
                                          convrot_stream_t stream) {
  convrot_status s = check_gemm_shape(M, N, K);
  if (s != CONVROT_OK) return s;
  if (M == 0) return CONVROT_OK;
  const size_t need = decoded_weight_bytes(N, K);
  if (ws == nullptr || ws_bytes < need) {
    return fail(CONVROT_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", ws_bytes, need);
  }
  if (reinterpret_cast<uintptr_t>(ws) & 255u) {
    return fail(CONVROT_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  }
  uint16_t* W_hat = static_cast<uint16_t*>(ws);
  s = dequant_derotate_impl(Wq, s_w, s_w_len, N, K, R, W_hat, f16, stream);
  if (s != CONVROT_OK) return s;
  return dense_linear_impl(x, f16, M, K, N, W_hat, bias, y, stream);
}

convrot_status convrot_linear_dequant(const convrot_bf16* x, int64_t M, int64_t K, int64_t N,
                                      convrot_rotation_t R, const int8_t* Wq, const float* s_w,
                                      int64_t s_w_len, const convrot_bf16* bias, convrot_bf16* y,
                                      void* ws, size_t ws_bytes, convrot_stream_t stream) {
  return linear_dequant_impl(x, false, M, K, N, R, Wq, s_w, s_w_len, bias, y, ws, ws_bytes, stream);
}

convrot_status convrot_linear_dequant_f16(const convrot_f16* x, int64_t M, int64_t K, int64_t N,
                                          convrot_rotation_t R, const int8_t* Wq, const float* s_w,
                                          int64_t s_w_len, const convrot_f16* bias, convrot_f16* y,
                                          void* ws, size_t ws_bytes, convrot_stream_t stream) {
  return linear_dequant_impl(x, true, M, K, N, R, Wq, s_w, s_w_len, bias, y, ws, ws_bytes, stream);
}

static convrot_status linear_int8_impl(const uint16_t* x, bool f16, int64_t M, int64_t K,
                                       int64_t N, convrot_rotation_t R, const int8_t* Wq,
                                       const float* s_w, int64_t s_w_len, const uint16_t* bias,
                                       uint16_t* y, void* ws, size_t ws_bytes,
                                       convrot_stream_t stream) {
  convrot_status s = check_gemm_shape(M, N, K);
  if (s != CONVROT_OK) return s;
  if (R == nullptr) return fail(CONVROT_ERR_INVALID_ARG, "rotation handle is NULL");
  s = check_rotation_shape(R, K);
  if (s != CONVROT_OK) return s;
  if (K > convrot::kMaxRotateK) {
    return fail(CONVROT_ERR_UNSUPPORTED, "K=%lld exceeds %lld", (long long)K,
                (long long)convrot::kMaxRotateK);
  }
  if (M == 0) return CONVROT_OK;
  if (ws == nullptr || ws_bytes < slice_bytes(1, K)) {
    return fail(CONVROT_ERR_WORKSPACE, "workspace of %zu bytes given, at least %zu needed",
                ws_bytes, slice_bytes(1, K));
  }
  if (reinterpret_cast<uintptr_t>(ws) & 255u) {
    return fail(CONVROT_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  }
  // as many tokens per slice as the workspace holds (all of M when it fits)
  int64_t rows = static_cast<int64_t>(ws_bytes / (static_cast<size_t>(K) + sizeof(float)));
  if (rows > M) rows = M;
  while (rows > 1 && slice_bytes(rows, K) > ws_bytes) --rows;
  int8_t* xq = static_cast<int8_t*>(ws);
  float* s_tok = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                          align256(static_cast<size_t>(rows) * static_cast<size_t>(K)));
  for (int64_t m0 = 0; m0 < M; m0 += rows) {
    const int64_t r = M - m0 < rows ? M - m0 : rows;
    s = rotate_quant_act_impl(x + m0 * K, f16, r, K, R, xq, s_tok, stream);
    if (s != CONVROT_OK) return s;
    s = gemm_common(xq, s_tok, Wq, s_w, s_w_len, bias, r, N, K, y + m0 * N, false, f16, stream);
    if (s != CONVROT_OK) return s;
  }
  return CONVROT_OK;
}

convrot_status convrot_linear_int8(const convrot_bf16* x, int64_t M, int64_t K, int64_t N,
                                   convrot_rotation_t R, const int8_t* Wq, const float* s_w,
                                   int64_t s_w_len, const convrot_bf16* bias, convrot_bf16* y,
                                   void* ws, size_t ws_bytes, convrot_stream_t stream) {
  return linear_int8_impl(x, false, M, K, N, R, Wq, s_w, s_w_len, bias, y, ws, ws_bytes, stream);
}

convrot_status convrot_linear_int8_f16(const convrot_f16* x, int64_t M, int64_t K, int64_t N,
                                       convrot_rotation_t R, const int8_t* Wq, const float* s_w,
                                       int64_t s_w_len, const convrot_f16* bias, convrot_f16* y,
                                       void* ws, size_t ws_bytes, convrot_stream_t stream) {
  return linear_int8_impl(x, true, M, K, N, R, Wq, s_w, s_w_len, bias, y, ws, ws_bytes, stream);
}

convrot_status convrot_selftest_wait_timeout(int limit_ms, convrot_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 1000) {
    return fail(CONVROT_ERR_INVALID_ARG, "limit_ms=%d must be in [1, 1000]", limit_ms);
  }
  int dev = -1;
  convrot_status s = current_device(&dev);
  if (s != CONVROT_OK) return s;
  return launched(convrot::launch_bounded_wait_selftest(
                      static_cast<uint64_t>(limit_ms) * 1000000ull, as_stream(stream)),
                  "selftest_wait_timeout launch");
}

convrot_status convrot_check_status(convrot_stream_t stream) {
  unsigned int st = 0;
  cudaError_t e = convrot::read_and_clear_status(&st, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "convrot_check_status");
  if (st & convrot::kStatusTimeout) {
    return fail(CONVROT_ERR_TIMEOUT, "a kernel gave up a bounded wait (timeout)");
  }
  if (st & convrot::kStatusBounds) {
    return fail(CONVROT_ERR_BOUNDS, "a kernel caught an out-of-range index and skipped it (debug build)");
  }
  return CONVROT_OK;
}

#if CONVROT_DEBUG
convrot_status convrot_debug_set_fault(int fault) {
  if (fault != CONVROT_FAULT_NONE && fault != CONVROT_FAULT_SKIP_STAGE &&
      fault != CONVROT_FAULT_SHORT_ROWS) {
    return fail(CONVROT_ERR_INVALID_ARG, "unknown fault %d", fault);
  }
  convrot::set_debug_fault(fault);
  return CONVROT_OK;
}
#endif

}  // extern "C"
