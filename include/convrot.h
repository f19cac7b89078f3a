/*
 * convrot.h -- C ABI of libconvrot, the ConvRot int8_tensorwise linear layer
 * for NVIDIA B200 (sm_100a).
 *
 * A ConvRot layer stores its weight W [N = out, K = in] as int8 codes with one
 * float32 scale per tensor, after a block-diagonal rotation B_R = diag(R, ..., R)
 * by an orthogonal G x G block R along the input dimension, G in {4, 16, 64, 256}
 * ("feat(quantization): share the int8_convrot scheme and read it for Krea-2 and
 * Z-Image", InvokeAI-7 PR #194, "Summary"; "Quantizing AI Models with
 * convert_to_quant", "How INT8 ConvRot Quantization Works" and "Determining the
 * Right ConvRot Group Size").  At run time the layer either
 *   - decodes the weight (dequantize + derotate) to bf16 and runs a dense
 *     matmul (the default path), or
 *   - in int8-compute mode rotates each token by the same R, quantizes it to
 *     int8 with one scale per token, multiplies int8 x int8 into int32 on the
 *     tensor cores and rescales to bf16 (Invoke docs, "int8 Compute").
 *
 * Conventions shared by every entry point:
 *   - Rotation direction: W_rot = W . B_R, x_rot = x . B_R, decode W_hat =
 *     s_w * Wq . B_R^T, so x_rot . W_rot^T = x . W^T.
 *   - All matrices are dense, row-major, with the contiguous dimension last:
 *     x [M, K], Wq [N, K], y [M, N].  bf16 tensors are passed as their 16-bit
 *     patterns (convrot_bf16).  Unless stated otherwise a pointer is a DEVICE
 *     pointer on the current CUDA device, 16-byte aligned.
 *   - The caller allocates and owns every tensor and workspace; the library
 *     owns only the device copy of R inside a rotation handle.  No entry point
 *     allocates device memory, except convrot_rotation_create.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL means the
 *     legacy default stream), except two that synchronize it and say so:
 *     convrot_check_status and the first call of a key in
 *     convrot_linear_checked.  Argument errors return at once, before any
 *     launch, and leave the outputs untouched.  A launch failure returns
 *     CONVROT_ERR_CUDA.  A wait inside a kernel that runs out of time (about a
 *     second) makes that kernel stop and record CONVROT_ERR_TIMEOUT in a device
 *     status word that convrot_check_status reports.
 *   - convrot_last_error_string() describes the last failure of this thread.
 *   - No C++ exception crosses this interface.
 */
#ifndef CONVROT_H_
#define CONVROT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum convrot_status {
  CONVROT_OK = 0,
  CONVROT_ERR_INVALID_ARG = 1,  /* null pointer, bad size, K % G != 0, non-orthogonal R, ... */
  CONVROT_ERR_UNSUPPORTED = 2,  /* device is not sm_100, G not in {4,16,64,256}, size limits */
  CONVROT_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  CONVROT_ERR_WORKSPACE = 4,    /* workspace missing or smaller than convrot_workspace_bytes() */
  CONVROT_ERR_TIMEOUT = 5,      /* a bounded wait inside a kernel ran out */
  CONVROT_ERR_ALIGNMENT = 6,    /* a pointer is not 16-byte aligned */
  CONVROT_ERR_BOUNDS = 7        /* debug library only (convrot_debug.h): a kernel caught an
                                   out-of-range index and skipped that access */
} convrot_status;

typedef uint16_t convrot_bf16;                     /* bfloat16 bit pattern */
typedef uint16_t convrot_f16;                      /* IEEE binary16 (fp16) bit pattern */
typedef void* convrot_stream_t;                    /* cudaStream_t */
typedef struct convrot_rotation_s* convrot_rotation_t;  /* opaque, owned by the library */

/* Workspace queries (convrot_workspace_bytes). */
#define CONVROT_OP_LINEAR_INT8 1         /* all M tokens in one pass */
#define CONVROT_OP_LINEAR_INT8_SLICED 2  /* slices of at most 2N tokens (see convrot_linear_int8) */
#define CONVROT_OP_LINEAR_DEQUANT 3      /* the decoded weight of convrot_linear_dequant */
#define CONVROT_OP_LINEAR_CHECKED 4      /* convrot_linear_checked, its first call included */

/* Library version, major * 10000 + minor * 100 + patch. */
int convrot_version(void);

/* 1 if CUDA device `device` is an sm_100 part the kernels are built for, else 0. */
int convrot_device_supported(int device);

/*
 * Rotation handle.  `R_host` is a HOST pointer to G*G float32 values, row-major
 * R[i][j] = R_host[i*G + j]; it is copied and may be freed after the call.
 * G must be 4, 16, 64 or 256 (powers of 4, "Determining the Right ConvRot Group
 * Size"; the loader in PR #10185 refuses any other group size), else
 * CONVROT_ERR_UNSUPPORTED.  R must be orthogonal: max |R R^T - I| <= 1e-5, else
 * CONVROT_ERR_INVALID_ARG.  The pages never say how R is built; when R equals
 * the normalized Sylvester-Hadamard matrix H_G / sqrt(G) bit for bit the kernels
 * use a fast Walsh-Hadamard butterfly, otherwise a dense G x G product.  The
 * handle's device data lives on the device current at creation; use it only
 * there.  Destroy with convrot_rotation_destroy (which synchronizes that device).
 */
convrot_status convrot_rotation_create(const float* R_host, int G, convrot_rotation_t* out);
convrot_status convrot_rotation_destroy(convrot_rotation_t R);
/* G and whether the butterfly path is used (1) or the dense path (0). */
convrot_status convrot_rotation_info(convrot_rotation_t R, int* G, int* is_sylvester);

/*
 * Offline weight quantization ("Quantizing AI Models with convert_to_quant",
 * "How INT8 ConvRot Quantization Works": --int8 --scaling_mode tensor --simple
 * --convrot --convrot-group-size G):
 *   W_rot = W . B_R;  s_w = max |W_rot| / 127;  Wq = clamp(rne(W_rot / s_w), -127, 127).
 * W [N, K] bf16 in; Wq [N, K] int8 and s_w (one float32, device) out.  K % G == 0,
 * K % 32 == 0, N >= 1.  s_w is used as the reduction target while the call runs.
 * An all-zero W gives s_w = 0 and zero codes.
 */
convrot_status convrot_quantize_weight(const convrot_bf16* W, int64_t N, int64_t K,
                                       convrot_rotation_t R, int8_t* Wq, float* s_w,
                                       convrot_stream_t stream);

/*
 * Default path, weight decode (PR #194 "Summary": each quantized layer
 * dequantizes and derotates per forward, the product [out, in/G, G] @ [G, G]):
 *   W_hat[n, :] = bf16_rn( s_w * Wq[n, :] . B_R^T ).
 * Wq [N, K] int8 and s_w (device) in; W_hat [N, K] bf16 out.  `s_w_len` is the
 * number of scales: 1 (per tensor) or N (one per output channel, applied along
 * the output axis).  K % G == 0, K % 32 == 0.  With the Sylvester R the result
 * is the correctly rounded bf16 of the exact value.
 */
convrot_status convrot_dequant_derotate(const int8_t* Wq, const float* s_w, int64_t s_w_len,
                                        int64_t N, int64_t K, convrot_rotation_t R,
                                        convrot_bf16* W_hat, convrot_stream_t stream);

/*
 * int8-compute step 1 (Invoke docs "int8 Compute", opening section: each layer
 * "rotates and quantizes its input to int8 per token"):
 *   x_rot = x[m, :] . B_R (float32);  s_tok[m] = max_k |x_rot| / 127;
 *   xq[m, :] = rne(x_rot / s_tok[m]) in [-127, 127]   (s_tok = 0 -> codes 0).
 * x [M, K] bf16 in; xq [M, K] int8 and s_tok [M] float32 out.  K % G == 0,
 * K % 32 == 0, K <= 32768, M >= 0 (M = 0 is a no-op).
 */
convrot_status convrot_rotate_quant_act(const convrot_bf16* x, int64_t M, int64_t K,
                                        convrot_rotation_t R, int8_t* xq, float* s_tok,
                                        convrot_stream_t stream);

/*
 * int8-compute steps 2-3 (Invoke docs "int8 Compute": "multiplies int8 by
 * int8" on the int8 tensor cores; outputs BF16):
 *   acc[m, n] = sum_k xq[m, k] * Wq[n, k]   (int32, exact)
 *   y[m, n]   = bf16_rn( float(acc) * (s_tok[m] * s_w[n or 0]) + bias[n] )
 * xq [M, K] int8, s_tok [M] f32, Wq [N, K] int8, s_w f32 (s_w_len = 1 or N),
 * bias [N] bf16 or NULL; y [M, N] bf16 out.  K % 16 == 0, K <= 131072,
 * N % 16 == 0, M >= 0.  No workspace is needed.
 */
convrot_status convrot_int8_gemm(const int8_t* xq, const float* s_tok, const int8_t* Wq,
                                 const float* s_w, int64_t s_w_len, const convrot_bf16* bias,
                                 int64_t M, int64_t N, int64_t K, convrot_bf16* y,
                                 convrot_stream_t stream);

/*
 * Diagnostic form of the GEMM above that stores the raw int32 accumulators
 * acc [M, N] instead of the rescaled bf16 output (same main loop, same limits).
 */
convrot_status convrot_int8_gemm_s32(const int8_t* xq, const int8_t* Wq, int64_t M, int64_t N,
                                     int64_t K, int32_t* acc, convrot_stream_t stream);

/*
 * The whole int8-compute forward (Invoke docs "int8 Compute"): rotate+quantize
 * x into the workspace, then the int8 GEMM with the fused epilogue.
 * x [M, K] bf16, Wq [N, K] int8, s_w (1 or N), bias [N] or NULL -> y [M, N] bf16.
 * `ws` (256-byte aligned) holds the int8 codes and per-token scales of a slice
 * of tokens: convrot_workspace_bytes(CONVROT_OP_LINEAR_INT8, M, N, K) bytes
 * take all M tokens in one pass; a smaller workspace makes the call process
 * the tokens in consecutive slices of as many rows as fit (the result is the
 * same bit for bit: every row is quantized and multiplied independently).
 * convrot_workspace_bytes(CONVROT_OP_LINEAR_INT8_SLICED, M, N, K) sizes slices
 * of at most 2N tokens, so that the codes never take more memory than the
 * N x K bf16 weight the default path decodes (Invoke docs "int8 Compute",
 * "Memory": the input is quantized in slices of at most twice the layer's
 * output width).  Less than one row's worth, or a misaligned workspace, is
 * CONVROT_ERR_WORKSPACE.  The same limits as the two steps apply.
 */
convrot_status convrot_linear_int8(const convrot_bf16* x, int64_t M, int64_t K, int64_t N,
                                   convrot_rotation_t R, const int8_t* Wq, const float* s_w,
                                   int64_t s_w_len, const convrot_bf16* bias, convrot_bf16* y,
                                   void* ws, size_t ws_bytes, convrot_stream_t stream);

/*
 * The int8-compute forward for callers that cannot allocate device memory.
 * (No counterpart on the pages: this is an interface of this library only.)
 * Callers such as a plugin inside a framework that owns all device memory and
 * offers its extensions no scratch allocator, or a serving path that must not
 * allocate (an allocation can synchronize the device and can fail with out of
 * memory mid-request), have no workspace to pass to convrot_linear_int8.  This
 * variant computes the same result with the same kernels, keeping the int8
 * codes and per-token scales in a static device array of
 * CONVROT_NOALLOC_SCRATCH_BYTES (32 MiB) that every GPU loading the library
 * holds until the process exits.  It allocates nothing itself.
 *   - Tokens whose codes and scales (round256(rows*K) + round256(4*rows)
 *     bytes) do not fit the array at once run in row slices, one after the
 *     other, with the same result.  Only a single token too large for it
 *     (round256(K) + 256 > CONVROT_NOALLOC_SCRATCH_BYTES, beyond any K the
 *     rotation accepts) is CONVROT_ERR_UNSUPPORTED.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and keeps it; make that first call before any
 *     stream capture, and do not call this entry point again after
 *     cudaDeviceReset in the same process (the kept address would be stale).
 *   - All calls share the array: calls that overlap on the GPU (other streams,
 *     other host threads) race and must be serialized by the caller.  Each call
 *     overwrites all of the scratch it reads, so nothing is carried over.
 *   - Other arguments, limits and errors are those of convrot_linear_int8.
 */
#define CONVROT_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
convrot_status convrot_linear_int8_noalloc(const convrot_bf16* x, int64_t M, int64_t K, int64_t N,
                                           convrot_rotation_t R, const int8_t* Wq,
                                           const float* s_w, int64_t s_w_len,
                                           const convrot_bf16* bias, convrot_bf16* y,
                                           convrot_stream_t stream);
/* Size of that static scratch in bytes (CONVROT_NOALLOC_SCRATCH_BYTES). */
size_t convrot_noalloc_scratch_bytes(void);

/*
 * The default path's matmul (Invoke docs "int8 Compute", opening section:
 * without int8 compute a layer unpacks its weight to BF16 or FP16 and
 * multiplies in that precision):
 *   y[m, n] = bf16_rn( sum_k x[m, k] * W[n, k] + bias[n] )
 * x [M, K] bf16, W [N, K] bf16 (typically W_hat of convrot_dequant_derotate),
 * bias [N] bf16 or NULL -> y [M, N] bf16.  The products are exact in fp32 and
 * are summed in fp32 on the tensor cores in an order of the kernel's choosing;
 * the bias is added in fp32 before the one rounding.  Limits: N % 16 == 0,
 * K % 16 == 0, K <= 131072, 16-byte aligned pointers; M == 0 is a no-op.
 */
convrot_status convrot_dense_linear(const convrot_bf16* x, int64_t M, int64_t K, int64_t N,
                                    const convrot_bf16* W, const convrot_bf16* bias,
                                    convrot_bf16* y, convrot_stream_t stream);

/*
 * The default path of a ConvRot int8 layer (Invoke docs "int8 Compute": a
 * layer that does not run in int8 dequantizes its weight on every forward):
 * convrot_dequant_derotate into the workspace, then convrot_dense_linear.
 * Arguments as convrot_linear_int8.  `ws` (256-byte aligned) holds the decoded
 * weight: convrot_workspace_bytes(CONVROT_OP_LINEAR_DEQUANT, M, N, K) =
 * 2*N*K rounded up to 256 bytes, else CONVROT_ERR_WORKSPACE.
 */
convrot_status convrot_linear_dequant(const convrot_bf16* x, int64_t M, int64_t K, int64_t N,
                                      convrot_rotation_t R, const int8_t* Wq, const float* s_w,
                                      int64_t s_w_len, const convrot_bf16* bias, convrot_bf16* y,
                                      void* ws, size_t ws_bytes, convrot_stream_t stream);

/*
 * The int8-compute forward with the first-call check against the default path
 * (Invoke docs "int8 Compute", "When something goes wrong" and "Memory"):
 *   - Calls are grouped by key: (device, N, K, G, 16-bit format, M bucket),
 *     with M bucket = ceil(log2(M)) (1 token: bucket 0).
 *   - The first call of a key runs convrot_linear_int8 into y, then the default
 *     path (convrot_linear_dequant) for the first R = min(M, CONVROT_CHECK_ROWS)
 *     rows, and compares the two on those R rows.  They match when no kernel
 *     reported a timeout, every y value is finite where the default path's is,
 *     and cosine(y, y_default) >= the threshold (convrot_check_min_cosine; the
 *     pages give none, the default is 0.99).  This call synchronizes `stream`
 *     and reads the device status word (convrot_check_status), so make it
 *     outside CUDA stream capture; it attributes any timeout recorded since
 *     the last status check to the int8 kernels.
 *   - On a mismatch, or when an int8-path launch fails, the call prints one
 *     warning to stderr, latches the device onto the default path for the rest
 *     of the process and overwrites y with the default path's result for all
 *     M rows.
 *   - Later calls of a checked key, on a device that is not latched, are
 *     convrot_linear_int8 (asynchronous); on a latched device every call is
 *     convrot_linear_dequant.
 *   - `path` (HOST pointer, may be NULL) receives CONVROT_PATH_INT8 or
 *     CONVROT_PATH_DEQUANT: the path whose result y holds.
 *   - `ws` (256-byte aligned): convrot_workspace_bytes(CONVROT_OP_LINEAR_CHECKED,
 *     M, N, K) bytes, the larger of the int8 forward's and the check's needs
 *     (the decoded weight, R rows of output and a few sums).
 * Argument errors are those of convrot_linear_int8 and latch nothing.
 */
#define CONVROT_CHECK_ROWS 256
#define CONVROT_PATH_INT8 1
#define CONVROT_PATH_DEQUANT 2
convrot_status convrot_linear_checked(const convrot_bf16* x, int64_t M, int64_t K, int64_t N,
                                      convrot_rotation_t R, const int8_t* Wq, const float* s_w,
                                      int64_t s_w_len, const convrot_bf16* bias, convrot_bf16* y,
                                      void* ws, size_t ws_bytes, int* path,
                                      convrot_stream_t stream);

/*
 * State of the check (host side, thread-safe).  convrot_check_state reports
 * for CUDA device `device` whether it is latched onto the default path (1/0)
 * and how many keys have been checked on it.  convrot_check_reset forgets
 * every checked key and latch on every device (as a restart would).
 * convrot_check_set_min_cosine sets the match threshold (0 < t <= 1.5; a value
 * above 1 makes every check fail, which lets a caller exercise the fallback
 * without a faulty kernel); convrot_check_min_cosine returns it.
 */
convrot_status convrot_check_state(int device, int* latched, int* checked_keys);
void convrot_check_reset(void);
convrot_status convrot_check_set_min_cosine(double threshold);
double convrot_check_min_cosine(void);

/*
 * fp16 forms.  The pages' int8 layers run with BF16 or FP16 activations and
 * refuse only FP32 (Invoke docs "int8 Compute": the opening section unpacks
 * each layer "to BF16 or FP16", and the table of layers that keep
 * dequantizing lists "Running in FP32" alone).  Each function below is its
 * bf16 namesake with every 16-bit float tensor in IEEE fp16 instead: the
 * input W or x is read exactly, and the outputs W_hat and y (and the bias) are
 * fp16, each value rounded once to nearest-even (fp16 overflow gives +-inf,
 * tiny values fp16 subnormals).  Arguments, limits and errors are the
 * namesake's; convrot_dequant_derotate_f16 is the correctly rounded fp16 of
 * the exact value with the Sylvester R.
 */
convrot_status convrot_quantize_weight_f16(const convrot_f16* W, int64_t N, int64_t K,
                                           convrot_rotation_t R, int8_t* Wq, float* s_w,
                                           convrot_stream_t stream);
convrot_status convrot_dequant_derotate_f16(const int8_t* Wq, const float* s_w, int64_t s_w_len,
                                            int64_t N, int64_t K, convrot_rotation_t R,
                                            convrot_f16* W_hat, convrot_stream_t stream);
convrot_status convrot_rotate_quant_act_f16(const convrot_f16* x, int64_t M, int64_t K,
                                            convrot_rotation_t R, int8_t* xq, float* s_tok,
                                            convrot_stream_t stream);
convrot_status convrot_int8_gemm_f16(const int8_t* xq, const float* s_tok, const int8_t* Wq,
                                     const float* s_w, int64_t s_w_len, const convrot_f16* bias,
                                     int64_t M, int64_t N, int64_t K, convrot_f16* y,
                                     convrot_stream_t stream);
convrot_status convrot_linear_int8_f16(const convrot_f16* x, int64_t M, int64_t K, int64_t N,
                                       convrot_rotation_t R, const int8_t* Wq, const float* s_w,
                                       int64_t s_w_len, const convrot_f16* bias, convrot_f16* y,
                                       void* ws, size_t ws_bytes, convrot_stream_t stream);
convrot_status convrot_dense_linear_f16(const convrot_f16* x, int64_t M, int64_t K, int64_t N,
                                        const convrot_f16* W, const convrot_f16* bias,
                                        convrot_f16* y, convrot_stream_t stream);
convrot_status convrot_linear_dequant_f16(const convrot_f16* x, int64_t M, int64_t K, int64_t N,
                                          convrot_rotation_t R, const int8_t* Wq, const float* s_w,
                                          int64_t s_w_len, const convrot_f16* bias, convrot_f16* y,
                                          void* ws, size_t ws_bytes, convrot_stream_t stream);
convrot_status convrot_linear_checked_f16(const convrot_f16* x, int64_t M, int64_t K, int64_t N,
                                          convrot_rotation_t R, const int8_t* Wq, const float* s_w,
                                          int64_t s_w_len, const convrot_f16* bias, convrot_f16* y,
                                          void* ws, size_t ws_bytes, int* path,
                                          convrot_stream_t stream);

/* Bytes of workspace an operation needs (0 if none); 0 for an unknown op. */
size_t convrot_workspace_bytes(int op, int64_t M, int64_t N, int64_t K);

/*
 * Synchronizes `stream`, then reads and clears the current device's status
 * word: CONVROT_ERR_TIMEOUT if a kernel gave up a wait since the last check,
 * CONVROT_ERR_BOUNDS if (debug library only) a kernel caught an out-of-range
 * index, CONVROT_ERR_CUDA if the synchronization reported an error, else
 * CONVROT_OK.
 */
convrot_status convrot_check_status(convrot_stream_t stream);

/*
 * Failure-detection self-test (no counterpart on the pages: it tests this
 * library's own timeout reporting).  Enqueues one small kernel whose bounded
 * wait can never be satisfied: it gives up after `limit_ms` milliseconds
 * (1..1000, else CONVROT_ERR_INVALID_ARG) and records a timeout in the
 * device status word, as a kernel whose pipeline stalled would.  Returns
 * CONVROT_OK once enqueued; the next convrot_check_status on the stream then
 * reports CONVROT_ERR_TIMEOUT and clears the word.  Nothing faults or hangs,
 * and the context stays usable.
 */
convrot_status convrot_selftest_wait_timeout(int limit_ms, convrot_stream_t stream);

/* Message of the last failure on the calling thread ("" if none). */
const char* convrot_last_error_string(void);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif /* CONVROT_H_ */
