// Block-diagonal rotation kernels of the ConvRot layer for sm_100a:
//   * per-token rotate + int8 quantize of activations (int8-compute step 1,
//     Invoke docs "int8 Compute", opening section),
//   * dequantize + derotate of an int8 weight to bf16 (default path,
//     InvokeAI-7 PR #194 "Summary"),
//   * offline weight quantization ("Quantizing AI Models with convert_to_quant",
//     "How INT8 ConvRot Quantization Works").
//
// Two implementations of the G x G product:
//   * R = H_G / sqrt(G) (Sylvester-Hadamard): an in-register fast Walsh-Hadamard
//     butterfly.  A thread owns 32 consecutive elements ("a chunk"): the
//     log2(min(G,32)) butterfly stages inside a chunk run in registers, the
//     remaining log2(G/32) stages pair chunks of neighbouring lanes through
//     warp shuffles.  The 1/sqrt(G) normalisation is a power of two and is
//     folded into the scales, so it never rounds.  These kernels are HBM-bound.
//   * any other orthogonal R: a shared-memory tiled product accumulated in
//     float64 (2G flops per element, ALU-bound; a correctness path).  Inputs
//     (bf16 or int8) and R (float32) are exact in float64, so each output is
//     the exact value up to one float64 rounding per term.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace convrot {
namespace {

constexpr int kChunk = 32;                 // elements one thread owns
constexpr float kRoundMagic = 12582912.0f; // 1.5 * 2^23: x + magic rounds x to an integer (RNE)
constexpr unsigned kFull = 0xffffffffu;

template <int G>
struct Norm {  // 1 / sqrt(G), exact
  static constexpr float value = G == 4 ? 0.5f : G == 16 ? 0.25f : G == 64 ? 0.125f : 0.0625f;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void load_bf16_chunk(const uint16_t* p, float (&v)[kChunk]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = __ldg(q + i);
    v[8 * i + 0] = bf16_lo(u.x);
    v[8 * i + 1] = bf16_hi(u.x);
    v[8 * i + 2] = bf16_lo(u.y);
    v[8 * i + 3] = bf16_hi(u.y);
    v[8 * i + 4] = bf16_lo(u.z);
    v[8 * i + 5] = bf16_hi(u.z);
    v[8 * i + 6] = bf16_lo(u.w);
    v[8 * i + 7] = bf16_hi(u.w);
  }
}

__device__ __forceinline__ void load_i8_chunk(const int8_t* p, float (&v)[kChunk]) {
  const int4* q = reinterpret_cast<const int4*>(p);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int4 u = __ldg(q + i);
    const int w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        v[16 * i + 4 * k + b] = static_cast<float>(static_cast<int8_t>((w[k] >> (8 * b)) & 0xff));
      }
    }
  }
}

// Butterfly stages whose partner lies in the same chunk (stride < min(G, 32)).
template <int G>
__device__ __forceinline__ void fwht_in_chunk(float (&v)[kChunk]) {
  constexpr int kTop = G < kChunk ? G : kChunk;
#pragma unroll
  for (int h = 1; h < kTop; h <<= 1) {
#pragma unroll
    for (int i = 0; i < kChunk; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
}

// Butterfly stages across the G/32 lanes that hold one group (G > 32).  Every
// lane of the warp must execute this (full-mask shuffles).
template <int G>
__device__ __forceinline__ void fwht_across_lanes(float (&v)[kChunk], uint32_t lane) {
#pragma unroll
  for (int m = 1; m < G / kChunk; m <<= 1) {
    const float sgn = (lane & m) ? -1.f : 1.f;  // upper partner keeps a - b
#pragma unroll
    for (int i = 0; i < kChunk; ++i) {
      const float p = __shfl_xor_sync(kFull, v[i], m);
      v[i] = fmaf(sgn, v[i], p);
    }
  }
}

template <int G>
__device__ __forceinline__ void fwht_chunk(float (&v)[kChunk], uint32_t lane) {
  fwht_in_chunk<G>(v);
  if constexpr (G > kChunk) fwht_across_lanes<G>(v, lane);
}

// Code of v * mul rounded half to even; |v * mul| <= 127.5 is required.
// Returns the code in the low byte (two's complement) of a 32-bit word.
__device__ __forceinline__ uint32_t round_code(float v, float mul) {
  return __float_as_uint(fmaf(v, mul, kRoundMagic));
}

__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// 32 codes of one chunk -> 32 bytes at dst (16-byte aligned).
__device__ __forceinline__ void store_codes(int8_t* dst, const float (&v)[kChunk], float mul) {
  uint32_t w[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    w[k] = pack4(round_code(v[4 * k], mul), round_code(v[4 * k + 1], mul),
                 round_code(v[4 * k + 2], mul), round_code(v[4 * k + 3], mul));
  }
  uint4* q = reinterpret_cast<uint4*>(dst);
  q[0] = make_uint4(w[0], w[1], w[2], w[3]);
  q[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// Slow but exact-division codes, for scales so small that 1/s overflows.
__device__ __forceinline__ void store_codes_div(int8_t* dst, const float (&v)[kChunk], float norm,
                                                float s) {
  uint32_t w[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t c[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      float q = rintf(__fdiv_rn(v[4 * k + b] * norm, s));
      q = fminf(fmaxf(q, -127.f), 127.f);
      c[b] = static_cast<uint32_t>(static_cast<int32_t>(q));
    }
    w[k] = pack4(c[0], c[1], c[2], c[3]);
  }
  uint4* q = reinterpret_cast<uint4*>(dst);
  q[0] = make_uint4(w[0], w[1], w[2], w[3]);
  q[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// bf16 bits of the exact product s * v rounded once to nearest-even.  The
// product is first rounded toward zero to float32 with the last bit forced to
// one when inexact ("round to odd"); rounding that to the 8-bit bf16 mantissa
// is then the correctly rounded result (float32 keeps >= 2 extra bits).
__device__ __forceinline__ float round_to_odd_product(float s, float v) {
  const float p = __fmul_rz(s, v);
  const float e = __fmaf_rn(s, v, -p);  // exact remainder
  return __uint_as_float(__float_as_uint(p) | (e != 0.f ? 1u : 0u));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float warp_max(float a) {
#pragma unroll
  for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, o));
  return a;
}

// ===========================================================================
// Sylvester path, activations: one team of `team_warps` warps per token.
// The token's rotated row stays in registers between the absmax and the pack.
// ===========================================================================
template <int G, int MAXC>
__global__ void __launch_bounds__(1024) rotate_quant_act_hadamard(
    const uint16_t* __restrict__ x, int64_t M, int K, int team_warps, int rows_per_cta,
    int8_t* __restrict__ xq, float* __restrict__ s_tok) {
  __shared__ float red[32];
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const int team = warp / team_warps;
  const int tpr = team_warps * 32;
  const int t = (warp % team_warps) * 32 + lane;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * rows_per_cta + team;
  const bool row_ok = row < M;  // uniform over the team
  const int nch = K / kChunk;
  const uint16_t* xr = x + row * K;

  float v[MAXC][kChunk];
#pragma unroll
  for (int j = 0; j < MAXC; ++j) {
    const int c = j * tpr + t;
    if (row_ok && c < nch) {
      load_bf16_chunk(xr + static_cast<int64_t>(c) * kChunk, v[j]);
    } else {
#pragma unroll
      for (int i = 0; i < kChunk; ++i) v[j][i] = 0.f;
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < MAXC; ++j) {
    fwht_chunk<G>(v[j], lane);
#pragma unroll
    for (int i = 0; i < kChunk; ++i) amax = fmaxf(amax, fabsf(v[j][i]));
  }
  amax = warp_max(amax);
  if (team_warps > 1) {
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = 0.f;
    for (int k = 0; k < team_warps; ++k) amax = fmaxf(amax, red[team * team_warps + k]);
  }
  if (!row_ok) return;

  constexpr float norm = Norm<G>::value;
  const float s = (amax * norm) / 127.f;  // s_tok = max |x_rot| / 127
  if (t == 0) s_tok[row] = s;
  const float inv = s > 0.f ? 1.f / s : 0.f;
  const float mul = norm * inv;  // exact: norm is a power of two
  int8_t* qr = xq + row * K;
  if (mul <= 3.0e38f) {
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
      const int c = j * tpr + t;
      if (c < nch) store_codes(qr + static_cast<int64_t>(c) * kChunk, v[j], mul);
    }
  } else {
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
      const int c = j * tpr + t;
      if (c < nch) store_codes_div(qr + static_cast<int64_t>(c) * kChunk, v[j], norm, s);
    }
  }
}

// ===========================================================================
// Sylvester path over a flat [rows, K] tensor, one chunk per thread per step.
// Groups never straddle rows (K % G == 0, K % 32 == 0).
// ===========================================================================
enum FlatMode { kFlatAbsmax = 0, kFlatQuant = 1, kFlatDequant = 2 };

template <int G, int MODE, bool PER_ROW_SCALE>
__global__ void __launch_bounds__(256) hadamard_flat(const void* __restrict__ in, int64_t nchunks,
                                                     int64_t chunks_per_row,
                                                     const float* __restrict__ scale,
                                                     void* __restrict__ out,
                                                     unsigned int* __restrict__ absmax_bits) {
  const uint32_t lane = threadIdx.x & 31;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t warp_stride = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  constexpr float norm = Norm<G>::value;
  float amax = 0.f;
  float mul = 0.f;
  if constexpr (MODE == kFlatQuant) {
    const float a = __uint_as_float(*absmax_bits);
    const float s = a / 127.f;
    mul = s > 0.f ? norm * (1.f / s) : 0.f;
  }
  for (int64_t base = warp_global * 32; base < nchunks; base += warp_stride * 32) {
    const int64_t c = base + lane;
    const bool ok = c < nchunks;
    float v[kChunk];
    if (ok) {
      if constexpr (MODE == kFlatDequant) {
        load_i8_chunk(static_cast<const int8_t*>(in) + c * kChunk, v);
      } else {
        load_bf16_chunk(static_cast<const uint16_t*>(in) + c * kChunk, v);
      }
    } else {
#pragma unroll
      for (int i = 0; i < kChunk; ++i) v[i] = 0.f;
    }
    fwht_chunk<G>(v, lane);
    if constexpr (MODE == kFlatAbsmax) {
#pragma unroll
      for (int i = 0; i < kChunk; ++i) amax = fmaxf(amax, fabsf(v[i]));
    } else if constexpr (MODE == kFlatQuant) {
      if (ok) store_codes(static_cast<int8_t*>(out) + c * kChunk, v, mul);
    } else {
      if (ok) {
        const float sw = PER_ROW_SCALE ? scale[c / chunks_per_row] : scale[0];
        const float sn = sw * norm;  // exact
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          w[k] = pack_bf16x2(round_to_odd_product(sn, v[2 * k]),
                             round_to_odd_product(sn, v[2 * k + 1]));
        }
        uint4* q = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + c * kChunk);
        q[0] = make_uint4(w[0], w[1], w[2], w[3]);
        q[1] = make_uint4(w[4], w[5], w[6], w[7]);
        q[2] = make_uint4(w[8], w[9], w[10], w[11]);
        q[3] = make_uint4(w[12], w[13], w[14], w[15]);
      }
    }
  }
  if constexpr (MODE == kFlatAbsmax) {
    __shared__ float red[8];
    amax = warp_max(amax);
    if (lane == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
      float m = 0.f;
      for (int k = 0; k < static_cast<int>(blockDim.x >> 5); ++k) m = fmaxf(m, red[k]);
      atomicMax(absmax_bits, __float_as_uint(m * norm));  // non-negative: bit order = value order
    }
  }
}

// ===========================================================================
// Dense-R path: out[r, :] = in[r, :] . Rm for every group-row r (G contiguous
// elements), Rm = R (rotation) or R^T (derotation).  A CTA computes 8192/G
// group-rows x G outputs; R is streamed through shared memory in 32-row slabs.
// ===========================================================================
enum DenseMode {
  kDenseAbsmaxRow = 0,    // absmax per token -> atomicMax(absmax_bits[token])
  kDenseAbsmaxAll = 1,    // one absmax for the tensor -> atomicMax(absmax_bits[0])
  kDenseQuantRow = 2,     // codes with the token's scale (absmax_bits[token] holds the absmax)
  kDenseQuantAll = 3,     // codes with the tensor scale
  kDenseDequant = 4,      // bf16 = RN(s_w * value)
};

template <int G, typename TIn, int MODE>
__global__ void __launch_bounds__(256) dense_rotate(const TIn* __restrict__ in, int64_t group_rows,
                                                    int64_t groups_per_token,
                                                    const float* __restrict__ Rm,
                                                    const float* __restrict__ scale,
                                                    int64_t scale_len, void* __restrict__ out,
                                                    unsigned int* __restrict__ absmax_bits) {
  constexpr int TC = G < 32 ? G : 32;  // threads along the output columns
  constexpr int CPT = G / TC;          // columns per thread
  constexpr int TR = 256 / TC;         // threads along the rows
  constexpr int TMR = 8192 / G;        // group-rows per CTA
  constexpr int RPT = TMR / TR;        // rows per thread
  constexpr int KC = G < 32 ? G : 32;  // R rows per slab

  extern __shared__ float smem[];
  float* xs = smem;             // [TMR][G]
  float* rs = smem + TMR * G;   // [KC][G]

  const int tx = threadIdx.x % TC;
  const int ty = threadIdx.x / TC;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * TMR;

  for (int i = threadIdx.x; i < TMR * G; i += 256) {
    const int64_t r = r0 + i / G;
    float val = 0.f;
    if (r < group_rows) {
      const TIn raw = in[r * G + (i % G)];
      if constexpr (sizeof(TIn) == 2) {
        val = __uint_as_float(static_cast<uint32_t>(raw) << 16);
      } else {
        val = static_cast<float>(raw);
      }
    }
    xs[i] = val;
  }

  double acc[RPT][CPT];
#pragma unroll
  for (int a = 0; a < RPT; ++a)
#pragma unroll
    for (int b = 0; b < CPT; ++b) acc[a][b] = 0.0;

  for (int k0 = 0; k0 < G; k0 += KC) {
    __syncthreads();
    for (int i = threadIdx.x; i < KC * G; i += 256) rs[i] = Rm[k0 * G + i];
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < KC; ++kk) {
      double rv[CPT];
#pragma unroll
      for (int b = 0; b < CPT; ++b) rv[b] = static_cast<double>(rs[kk * G + tx + b * TC]);
#pragma unroll
      for (int a = 0; a < RPT; ++a) {
        const double xv = static_cast<double>(xs[(ty + a * TR) * G + k0 + kk]);
#pragma unroll
        for (int b = 0; b < CPT; ++b) acc[a][b] = fma(xv, rv[b], acc[a][b]);
      }
    }
  }

#pragma unroll
  for (int a = 0; a < RPT; ++a) {
    const int64_t r = r0 + ty + a * TR;
    const bool ok = r < group_rows;
    if constexpr (MODE == kDenseAbsmaxRow || MODE == kDenseAbsmaxAll) {
      float m = 0.f;
#pragma unroll
      for (int b = 0; b < CPT; ++b) m = fmaxf(m, static_cast<float>(fabs(acc[a][b])));
#pragma unroll
      for (int o = TC / 2; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
      if (ok && tx == 0) {
        const int64_t idx = MODE == kDenseAbsmaxRow ? r / groups_per_token : 0;
        atomicMax(absmax_bits + idx, __float_as_uint(m));
      }
    } else if constexpr (MODE == kDenseQuantRow || MODE == kDenseQuantAll) {
      if (ok) {
        const int64_t idx = MODE == kDenseQuantRow ? r / groups_per_token : 0;
        // the code decision in float32: rne(float(x_rot) / s) with IEEE division
        const float s = __uint_as_float(absmax_bits[idx]) / 127.f;
        int8_t* q = static_cast<int8_t*>(out) + r * G;
#pragma unroll
        for (int b = 0; b < CPT; ++b) {
          float c = s > 0.f ? rintf(__fdiv_rn(static_cast<float>(acc[a][b]), s)) : 0.f;
          c = fminf(fmaxf(c, -127.f), 127.f);
          q[tx + b * TC] = static_cast<int8_t>(static_cast<int32_t>(c));
        }
      }
    } else {  // kDenseDequant
      if (ok) {
        const float sw = scale_len == 1 ? scale[0] : scale[r / groups_per_token];
        uint16_t* o = static_cast<uint16_t*>(out) + r * G;
#pragma unroll
        for (int b = 0; b < CPT; ++b) {
          const __nv_bfloat16 h = __double2bfloat16(static_cast<double>(sw) * acc[a][b]);
          o[tx + b * TC] = *reinterpret_cast<const uint16_t*>(&h);
        }
      }
    }
  }
}

// s[i] = absmax[i] / 127 (the absmax was accumulated in the same buffer as bits).
__global__ void finalize_scales(float* __restrict__ s, int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) s[i] = s[i] / 127.f;
}

template <int G>
cudaError_t rqa_hadamard(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* s_tok,
                         cudaStream_t stream) {
  // A token's row is held by a team of ceil(K / 1024) warps, one 32-element
  // chunk per lane (64 registers), so many teams stay resident per SM and the
  // load, butterfly and store phases of different teams overlap.
  const int nch = static_cast<int>(K / kChunk);
  const int team_warps = (nch + 31) / 32;
  const int rows_per_cta = team_warps >= 8 ? 1 : 8 / team_warps;
  const int64_t grid = (M + rows_per_cta - 1) / rows_per_cta;
  rotate_quant_act_hadamard<G, 1><<<static_cast<unsigned>(grid), 32 * team_warps * rows_per_cta,
                                    0, stream>>>(x, M, static_cast<int>(K), team_warps,
                                                 rows_per_cta, xq, s_tok);
  return cudaGetLastError();
}

template <int G, typename TIn, int MODE>
cudaError_t dense_launch(const TIn* in, int64_t group_rows, int64_t groups_per_token,
                         const float* Rm, const float* scale, int64_t scale_len, void* out,
                         unsigned int* absmax_bits, cudaStream_t stream) {
  constexpr int TMR = 8192 / G;
  constexpr int KC = G < 32 ? G : 32;
  const size_t smem = sizeof(float) * (TMR * G + KC * G);
  auto kern = dense_rotate<G, TIn, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t grid = (group_rows + TMR - 1) / TMR;
  kern<<<static_cast<unsigned>(grid), 256, smem, stream>>>(in, group_rows, groups_per_token, Rm,
                                                           scale, scale_len, out, absmax_bits);
  return cudaGetLastError();
}

template <int G, int MODE, bool PER_ROW>
cudaError_t flat_launch(const void* in, int64_t nchunks, int64_t chunks_per_row,
                        const float* scale, void* out, unsigned int* absmax_bits,
                        cudaStream_t stream) {
  const int64_t warps = (nchunks + 31) / 32;
  int64_t grid = (warps + 7) / 8;  // one chunk per thread
  if (grid < 1) grid = 1;
  hadamard_flat<G, MODE, PER_ROW><<<static_cast<unsigned>(grid), 256, 0, stream>>>(
      in, nchunks, chunks_per_row, scale, out, absmax_bits);
  return cudaGetLastError();
}

template <typename F>
cudaError_t by_group_size(int G, F&& f) {
  switch (G) {
    case 4: return f(std::integral_constant<int, 4>{});
    case 16: return f(std::integral_constant<int, 16>{});
    case 64: return f(std::integral_constant<int, 64>{});
    case 256: return f(std::integral_constant<int, 256>{});
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_rotate_quant_act(const convrot_rotation_s* R, const uint16_t* x, int64_t M,
                                    int64_t K, int8_t* xq, float* s_tok, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  if (R->is_sylvester) {
    return by_group_size(R->G, [&](auto g) {
      return rqa_hadamard<decltype(g)::value>(x, M, K, xq, s_tok, stream);
    });
  }
  unsigned int* amax = reinterpret_cast<unsigned int*>(s_tok);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float) * M, stream);
  if (e != cudaSuccess) return e;
  const int64_t gpt = K / R->G;
  e = by_group_size(R->G, [&](auto g) {
    constexpr int Gv = decltype(g)::value;
    cudaError_t r = dense_launch<Gv, uint16_t, kDenseAbsmaxRow>(x, M * gpt, gpt, R->R_dev, nullptr,
                                                                0, nullptr, amax, stream);
    if (r != cudaSuccess) return r;
    return dense_launch<Gv, uint16_t, kDenseQuantRow>(x, M * gpt, gpt, R->R_dev, nullptr, 0, xq,
                                                      amax, stream);
  });
  if (e != cudaSuccess) return e;
  finalize_scales<<<static_cast<unsigned>((M + 255) / 256), 256, 0, stream>>>(s_tok, M);
  return cudaGetLastError();
}

cudaError_t launch_dequant_derotate(const convrot_rotation_s* R, const int8_t* Wq,
                                    const float* s_w, int64_t s_w_len, int64_t N, int64_t K,
                                    uint16_t* W_hat, cudaStream_t stream) {
  if (R->is_sylvester) {
    const int64_t nchunks = N * K / kChunk;
    return by_group_size(R->G, [&](auto g) {
      constexpr int Gv = decltype(g)::value;
      if (s_w_len == 1) {
        return flat_launch<Gv, kFlatDequant, false>(Wq, nchunks, K / kChunk, s_w, W_hat, nullptr,
                                                    stream);
      }
      return flat_launch<Gv, kFlatDequant, true>(Wq, nchunks, K / kChunk, s_w, W_hat, nullptr,
                                                 stream);
    });
  }
  const int64_t gpt = K / R->G;
  return by_group_size(R->G, [&](auto g) {
    return dense_launch<decltype(g)::value, int8_t, kDenseDequant>(
        Wq, N * gpt, gpt, R->Rt_dev, s_w, s_w_len, W_hat, nullptr, stream);
  });
}

cudaError_t launch_quantize_weight(const convrot_rotation_s* R, const uint16_t* W, int64_t N,
                                   int64_t K, int8_t* Wq, float* s_w, cudaStream_t stream) {
  unsigned int* amax = reinterpret_cast<unsigned int*>(s_w);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), stream);
  if (e != cudaSuccess) return e;
  if (R->is_sylvester) {
    const int64_t nchunks = N * K / kChunk;
    e = by_group_size(R->G, [&](auto g) {
      constexpr int Gv = decltype(g)::value;
      cudaError_t r = flat_launch<Gv, kFlatAbsmax, false>(W, nchunks, K / kChunk, nullptr,
                                                          nullptr, amax, stream);
      if (r != cudaSuccess) return r;
      return flat_launch<Gv, kFlatQuant, false>(W, nchunks, K / kChunk, nullptr, Wq, amax,
                                                stream);
    });
  } else {
    const int64_t gpt = K / R->G;
    e = by_group_size(R->G, [&](auto g) {
      constexpr int Gv = decltype(g)::value;
      cudaError_t r = dense_launch<Gv, uint16_t, kDenseAbsmaxAll>(W, N * gpt, gpt, R->R_dev,
                                                                  nullptr, 0, nullptr, amax, stream);
      if (r != cudaSuccess) return r;
      return dense_launch<Gv, uint16_t, kDenseQuantAll>(W, N * gpt, gpt, R->R_dev, nullptr, 0, Wq,
                                                        amax, stream);
    });
  }
  if (e != cudaSuccess) return e;
  finalize_scales<<<1, 32, 0, stream>>>(s_w, 1);
  return cudaGetLastError();
}

}  // namespace convrot
