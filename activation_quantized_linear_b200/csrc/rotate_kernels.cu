// Block-diagonal rotation kernels of the ConvRot layer for sm_100a:
//   * per-token rotate + int8 quantize of activations (int8-compute step 1,
//     Invoke docs "int8 Compute", opening section),
//   * dequantize + derotate of an int8 weight to bf16 (default path,
//     InvokeAI-7 PR #194 "Summary"),
//   * offline weight quantization ("Quantizing AI Models with convert_to_quant",
//     "How INT8 ConvRot Quantization Works").
//
// Two implementations of the G x G product:
//   * R = H_G / sqrt(G) (Sylvester-Hadamard): a fast Walsh-Hadamard butterfly.
//     A lane owns 32 consecutive elements as 16 packed float pairs and runs the
//     butterfly stages two elements per instruction (sm_100 f32x2 arithmetic);
//     for G = 256 the last three stages follow one exchange through shared
//     memory, for G = 64 the last one a warp shuffle.  All loads are issued
//     before any arithmetic and many warps stay resident.  The 1/sqrt(G) factor
//     is a power of two folded into the scales, so it never rounds.  These
//     kernels are HBM-bound.
//   * any other orthogonal R: a shared-memory tiled product accumulated in
//     float64 (2G flops per element, ALU-bound; a correctness path).  Inputs
//     (bf16 or int8) and R (float32) are exact in float64, so each output is
//     the exact value up to one float64 rounding per term.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace convrot {
namespace {

constexpr int kVec = 32;                   // elements one thread owns
constexpr int kPairs = kVec / 2;           // held as 16 packed float pairs (2i, 2i + 1)
constexpr float kRoundMagic = 12582912.0f; // 1.5 * 2^23: x + magic rounds x to an integer (RNE)
constexpr unsigned kFull = 0xffffffffu;

template <int G>
struct Norm {  // 1 / sqrt(G), exact
  static constexpr float value = G == 4 ? 0.5f : G == 16 ? 0.25f : G == 64 ? 0.125f : 0.0625f;
};

// ---------------------------------------------------------------- packed pairs
// sm_100 executes two float32 operations per instruction on a 64-bit register
// pair; the butterflies, the scaling and the code rounding use these forms.
// A pair is a 64-bit register pair; pack and unpack only name its halves.
__device__ __forceinline__ uint64_t pk(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ uint64_t pku(uint32_t lo, uint32_t hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
  return d;
}
__device__ __forceinline__ void unpk(uint64_t p, uint32_t& lo, uint32_t& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(p));
}
__device__ __forceinline__ float plo(uint64_t p) {
  uint32_t lo, hi;
  unpk(p, lo, hi);
  return __uint_as_float(lo);
}
__device__ __forceinline__ float phi(uint64_t p) {
  uint32_t lo, hi;
  unpk(p, lo, hi);
  return __uint_as_float(hi);
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t mulrz2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// ---------------------------------------------------------------- shared memory
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void sts64(uint32_t addr, uint64_t a) {
  asm volatile("st.shared.b64 [%0], %1;" ::"r"(addr), "l"(a) : "memory");
}
__device__ __forceinline__ uint64_t lds64(uint32_t addr) {
  uint64_t a;
  asm volatile("ld.shared.b64 %0, [%1];" : "=l"(a) : "r"(addr) : "memory");
  return a;
}

// ---------------------------------------------------------------- loads
// raw words -> P[i] = (p[2i], p[2i + 1]) as floats.
__device__ __forceinline__ void widen_bf16_32(const uint4 (&u)[4], uint64_t (&P)[kPairs]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t w[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      P[4 * j + k] = pku(w[k] << 16, w[k] & 0xffff0000u);
    }
  }
}

// raw fp16 words -> P[i] = (p[2i], p[2i + 1]) as floats (exact).
__device__ __forceinline__ void widen_f16_32(const uint4 (&u)[4], uint64_t (&P)[kPairs]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t w[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
      P[4 * j + k] = pk(f.x, f.y);
    }
  }
}

// 16-bit float input: bf16 (kF16 = false) or fp16 (kF16 = true).
template <bool kF16>
__device__ __forceinline__ void widen16_32(const uint4 (&u)[4], uint64_t (&P)[kPairs]) {
  if constexpr (kF16) {
    widen_f16_32(u, P);
  } else {
    widen_bf16_32(u, P);
  }
}

// 16-bit words -> P[i] = (p[2i] + p[2i + 1], p[2i] - p[2i + 1]): the widening
// and butterfly bit 0 together.  The high element is widened to float32; the
// low one enters the sm_100 mixed-precision add and subtract as a 16-bit
// operand, which is converted exactly, so each result is the float32 sum
// rounded once, as in fwht32's own bit-0 stage.
template <bool kF16>
__device__ __forceinline__ void widen_stage0_32(const uint4 (&u)[4], uint64_t (&P)[kPairs]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t w[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float sum, dif;
      if constexpr (kF16) {
        asm("{\n\t.reg .b16 lo, hi;\n\t.reg .f32 h;\n\tmov.b32 {lo, hi}, %2;\n\t"
            "cvt.f32.f16 h, hi;\n\t"
            "add.rn.f32.f16 %0, lo, h;\n\t"
            "sub.rn.f32.f16 %1, lo, h;\n\t}"
            : "=f"(sum), "=f"(dif)
            : "r"(w[k]));
      } else {
        const float h = __uint_as_float(w[k] & 0xffff0000u);
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
            "add.rn.f32.bf16 %0, lo, %3;\n\t"
            "sub.rn.f32.bf16 %1, lo, %3;\n\t}"
            : "=f"(sum), "=f"(dif)
            : "r"(w[k]), "f"(h));
      }
      P[4 * j + k] = pk(sum, dif);
    }
  }
}

// raw int8 words -> P after butterfly bits 0 and 1: each word holds four
// elements b0..b3, and dp4a against the +-1 sign words of the 4-point
// transform gives its four outputs as exact integers (|y| <= 508).  The
// accumulator 0x4B400000 is 1.5 * 2^23 as a float, so each result read as a
// float is 1.5 * 2^23 + y exactly; one packed subtraction leaves y.
//   P[2k] = (b0 + b1 + b2 + b3, b0 - b1 + b2 - b3),
//   P[2k + 1] = (b0 + b1 - b2 - b3, b0 - b1 - b2 + b3)   (word k).
__device__ __forceinline__ void widen_i8_wht4_32(const uint4 (&u)[2], uint64_t (&P)[kPairs]) {
  constexpr int kMagicBits = 0x4B400000;
  const uint64_t magic2 = pk(kRoundMagic, kRoundMagic);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int w[4] = {static_cast<int>(u[j].x), static_cast<int>(u[j].y),
                      static_cast<int>(u[j].z), static_cast<int>(u[j].w)};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int y0 = __dp4a(w[k], 0x01010101, kMagicBits);
      const int y1 = __dp4a(w[k], static_cast<int>(0xFF01FF01u), kMagicBits);
      const int y2 = __dp4a(w[k], static_cast<int>(0xFFFF0101u), kMagicBits);
      const int y3 = __dp4a(w[k], static_cast<int>(0x01FFFF01u), kMagicBits);
      P[8 * j + 2 * k] = sub2(pku(y0, y1), magic2);
      P[8 * j + 2 * k + 1] = sub2(pku(y2, y3), magic2);
    }
  }
}

// ---------------------------------------------------------------- butterflies
// Unnormalised Walsh-Hadamard transform of every G-group, y = x . H_G, for the
// 32-element chunk of each lane (pairs P[i] = elements (2i, 2i + 1)).
//   bit 0: the two halves of each pair;   bits 1..4: across pairs (packed);
//   G == 64: bit 5 across lanes l and l ^ 1 (warp shuffle);
//   G == 256: bits 5..7 after one exchange through shared memory: the 8 lanes
//   of a group each write their 32 elements as 8 slots of 16 bytes and read
//   slot t (elements 4t .. 4t + 3) of every lane of the group.  Slot m of
//   lane s sits at 9 s + m (rows padded to 9 slots) and the groups are 1160
//   bytes apart (8 more than their 72 slots), so the 64-bit halves that each
//   access moves (a pair register, never a packed quad) hit 16 distinct bank
//   pairs in every 16-lane phase, on both sides; every address is a per-lane
//   base plus a constant.  Afterwards lane t holds in P[2 s + q] the elements
//   (32 s + 4t + 2q, 32 s + 4t + 2q + 1), s = 0..7.
constexpr int kXchGroupBytes = 8 * 9 * 16 + 8;
constexpr int kXchBytesPerWarp = 4 * kXchGroupBytes;  // 4 groups

// kDone: element bits already transformed by the widening (0; 1 after
// widen_stage0_32; 2 after widen_i8_wht4_32).
template <int G, int kDone>
__device__ __forceinline__ void fwht32(uint64_t (&P)[kPairs], uint32_t xch, uint32_t lane) {
  static_assert(kDone >= 0 && kDone <= 2, "stages done by the widening");
  if constexpr (kDone == 0) {
#pragma unroll
    for (int i = 0; i < kPairs; ++i) {  // bit 0
      const float a = plo(P[i]), b = phi(P[i]);
      P[i] = pk(a + b, a - b);
    }
  }
  constexpr int kTop = (G < kVec ? G : kVec) / 2;  // pair-index stages (bits 1..)
#pragma unroll
  for (int h = kDone == 2 ? 2 : 1; h < kTop; h <<= 1) {
#pragma unroll
    for (int i = 0; i < kPairs; ++i) {
      if ((i & h) == 0) {
        const uint64_t a = P[i], b = P[i + h];
        P[i] = add2(a, b);
        P[i + h] = sub2(a, b);
      }
    }
  }
  if constexpr (G == 64) {
    const float sg = (lane & 1) ? -1.f : 1.f;  // the upper lane keeps a - b
    const uint64_t sgn = pk(sg, sg);
#pragma unroll
    for (int i = 0; i < kPairs; ++i) {
      const float lo = __shfl_xor_sync(kFull, plo(P[i]), 1);
      const float hi = __shfl_xor_sync(kFull, phi(P[i]), 1);
      P[i] = fma2(sgn, P[i], pk(lo, hi));
    }
  }
  if constexpr (G == 256) {
    const uint32_t t = lane & 7;
    const uint32_t g = xch + (lane >> 3) * kXchGroupBytes;
    const uint32_t wbase = g + 144 * t, rbase = g + 16 * t;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      sts64(wbase + 16 * m, P[2 * m]);
      sts64(wbase + 16 * m + 8, P[2 * m + 1]);
    }
    __syncwarp();
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      P[2 * s] = lds64(rbase + 144 * s);
      P[2 * s + 1] = lds64(rbase + 144 * s + 8);
    }
    __syncwarp();
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {  // bits 5..7: across source lanes
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        if ((s & h) == 0) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const uint64_t a = P[2 * s + q], b = P[2 * (s + h) + q];
            P[2 * s + q] = add2(a, b);
            P[2 * (s + h) + q] = sub2(a, b);
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------- outputs
__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Writes the low byte of each half of R (a code in two's complement) where
// fwht32 left that element; `base` = first element of the lane's chunk.
template <int G>
__device__ __forceinline__ void store_code_bytes(int8_t* base, const uint64_t (&R)[kPairs],
                                                 uint32_t lane) {
  uint32_t w[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t a0, a1, b0, b1;
    unpk(R[2 * j], a0, a1);
    unpk(R[2 * j + 1], b0, b1);
    w[j] = pack4(a0, a1, b0, b1);
  }
  if constexpr (G == 256) {
    const uint32_t t = lane & 7;
    int8_t* grp = base - kVec * t;
#pragma unroll
    for (int s = 0; s < 8; ++s) *reinterpret_cast<uint32_t*>(grp + 32 * s + 4 * t) = w[s];
  } else {
    uint4* q = reinterpret_cast<uint4*>(base);
    q[0] = make_uint4(w[0], w[1], w[2], w[3]);
    q[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

// Codes rne(v * mul) of the 32 values (|v * mul| <= 127.5): one packed FMA
// against 1.5 * 2^23 leaves each code in the low byte of its float.
template <int G>
__device__ __forceinline__ void store_codes32(int8_t* base, const uint64_t (&P)[kPairs], float mul,
                                             uint32_t lane) {
  const uint64_t m2 = pk(mul, mul), magic2 = pk(kRoundMagic, kRoundMagic);
  uint64_t R[kPairs];
#pragma unroll
  for (int i = 0; i < kPairs; ++i) R[i] = fma2(P[i], m2, magic2);
  store_code_bytes<G>(base, R, lane);
}

// Exact-division codes rne(v * norm / s), for scales so small that 1/s overflows.
template <int G>
__device__ __forceinline__ void store_codes32_div(int8_t* base, const uint64_t (&P)[kPairs],
                                                  float norm, float s, uint32_t lane) {
  uint64_t R[kPairs];
#pragma unroll
  for (int i = 0; i < kPairs; ++i) {
    const float a = fminf(fmaxf(rintf(__fdiv_rn(plo(P[i]) * norm, s)), -127.f), 127.f);
    const float b = fminf(fmaxf(rintf(__fdiv_rn(phi(P[i]) * norm, s)), -127.f), 127.f);
    R[i] = pk(a + kRoundMagic, b + kRoundMagic);
  }
  store_code_bytes<G>(base, R, lane);
}

// The exact products s * v of a pair, each rounded once to nearest-even into a
// 16-bit float: the product is rounded toward zero to float32 and its last
// bit forced to one when inexact ("round to odd"); float32 keeps at least two
// bits more than bf16 and fp16 (normal or subnormal results alike), so
// rounding that to the 16-bit format is the correctly rounded result.
__device__ __forceinline__ void odd_product2(uint64_t s2, uint64_t neg_s2, uint64_t v, uint32_t& lo,
                                             uint32_t& hi) {
  const uint64_t p = mulrz2(s2, v);
  const uint64_t e = fma2(neg_s2, v, p);  // exact p - s*v
  uint32_t e_lo, e_hi;
  unpk(p, lo, hi);
  unpk(e, e_lo, e_hi);
  // the remainder is +0 exactly when the product is exact (x - x rounds to +0)
  asm("{\n\t.reg .pred q;\n\t"
      "setp.ne.b32 q, %2, 0;\n\t@q or.b32 %0, %0, 1;\n\t"
      "setp.ne.b32 q, %3, 0;\n\t@q or.b32 %1, %1, 1;\n\t}"
      : "+r"(lo), "+r"(hi)
      : "r"(e_lo), "r"(e_hi));
}

// Round-to-odd without the remainder (bf16 output): p | 1 on the product
// rounded toward zero.  Exact whenever no product s * v is itself a bf16
// midpoint: v is an integer (|v| <= 127 G < 2^15), so s * v has at least as
// many significant bits as s's mantissa without its trailing zeros; with fewer
// than 15 trailing zeros that is more than the 9 bits of a midpoint (s normal,
// so the products stay in bf16's normal range).  p | 1 is then correct whether
// or not the product was exact, since an exact p is no midpoint.  (fp16 output
// has no such shortcut: its subnormal midpoints sit at fixed multiples of
// 2^-25, which exact products can hit.)
__device__ __forceinline__ bool odd_rounding_is_exact(float s) {
  const uint32_t b = __float_as_uint(s);
  return (b & 0x7FFFu) != 0 && (b & 0x7F800000u) != 0;
}

template <bool kF16>
__device__ __forceinline__ uint32_t pack16x2(uint32_t lo, uint32_t hi) {
  if constexpr (kF16) {
    const __half2 h = __floats2half2_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<const uint32_t*>(&h);
  } else {
    const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<const uint32_t*>(&h);
  }
}

// 16-bit words of the 32 products s * P (pairs 2i, 2i + 1 in w[i]), each
// rounded once: bf16 (kF16 = false) or fp16.
template <bool kF16>
__device__ __forceinline__ void products16_32(uint32_t (&w)[kPairs], const uint64_t (&P)[kPairs],
                                              float sn) {
  const uint64_t s2 = pk(sn, sn);
  if (!kF16 && odd_rounding_is_exact(sn)) {
#pragma unroll
    for (int i = 0; i < kPairs; ++i) {
      uint32_t lo, hi;
      unpk(mulrz2(s2, P[i]), lo, hi);
      w[i] = pack16x2<false>(lo | 1u, hi | 1u);
    }
  } else {
    const uint64_t neg_s2 = pk(-sn, -sn);
#pragma unroll
    for (int i = 0; i < kPairs; ++i) {
      uint32_t lo, hi;
      odd_product2(s2, neg_s2, P[i], lo, hi);
      w[i] = pack16x2<kF16>(lo, hi);
    }
  }
}

template <int G>
__device__ __forceinline__ void store_words16(uint16_t* base, const uint32_t (&w)[kPairs],
                                                 uint32_t lane) {
  if constexpr (G == 256) {
    const uint32_t t = lane & 7;
    uint16_t* grp = base - kVec * t;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      *reinterpret_cast<uint2*>(grp + 32 * s + 4 * t) = make_uint2(w[2 * s], w[2 * s + 1]);
    }
  } else {
    uint4* q = reinterpret_cast<uint4*>(base);
#pragma unroll
    for (int j = 0; j < 4; ++j) q[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  }
}

__device__ __forceinline__ float absmax32(const uint64_t (&P)[kPairs]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < kPairs; ++i) m = fmaxf(m, fmaxf(fabsf(plo(P[i])), fabsf(phi(P[i]))));
  return m;
}

// Max over the warp of non-negative floats (never NaN: the absmax drops NaN
// inputs); their bit patterns order like their values.
__device__ __forceinline__ float warp_max(float a) {
  return __uint_as_float(__reduce_max_sync(kFull, __float_as_uint(a)));
}

template <int G>
__host__ __device__ constexpr int xch_bytes_per_warp() {
  return G == 256 ? kXchBytesPerWarp : 0;
}

// ===========================================================================
// Sylvester path, activations: a team of `team_warps` warps per token, one
// 32-element chunk per lane, all loads issued before any arithmetic.  The
// token's rotated row stays in registers between the absmax and the pack.
// ===========================================================================
// cp.async groups: commit the copies issued so far, wait for all of them.
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// A warp stages 32 consecutive chunks of kParts 16-byte units each (bf16:
// 4, int8: 2) in a slot of its own.  Copy j of lane i moves unit 32 j + i, so
// each copy instruction reads 512 contiguous bytes; lane L later reads its
// units kParts * L + k.  Unit (L, k) sits at position kParts * L + (L >> s) + k,
// s = log2(8 / kParts): the gaps make both sides conflict-free (8 lanes of a
// phase hit 8 distinct 16-byte bank groups) and both sides' addresses a
// per-lane base plus a constant: the copy's position is i + (i >> 3) + 36 j,
// the read's kParts * L + (L >> s) + k.
constexpr int kStageUnitsPerWarp = 144;  // positions 0 .. 142
constexpr int kStageBytesPerWarp = kStageUnitsPerWarp * 16;

__device__ __forceinline__ uint32_t stage_copy_offset(uint32_t lane) {
  return (lane + (lane >> 3)) * 16;
}
template <int kParts>
__device__ __forceinline__ uint32_t stage_read_offset(uint32_t lane) {
  return (kParts * lane + (lane >> (kParts == 4 ? 1 : 2))) * 16;
}

// Copies j = 0 .. kParts-1 of one lane: 16 bytes from src + 512 j to
// dst + 576 j, each only when 32 / kParts * j < lim (the unit's chunk exists).
template <int kParts>
__device__ __forceinline__ void stage_copies(uint32_t dst, const uint8_t* src, int lim) {
#pragma unroll
  for (int j = 0; j < kParts; ++j) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.lt.s32 p, %2, %3;\n\t"
        "@p cp.async.cg.shared.global [%0], [%1], 16;\n\t}"
        ::"r"(dst + 576 * j), "l"(src + 512 * j), "r"((32 / kParts) * j), "r"(lim)
        : "memory");
  }
  cp_async_commit();
}

template <int kParts>
__device__ __forceinline__ void unstage_chunk(uint32_t src, uint4 (&v)[kParts]) {
#pragma unroll
  for (int k = 0; k < kParts; ++k) {
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v[k].x), "=r"(v[k].y), "=r"(v[k].z), "=r"(v[k].w)
                 : "r"(src + 16 * k)
                 : "memory");
  }
}

// The named barrier of team `team` (ID 1 + team) for the kTeams teams of a
// CTA, its ID an immediate: ptxas then reserves only those IDs, where a
// register-valued ID reserves all 16 of the CTA, and the occupancy
// calculation admitted only 4 CTAs of 5 warps per SM although registers and
// shared memory allow 5.  kTeams == 0: one-warp teams, no barrier.
template <int kTeams>
__device__ __forceinline__ void team_barrier(int team, int nthreads) {
  static_assert(kTeams == 0 || kTeams == 1 || kTeams == 2 || kTeams == 4, "teams per CTA");
  if constexpr (kTeams == 1) {
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
  } else if constexpr (kTeams == 2) {
    if (team == 0) {
      asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
    } else {
      asm volatile("bar.sync 2, %0;" ::"r"(nthreads) : "memory");
    }
  } else if constexpr (kTeams == 4) {
    switch (team) {
      case 0: asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory"); break;
      case 1: asm volatile("bar.sync 2, %0;" ::"r"(nthreads) : "memory"); break;
      case 2: asm volatile("bar.sync 3, %0;" ::"r"(nthreads) : "memory"); break;
      default: asm volatile("bar.sync 4, %0;" ::"r"(nthreads) : "memory"); break;
    }
  }
}

// Register budgets by CTA size: kMaxThreads threads, kMinBlocks CTAs per SM
// (256, 3) and (384, 2) leave room for 85 registers; (1024, 1) keeps 64, so
// that teams of up to 512 threads still fit two CTAs per SM.  kTeams: teams
// (token rows) per CTA, 0 for one-warp teams.
template <int G, int kMaxThreads, int kMinBlocks, bool kF16, int kTeams>
__global__ void __launch_bounds__(kMaxThreads, kMinBlocks) rotate_quant_act_hadamard(
    const uint16_t* __restrict__ x, int64_t M, int K, int team_warps, int rows_per_cta,
    int8_t* __restrict__ xq, float* __restrict__ s_tok, unsigned int* __restrict__ status,
    int fault) {
  extern __shared__ __align__(16) uint8_t smem_all[];
  __shared__ float red[2][32];
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const int team = warp / team_warps;
  const int t0 = (warp % team_warps) * 32;
  const int t = t0 + static_cast<int>(lane);  // chunk within the token
  const int nch = K / kVec;
  const int nwarps = blockDim.x >> 5;
  const uint32_t slot = smem_addr(smem_all) + warp * kStageBytesPerWarp;
  const uint32_t xch = smem_addr(smem_all) + nwarps * kStageBytesPerWarp + warp * xch_bytes_per_warp<G>();
  const uint32_t cp_dst = slot + stage_copy_offset(lane);
  const uint32_t rd_src = slot + stage_read_offset<4>(lane);
  // copy j of this lane holds part of chunk t0 + 8 j + lane / 4 of the row
  const int lim = nch - t0 - static_cast<int>(lane >> 2);
  const uint8_t* xb = reinterpret_cast<const uint8_t*>(x) + (static_cast<int64_t>(t0) * 64 + 16 * lane);
  const int64_t row_bytes = static_cast<int64_t>(K) * 2;
  constexpr float norm = Norm<G>::value;

  // The CTA walks row blocks blockIdx.x, blockIdx.x + gridDim.x, ...; the next
  // block's chunks are copied into shared memory while this one is transformed.
  // Lanes without a chunk (the row's tail, rows past M) copy nothing and
  // transform stale data; whole groups share `ok`, and their results are dropped.
  const int bar_threads = team_warps * 32;
  const int64_t row_step = static_cast<int64_t>(gridDim.x) * rows_per_cta;
  // launched chained to the previous kernel: global memory only after it completes
  ptx::grid_dependency_wait();
  ptx::grid_dependents_launch();
  const int64_t src_step = row_step * row_bytes;
  int64_t row = static_cast<int64_t>(blockIdx.x) * rows_per_cta + team;
  const uint8_t* src = xb + row * row_bytes;
  stage_copies<4>(cp_dst, src, row < M ? lim : 0);
  for (int it = 0; row - team < M; row += row_step, ++it) {
    const bool ok = row < M && t < nch;  // row < M is uniform over the team
    uint4 u[4];
    cp_async_wait_all();
    __syncwarp();  // the lanes' copies landed: every lane's units are visible
    unstage_chunk<4>(rd_src, u);
    uint64_t P[kPairs];
    widen_stage0_32<kF16>(u, P);
    __syncwarp();  // every lane has read its units before the slot is refilled
    src += src_step;
    stage_copies<4>(cp_dst, src, row + row_step < M ? lim : 0);
    fwht32<G, 1>(P, xch, lane);
    float amax = warp_max(ok ? absmax32(P) : 0.f);
    if (kTeams > 0) {
      float* rb_red = red[it & 1];
      if (lane == 0) rb_red[warp] = amax;
      // the team's warps only: teams of one CTA run independently
      team_barrier<kTeams>(team, bar_threads);
      amax = warp_max(static_cast<int>(lane) < team_warps ? rb_red[team * team_warps + lane] : 0.f);
    }
    if (!ok) continue;
    // debug build: the token's codes and scale must lie inside xq and s_tok
    const int64_t row_limit = CONVROT_DEBUG && fault == kFaultShortRows ? M - 1 : M;
    if (!in_bounds(row < row_limit && (t + 1) * kVec <= K, status)) continue;
    // s_tok = max |x_rot| / 127, correctly rounded without a division.  With
    // a = amax * norm (exact) and m any float32 rounding midpoint of a / 127,
    // a - 127 m is an odd multiple of half the quotient's ulp (a's bits are
    // even multiples of it, 127 times an odd multiple is odd), so a / 127 lies
    // at least 2^-31 (relative) from every midpoint, and 2^-150 / 127 away when
    // the quotient is subnormal.  The float64 product a * RN(1/127) is within
    // 2^-52 (relative) of a / 127, so its one rounding to float32 is RN(a / 127).
    const float sc = static_cast<float>(static_cast<double>(amax * norm) * (1.0 / 127.0));
    if (t == 0) s_tok[row] = sc;
    const float mul = norm * (sc > 0.f ? 1.f / sc : 0.f);  // exact scaling: norm is a power of two
    int8_t* dst = xq + row * K + static_cast<int64_t>(t) * kVec;
    if (mul <= 3.0e38f) {
      store_codes32<G>(dst, P, mul, lane);
    } else {
      store_codes32_div<G>(dst, P, norm, sc, lane);
    }
  }
}

// ===========================================================================
// Sylvester path over a flat [rows, K] tensor, one 32-element chunk per
// thread.  Groups never straddle rows (K % G == 0, K % 32 == 0).
// ===========================================================================
enum FlatMode { kFlatAbsmax = 0, kFlatQuant = 1, kFlatDequant = 2 };

// Per-warp shared memory of the flat kernel besides its staging slot: the
// G = 256 exchange, or the output slot of the decode at G < 256.
template <int G, int MODE>
__host__ __device__ constexpr int flat_aux_bytes() {
  return G == 256 ? kXchBytesPerWarp : (MODE == kFlatDequant ? kStageBytesPerWarp : 0);
}

// kF16: the 16-bit float format of W (absmax / quant) or of W_hat (decode).
template <int G, int MODE, bool PER_ROW_SCALE, bool kF16>
__global__ void __launch_bounds__(256, MODE == kFlatDequant ? 3 : 4) hadamard_flat(const void* __restrict__ in, int64_t nchunks,
                                                     uint64_t row_mul, int row_shift,
                                                     const float* __restrict__ scale,
                                                     void* __restrict__ out,
                                                     unsigned int* __restrict__ absmax_bits,
                                                     unsigned int* __restrict__ status, int fault) {
  constexpr int kParts = MODE == kFlatDequant ? 2 : 4;  // 16-byte parts of a chunk
  extern __shared__ __align__(16) uint8_t smem_all[];
  const uint32_t lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint32_t slot = smem_addr(smem_all) + warp * kStageBytesPerWarp;
  // G = 256: the butterfly exchange; decode at G < 256: the output slot
  const uint32_t aux =
      smem_addr(smem_all) + (blockDim.x >> 5) * kStageBytesPerWarp + warp * flat_aux_bytes<G, MODE>();
  const uint32_t cp_dst = slot + stage_copy_offset(lane);
  const uint32_t rd_src = slot + stage_read_offset<kParts>(lane);
  const int64_t blocks = (nchunks + blockDim.x - 1) / blockDim.x;
  // copy j of this lane holds part of chunk b * blockDim.x + 32 warp + (32 / kParts) j + lane / kParts
  const uint8_t* src = static_cast<const uint8_t*>(in) +
                       (static_cast<int64_t>(warp) * 32 * kParts + lane) * 16;
  const int64_t lim0 = nchunks - warp * 32 - static_cast<int>(lane / kParts);
  const int64_t block_bytes = static_cast<int64_t>(blockDim.x) * kParts * 16;
  constexpr float norm = Norm<G>::value;

  // Chunk c = b * blockDim.x + thread for blocks b = blockIdx.x, + gridDim.x, ...;
  // the next block's chunks are copied into shared memory while this one is
  // transformed.  Lanes past the end copy nothing and transform stale data
  // (whole groups share `ok`); their results are dropped.
  // debug build: the chunks this kernel may write (the last 256 elements,
  // 8 chunks, fewer under the short-rows fault).  At G = 256 a lane's stores
  // cover its whole group of 8 chunks, so its check covers the group.
  const int64_t chunk_limit = CONVROT_DEBUG && fault == kFaultShortRows ? nchunks - 8 : nchunks;
  auto stage = [&](int64_t b) {
    const int64_t lim = lim0 - b * blockDim.x;
    stage_copies<kParts>(cp_dst, src + b * block_bytes,
                         lim > 32 ? 32 : static_cast<int>(lim < 0 ? 0 : lim));
  };
  // launched chained to the previous kernel: global memory only after it completes
  ptx::grid_dependency_wait();
  ptx::grid_dependents_launch();
  float mul = 0.f, s = 0.f, run_max = 0.f;
  if constexpr (MODE == kFlatQuant) {
    s = __uint_as_float(*absmax_bits) / 127.f;
    mul = s > 0.f ? norm * (1.f / s) : 0.f;
  }
  int64_t b = blockIdx.x;
  stage(b);
  for (; b < blocks; b += gridDim.x) {
    const int64_t c = b * blockDim.x + threadIdx.x;
    const bool ok = c < nchunks;
    uint4 u[kParts];
    cp_async_wait_all();
    __syncwarp();  // the lanes' copies landed: every lane's units are visible
    unstage_chunk<kParts>(rd_src, u);
    uint64_t P[kPairs];
    if constexpr (MODE == kFlatDequant) {
      widen_i8_wht4_32(u, P);
    } else {
      widen16_32<kF16>(u, P);
    }
    __syncwarp();  // every lane has read its units before the slot is refilled
    stage(b + gridDim.x);
    if constexpr (MODE == kFlatDequant) {
      fwht32<G, 2>(P, aux, lane);
    } else {
      fwht32<G, 0>(P, aux, lane);
    }

    if constexpr (MODE == kFlatAbsmax) {
      if (ok) run_max = fmaxf(run_max, absmax32(P));
    } else if constexpr (MODE == kFlatQuant) {
      if (ok && in_bounds((G == 256 ? (c | 7) : c) < chunk_limit, status)) {
        int8_t* dst = static_cast<int8_t*>(out) + c * kVec;
        if (mul <= 3.0e38f) {
          store_codes32<G>(dst, P, mul, lane);
        } else {
          store_codes32_div<G>(dst, P, norm, s, lane);
        }
      }
    } else {
      // output row of chunk c: c / (K / 32) as a multiply and shift (row_reciprocal)
      const float sw =
          PER_ROW_SCALE ? scale[((ok ? static_cast<uint64_t>(c) : 0ull) * row_mul) >> row_shift] : scale[0];
      const bool store_ok = in_bounds(!ok || (G == 256 ? (c | 7) : c) < chunk_limit, status);
      uint32_t w[kPairs];
      products16_32<kF16>(w, P, sw * norm);
      if constexpr (G == 256) {
        if (ok && store_ok) store_words16<G>(static_cast<uint16_t*>(out) + c * kVec, w, lane);
      } else {
        // A lane's 64 output bytes are 4 units of the warp's 2 KB; through the
        // output slot, store j of lane i writes unit 32 j + i (512 contiguous
        // bytes per instruction) when its chunk exists.
        const uint32_t wr = aux + stage_read_offset<4>(lane);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(wr + 16 * k),
                       "r"(w[4 * k]), "r"(w[4 * k + 1]), "r"(w[4 * k + 2]), "r"(w[4 * k + 3])
                       : "memory");
        }
        __syncwarp();
        const int64_t chunk0 = b * blockDim.x + warp * 32;
        const int64_t olim = nchunks - chunk0 - static_cast<int>(lane >> 2);
        uint8_t* dst = static_cast<uint8_t*>(out) + chunk0 * 64 + lane * 16;
        const uint32_t rd = aux + stage_copy_offset(lane);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (8 * j < olim && in_bounds(chunk0 + 8 * j + static_cast<int>(lane >> 2) < chunk_limit, status)) {
            uint4 v;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(rd + 576 * j)
                         : "memory");
            *reinterpret_cast<uint4*>(dst + 512 * j) = v;
          }
        }
        __syncwarp();  // the slot is read out before the next block writes it
      }
    }
  }
  if constexpr (MODE == kFlatAbsmax) {
    __shared__ float red[8];
    const float amax = warp_max(run_max);
    if (lane == 0) red[warp] = amax;
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

// kF16: the 16-bit float format of a uint16_t input, and of the decoded output.
template <int G, typename TIn, int MODE, bool kF16>
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
        val = kF16 ? __half2float(__ushort_as_half(raw))
                   : __uint_as_float(static_cast<uint32_t>(raw) << 16);
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
          const double v = static_cast<double>(sw) * acc[a][b];
          if constexpr (kF16) {
            o[tx + b * TC] = __half_as_ushort(__double2half(v));
          } else {
            const __nv_bfloat16 h = __double2bfloat16(v);
            o[tx + b * TC] = *reinterpret_cast<const uint16_t*>(&h);
          }
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

// Launches `kern` chained to the previous kernel of the stream (programmatic
// dependent launch): it may be scheduled while that kernel drains and waits
// on the device before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kern)(KArgs...), int64_t grid, int block, size_t smem,
                           cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(block));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Opts the kernel in to `bytes` of dynamic shared memory (the default limit,
// 48 KB, counts the kernel's static shared memory too).
template <typename Kern>
cudaError_t allow_smem(Kern kern, size_t bytes) {
  if (bytes == 0) return cudaSuccess;
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

template <int G, int kMaxThreads, int kMinBlocks, bool kF16, int kTeams>
cudaError_t rqa_launch(const uint16_t* x, int64_t M, int K, int team_warps, int rows_per_cta,
                       int8_t* xq, float* s_tok, cudaStream_t stream) {
  const int warps = team_warps * rows_per_cta;
  const size_t smem = static_cast<size_t>(warps) * (kStageBytesPerWarp + xch_bytes_per_warp<G>());
  cudaError_t e = allow_smem(rotate_quant_act_hadamard<G, kMaxThreads, kMinBlocks, kF16, kTeams>, smem);
  if (e != cudaSuccess) return e;
  // enough CTAs to fill every SM (register-limited occupancy), each looping
  // over row blocks with a one-block-ahead prefetch
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rotate_quant_act_hadamard<G, kMaxThreads, kMinBlocks, kF16, kTeams>,
                                                    32 * warps, smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (M + rows_per_cta - 1) / rows_per_cta;
  const int64_t cap = static_cast<int64_t>(sm_count()) * (per_sm > 0 ? per_sm : 1);
  const int64_t grid = blocks < cap ? blocks : cap;
  unsigned int* status = nullptr;
  e = status_word(&status);
  if (e != cudaSuccess) return e;
  return launch_chained(rotate_quant_act_hadamard<G, kMaxThreads, kMinBlocks, kF16, kTeams>, grid, 32 * warps, smem,
                        stream, x, M, K, team_warps, rows_per_cta, xq, s_tok, status, debug_fault());
}

template <int G, bool kF16>
cudaError_t rqa_hadamard(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* s_tok,
                         cudaStream_t stream) {
  // A token's row is held by a team of ceil(K / 1024) warps, one 32-element
  // chunk per lane; small rows share a CTA (8 warps).
  const int nch = static_cast<int>(K / kVec);
  const int team_warps = (nch + 31) / 32;
  const int rows_per_cta = team_warps >= 8 ? 1 : 8 / team_warps;
  const int warps = team_warps * rows_per_cta;
  const int k = static_cast<int>(K);
  // 9-10 warps fit three CTAs per SM only at 64 registers; 11-12 fit two
  // CTAs either way, so they take the larger budget
  // teams per CTA: 8 one-warp teams (no barrier), 4 of 2 warps, 2 of 3-4,
  // else 1
  if (warps <= 8) {
    if (team_warps == 1) {
      return rqa_launch<G, 256, 3, kF16, 0>(x, M, k, team_warps, rows_per_cta, xq, s_tok, stream);
    }
    if (rows_per_cta == 4) {
      return rqa_launch<G, 256, 3, kF16, 4>(x, M, k, team_warps, rows_per_cta, xq, s_tok, stream);
    }
    if (rows_per_cta == 2) {
      return rqa_launch<G, 256, 3, kF16, 2>(x, M, k, team_warps, rows_per_cta, xq, s_tok, stream);
    }
    return rqa_launch<G, 256, 3, kF16, 1>(x, M, k, team_warps, rows_per_cta, xq, s_tok, stream);
  }
  if (warps >= 11 && warps <= 12) {
    return rqa_launch<G, 384, 2, kF16, 1>(x, M, k, team_warps, rows_per_cta, xq, s_tok, stream);
  }
  return rqa_launch<G, 1024, 1, kF16, 1>(x, M, k, team_warps, rows_per_cta, xq, s_tok, stream);
}

// Multiplier m and shift k with floor(c * m / 2^k) == c / d for every
// 0 <= c < 2^31 (1 <= d < 2^31): k = 31 + ceil(log2 d), m = ceil(2^k / d).  With
// e = m d - 2^k < d, c m / 2^k = c / d + c e / (d 2^k), and the second term is
// below 2^31 / 2^k = 2^-ceil(log2 d) <= 1 / d, too small to carry c / d past
// the next integer.
void row_reciprocal(uint64_t d, uint64_t* m, int* k) {
  int l = 0;
  while ((1ull << l) < d) ++l;
  *k = 31 + l;
  *m = ((1ull << *k) + d - 1) / d;
}

template <int G, int MODE, bool PER_ROW, bool kF16>
cudaError_t flat_launch(const void* in, int64_t nchunks, int64_t chunks_per_row,
                        const float* scale, void* out, unsigned int* absmax_bits,
                        cudaStream_t stream) {
  constexpr int kThreadsFlat = 256;
  const size_t smem = (kThreadsFlat / 32) * (kStageBytesPerWarp + flat_aux_bytes<G, MODE>());
  cudaError_t e = allow_smem(hadamard_flat<G, MODE, PER_ROW, kF16>, smem);
  if (e != cudaSuccess) return e;
  // one chunk per thread and block; enough CTAs to fill every SM, each looping
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, hadamard_flat<G, MODE, PER_ROW, kF16>,
                                                    kThreadsFlat, smem);
  if (e != cudaSuccess) return e;
  const int64_t cap = static_cast<int64_t>(sm_count()) * (per_sm > 0 ? per_sm : 1);
  int64_t grid = (nchunks + kThreadsFlat - 1) / kThreadsFlat;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  uint64_t row_mul = 0;
  int row_shift = 0;
  if (PER_ROW) {
    // the reciprocal is exact below 2^31 chunks (64 G weights: beyond any HBM)
    if (nchunks >= (1ll << 31) || chunks_per_row < 1) return cudaErrorInvalidValue;
    row_reciprocal(static_cast<uint64_t>(chunks_per_row), &row_mul, &row_shift);
  }
  unsigned int* status = nullptr;
  e = status_word(&status);
  if (e != cudaSuccess) return e;
  return launch_chained(hadamard_flat<G, MODE, PER_ROW, kF16>, grid, kThreadsFlat, smem, stream, in,
                        nchunks, row_mul, row_shift, scale, out, absmax_bits, status, debug_fault());
}

template <int G, typename TIn, int MODE, bool kF16>
cudaError_t dense_launch(const TIn* in, int64_t group_rows, int64_t groups_per_token,
                         const float* Rm, const float* scale, int64_t scale_len, void* out,
                         unsigned int* absmax_bits, cudaStream_t stream) {
  constexpr int TMR = 8192 / G;
  constexpr int KC = G < 32 ? G : 32;
  const size_t smem = sizeof(float) * (TMR * G + KC * G);
  auto kern = dense_rotate<G, TIn, MODE, kF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t grid = (group_rows + TMR - 1) / TMR;
  kern<<<static_cast<unsigned>(grid), 256, smem, stream>>>(in, group_rows, groups_per_token, Rm,
                                                           scale, scale_len, out, absmax_bits);
  return cudaGetLastError();
}

// Calls f(std::integral_constant<bool, f16>{}).
template <typename F>
cudaError_t by_format(bool f16, F&& f) {
  return f16 ? f(std::true_type{}) : f(std::false_type{});
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

cudaError_t launch_rotate_quant_act(const convrot_rotation_s* R, const uint16_t* x, bool f16,
                                    int64_t M, int64_t K, int8_t* xq, float* s_tok,
                                    cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  if (R->is_sylvester) {
    return by_format(f16, [&](auto fmt) {
      return by_group_size(R->G, [&](auto g) {
        return rqa_hadamard<decltype(g)::value, decltype(fmt)::value>(x, M, K, xq, s_tok, stream);
      });
    });
  }
  unsigned int* amax = reinterpret_cast<unsigned int*>(s_tok);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float) * M, stream);
  if (e != cudaSuccess) return e;
  const int64_t gpt = K / R->G;
  e = by_format(f16, [&](auto fmt) {
    constexpr bool F = decltype(fmt)::value;
    return by_group_size(R->G, [&](auto g) {
      constexpr int Gv = decltype(g)::value;
      cudaError_t r = dense_launch<Gv, uint16_t, kDenseAbsmaxRow, F>(
          x, M * gpt, gpt, R->R_dev, nullptr, 0, nullptr, amax, stream);
      if (r != cudaSuccess) return r;
      return dense_launch<Gv, uint16_t, kDenseQuantRow, F>(x, M * gpt, gpt, R->R_dev, nullptr, 0,
                                                           xq, amax, stream);
    });
  });
  if (e != cudaSuccess) return e;
  finalize_scales<<<static_cast<unsigned>((M + 255) / 256), 256, 0, stream>>>(s_tok, M);
  return cudaGetLastError();
}

cudaError_t launch_dequant_derotate(const convrot_rotation_s* R, const int8_t* Wq,
                                    const float* s_w, int64_t s_w_len, int64_t N, int64_t K,
                                    uint16_t* W_hat, bool f16, cudaStream_t stream) {
  return by_format(f16, [&](auto fmt) {
    constexpr bool F = decltype(fmt)::value;
    if (R->is_sylvester) {
      const int64_t nchunks = N * K / kVec;
      return by_group_size(R->G, [&](auto g) {
        constexpr int Gv = decltype(g)::value;
        if (s_w_len == 1) {
          return flat_launch<Gv, kFlatDequant, false, F>(Wq, nchunks, K / kVec, s_w, W_hat,
                                                         nullptr, stream);
        }
        return flat_launch<Gv, kFlatDequant, true, F>(Wq, nchunks, K / kVec, s_w, W_hat, nullptr,
                                                      stream);
      });
    }
    const int64_t gpt = K / R->G;
    return by_group_size(R->G, [&](auto g) {
      return dense_launch<decltype(g)::value, int8_t, kDenseDequant, F>(
          Wq, N * gpt, gpt, R->Rt_dev, s_w, s_w_len, W_hat, nullptr, stream);
    });
  });
}

cudaError_t launch_quantize_weight(const convrot_rotation_s* R, const uint16_t* W, bool f16,
                                   int64_t N, int64_t K, int8_t* Wq, float* s_w,
                                   cudaStream_t stream) {
  unsigned int* amax = reinterpret_cast<unsigned int*>(s_w);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), stream);
  if (e != cudaSuccess) return e;
  e = by_format(f16, [&](auto fmt) {
    constexpr bool F = decltype(fmt)::value;
    if (R->is_sylvester) {
      const int64_t nchunks = N * K / kVec;
      return by_group_size(R->G, [&](auto g) {
        constexpr int Gv = decltype(g)::value;
        cudaError_t r = flat_launch<Gv, kFlatAbsmax, false, F>(W, nchunks, K / kVec, nullptr,
                                                               nullptr, amax, stream);
        if (r != cudaSuccess) return r;
        return flat_launch<Gv, kFlatQuant, false, F>(W, nchunks, K / kVec, nullptr, Wq, amax,
                                                     stream);
      });
    }
    const int64_t gpt = K / R->G;
    return by_group_size(R->G, [&](auto g) {
      constexpr int Gv = decltype(g)::value;
      cudaError_t r = dense_launch<Gv, uint16_t, kDenseAbsmaxAll, F>(W, N * gpt, gpt, R->R_dev,
                                                                     nullptr, 0, nullptr, amax,
                                                                     stream);
      if (r != cudaSuccess) return r;
      return dense_launch<Gv, uint16_t, kDenseQuantAll, F>(W, N * gpt, gpt, R->R_dev, nullptr, 0,
                                                           Wq, amax, stream);
    });
  });
  if (e != cudaSuccess) return e;
  finalize_scales<<<1, 32, 0, stream>>>(s_w, 1);
  return cudaGetLastError();
}

}  // namespace convrot
