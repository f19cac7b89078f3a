// Few-token int8 product of the ConvRot layer's int8 compute (Invoke docs
// "int8 Compute", opening section: each layer "multiplies int8 by int8"), for
// up to kGemvMaxTokens tokens:
//
//   acc[m, n] = sum_k xq[m, k] * Wq[n, k]                       (exact int32)
//   y[m, n]   = bf16_rn(float(acc) * (s_tok[m] * s_w[n|0]) + bias[n])
//
// the same values as the tensor-core GEMMs (the epilogue is the same single
// FMA and rounding).  With this few tokens the weight stream is the whole
// cost, and the tensor-core kernels' set-up, ring fill and split-K reduction
// across a cluster are what bound them.  Here every warp takes whole weight
// rows: each lane loads 16-byte pieces of the row (one 512-byte load per warp
// instruction, kUnroll of them in flight per lane), and dp4a against the
// tokens' codes, staged once per CTA in shared memory, gives the dot products;
// one warp reduction per token ends the row.  The first row's weight loads are
// issued before the chained wait: no kernel of this library that can precede
// this one in a chained launch writes an int8 weight (the weight quantizer
// ends with a plain launch), so they overlap the previous kernel's drain; the
// codes, scales and bias are read after it.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace convrot {
namespace {

constexpr int kUnroll = 8;                  // 16-byte pieces per lane per row block
constexpr int kBlockPieces = 32 * kUnroll;  // a row block: 4 KB of the weight row
constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;

struct GemvParams {
  const int8_t* x;       // xq [M, K]
  const int8_t* w;       // Wq [N, K]
  const float* s_tok;    // [M]
  const float* s_w;      // [1] or [N]
  const uint16_t* bias;  // [N] or null, in the output's format
  void* out;             // y [M, N] (16-bit) or acc [M, N] (int32)
  int M;
  int64_t N;
  int K;
  int per_channel_scale;
  int out_s32;
  int out_f16;
  unsigned int* status;  // device status word (bit 1: debug bounds)
  int fault;             // debug build: injected fault (kFaultShortRows)
};

// Lane `lane`'s kUnroll pieces of row block `blk` of weight row `row`: piece
// q = blk * kBlockPieces + u * 32 + lane; pieces past the row read as zero.
__device__ __forceinline__ void load_block(uint4 (&wv)[kUnroll], const int8_t* w, int64_t row, int K,
                                           int pieces, int blk, int lane) {
  const uint4* wr = reinterpret_cast<const uint4*>(w + row * K);
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const int q = blk * kBlockPieces + u * 32 + lane;
    wv[u] = q < pieces ? __ldg(wr + q) : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <int MT>
__global__ void __launch_bounds__(kThreads) int8_gemv_dp4a(const GemvParams p) {
  extern __shared__ __align__(16) int8_t xs[];  // the tokens' codes [MT][K] (rows past M zero)
  const int lane = static_cast<int>(threadIdx.x & 31);
  const int64_t first = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  const int64_t step = static_cast<int64_t>(gridDim.x) * kWarps;
  const int pieces = p.K / 16;
  const int blocks = (pieces + kBlockPieces - 1) / kBlockPieces;

  uint4 wv[kUnroll];
  if (first < p.N) load_block(wv, p.w, first, p.K, pieces, 0, lane);  // before the wait
  ptx::grid_dependency_wait();
  ptx::grid_dependents_launch();

  const uint4* xg = reinterpret_cast<const uint4*>(p.x);
  uint4* xs4 = reinterpret_cast<uint4*>(xs);
  const int xpieces = p.M * pieces;
  for (int i = static_cast<int>(threadIdx.x); i < MT * pieces; i += kThreads) {
    xs4[i] = i < xpieces ? xg[i] : make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();

  // debug build: the token rows this kernel may write (one fewer under the
  // short-rows fault)
  const int m_limit = CONVROT_DEBUG && p.fault == kFaultShortRows ? p.M - 1 : p.M;
  for (int64_t n = first; n < p.N; n += step) {
    int acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0;
    for (int blk = 0; blk < blocks; ++blk) {
      if (n != first || blk != 0) load_block(wv, p.w, n, p.K, pieces, blk, lane);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int q = blk * kBlockPieces + u * 32 + lane;
        if (q < pieces) {
          const uint4 wq = wv[u];
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const uint4 xv = xs4[m * pieces + q];
            int a = acc[m];
            a = __dp4a(static_cast<int>(wq.x), static_cast<int>(xv.x), a);
            a = __dp4a(static_cast<int>(wq.y), static_cast<int>(xv.y), a);
            a = __dp4a(static_cast<int>(wq.z), static_cast<int>(xv.z), a);
            a = __dp4a(static_cast<int>(wq.w), static_cast<int>(xv.w), a);
            acc[m] = a;
          }
        }
      }
    }
    // lane m takes token m's sum (|acc| <= 127^2 * K < 2^31 for K <= 131072)
    int mine = 0;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int s = __reduce_add_sync(0xffffffffu, acc[m]);
      if (m == lane) mine = s;
    }
    if (lane < p.M && in_bounds(lane < m_limit, p.status)) {
      const int64_t o = static_cast<int64_t>(lane) * p.N + n;
      if (p.out_s32) {
        static_cast<int32_t*>(p.out)[o] = mine;
      } else {
        const float sw = p.per_channel_scale ? p.s_w[n] : p.s_w[0];
        float bn = 0.f;
        if (p.bias != nullptr) {
          bn = p.out_f16 ? __half2float(__ushort_as_half(p.bias[n]))
                         : __uint_as_float(static_cast<uint32_t>(p.bias[n]) << 16);
        }
        const float y = fmaf(__int2float_rn(mine), p.s_tok[lane] * sw, bn);
        uint16_t bits;
        if (p.out_f16) {
          bits = __half_as_ushort(__float2half_rn(y));
        } else {
          const __nv_bfloat16 h = __float2bfloat16_rn(y);
          bits = *reinterpret_cast<const uint16_t*>(&h);
        }
        static_cast<uint16_t*>(p.out)[o] = bits;
      }
    }
  }
}

template <int MT>
cudaError_t launch_mt(const GemvParams& p, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(MT) * p.K;
  auto kern = int8_gemv_dp4a<MT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess) return e;
  // one warp per weight row while they fit on the SMs at once, else each
  // warp loops over rows
  const int64_t want = (p.N + kWarps - 1) / kWarps;
  const int64_t cap = static_cast<int64_t>(sm_count()) * (per_sm > 0 ? per_sm : 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(want < cap ? want : cap));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

bool int8_gemv_applies(const GemmArgs& a) {
  if (a.ops16 || a.M < 1 || a.M > kGemvMaxTokens || a.K % 16 != 0) return false;
  const int64_t rows = a.M <= 1 ? 1 : 2;  // launch_mt's MT
  return rows * a.K <= kGemvMaxCodeBytes;
}

cudaError_t launch_int8_gemv(const GemmArgs& a, cudaStream_t stream) {
  GemvParams p;
  cudaError_t e = status_word(&p.status);
  if (e != cudaSuccess) return e;
  p.x = a.A;
  p.w = a.B;
  p.s_tok = a.s_tok;
  p.s_w = a.s_w;
  p.bias = a.bias;
  p.out = a.out;
  p.M = static_cast<int>(a.M);
  p.N = a.N;
  p.K = static_cast<int>(a.K);
  p.per_channel_scale = a.s_w_len > 1 ? 1 : 0;
  p.out_s32 = a.out_s32 ? 1 : 0;
  p.out_f16 = a.out_f16 ? 1 : 0;
  p.fault = debug_fault();
  static_assert(kGemvMaxTokens == 2, "token counts instantiated below");
  if (a.M <= 1) return launch_mt<1>(p, stream);
  return launch_mt<2>(p, stream);
}

}  // namespace convrot
