// int8 GEMM for few tokens (M <= 128): the weight is the MMA's 128-row operand
// and the tokens its N dimension, so tensor-core work scales with the real
// token count and the kernel streams the weight at HBM speed.
//
//   D[n, m] = sum_k Wq[n, k] * xq[m, k]   (n: 128 weight rows per CTA, m: NT >= M tokens)
//
// K is split over a cluster of S CTAs (S <= 8) that share one 128-row block of
// the weight; each CTA accumulates its K range in TMEM, parks the int32
// partial in its shared memory, and after a cluster barrier every CTA sums
// the S partials of its share of the rows through distributed shared memory
// and applies the rescale/bias epilogue (or stores int32).  No global
// scratch.  Same warp roles and bounded waits as the main GEMM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace convrot {
namespace {

constexpr int kRows = 128;    // weight rows per CTA = MMA M
constexpr int kBK = 128;      // bytes per stage along K
constexpr int kUmmaK = 32;
constexpr int kThreads = 192;
constexpr uint64_t kWaitNs = 1000000000ull;

struct SkinnyParams {
  const float* s_tok;
  const float* s_w;
  const uint16_t* bias;
  void* out;
  int64_t M, N;
  int num_kb;        // k-blocks of the whole K
  int kb_per_split;  // k-blocks per cluster rank
  int splits;        // cluster size S
  int per_channel_scale;
  int out_s32;
  int out_f16;  // y and bias fp16 (else bf16)
  unsigned int* status;
};

template <int NT>
struct SkinnyCfg {
  static constexpr int kAStage = kRows * kBK;
  static constexpr int kBStage = NT * kBK;
  static constexpr int kStageBytes = kAStage + kBStage;
  // as many stages as fit (a CTA's whole K range in flight at once); the int32
  // partial reuses the ring once the mainloop has drained it
  static constexpr int kFit = (232448 - 1024 - 256) / kStageBytes;
  static constexpr int kStages = kFit > 12 ? 12 : kFit;
  static constexpr int kPartStride = NT + 4;  // int32 per partial row (padded: no bank conflicts)
  static constexpr int kPartBytes = kRows * kPartStride * 4;
  static_assert(kPartBytes <= kStages * kStageBytes, "partial must fit in the ring");
  static constexpr size_t kSmem = 1024 + kStages * kStageBytes + 256;
  static constexpr uint32_t kTmemCols = NT < 32 ? 32 : NT;
  static constexpr uint32_t kIdesc = ptx::idesc_i8(kRows, NT);
};

template <int STAGES>
struct SkinnyBars {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    int8_gemm_skinny(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                     const SkinnyParams p) {
  using C = SkinnyCfg<NT>;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * C::kAStage;
  int32_t* part = reinterpret_cast<int32_t*>(smem);  // after the mainloop only
  auto* bars = reinterpret_cast<SkinnyBars<kStages>*>(smem + kStages * C::kStageBytes);
  volatile uint32_t* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int block = static_cast<int>(blockIdx.x) / p.splits;  // 128-row block of the weight
  const int kb0 = static_cast<int>(rank) * p.kb_per_split;
  const int kb1 = min(p.num_kb, kb0 + p.kb_per_split);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&bars->full[s], 1);
      ptx::mbar_init(&bars->empty[s], 1);
    }
    ptx::mbar_init(&bars->acc_full, 1);
    bars->abort_flag = 0;
    ptx::fence_mbarrier_init();
    ptx::tma_prefetch_desc(&tmW);
    ptx::tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&bars->tmem_base, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // the set-up above overlaps the previous kernel of the stream; every global
  // access below comes after it
  ptx::grid_dependency_wait();
  ptx::grid_dependents_launch();

  if (threadIdx.x == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!ptx::mbar_wait(&bars->empty[stage], phase ^ 1u, ptx::globaltimer_ns() + kWaitNs)) {
        atomicOr(p.status, 1u);
        *abort_flag = 1;
        break;
      }
      ptx::mbar_arrive_expect_tx(&bars->full[stage], C::kStageBytes);
      ptx::tma_load_2d(sA + stage * C::kAStage, &tmW, &bars->full[stage], kb * kBK, block * kRows);
      ptx::tma_load_2d(sB + stage * C::kBStage, &tmX, &bars->full[stage], kb * kBK, 0);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  } else if (threadIdx.x == 32) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!ptx::mbar_wait(&bars->full[stage], phase, ptx::globaltimer_ns() + kWaitNs)) {
        atomicOr(p.status, 1u);
        *abort_flag = 1;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t a_addr = ptx::smem_u32(sA + stage * C::kAStage);
      const uint32_t b_addr = ptx::smem_u32(sB + stage * C::kBStage);
#pragma unroll
      for (int k = 0; k < kBK / kUmmaK; ++k) {
        ptx::mma_i8(tmem, ptx::smem_desc_k_sw128(a_addr + k * kUmmaK),
                    ptx::smem_desc_k_sw128(b_addr + k * kUmmaK), C::kIdesc,
                    (kb > kb0 || k > 0) ? 1u : 0u);
      }
      ptx::mma_commit(&bars->empty[stage]);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    // publishes the accumulator once every MMA issued above has completed
    ptx::mma_commit(&bars->acc_full);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ partial -> shared memory
    const int quarter = warp & 3;
    const int row = quarter * 32 + static_cast<int>(lane);
    const bool ready =
        __all_sync(0xffffffffu, ptx::mbar_wait(&bars->acc_full, 0, ptx::globaltimer_ns() + kWaitNs));
    ptx::tc_fence_after();
    const uint32_t t_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int32_t* dst = part + row * C::kPartStride;
    if (kb1 <= kb0 || !ready || *abort_flag) {
      if (!ready && lane == 0) atomicOr(p.status, 1u);
#pragma unroll
      for (int c = 0; c < NT; c += 4) *reinterpret_cast<int4*>(dst + c) = make_int4(0, 0, 0, 0);
    } else if constexpr (NT == 16) {
      uint32_t r[16];
      ptx::tmem_ld_32x32b_x16(t_base, r);
      ptx::tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 16; c += 4) {
        *reinterpret_cast<uint4*>(dst + c) = make_uint4(r[c], r[c + 1], r[c + 2], r[c + 3]);
      }
    } else {
#pragma unroll 1
      for (int c0 = 0; c0 < NT; c0 += 32) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(t_base + c0, r);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          *reinterpret_cast<uint4*>(dst + c0 + c) = make_uint4(r[c], r[c + 1], r[c + 2], r[c + 3]);
        }
      }
    }
  }

  // ---------------------------------------------------------------- split-K reduction
  ptx::tc_fence_before();
  ptx::cluster_sync();  // every CTA's partial is in its shared memory
  {
    // this CTA finishes rows [r0, r0 + rows) of the block, for all tokens
    const int rows = kRows / p.splits;
    const int r0 = static_cast<int>(rank) * rows;
    const uint32_t part_local = ptx::smem_u32(part);
    const int items = rows * (NT / 4);  // (row, 4 tokens) items
    for (int it = threadIdx.x; it < items; it += kThreads) {
      const int rr = r0 + it % rows;   // consecutive threads -> consecutive weight rows
      const int m4 = (it / rows) * 4;  // first of 4 tokens
      int32_t acc[4] = {0, 0, 0, 0};
      const uint32_t off = static_cast<uint32_t>((rr * C::kPartStride + m4) * 4);
      for (int s = 0; s < p.splits; ++s) {
        const uint4 v = ptx::ld_cluster_v4(ptx::mapa_shared(part_local + off, static_cast<uint32_t>(s)));
        acc[0] += static_cast<int32_t>(v.x);
        acc[1] += static_cast<int32_t>(v.y);
        acc[2] += static_cast<int32_t>(v.z);
        acc[3] += static_cast<int32_t>(v.w);
      }
      const int64_t n = static_cast<int64_t>(block) * kRows + rr;
      if (n >= p.N) continue;
      const float sw = p.out_s32 ? 0.f : (p.per_channel_scale ? p.s_w[n] : p.s_w[0]);
      float bn = 0.f;
      if (!p.out_s32 && p.bias) {
        bn = p.out_f16 ? __half2float(__ushort_as_half(p.bias[n]))
                       : __uint_as_float(static_cast<uint32_t>(p.bias[n]) << 16);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t m = m4 + j;
        if (m >= p.M) break;
        if (p.out_s32) {
          static_cast<int32_t*>(p.out)[m * p.N + n] = acc[j];
        } else {
          const float y = fmaf(__int2float_rn(acc[j]), p.s_tok[m] * sw, bn);
          uint16_t bits;
          if (p.out_f16) {
            bits = __half_as_ushort(__float2half_rn(y));
          } else {
            const __nv_bfloat16 h = __float2bfloat16_rn(y);
            bits = *reinterpret_cast<const uint16_t*>(&h);
          }
          static_cast<uint16_t*>(p.out)[m * p.N + n] = bits;
        }
      }
    }
  }
  ptx::cluster_sync();  // peers' partials stay alive until every CTA has read them
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

bool encode_rows(CUtensorMap* map, const int8_t* base, int64_t rows, int64_t K, int box_rows) {
  return encode_tma_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, static_cast<uint64_t>(K),
                       static_cast<uint64_t>(rows), static_cast<uint64_t>(K), kBK,
                       static_cast<uint32_t>(box_rows));
}

template <int NT>
cudaError_t launch_nt(const GemmArgs& a, SkinnyParams p, cudaStream_t stream) {
  using C = SkinnyCfg<NT>;
  CUtensorMap tmW, tmX;
  if (!encode_rows(&tmW, a.B, a.N, a.K, kRows) || !encode_rows(&tmX, a.A, a.M, a.K, NT)) {
    return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(int8_gemm_skinny<NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  const int blocks = static_cast<int>((a.N + kRows - 1) / kRows);
  int splits = sm_count() / blocks;  // one wave of CTAs
  splits = splits < 1 ? 1 : (splits > 8 ? 8 : splits);
  if (splits > p.num_kb) splits = p.num_kb;
  while (kRows % splits) --splits;  // each rank finishes an equal share of the 128 rows
  p.splits = splits;
  p.kb_per_split = (p.num_kb + splits - 1) / splits;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks * splits));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, int8_gemm_skinny<NT>, tmW, tmX, p);
}

}  // namespace

cudaError_t launch_int8_gemm_skinny(const GemmArgs& a, cudaStream_t stream) {
  SkinnyParams p;
  cudaError_t e = status_word(&p.status);
  if (e != cudaSuccess) return e;
  p.s_tok = a.s_tok;
  p.s_w = a.s_w;
  p.bias = a.bias;
  p.out = a.out;
  p.M = a.M;
  p.N = a.N;
  p.num_kb = static_cast<int>((a.K + kBK - 1) / kBK);
  p.per_channel_scale = a.s_w_len > 1 ? 1 : 0;
  p.out_s32 = a.out_s32 ? 1 : 0;
  p.out_f16 = a.out_f16 ? 1 : 0;
  if (a.M <= 16) return launch_nt<16>(a, p, stream);
  if (a.M <= 32) return launch_nt<32>(a, p, stream);
  if (a.M <= 64) return launch_nt<64>(a, p, stream);
  return launch_nt<128>(a, p, stream);
}

}  // namespace convrot
