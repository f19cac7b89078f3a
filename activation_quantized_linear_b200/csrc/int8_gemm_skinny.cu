// int8 GEMM for few tokens (M <= 128): the weight is the MMA's 128-row operand
// and the tokens its N dimension, so tensor-core work scales with the real
// token count and the kernel streams the weight at HBM speed.
//
//   D[n, m] = sum_k Wq[n, k] * xq[m, k]   (n: 128 weight rows per CTA, m: NT >= M tokens)
//
// K is split over a cluster of S CTAs (S <= 8) that share one 128-row block of
// the weight; each CTA accumulates its K range in TMEM and parks the int32
// partial in its shared memory.  After a cluster barrier every CTA pushes the
// rows each peer finishes into that peer's shared memory with one bulk copy
// per peer (completed on the peer's mbarrier), then sums the S partials of its
// own 128 / S rows from local shared memory and applies the rescale/bias
// epilogue (or stores int32).  No global scratch.  Same warp roles and bounded
// waits as the main GEMM.
//
// Bulk copies rather than per-thread loads through the cluster window: with
// every thread pulling 16-byte pieces of its peers' partials the reduction
// ran at a few bytes per clock per SM and took half of the kernel at 128
// tokens; keeping more such loads in flight made it slower still.
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
  unsigned int* status;  // bit 0: a wait ran out; bit 1: debug bounds
  int fault;             // debug build: injected fault (kFaultSkipStage, kFaultShortRows)
};

template <int NT>
struct SkinnyCfg {
  static constexpr int kAStage = kRows * kBK;
  static constexpr int kBStage = NT * kBK;
  static constexpr int kStageBytes = kAStage + kBStage;
  // epilogue factors staged during the mainloop: s_tok of the NT tokens, s_w
  // and bias of the block's rows (f32)
  static constexpr int kEpiBytes = (NT + 2 * kRows) * 4;
  static constexpr int kPartStride = NT + 4;  // int32 per partial row (padded: no bank conflicts)
  static constexpr int kPartBytes = kRows * kPartStride * 4;
  // Two CTAs per SM when the ring that fits half of the SM's shared memory
  // still holds the int32 partial and the peers' slices (NT <= 64): a CTA of
  // the next launch then lands beside one of this launch, issues its weight
  // loads while this one finishes, and a weight of more 128-row blocks than
  // SMs runs in one wave.  Otherwise as many stages as fit one CTA per SM.
  // The partial reuses the ring once the mainloop has drained it.
  static constexpr int kHalfFit = (115712 - 1024 - 256 - kEpiBytes) / kStageBytes;
  static constexpr int kFit = (232448 - 1024 - 256 - kEpiBytes) / kStageBytes;
  static constexpr bool kTwoPerSm = 2 * kPartBytes <= kHalfFit * kStageBytes;
  static constexpr int kStages = kTwoPerSm ? kHalfFit : (kFit > 12 ? 12 : kFit);
  // the partial and, after it, the slices the peers push (one per rank)
  static_assert(2 * kPartBytes <= kStages * kStageBytes, "partial and slices must fit in the ring");
  static constexpr size_t kSmem = 1024 + kStages * kStageBytes + 256 + kEpiBytes;
  static constexpr uint32_t kTmemCols = NT < 32 ? 32 : NT;
  static constexpr uint32_t kIdesc = ptx::idesc_i8(kRows, NT);
};

template <int STAGES>
struct SkinnyBars {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t recv_full;  // the peers' slices have landed
  uint32_t tmem_base;
  uint32_t abort_flag;
};

template <int NT>
__global__ void __launch_bounds__(kThreads, SkinnyCfg<NT>::kTwoPerSm ? 2 : 1)
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
  int32_t* recv = part + kRows * C::kPartStride;     // [splits][rows][kPartStride]
  auto* bars = reinterpret_cast<SkinnyBars<kStages>*>(smem + kStages * C::kStageBytes);
  volatile uint32_t* abort_flag = &bars->abort_flag;
  float* ep_tok = reinterpret_cast<float*>(smem + kStages * C::kStageBytes + 256);  // [NT]
  float* ep_sw = ep_tok + NT;      // [rows], this CTA's share of the block
  float* ep_bias = ep_sw + kRows;  // [rows]

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int block = static_cast<int>(blockIdx.x) / p.splits;  // 128-row block of the weight
  const int kb0 = static_cast<int>(rank) * p.kb_per_split;
  const int kb1 = min(p.num_kb, kb0 + p.kb_per_split);
  // after the split-K reduction this CTA finishes rows [r0, r0 + rows) of the block
  const int rows = kRows / p.splits;
  const int r0 = static_cast<int>(rank) * rows;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&bars->full[s], 1);
      ptx::mbar_init(&bars->empty[s], 1);
    }
    ptx::mbar_init(&bars->acc_full, 1);
    ptx::mbar_init(&bars->recv_full, 1);
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
  // The int8 weight is never written by the kernel this one is chained to
  // (the library's weight quantizer ends with a plain launch), so the
  // producer issues the weight loads of its first stages before waiting on
  // that kernel: they stream while it drains.  The tokens' codes come after.
  const int early = kb1 - kb0 < kStages ? (kb1 > kb0 ? kb1 - kb0 : 0) : kStages;
  // debug build: the skipped-stage fault leaves stage 0 empty (no expected
  // bytes, no copies), so the MMA issuer's bounded wait on it runs out
  const bool skip0 = CONVROT_DEBUG && p.fault == kFaultSkipStage;
  if (threadIdx.x == 0) {
    for (int i = 0; i < early; ++i) {  // fresh ring: every stage is free
      if (skip0 && i == 0) continue;
      ptx::mbar_arrive_expect_tx(&bars->full[i], C::kStageBytes);
      ptx::tma_load_2d(sA + i * C::kAStage, &tmW, &bars->full[i], (kb0 + i) * kBK, block * kRows);
    }
  }
  // the set-up above overlaps the previous kernel of the stream; every other
  // global access below comes after it
  ptx::grid_dependency_wait();
  ptx::grid_dependents_launch();

  if (threadIdx.x == 0) {
    // ------------------------------------------------------------ producer
    // the early stages' codes first (always, so every issued stage completes)
    for (int i = 0; i < early; ++i) {
      if (skip0 && i == 0) continue;
      ptx::tma_load_2d(sB + i * C::kBStage, &tmX, &bars->full[i], (kb0 + i) * kBK, 0);
    }
    int stage = early == kStages ? 0 : early;
    uint32_t phase = early == kStages ? 1u : 0u;
    for (int kb = kb0 + early; kb < kb1; ++kb) {
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
    // ------------------------------------------------------------ epilogue factors
    // read while the mainloop streams the weight, so the reduction below
    // touches no global memory before its stores
    if (!p.out_s32) {
      const int t = static_cast<int>(threadIdx.x) - 64;
      for (int m = t; m < NT; m += kThreads - 64) ep_tok[m] = m < p.M ? p.s_tok[m] : 0.f;
      for (int r = t; r < rows; r += kThreads - 64) {
        const int64_t n = static_cast<int64_t>(block) * kRows + r0 + r;
        float sw = 0.f, bn = 0.f;
        if (n < p.N) {
          sw = p.per_channel_scale ? p.s_w[n] : p.s_w[0];
          if (p.bias) {
            bn = p.out_f16 ? __half2float(__ushort_as_half(p.bias[n]))
                           : __uint_as_float(static_cast<uint32_t>(p.bias[n]) << 16);
          }
        }
        ep_sw[r] = sw;
        ep_bias[r] = bn;
      }
    }
    // ------------------------------------------------------------ partial -> shared memory
    const int quarter = warp & 3;
    const int row = quarter * 32 + static_cast<int>(lane);
    const bool ready =
        __all_sync(0xffffffffu, ptx::mbar_wait(&bars->acc_full, 0, ptx::globaltimer_ns() + kWaitNs));
    ptx::tc_fence_after();
    const uint32_t t_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int32_t* dst = part + row * C::kPartStride;
    if (p.splits == 1) {
      // one CTA holds the whole K: each thread drains its weight row n from
      // TMEM straight to y[:, n] (a warp's 32 rows are 32 consecutive outputs
      // of a token); the factors staged above are read after the four
      // epilogue warps' barrier, which every one of them reaches.  After a
      // timeout nothing is stored (the status word reports it).
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const bool drain = ready && !__any_sync(0xffffffffu, *abort_flag != 0);
      // debug build: the tokens this kernel may write (one fewer under the
      // short-rows fault)
      const int64_t m_limit = CONVROT_DEBUG && p.fault == kFaultShortRows ? p.M - 1 : p.M;
      const int64_t n = static_cast<int64_t>(block) * kRows + row;
      const float sw = p.out_s32 ? 0.f : ep_sw[row];
      const float bn = p.out_s32 ? 0.f : ep_bias[row];
#pragma unroll 1
      for (int c0 = 0; drain && c0 < NT; c0 += 16) {
        uint32_t r[16];
        ptx::tmem_ld_32x32b_x16(t_base + c0, r);
        ptx::tmem_ld_wait();
        if (n >= p.N) continue;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int64_t m = c0 + j;
          if (m >= p.M) break;
          if (!in_bounds(m < m_limit && n < p.N, p.status)) continue;
          if (p.out_s32) {
            static_cast<int32_t*>(p.out)[m * p.N + n] = static_cast<int32_t>(r[j]);
          } else {
            const float y = fmaf(__int2float_rn(static_cast<int32_t>(r[j])), ep_tok[m] * sw, bn);
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
    } else if (kb1 <= kb0 || !ready || *abort_flag) {
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
  const uint32_t slice_words = static_cast<uint32_t>(rows * C::kPartStride);
  if (warp >= 2) ptx::fence_proxy_async_smem();  // the partial, for the bulk copies below
  if (threadIdx.x == 0 && p.splits > 1) {
    // armed before the barrier: no peer pushes before every CTA has passed it
    ptx::mbar_arrive_expect_tx(&bars->recv_full, static_cast<uint32_t>(p.splits - 1) * slice_words * 4u);
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();  // every CTA's partial (and the staged factors) in shared memory
  if (p.splits > 1) {
    // push rank o's rows of this CTA's partial into slot [rank] of rank o
    if (threadIdx.x == 0) {
      for (int o = 0; o < p.splits; ++o) {
        if (o == static_cast<int>(rank)) continue;
        ptx::bulk_copy_to_peer(
            ptx::mapa_shared(ptx::smem_u32(recv + rank * slice_words), static_cast<uint32_t>(o)),
            ptx::smem_u32(part + o * slice_words), slice_words * 4u,
            ptx::mapa_shared(ptx::smem_u32(&bars->recv_full), static_cast<uint32_t>(o)));
      }
    }
    if (!ptx::mbar_wait(&bars->recv_full, 0, ptx::globaltimer_ns() + kWaitNs) && lane == 0) {
      atomicOr(p.status, 1u);
    }
  }
  // every copy into this CTA has landed; once all ranks have arrived, every
  // copy out of this CTA has too, and its shared memory may be released
  __syncwarp();
  ptx::cluster_arrive();
  if (p.splits > 1) {
    // (row, 4 tokens) items; consecutive threads take consecutive weight rows
    const int items = rows * (NT / 4);
    for (int it = threadIdx.x; it < items; it += kThreads) {
      const int r = it % rows;
      const int m4 = (it / rows) * 4;  // first of 4 tokens
      int4 acc = *reinterpret_cast<const int4*>(part + (r0 + r) * C::kPartStride + m4);
      for (int s = 0; s < p.splits; ++s) {
        if (s == static_cast<int>(rank)) continue;
        const int4 v = *reinterpret_cast<const int4*>(recv + s * slice_words + r * C::kPartStride + m4);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      const int32_t a4[4] = {acc.x, acc.y, acc.z, acc.w};
      const int64_t n = static_cast<int64_t>(block) * kRows + r0 + r;
      if (n >= p.N) continue;
      const float sw = p.out_s32 ? 0.f : ep_sw[r];
      const float bn = p.out_s32 ? 0.f : ep_bias[r];
      const int64_t m_limit = CONVROT_DEBUG && p.fault == kFaultShortRows ? p.M - 1 : p.M;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t m = m4 + j;
        if (m >= p.M) break;
        if (!in_bounds(m < m_limit, p.status)) continue;
        if (p.out_s32) {
          static_cast<int32_t*>(p.out)[m * p.N + n] = a4[j];
        } else {
          const float y = fmaf(__int2float_rn(a4[j]), ep_tok[m] * sw, bn);
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
  __syncwarp();
  ptx::cluster_wait();
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
  // as many CTAs as fit in one wave: two per SM when the ring is sized for it
  // (chained few-token launches over 3840 x 11520 and 10240 x 3840 weights
  // measured 6 and 10 % faster than with one CTA per SM's worth of splits)
  int splits = (C::kTwoPerSm ? 2 : 1) * sm_count() / blocks;
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
  if (int8_gemv_applies(a)) return launch_int8_gemv(a, stream);
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
  p.fault = debug_fault();
  if (a.M <= 16) return launch_nt<16>(a, p, stream);
  if (a.M <= 32) return launch_nt<32>(a, p, stream);
  if (a.M <= 64) return launch_nt<64>(a, p, stream);
  return launch_nt<128>(a, p, stream);
}

}  // namespace convrot
