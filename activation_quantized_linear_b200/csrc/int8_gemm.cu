// int8 x int8 -> int32 GEMM on the sm_100a tensor cores with the ConvRot
// rescale epilogue fused (Invoke docs "int8 Compute", opening section: each
// layer "multiplies int8 by int8" on the int8 tensor cores):
//
//   acc[m, n] = sum_k xq[m, k] * Wq[n, k]                       (exact int32)
//   y[m, n]   = bf16_rn(float(acc) * (s_tok[m] * s_w[n|0]) + bias[n])
//
// Structure (persistent; one CTA per SM, CTA pairs as clusters of two SMs):
//   warp 0      TMA producer: A and B int8 tiles of 128-byte rows, 128-byte
//               swizzle, into a shared-memory ring;
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma
//               kind::i8 (K = 32 per instruction) into one of two 256-column
//               int32 accumulators; tcgen05.commit frees the stage / publishes
//               the accumulator;
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, rescale, bias, bf16,
//               128-bit global stores; then release the accumulator so the MMA
//               of the next tile overlaps this tile's epilogue.
// A CTA pair (cta_group::2) works on 256 x 256 tiles: each CTA loads its 128
// rows of A and 128 rows of B (no multicast), the even CTA issues M=256 x
// N=256 MMAs whose accumulators are split across the two CTAs' TMEM, and
// commits signal both CTAs' barriers.  A pair moves 2/3 of the operand bytes
// per MMA that two single CTAs would.  (Up to 128 tokens take the swap-AB
// kernel in int8_gemm_skinny.cu instead.)
// The same pipeline with 16-bit operands (kind::f16, fp32 accumulator, no
// scales: y = f16(acc + bias)) is the dense linear of the default path, which
// multiplies by the decoded weight (gemm16_tcgen05).
// Every mbarrier wait is bounded by the global timer.  A wait that runs out
// records CONVROT_ERR_TIMEOUT in the device status word; the CTA then stops
// issuing work, drains what it issued and frees its TMEM before returning.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace convrot {
namespace {

constexpr int BM = 128;       // accumulator rows per CTA (TMEM lanes)
constexpr int BN = 256;       // accumulator columns per tile
constexpr int BK = 128;       // bytes per operand row per stage; one 128-byte swizzle row
constexpr int UMMA_K = 32;    // bytes of K per MMA (32 int8 or 16 16-bit elements)
constexpr int A_STAGE = BM * BK;
constexpr int ACC_COLS = BN;  // 32-bit accumulator columns per tile
constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s per wait

// Operand kinds: int8 (int32 accumulator, ConvRot epilogue), or bf16 / fp16
// (fp32 accumulator, bias only).
constexpr int kKindI8 = 0, kKindBF16 = 1, kKindF16 = 2;

// A cluster of two CTAs per tile of 256 x 256 (cta_group::2); each CTA loads
// its 128 rows of A and its 128 rows of B per stage, 6 stages, and only the
// even CTA issues the MMAs.  The geometry is in bytes, the same for every kind.
struct Cfg {
  static constexpr int kBRows = BN / 2;  // B rows loaded per CTA
  static constexpr int kBStage = kBRows * BK;
  static constexpr int kStageBytes = A_STAGE + kBStage;
  static constexpr int kStages = 6;
  static constexpr int kTileM = 2 * BM;
  // each epilogue warp's copy of a tile's 256 bias values and 256 weight
  // scales (float)
  static constexpr int kEpiWarpBytes = 2 * BN * 4;
  // each epilogue warp's 32 x 32 tile of 16-bit outputs, staged so that the
  // global stores write whole 64-byte row segments
  static constexpr int kEpiStageBytes = 32 * 64;
  static constexpr size_t kSmem =
      1024 + kStages * kStageBytes + 256 + 4 * kEpiWarpBytes + 4 * kEpiStageBytes;
  // bytes that complete one stage on the leader's full barrier (both CTAs' loads)
  static constexpr uint32_t kTxBytes = 2 * kStageBytes;
};

template <int kKind>
struct KindCfg {
  static constexpr uint32_t kIdesc = kKind == kKindI8
                                         ? ptx::idesc_i8(Cfg::kTileM, BN)
                                         : ptx::idesc_f16(Cfg::kTileM, BN, kKind == kKindF16);
  static constexpr int kStageK = kKind == kKindI8 ? BK : BK / 2;  // K elements per stage
};

struct Params {
  const float* s_tok;
  const float* s_w;
  const uint16_t* bias;
  void* out;
  int64_t M, N;
  int num_kb;
  int m_tiles, n_tiles;
  int group_m;
  int per_channel_scale;
  int out_s32;
  int out_f16;           // y and bias fp16 (else bf16)
  unsigned int* status;  // device status word (bit 0: a wait ran out; bit 1: debug bounds)
  int fault;             // debug build: injected fault (kFaultSkipStage, kFaultShortRows)
};

template <int STAGES>
struct Barriers {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

// Tile raster: groups of `group_m` M-tiles sweep all N-tiles, M fastest, so
// the tiles in flight share their weight (B) tiles; with group_m = m_tiles
// every weight tile is read once while all of A stays in L2.
__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int group_m, int& mb,
                                            int& nb) {
  const int per_group = group_m * n_tiles;
  const int g = tile / per_group;
  const int first_m = g * group_m;
  const int gm = min(group_m, m_tiles - first_m);
  const int local = tile - g * per_group;
  mb = first_m + local % gm;
  nb = local / gm;
}

__device__ __forceinline__ void record_timeout(volatile uint32_t* abort_flag, unsigned int* status) {
  atomicOr(status, 1u);
  *abort_flag = 1u;
}

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity) {
  return ptx::mbar_wait(bar, parity, ptx::globaltimer_ns() + kWaitNs);
}

// 32 outputs of one row: y = f16(float(acc) * scale [* s_w_row] + bias), in bf16
// or fp16 (f16), rounded once from the fp32 FMA.  The accumulator columns hold
// int32 (kF32Acc = false) or fp32 (true: scale is 1, so y = f16(acc + bias)).
__device__ __forceinline__ float widen16(uint16_t v, bool f16) {
  return f16 ? __half2float(__ushort_as_half(v)) : __uint_as_float(static_cast<uint32_t>(v) << 16);
}

// 32 outputs of one row: y = f16(float(acc) * scale [* s_w[col]] + bias[col]),
// in bf16 or fp16 (f16), rounded once from the fp32 FMA, with the tile's bias
// and weight scales read from the warp's shared-memory copy (float; `bias`
// null: none, `s_w` null: per tensor), as 16 words of two 16-bit values.  The
// accumulator columns hold int32 (kF32Acc = false) or fp32 (true: scale is 1,
// so y = f16(acc + bias)).  Columns past a half-filled chunk read staged
// zeros and are not stored.
template <bool kF32Acc>
__device__ __forceinline__ void row32_words(uint32_t (&w)[16], const uint32_t (&r)[32], float scale,
                                            const float* s_w, const float* bias, bool f16) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int col = 2 * i;
    float lo = kF32Acc ? __uint_as_float(r[2 * i]) : __int2float_rn(static_cast<int32_t>(r[2 * i]));
    float hi = kF32Acc ? __uint_as_float(r[2 * i + 1])
                       : __int2float_rn(static_cast<int32_t>(r[2 * i + 1]));
    const float sl = s_w ? scale * s_w[col] : scale;
    const float sh = s_w ? scale * s_w[col + 1] : scale;
    const float bl = bias ? bias[col] : 0.f, bh = bias ? bias[col + 1] : 0.f;
    lo = fmaf(lo, sl, bl);
    hi = fmaf(hi, sh, bh);
    if (f16) {
      const __half2 h = __floats2half2_rn(lo, hi);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    } else {
      const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
}

// 16-byte unit k of row r (0..31) of an epilogue warp's 32 x 32 staging tile
// of 16-bit outputs (64-byte rows).  The unit index is XOR-ed with bits 1..2 of
// the row: a quarter-warp writing one unit of rows r..r+7, or reading the four
// units of two rows, then touches eight distinct 16-byte bank groups.
__device__ __forceinline__ int stage_unit(int r, int k) { return r * 4 + (k ^ ((r >> 1) & 3)); }

__device__ __forceinline__ void store_s32_row32(int32_t* dst, const uint32_t (&r)[32], int valid) {
  uint4* q = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i < 4 || valid == 32) q[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
  }
}

template <int kKind>
__device__ __forceinline__ void gemm_pair(const CUtensorMap& tmA, const CUtensorMap& tmB,
                                          const Params& p) {
  using C = Cfg;
  using KC = KindCfg<kKind>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kStages * A_STAGE;
  auto* bars = reinterpret_cast<Barriers<C::kStages>*>(smem + C::kStages * C::kStageBytes);
  static_assert(sizeof(Barriers<C::kStages>) <= 256, "barriers must fit their 256 bytes");
  float* ep_all = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes + 256);
  volatile uint32_t* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();  // CTA within the pair
  const bool leader = rank == 0;
  const int unit = static_cast<int>(blockIdx.x >> 1);
  const int units = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(&bars->full[s], 1);
      ptx::mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&bars->acc_full[a], 1);
      ptx::mbar_init(&bars->acc_empty[a], 2 * kEpiWarps);
    }
    ptx::mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    ptx::fence_mbarrier_init();
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(&bars->tmem_base, TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();  // both CTAs' barriers initialised before any cross-CTA signal
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int num_tiles = p.m_tiles * p.n_tiles;
  // The int8 weight (B) is never written by the kernel this one is chained
  // to (nothing in this library writes int8 weights in a chained launch: the
  // weight quantizer ends with a plain launch), so the producer issues the
  // weight loads of its first stages before waiting on that kernel; they fill
  // the ring while it drains.  The 16-bit GEMM's B is the decoded weight,
  // which the decode right before it writes, so it waits first.
  constexpr bool kEarlyB = kKind == kKindI8;
  // debug build: the skipped-stage fault leaves the first tile's stage 0
  // empty in both CTAs (no expected bytes, no copies), so the MMA issuer's
  // bounded wait on it runs out and the kernel takes its abort path
  const bool skip0 = CONVROT_DEBUG && p.fault == kFaultSkipStage;
  int early = 0;  // stages of the first tile whose B load is already issued
  if (kEarlyB && threadIdx.x == 0 && unit < num_tiles) {
    int mb, nb;
    tile_coords(unit, p.m_tiles, p.n_tiles, p.group_m, mb, nb);
    const int b_row = nb * BN + static_cast<int>(rank) * C::kBRows;
    early = p.num_kb < C::kStages ? p.num_kb : C::kStages;
    for (int kb = 0; kb < early; ++kb) {  // fresh ring: every stage is free
      if (skip0 && kb == 0) continue;
      if (leader) ptx::mbar_arrive_expect_tx(&bars->full[kb], C::kTxBytes);
      ptx::tma_load_2d_pair(sB + kb * C::kBStage, &tmB, &bars->full[kb], kb * KC::kStageK, b_row);
    }
  }
  // the set-up above overlaps the previous kernel of the stream; every other
  // global access below comes after it (the whole grid is resident, so the
  // next kernel may be scheduled right away)
  ptx::grid_dependency_wait();
  ptx::grid_dependents_launch();

  if (threadIdx.x == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    int last_stage = -1;
    uint32_t last_phase = 0;
    if (early > 0) {
      // the first tile's early stages: their B is in flight, add A (always,
      // so that every issued stage completes before the CTA can exit)
      int mb, nb;
      tile_coords(unit, p.m_tiles, p.n_tiles, p.group_m, mb, nb);
      const int a_row = mb * C::kTileM + static_cast<int>(rank) * BM;
      for (int kb = 0; kb < early; ++kb) {
        if (skip0 && kb == 0) continue;
        ptx::tma_load_2d_pair(sA + kb * A_STAGE, &tmA, &bars->full[kb], kb * KC::kStageK, a_row);
      }
      last_stage = early - 1;
      stage = early == C::kStages ? 0 : early;
      phase = early == C::kStages ? 1u : 0u;
    }
    for (int tile = unit; tile < num_tiles && !*abort_flag; tile += units) {
      int mb, nb;
      tile_coords(tile, p.m_tiles, p.n_tiles, p.group_m, mb, nb);
      const int a_row = mb * C::kTileM + static_cast<int>(rank) * BM;
      const int b_row = nb * BN + static_cast<int>(rank) * C::kBRows;
      for (int kb = tile == unit ? early : 0; kb < p.num_kb; ++kb) {
        if (!wait_bounded(&bars->empty[stage], phase ^ 1u)) {
          record_timeout(abort_flag, p.status);
          break;
        }
        if (skip0 && tile == unit && kb == 0) {  // (a form without early loads)
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
          continue;
        }
        if (leader) ptx::mbar_arrive_expect_tx(&bars->full[stage], C::kTxBytes);
        ptx::tma_load_2d_pair(sA + stage * A_STAGE, &tmA, &bars->full[stage], kb * KC::kStageK, a_row);
        ptx::tma_load_2d_pair(sB + stage * C::kBStage, &tmB, &bars->full[stage], kb * KC::kStageK,
                              b_row);
        last_stage = stage;
        last_phase = phase;
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (*abort_flag && last_stage >= 0 && leader) {
      // let the last copy land before the CTA's shared memory goes away
      ptx::mbar_wait(&bars->full[last_stage], last_phase, ptx::globaltimer_ns() + 10000000ull);
    }
  } else if (threadIdx.x == 32 && leader) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;
    bool issued = false;
    for (int tile = unit; tile < num_tiles && !*abort_flag; tile += units, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!wait_bounded(&bars->acc_empty[acc], acc_phase ^ 1u)) {
        record_timeout(abort_flag, p.status);
        break;
      }
      ptx::tc_fence_after();
      const uint32_t d_tmem = tmem + acc * ACC_COLS;
      bool ok = true;
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!wait_bounded(&bars->full[stage], phase)) {
          record_timeout(abort_flag, p.status);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a_addr = ptx::smem_u32(sA + stage * A_STAGE);
        const uint32_t b_addr = ptx::smem_u32(sB + stage * C::kBStage);
#pragma unroll
        for (int k = 0; k < BK / UMMA_K; ++k) {
          const uint64_t ad = ptx::smem_desc_k_sw128(a_addr + k * UMMA_K);
          const uint64_t bd = ptx::smem_desc_k_sw128(b_addr + k * UMMA_K);
          if constexpr (kKind == kKindI8) {
            ptx::mma_i8_pair(d_tmem, ad, bd, KC::kIdesc, (kb | k) != 0 ? 1u : 0u);
          } else {
            ptx::mma_f16_pair(d_tmem, ad, bd, KC::kIdesc, (kb | k) != 0 ? 1u : 0u);
          }
        }
        issued = true;
        ptx::mma_commit_pair(&bars->empty[stage]);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      ptx::mma_commit_pair(&bars->acc_full[acc]);
    }
    if (*abort_flag && issued) {
      // every MMA issued so far must finish before TMEM is released
      ptx::mma_commit_pair_local(&bars->drain);
      ptx::mbar_wait(&bars->drain, 0, ptx::globaltimer_ns() + 10000000ull);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may read: 32*quarter ..
    const int row = quarter * 32 + static_cast<int>(lane);
    // this warp's copy of the tile's factors: bias [BN], weight scales [BN]
    float* ep_bias = ep_all + (warp - 2) * (C::kEpiWarpBytes / 4);
    float* ep_sw = ep_bias + BN;
    uint4* ep_stage = reinterpret_cast<uint4*>(ep_all + 4 * (C::kEpiWarpBytes / 4)) +
                      (warp - 2) * (C::kEpiStageBytes / 16);
    const bool has_bias = p.bias != nullptr;
    const bool chan_sw = kKind == kKindI8 && p.per_channel_scale && !p.out_s32;
    int local = 0;
    for (int tile = unit; tile < num_tiles; tile += units, ++local) {
      int mb, nb;
      tile_coords(tile, p.m_tiles, p.n_tiles, p.group_m, mb, nb);
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      // Stage the tile's bias and per-channel scales before waiting for its
      // accumulator, so the loads overlap the tile's MMAs instead of
      // following each 32-column chunk: lane i takes columns 8i .. 8i + 7
      // (N % 16 == 0, so such a group is wholly inside or outside N).
      __syncwarp();  // the previous tile's copy is no longer read
      {
        const int64_t col = static_cast<int64_t>(nb) * BN + 8 * lane;
        const bool in_n = col < p.N;
        float b8[8], s8[8];
        if (has_bias && in_n) {
          const uint4 v = *reinterpret_cast<const uint4*>(p.bias + col);
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            b8[2 * k] = widen16(static_cast<uint16_t>(wv[k] & 0xffffu), p.out_f16 != 0);
            b8[2 * k + 1] = widen16(static_cast<uint16_t>(wv[k] >> 16), p.out_f16 != 0);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) b8[k] = 0.f;
        }
        if (chan_sw && in_n) {
          const float4 a = *reinterpret_cast<const float4*>(p.s_w + col);
          const float4 b = *reinterpret_cast<const float4*>(p.s_w + col + 4);
          s8[0] = a.x; s8[1] = a.y; s8[2] = a.z; s8[3] = a.w;
          s8[4] = b.x; s8[5] = b.y; s8[6] = b.z; s8[7] = b.w;
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) s8[k] = 0.f;
        }
        *reinterpret_cast<float4*>(ep_bias + 8 * lane) = make_float4(b8[0], b8[1], b8[2], b8[3]);
        *reinterpret_cast<float4*>(ep_bias + 8 * lane + 4) = make_float4(b8[4], b8[5], b8[6], b8[7]);
        *reinterpret_cast<float4*>(ep_sw + 8 * lane) = make_float4(s8[0], s8[1], s8[2], s8[3]);
        *reinterpret_cast<float4*>(ep_sw + 8 * lane + 4) = make_float4(s8[4], s8[5], s8[6], s8[7]);
      }
      __syncwarp();
      const bool ready = __all_sync(0xffffffffu, wait_bounded(&bars->acc_full[acc], acc_phase));
      if (!ready) {
        if (lane == 0) record_timeout(abort_flag, p.status);
        break;
      }
      ptx::tc_fence_after();
      const int64_t m = static_cast<int64_t>(mb) * C::kTileM + rank * BM + row;
      const bool row_ok = m < p.M;
      // debug build: the rows this kernel may write (one fewer under the
      // short-rows fault)
      const int64_t m_limit = CONVROT_DEBUG && p.fault == kFaultShortRows ? p.M - 1 : p.M;
      float scale = kKind == kKindI8 ? 0.f : 1.f;
      if (kKind == kKindI8 && !p.out_s32 && row_ok) {
        scale = p.s_tok[m] * (p.per_channel_scale ? 1.f : p.s_w[0]);
      }
      const uint32_t t_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * ACC_COLS;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(t_base + c * 32, r);
        ptx::tmem_ld_wait();
        const int64_t n0 = static_cast<int64_t>(nb) * BN + c * 32;
        const int valid = n0 + 32 <= p.N ? 32 : (n0 + 16 <= p.N ? 16 : 0);  // warp-uniform
        if (valid == 0) continue;
        if (kKind == kKindI8 && p.out_s32) {
          if (row_ok && in_bounds(m < m_limit && n0 + valid <= p.N, p.status)) {
            store_s32_row32(static_cast<int32_t*>(p.out) + m * p.N + n0, r, valid);
          }
          continue;
        }
        // Lane i computes row i of the warp's 32 x 32 chunk and stages it;
        // then each store instruction writes 8 rows x 64 contiguous bytes
        // (lane i: row 8 j + i / 4, unit i % 4), where one row per lane
        // would touch 32 lines with 16 bytes each.
        uint32_t w[16];
        row32_words<kKind != kKindI8>(w, r, scale, chan_sw ? ep_sw + c * 32 : nullptr,
                                      has_bias ? ep_bias + c * 32 : nullptr, p.out_f16 != 0);
        __syncwarp();  // the previous chunk's staged rows are read out
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          ep_stage[stage_unit(static_cast<int>(lane), k)] =
              make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
        __syncwarp();
        const int unit_k = static_cast<int>(lane & 3);
        const int64_t m_warp = m - static_cast<int64_t>(lane);  // row 0 of the warp's 32
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int rr = 8 * j + static_cast<int>(lane >> 2);
          const int64_t mm = m_warp + rr;
          const uint4 v = ep_stage[stage_unit(rr, unit_k)];
          if (mm < p.M && 8 * unit_k < valid &&
              in_bounds(mm < m_limit && n0 + valid <= p.N, p.status)) {
            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + mm * p.N + n0 + 8 * unit_k) = v;
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_leader(&bars->acc_empty[acc]);
    }
  }

  ptx::tc_fence_before();
  ptx::cluster_sync();  // the leader's MMAs into this CTA's TMEM are complete
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    int8_gemm_tcgen05(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const Params p) {
  gemm_pair<kKindI8>(tmA, tmB, p);
}

// x [M, K] and W [N, K] both bf16 (kF16 = false) or both fp16
template <bool kF16>
__global__ void __launch_bounds__(kThreads, 1)
    gemm16_tcgen05(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const Params p) {
  gemm_pair<kF16 ? kKindF16 : kKindBF16>(tmA, tmB, p);
}

// int8 [rows, K] row-major, box of `box_rows` x 128 bytes, 128-byte swizzle,
// zero fill outside the tensor.
bool encode_operand(CUtensorMap* map, const int8_t* base, int64_t rows, int64_t K, int box_rows) {
  return encode_tma_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, static_cast<uint64_t>(K),
                       static_cast<uint64_t>(rows), static_cast<uint64_t>(K), BK,
                       static_cast<uint32_t>(box_rows));
}

// bf16 / fp16 [rows, K] row-major, box of `box_rows` x 64 elements (128 bytes),
// 128-byte swizzle, zero fill outside the tensor.
bool encode_operand16(CUtensorMap* map, const uint16_t* base, bool f16, int64_t rows, int64_t K,
                      int box_rows) {
  return encode_tma_2d(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                       base, static_cast<uint64_t>(K), static_cast<uint64_t>(rows),
                       static_cast<uint64_t>(K) * 2, BK / 2, static_cast<uint32_t>(box_rows));
}

cudaError_t launch_pair(const GemmArgs& a, Params p, cudaStream_t stream) {
  using C = Cfg;
  CUtensorMap tmA, tmB;
  const bool ok = a.ops16 ? encode_operand16(&tmA, a.A16, a.out_f16, a.M, a.K, BM) &&
                                encode_operand16(&tmB, a.B16, a.out_f16, a.N, a.K, C::kBRows)
                          : encode_operand(&tmA, a.A, a.M, a.K, BM) &&
                                encode_operand(&tmB, a.B, a.N, a.K, C::kBRows);
  if (!ok) return cudaErrorInvalidValue;
  void (*kernel)(CUtensorMap, CUtensorMap, Params) =
      !a.ops16 ? int8_gemm_tcgen05 : (a.out_f16 ? gemm16_tcgen05<true> : gemm16_tcgen05<false>);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  p.m_tiles = static_cast<int>((a.M + C::kTileM - 1) / C::kTileM);
  // all M-tiles per column sweep when A (M x K elements) fits in half of L2
  p.group_m = a.M * a.K * (a.ops16 ? 2 : 1) <= (64ll << 20) ? p.m_tiles : 8;
  const int tiles = p.m_tiles * p.n_tiles;
  const int per_unit = 2;  // CTAs per cluster
  const int max_units = sm_count() / per_unit;
  const int units = tiles < max_units ? tiles : max_units;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(units * per_unit));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = per_unit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, p);
}

}  // namespace

cudaError_t launch_int8_gemm(const GemmArgs& a, cudaStream_t stream) {
  if (a.M == 0) return cudaSuccess;
  Params p;
  cudaError_t se = status_word(&p.status);
  if (se != cudaSuccess) return se;
  p.s_tok = a.s_tok;
  p.s_w = a.s_w;
  p.bias = a.bias;
  p.out = a.out;
  p.M = a.M;
  p.N = a.N;
  p.num_kb = static_cast<int>((a.K + BK - 1) / BK);
  p.n_tiles = static_cast<int>((a.N + BN - 1) / BN);
  p.per_channel_scale = a.s_w_len > 1 ? 1 : 0;
  p.out_s32 = a.out_s32 ? 1 : 0;
  p.out_f16 = a.out_f16 ? 1 : 0;
  p.fault = debug_fault();
  // few tokens: the weight-streaming swap-AB kernel; otherwise CTA pairs
  // (256-row tiles) once there is more than one 128-row block of tokens
  if (a.M <= BM) return launch_int8_gemm_skinny(a, stream);
  return launch_pair(a, p, stream);
}

cudaError_t launch_gemm16(const GemmArgs& a, cudaStream_t stream) {
  if (a.M == 0) return cudaSuccess;
  Params p;
  cudaError_t se = status_word(&p.status);
  if (se != cudaSuccess) return se;
  p.s_tok = nullptr;
  p.s_w = nullptr;
  p.bias = a.bias;
  p.out = a.out;
  p.M = a.M;
  p.N = a.N;
  p.num_kb = static_cast<int>((2 * a.K + BK - 1) / BK);
  p.n_tiles = static_cast<int>((a.N + BN - 1) / BN);
  p.per_channel_scale = 0;
  p.out_s32 = 0;
  p.out_f16 = a.out_f16 ? 1 : 0;
  p.fault = debug_fault();
  return launch_pair(a, p, stream);
}

}  // namespace convrot
