// int8 x int8 -> int32 GEMM on the sm_100a tensor cores with the ConvRot
// rescale epilogue fused (Invoke docs "int8 Compute", opening section: each
// layer "multiplies int8 by int8" on the int8 tensor cores):
//
//   acc[m, n] = sum_k xq[m, k] * Wq[n, k]                       (exact int32)
//   y[m, n]   = bf16_rn(float(acc) * (s_tok[m] * s_w[n|0]) + bias[n])
//
// Structure (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: 128 x 128 A and 256 x 128 B int8 tiles, 128-byte
//               swizzle, into a 4-stage shared-memory ring (48 KB per stage);
//   warp 1      allocates 512 TMEM columns, one thread issues
//               tcgen05.mma.cta_group::1.kind::i8 (M=128, N=256, K=32) into one
//               of two 256-column int32 accumulators, tcgen05.commit frees the
//               stage / publishes the accumulator;
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, rescale, bias, bf16,
//               128-bit global stores; then release the accumulator so the MMA
//               of the next tile overlaps this tile's epilogue.
// Every mbarrier wait is bounded by the global timer.  A wait that runs out
// records CONVROT_ERR_TIMEOUT in the device status word; the CTA then stops
// issuing work, drains what it issued and frees its TMEM before returning.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace convrot {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;  // bytes = int8 elements; one 128-byte swizzle row
constexpr int UMMA_K = 32;
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK;
constexpr int B_STAGE = BN * BK;
constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
constexpr int ACC_COLS = BN;        // int32 accumulator columns per tile
constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kGroupM = 8;          // tile raster: 8 M-tiles share a column sweep
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s per wait
constexpr size_t kSmemBytes = 1024 /*align slack*/ + STAGES * STAGE_BYTES + 256 /*barriers*/;

struct Params {
  const float* s_tok;
  const float* s_w;
  const uint16_t* bias;
  void* out;
  int64_t M, N;
  int num_kb;
  int m_tiles, n_tiles;
  int per_channel_scale;
  int out_s32;
  unsigned int* status;  // device status word (bit 0: a wait ran out)
};

struct Barriers {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int& mb, int& nb) {
  const int per_group = kGroupM * n_tiles;
  const int g = tile / per_group;
  const int first_m = g * kGroupM;
  const int gm = min(kGroupM, m_tiles - first_m);
  const int local = tile - g * per_group;
  mb = first_m + local % gm;
  nb = local / gm;
}

__device__ __forceinline__ void record_timeout(Barriers* bars, unsigned int* status) {
  atomicOr(status, 1u);
  *reinterpret_cast<volatile uint32_t*>(&bars->abort_flag) = 1u;
}

__device__ __forceinline__ bool aborted(Barriers* bars) {
  return *reinterpret_cast<volatile uint32_t*>(&bars->abort_flag) != 0u;
}

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity) {
  return ptx::mbar_wait(bar, parity, ptx::globaltimer_ns() + kWaitNs);
}

__device__ __forceinline__ void store_bf16_row32(uint16_t* dst, const uint32_t (&r)[32], float scale,
                                                 const float* s_w_row, const uint16_t* bias,
                                                 int valid) {
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float lo = __int2float_rn(static_cast<int32_t>(r[2 * i]));
    float hi = __int2float_rn(static_cast<int32_t>(r[2 * i + 1]));
    const float sl = s_w_row ? scale * s_w_row[2 * i] : scale;
    const float sh = s_w_row ? scale * s_w_row[2 * i + 1] : scale;
    float bl = 0.f, bh = 0.f;
    if (bias) {
      bl = __uint_as_float(static_cast<uint32_t>(bias[2 * i]) << 16);
      bh = __uint_as_float(static_cast<uint32_t>(bias[2 * i + 1]) << 16);
    }
    lo = fmaf(lo, sl, bl);
    hi = fmaf(hi, sh, bh);
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  uint4* q = reinterpret_cast<uint4*>(dst);
  q[0] = make_uint4(w[0], w[1], w[2], w[3]);
  q[1] = make_uint4(w[4], w[5], w[6], w[7]);
  if (valid == 32) {
    q[2] = make_uint4(w[8], w[9], w[10], w[11]);
    q[3] = make_uint4(w[12], w[13], w[14], w[15]);
  }
}

__device__ __forceinline__ void store_s32_row32(int32_t* dst, const uint32_t (&r)[32], int valid) {
  uint4* q = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i < 4 || valid == 32) q[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    int8_gemm_tcgen05(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE;
  Barriers* bars = reinterpret_cast<Barriers*>(smem + STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&bars->full[s], 1);
      ptx::mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&bars->acc_full[a], 1);
      ptx::mbar_init(&bars->acc_empty[a], kEpiThreads);
    }
    ptx::mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    ptx::fence_mbarrier_init();
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&bars->tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  const int num_tiles = p.m_tiles * p.n_tiles;

  if (threadIdx.x == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    int last_stage = -1;
    uint32_t last_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles && !aborted(bars); tile += gridDim.x) {
      int mb, nb;
      tile_coords(tile, p.m_tiles, p.n_tiles, mb, nb);
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!wait_bounded(&bars->empty[stage], phase ^ 1u)) {
          record_timeout(bars, p.status);
          break;
        }
        ptx::mbar_arrive_expect_tx(&bars->full[stage], STAGE_BYTES);
        ptx::tma_load_2d(sA + stage * A_STAGE, &tmA, &bars->full[stage], kb * BK, mb * BM);
        ptx::tma_load_2d(sB + stage * B_STAGE, &tmB, &bars->full[stage], kb * BK, nb * BN);
        last_stage = stage;
        last_phase = phase;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (aborted(bars) && last_stage >= 0) {
      // let the last copy land before the CTA's shared memory goes away
      ptx::mbar_wait(&bars->full[last_stage], last_phase, ptx::globaltimer_ns() + 10000000ull);
    }
  } else if (threadIdx.x == 32) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = ptx::idesc_i8(BM, BN);
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;
    bool issued = false;
    for (int tile = blockIdx.x; tile < num_tiles && !aborted(bars); tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!wait_bounded(&bars->acc_empty[acc], acc_phase ^ 1u)) {
        record_timeout(bars, p.status);
        break;
      }
      ptx::tc_fence_after();
      const uint32_t d_tmem = tmem + acc * ACC_COLS;
      bool ok = true;
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!wait_bounded(&bars->full[stage], phase)) {
          record_timeout(bars, p.status);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a_addr = ptx::smem_u32(sA + stage * A_STAGE);
        const uint32_t b_addr = ptx::smem_u32(sB + stage * B_STAGE);
#pragma unroll
        for (int k = 0; k < BK / UMMA_K; ++k) {
          const uint64_t ad = ptx::smem_desc_k_sw128(a_addr + k * UMMA_K);
          const uint64_t bd = ptx::smem_desc_k_sw128(b_addr + k * UMMA_K);
          ptx::mma_i8(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
        }
        issued = true;
        ptx::mma_commit(&bars->empty[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      ptx::mma_commit(&bars->acc_full[acc]);
    }
    if (aborted(bars) && issued) {
      // every MMA issued so far must finish before TMEM is released
      ptx::mma_commit(&bars->drain);
      ptx::mbar_wait(&bars->drain, 0, ptx::globaltimer_ns() + 10000000ull);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may read: 32*quarter ..
    const int row = quarter * 32 + static_cast<int>(lane);
    int local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      int mb, nb;
      tile_coords(tile, p.m_tiles, p.n_tiles, mb, nb);
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const bool ready = __all_sync(0xffffffffu, wait_bounded(&bars->acc_full[acc], acc_phase));
      if (!ready) {
        if (lane == 0) record_timeout(bars, p.status);
        break;
      }
      ptx::tc_fence_after();
      const int64_t m = static_cast<int64_t>(mb) * BM + row;
      const bool row_ok = m < p.M;
      float scale = 0.f;
      if (!p.out_s32 && row_ok) scale = p.s_tok[m] * (p.per_channel_scale ? 1.f : p.s_w[0]);
      const uint32_t t_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * ACC_COLS;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(t_base + c * 32, r);
        ptx::tmem_ld_wait();
        const int64_t n0 = static_cast<int64_t>(nb) * BN + c * 32;
        const int valid = n0 + 32 <= p.N ? 32 : (n0 + 16 <= p.N ? 16 : 0);
        if (row_ok && valid) {
          if (p.out_s32) {
            store_s32_row32(static_cast<int32_t*>(p.out) + m * p.N + n0, r, valid);
          } else {
            store_bf16_row32(static_cast<uint16_t*>(p.out) + m * p.N + n0, r, scale,
                             p.per_channel_scale ? p.s_w + n0 : nullptr,
                             p.bias ? p.bias + n0 : nullptr, valid);
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->acc_empty[acc]);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// int8 [rows, K] row-major, box of `box_rows` x 128 bytes, 128-byte swizzle,
// zero fill outside the tensor.
bool encode_operand(CUtensorMap* map, const int8_t* base, int64_t rows, int64_t K, int box_rows) {
  return encode_tma_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, static_cast<uint64_t>(K),
                       static_cast<uint64_t>(rows), static_cast<uint64_t>(K), BK,
                       static_cast<uint32_t>(box_rows));
}

}  // namespace

cudaError_t launch_int8_gemm(const GemmArgs& a, cudaStream_t stream) {
  if (a.M == 0) return cudaSuccess;
  CUtensorMap tmA, tmB;
  if (!encode_operand(&tmA, a.A, a.M, a.K, BM) || !encode_operand(&tmB, a.B, a.N, a.K, BN)) {
    return cudaErrorInvalidValue;
  }
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(int8_gemm_tcgen05,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
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
  p.m_tiles = static_cast<int>((a.M + BM - 1) / BM);
  p.n_tiles = static_cast<int>((a.N + BN - 1) / BN);
  p.per_channel_scale = a.s_w_len > 1 ? 1 : 0;
  p.out_s32 = a.out_s32 ? 1 : 0;
  const int tiles = p.m_tiles * p.n_tiles;
  const int grid = tiles < sm_count() ? tiles : sm_count();
  int8_gemm_tcgen05<<<grid, kThreads, kSmemBytes, stream>>>(tmA, tmB, p);
  return cudaGetLastError();
}

}  // namespace convrot
