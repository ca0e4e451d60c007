// gemm_sm100.cuh — W4A4 block-scaled FP4 GEMM on sm_100a tensor cores.
//
//   Y[m][n] = (1 / (g_a * g_b)) * sum_k val(A)[m][k] dec(sfA)[m][k/16]
//                                     * val(B)[n][k] dec(sfB)[n][k/16]
// News article "Qwen3.8-27B最激进4bit量化开源，权重显存暴降2.9倍！" §02: W4A4
// quantizes weights and activations so the GEMM runs on hardware-native 4-bit
// tensor cores; the per-16 E4M3 scales are applied inside the MMA and the two
// FP32 globals in the epilogue.
//
// Design (one CTA per SM, persistent over 128x256 output tiles):
//   warp 0  TMA producer: A (128 rows x 128 B), B (256 x 128 B) with 128-byte
//           swizzle, and the two scale tiles (whole 512-byte atoms) into a
//           4-stage shared-memory ring guarded by full/empty mbarriers;
//   warp 1  allocates 512 tensor-memory columns; one thread copies each
//           stage's scale atoms into tensor memory (tcgen05.cp 32x128b.warpx4)
//           and issues 4 x tcgen05.mma.kind::mxf4nvf4.block16 (K = 64 each)
//           per 256-element k-tile into a 128x256 FP32 accumulator;
//   warps 2..9  epilogue: two warps per tensor-memory lane quarter, each
//           drains 128 accumulator columns into registers, releases the
//           accumulator (so the next tile's MMAs start at once), then scales
//           by 1/(g_a g_b), converts and stores its row.
// Every mbarrier wait is bounded in time; on expiry the kernel records a fault
// word, every role stops, in-flight copies and MMAs are drained (again with a
// bound) and tensor memory is released before the CTA exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace nvfp4 {

// Nonzero after a bounded wait expired in any kernel; read and cleared by
// nvfp4_read_fault. Bits name the role that gave up.
__device__ unsigned int g_fault_word;

namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 256;                       // FP4 elements per k-tile
constexpr int BK_BYTES = BK / 2;              // 128 bytes: one swizzle row
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK_BYTES;        // 16 KiB
constexpr int B_BYTES = BN * BK_BYTES;        // 32 KiB
constexpr int SFA_BYTES = BM * (BK / 16);     // 2 KiB = 4 atoms
constexpr int SFB_BYTES = BN * (BK / 16);     // 4 KiB = 2 row blocks x 4 atoms
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;               // [0, 256): FP32 accumulator
constexpr uint32_t SFA_COL = 256;             // 2 buffers x 16 columns
constexpr uint32_t SFB_COL = 288;             // 2 buffers x 32 columns
constexpr int GROUP_M = 8;                    // tile raster: 8 M-blocks per band
constexpr size_t SMEM_BYTES = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait
constexpr uint64_t kDrainLimitNs = 100000000ull;  // 0.1 s for the abort drain

// Instruction descriptor, kind::mxf4nvf4: A/B format E2M1 (1) at bits 7 and
// 10, both K-major, N>>3 at bit 17, scale format UE4M3 (0) at bit 23, M>>4 at
// bit 24, scale-factor ids 0, dense K = 64.
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                           (static_cast<uint32_t>(BM >> 4) << 24);

enum : uint32_t { kFaultProducer = 1u, kFaultMma = 2u, kFaultEpilogue = 4u };

struct Params {
  int M, N, K;
  int num_m_blk, num_n_blk, num_k_tiles;
  const float* a_global;
  const float* b_global;
  void* y;
  int64_t ldy;
  int y_fp32;
};

// Band rasterization: consecutive tiles walk GROUP_M M-blocks down one
// N-column band, so the CTAs resident at one time share A and B tiles in L2.
__device__ __forceinline__ void tile_coords(int t, const Params& p, int& mb, int& nb) {
  const int per_group = GROUP_M * p.num_n_blk;
  const int group = t / per_group;
  const int first_m = group * GROUP_M;
  const int gsize = min(p.num_m_blk - first_m, GROUP_M);
  const int r = t - group * per_group;
  mb = first_m + r % gsize;
  nb = r / gsize;
}

// Bounded wait: true when the phase of parity `parity` completed; false when
// another role aborted or the time limit passed (then this role aborts too).
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity,
                                             volatile uint32_t* abort_flag, uint32_t who) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1u;
      atomicOr(&g_fault_word, who);
      return false;
    }
  }
}

// Used only while aborting: wait for in-flight asynchronous work, bounded.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (ptx::globaltimer_ns() - t0 > kDrainLimitNs) return;
  }
}

// Scale 32 accumulator columns of one output row by alpha and store them
// (bf16 or fp32), 16-byte vectors where the whole vector is inside N.
__device__ __forceinline__ void store_cols(const uint32_t (&r)[32], const Params& p, int64_t row,
                                           int col0, float alpha) {
  if (p.y_fp32) {
    float* yrow = reinterpret_cast<float*>(p.y) + row * p.ldy;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int col = col0 + v * 4;
      float o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = __uint_as_float(r[v * 4 + e]) * alpha;
      if (col + 4 <= p.N) {
        *reinterpret_cast<float4*>(yrow + col) = make_float4(o[0], o[1], o[2], o[3]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (col + e < p.N) yrow[col + e] = o[e];
      }
    }
  } else {
    uint16_t* yrow = reinterpret_cast<uint16_t*>(p.y) + row * p.ldy;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int col = col0 + v * 8;
      uint32_t packed[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[v * 8 + 2 * e]) * alpha,
                                                        __uint_as_float(r[v * 8 + 2 * e + 1]) * alpha);
        packed[e] = *reinterpret_cast<const uint32_t*>(&b2);
      }
      if (col + 8 <= p.N) {
        *reinterpret_cast<uint4*>(yrow + col) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (col + e < p.N)
            yrow[col + e] = static_cast<uint16_t>((packed[e >> 1] >> (16 * (e & 1))) & 0xFFFFu);
      }
    }
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmSFA,
                const __grid_constant__ CUtensorMap tmSFB, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tmem_full = empty + STAGES;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* drain = tmem_empty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(tmem_full, 1);
    ptx::mbar_init(tmem_empty, NUM_EPI_WARPS);
    ptx::mbar_init(drain, 1);
    *abort_flag = 0u;
    ptx::fence_mbarrier_init();
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
    ptx::tma_prefetch_desc(&tmSFA);
    ptx::tma_prefetch_desc(&tmSFB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_holder, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int num_tiles = p.num_m_blk * p.num_n_blk;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t pending = 0, pending_parity = 0;  // stages loaded, not yet seen free
      bool aborted = false;
      for (int t = blockIdx.x; t < num_tiles && !aborted; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        for (int kt = 0; kt < p.num_k_tiles; ++kt) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, kFaultProducer)) {
            aborted = true;
            break;
          }
          pending &= ~(1u << stage);
          uint8_t* st = smem + stage * STAGE_BYTES;
          ptx::mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          ptx::tma_load_2d(st, &tmA, &full[stage], kt * BK_BYTES, mb * BM);
          ptx::tma_load_2d(st + A_BYTES, &tmB, &full[stage], kt * BK_BYTES, nb * BN);
          ptx::tma_load_3d(st + A_BYTES + B_BYTES, &tmSFA, &full[stage], 0, kt * 4, mb);
          ptx::tma_load_3d(st + A_BYTES + B_BYTES + SFA_BYTES, &tmSFB, &full[stage], 0, kt * 4,
                           nb * 2);
          pending |= 1u << stage;
          pending_parity = (pending_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (aborted) {
        // let every issued copy land before the CTA can exit
        for (int s = 0; s < STAGES; ++s)
          if (pending & (1u << s)) drain_wait(&full[s], (pending_parity >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t smem_base = ptx::smem_u32(smem);
      uint32_t stage = 0, phase = 0, acc_phase = 0, sf_buf = 0;
      bool aborted = false;
      for (int t = blockIdx.x; t < num_tiles && !aborted; t += gridDim.x) {
        if (!wait_bounded(tmem_empty, acc_phase ^ 1u, abort_flag, kFaultMma)) {
          aborted = true;
          break;
        }
        ptx::tc_fence_after();
        for (int kt = 0; kt < p.num_k_tiles; ++kt) {
          if (!wait_bounded(&full[stage], phase, abort_flag, kFaultMma)) {
            aborted = true;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sa = smem_base + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          const uint32_t ssfa = sb + B_BYTES;
          const uint32_t ssfb = ssfa + SFA_BYTES;
          const uint32_t tsfa = tmem + SFA_COL + sf_buf * 16u;
          const uint32_t tsfb = tmem + SFB_COL + sf_buf * 32u;
          // scale atoms -> tensor memory: 4 columns per 128 rows per K=64 step
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            ptx::tc_cp_32x128b_warpx4(tsfa + 4u * j, ptx::smem_desc(ssfa + 512u * j, 0, 128, 0));
            ptx::tc_cp_32x128b_warpx4(tsfb + 8u * j, ptx::smem_desc(ssfb + 512u * j, 0, 128, 0));
            ptx::tc_cp_32x128b_warpx4(tsfb + 8u * j + 4u,
                                      ptx::smem_desc(ssfb + 2048u + 512u * j, 0, 128, 0));
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t adesc = ptx::smem_desc(sa + 32u * j, 16, 1024, 2);
            const uint64_t bdesc = ptx::smem_desc(sb + 32u * j, 16, 1024, 2);
            ptx::tc_mma_nvf4(tmem + ACC_COL, adesc, bdesc, IDESC, tsfa + 4u * j, tsfb + 8u * j,
                             (kt | j) != 0 ? 1u : 0u);
          }
          ptx::tc_commit(&empty[stage]);  // frees the stage when these MMAs finish
          sf_buf ^= 1u;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (aborted) break;
        ptx::tc_commit(tmem_full);  // accumulator ready when all MMAs finish
        acc_phase ^= 1u;
      }
      if (aborted) {
        ptx::tc_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue --
    const int q = warp & 3;                 // tensor-memory lane quarter
    const int half = (warp - 2) >> 2;       // accumulator columns [128*half, +128)
    const float alpha = 1.0f / (__ldg(p.a_global) * __ldg(p.b_global));
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      if (!wait_bounded(tmem_full, acc_phase, abort_flag, kFaultEpilogue)) break;
      ptx::tc_fence_after();
      uint32_t r0[32], r1[32], r2[32], r3[32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + ACC_COL + half * 128u;
      ptx::tc_ld_32x32b_x32(taddr + 0u, r0);
      ptx::tc_ld_32x32b_x32(taddr + 32u, r1);
      ptx::tc_ld_32x32b_x32(taddr + 64u, r2);
      ptx::tc_ld_32x32b_x32(taddr + 96u, r3);
      ptx::tc_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(tmem_empty);
      acc_phase ^= 1u;

      const int64_t row = static_cast<int64_t>(mb) * BM + q * 32 + lane;
      if (row >= p.M) continue;
      const int col0 = nb * BN + half * 128;
      store_cols(r0, p, row, col0 + 0, alpha);
      store_cols(r1, p, row, col0 + 32, alpha);
      store_cols(r2, p, row, col0 + 64, alpha);
      store_cols(r3, p, row, col0 + 96, alpha);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace gemm
}  // namespace nvfp4
