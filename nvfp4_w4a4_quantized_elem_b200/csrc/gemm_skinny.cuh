// gemm_skinny.cuh — the W4A4 GEMM for few tokens (M <= 64): decode steps.
//
// Same product as gemm_sm100.cuh (Y = dequant(A) dequant(B)^T / (g_a g_b)),
// computed as Y^T = B A^T so that the weights fill the 128-row MMA side and
// the tokens are the MMA N (16, 32 or 64): the tensor cores then do no work on
// padded token rows, and the kernel streams the weights at memory speed.
// News article "Qwen3.8-27B最激进4bit量化开源，权重显存暴降2.9倍！" §02
// (W4A4 on 4-bit tensor cores); decode throughput is one of the serving
// numbers the pages report (§04).
//
// One CTA per SM. With at least as many weight tiles (128 rows each) as
// CTAs, a CTA takes whole tiles. With fewer, the work is split stream-K
// fashion: the W x KT (tile, k-tile) iterations are dealt out in G equal
// contiguous shares, so every SM streams weights; a share may end inside one
// tile and continue into the next. A segment that is only part of a tile
// writes its FP32 partial (already scaled by 1/(g_a g_b)) to the slab of
// its (tile, contributor) slot; then each epilogue warp counts itself in on
// the counter of its 32 output columns, and the warp that arrives last for
// those columns sums the tile's slabs in contributor (= k) order, writes Y
// and resets the counter. The result is the same on every run, and no warp
// ever waits for another.
// Launched with programmatic stream serialisation: tensor-memory allocation
// and barrier set-up overlap the previous kernel; every global access waits
// for it, except that, when the caller guarantees the weights were written
// before that kernel started (`early_w`), the first ring's worth of weight
// tiles is requested before the wait.
//   warp 0     TMA producer: W tile (128 rows x 128 B, 128-byte swizzle), the
//              token tile (BNT rows), and both tiles' scale atoms, into a
//              ring of up to 8 stages.
//   warp 1     allocates tensor memory; one thread issues 4 MMAs
//              (kind::mxf4nvf4.block16, M = 128, N = BNT, K = 64) per k-tile.
//   warps 2-3  copy the stage's scale atoms into that stage's tensor-memory
//              scale buffer (tcgen05.cp 32x128b.warpx4, ~50 cycles each
//              whatever the size): with only ~18 KiB of weights per k-tile
//              the copies would otherwise set the pace of the weight stream.
//              A buffer is reused only when its stage is refilled, so the
//              copy warps wait for nothing but the data.
//   warps 4-7  epilogue: each thread owns one weight row (= one output
//              column n) and drains its BNT token values 32 at a time; for a
//              fixed token the 32 lanes write 32 consecutive columns.
//   warps 8-11 (in-kernel token quantization, m <= XR: nvfp4_linear of a
//              decode step) the producer brings each k-tile of the bf16
//              tokens instead of their codes and scales, and these warps
//              quantize it into the stage (X's global first: static, from
//              the amax pass's partials, or the max over X taken together
//              with the epilogue warps); the MMA and copy warps wait for them.
// Every wait is bounded; on expiry the fault word is set, copies and MMAs in
// flight are drained (bounded) and tensor memory is freed before exit.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "fault.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace nvfp4 {

namespace skinny {

constexpr int BW = 128;           // weight rows per tile (MMA M)
constexpr int BK = 256;           // FP4 elements per k-tile
constexpr int BK_BYTES = BK / 2;
constexpr int SF_WARP0 = 2;       // warps 2, 3 copy scales
constexpr int EPI_WARP0 = 4;      // warps 4..7 drain the accumulator
constexpr int XQ_WARP0 = 8;       // warps 8..11 quantize the tokens (in-kernel mode)
constexpr int XQ_THREADS = 128;
// One CTA per SM with the deepest ring that fits: in a decode layer
// sequence the ring's first stages are requested before the grid-dependency
// wait, and the deeper the ring the more of the weight stream overlaps the
// wait for the previous layer and this layer's quantizer (measured on a
// graph of 8 decode steps: 8 stages beat a half-SM CTA with 5 stages that
// let the next layer's CTA start beside it, by 0.3-1.2 us per step).
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_BUF_COLS = 32;  // per scale buffer: weights 16, tokens 16
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kDrainLimitNs = 100000000ull;
// dynamic shared memory per CTA (of the 227 KiB a CTA may use)
constexpr size_t kSmemPerCta = 220 * 1024;
constexpr int kMaxSplits = 8;     // stream-K: at most this many CTAs per weight tile
constexpr int kMaxContrib = kMaxSplits + 1;  // contributor slots per tile (host-checked)
// tokens summed per round of slab loads: every load of a round is issued
// before its first add, so a round costs one L2 round trip
template <int BNT, bool FUSED>
__host__ __device__ constexpr int sum_tokens() { return FUSED || BNT == 16 ? 8 : 16; }

enum : uint32_t { kFaultProducer = 16u, kFaultMma = 32u, kFaultEpilogue = 64u, kFaultScales = 128u };

constexpr int XR = 8;             // in-kernel mode: bf16 token rows per stage (m <= XR)
// in-kernel mode, dynamic global: X of at most quant::kSelfAmaxBytes (64 KiB)
// takes its max inside the kernel, in one round of loads by warps 4..11
// (larger X comes with the amax pass's partial maxima: a second round, 148
// CTAs each reading all of X, measured slower than the amax pass)
constexpr int XMAX_THREADS = 256;

// FUSED: the tokens (m <= XR) arrive in bf16 (one [XR][256] tile per stage, by
// TMA with the weights) and warps 8..11 quantize them into the stage, in the
// code and scale layouts the TMA would have written (see skinny_kernel).
template <int BNT, bool FUSED>
struct Cfg {
  static_assert(BNT == 16 || BNT == 32 || BNT == 64, "token tile (few-token kernel: m <= 64)");
  static_assert(!FUSED || BNT == 16, "in-kernel token quantization: m <= XR, one 16-token tile");
  static constexpr int THREADS = FUSED ? 32 * XQ_WARP0 + XQ_THREADS : 32 * XQ_WARP0;
  static constexpr int A_BYTES = BW * BK_BYTES;             // 16 KiB of weights
  static constexpr int B_BYTES = (BNT < 8 ? 8 : BNT) * BK_BYTES;
  static constexpr int SFB_BLOCKS = (BNT + 127) / 128;      // 128-row scale blocks of tokens
  static constexpr int SFA_BYTES = 2048;
  static constexpr int SFB_BYTES = 2048 * SFB_BLOCKS;
  static constexpr int XRAW_OFF = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int XRAW_BYTES = FUSED ? XR * BK * 2 : 0;  // bf16 tokens of one k-tile
  static constexpr int STAGE_RAW = XRAW_OFF + XRAW_BYTES;
  // bytes the TMA brings into a stage
  static constexpr int TMA_BYTES = FUSED ? A_BYTES + SFA_BYTES + XRAW_BYTES : STAGE_RAW;
  static constexpr int STAGE_BYTES = (STAGE_RAW + 1023) / 1024 * 1024;
  // after the ring: barriers, then (FUSED) X's global, warp maxima and its
  // 128-entry table of g / dec(s)
  static constexpr int TAIL_BYTES = 1536;
  static constexpr int STAGES_FIT =
      static_cast<int>((kSmemPerCta - 1024 - TAIL_BYTES) / STAGE_BYTES);
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr size_t SMEM_BYTES =
      1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + TAIL_BYTES;
  static_assert(SMEM_BYTES <= kSmemPerCta, "shared memory per CTA");
  // two BNT-column accumulators (a segment's MMAs run while the epilogue
  // drains the previous segment), then one scale buffer per stage
  static constexpr int NSF = STAGES;
  static constexpr uint32_t SF_COL = 2u * BNT;
  static_assert(SF_COL + NSF * SF_BUF_COLS <= TMEM_COLS, "scale buffers exceed tensor memory");
  static constexpr uint32_t SFB_COLS = 4u * SFB_BLOCKS;     // per K = 64 step
  // kind::mxf4nvf4, E2M1 x E2M1, both K-major, N = BNT, UE4M3 scales, M = 128
  static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) |
                                    (static_cast<uint32_t>(BNT >> 3) << 17) |
                                    (static_cast<uint32_t>(BW >> 4) << 24);
};

struct Params {
  int M, N, K;              // Y is [M][N]; weights are [N][K], tokens [M][K]
  int num_w_tiles, num_k_tiles;
  int stream_k;             // 1: contiguous shares of the tile x k-tile iterations
  const float* a_global;    // tokens' global
  const float* b_global;    // weights' global
  void* y;                  // direct mode: [M][ldy] bf16 / fp32
  int64_t ldy;
  int y_fp32;
  float* partial;           // stream-K: [num_w_tiles][kMaxContrib][M][BW] FP32 slabs
  unsigned int* tile_count; // stream-K: [num_w_tiles * 4], zero before and after a launch
  int early_w;              // weights may be read before the previous kernel finishes
  // Failure-detection self-test only (0 in every product call): the
  // producer issues nothing for the first ring stage, so its full barrier
  // never completes and every role's bounded wait runs into its limit.
  int stall_first_stage;
  uint64_t wait_limit_ns;   // per-wait limit; 0 = kWaitLimitNs
  // FUSED only: X's global scale, in the order nvfp4_quantize takes it: the
  // static global x_global_in; else 2688 / max|X| over the amax pass's
  // x_nparts partial maxima; else (x_nparts == 0) over X itself, which the
  // host bounds to kSelfAmaxBytes. CTA 0 writes it to x_global_out if set.
  const uint16_t* x;        // bf16 [M][ldx] (read for the max; tiles come by TMA)
  int64_t ldx;
  const float* x_global_in;
  const float* x_partials;
  int x_nparts;
  float* x_global_out;
};

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity,
                                             volatile uint32_t* abort_flag, uint32_t who,
                                             uint64_t limit_ns = kWaitLimitNs) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1u;
      atomicOr(&g_fault_word, who);
      return false;
    }
  }
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (ptx::globaltimer_ns() - t0 > kDrainLimitNs) return;
  }
}

__device__ __forceinline__ void tc_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// FP32 bits of max|x| over the 16-byte chunks i = part, part + nparts, ... of
// the bf16 X [M][ldx] (row length K): rounds of 16 predicated loads per thread.
__device__ __forceinline__ uint32_t x_max_part(const uint16_t* x, int64_t ldx, int M, int K,
                                               uint32_t part, uint32_t nparts) {
  const uint32_t chunks = static_cast<uint32_t>(K >> 3);
  const uint32_t total = static_cast<uint32_t>(M) * chunks;
  uint32_t m = 0;
  for (uint32_t i = part; i < total; i += 16u * nparts) {
    uint4 v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const uint32_t e = i + static_cast<uint32_t>(u) * nparts;
      const uint32_t r = e / chunks;
      const uint32_t c = e - r * chunks;
      v[u] = e < total ? __ldg(reinterpret_cast<const uint4*>(
                             x + static_cast<uint64_t>(r) * static_cast<uint64_t>(ldx) + c * 8u))
                       : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) m = max(m, quant::absmax_bits8(v[u]) << 16);
  }
  return m;
}

// The CTA that owns stream-K iteration `it` (shares are [c T / G, (c+1) T / G)).
__device__ __forceinline__ int cta_of(int64_t it, int64_t T, int64_t G) {
  return static_cast<int>(((it + 1) * G - 1) / T);
}

// This CTA's segments, in issue order: (weight tile, [k0, k1)).
struct SegIter {
  int64_t i, i1;  // stream-K: next iteration and end of this CTA's share
  int wt, k0, k1;
  bool valid;
  __device__ __forceinline__ void load(const Params& p) {
    valid = i < i1;
    if (valid) {
      wt = static_cast<int>(i / p.num_k_tiles);
      k0 = static_cast<int>(i - static_cast<int64_t>(wt) * p.num_k_tiles);
      k1 = static_cast<int>(min(static_cast<int64_t>(p.num_k_tiles), k0 + (i1 - i)));
    }
  }
  __device__ __forceinline__ void first(const Params& p) {
    if (p.stream_k) {
      const int64_t T = static_cast<int64_t>(p.num_w_tiles) * p.num_k_tiles;
      const int64_t G = gridDim.x;
      i = static_cast<int64_t>(blockIdx.x) * T / G;
      i1 = (static_cast<int64_t>(blockIdx.x) + 1) * T / G;
      load(p);
    } else {
      wt = blockIdx.x;
      k0 = 0;
      k1 = p.num_k_tiles;
      valid = wt < p.num_w_tiles;
    }
  }
  __device__ __forceinline__ void next(const Params& p) {
    if (p.stream_k) {
      i += k1 - k0;
      load(p);
    } else {
      wt += gridDim.x;
      valid = wt < p.num_w_tiles;
    }
  }
};

// Issue order of the producer: (segment, k-tile) pairs of this CTA.
struct WorkIter {
  SegIter sg;
  int kt;
  __device__ __forceinline__ void start(const Params& p) {
    sg.first(p);
    kt = sg.k0;
  }
  __device__ __forceinline__ void next(const Params& p) {
    if (++kt >= sg.k1) {
      sg.next(p);
      kt = sg.k0;
    }
  }
};

// One output column of a stream-K tile for T tokens from m0: the
// NC contributors' FP32 slabs ([M][BW] each, `slab` floats apart) added in
// contributor (= k) order. Every load is issued before the first add, so a
// round costs one L2 round trip rather than one per contributor; rows past M
// are clamped to a valid row and their sums are not stored.
template <int NC, int T>
__device__ __forceinline__ void sum_slabs(const float* col, int64_t slab, int m0, int M,
                                          float (&acc)[T]) {
  float v[NC][T];
#pragma unroll
  for (int j = 0; j < NC; ++j)
#pragma unroll
    for (int i = 0; i < T; ++i)
      v[j][i] = __ldcg(col + j * slab + static_cast<int64_t>(min(m0 + i, M - 1)) * BW);
#pragma unroll
  for (int i = 0; i < T; ++i) {
    float a = v[0][i];
#pragma unroll
    for (int j = 1; j < NC; ++j) a += v[j][i];
    acc[i] = a;
  }
}

template <int BNT, bool FUSED>
__global__ void __launch_bounds__(Cfg<BNT, FUSED>::THREADS, 1)
    skinny_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const __grid_constant__ CUtensorMap tmSFW,
                  const __grid_constant__ CUtensorMap tmSFX, const Params p) {
  using C = Cfg<BNT, FUSED>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tmem_full = empty + C::STAGES;   // [2]: one per accumulator
  uint64_t* tmem_empty = tmem_full + 2;      // [2]
  uint64_t* drain = tmem_empty + 2;
  uint64_t* sf_full = drain + 1;
  uint64_t* drain_sf = sf_full + C::NSF;
  uint64_t* xready = drain_sf + 1;           // FUSED: [STAGES] tokens quantized into the stage
  uint64_t* g_ready = xready + C::STAGES;    // FUSED: X's global and its table are ready
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(g_ready + 1);
  volatile uint32_t* abort_flag = tmem_holder + 1;
  float* s_gx = reinterpret_cast<float*>(tmem_holder + 2);      // FUSED: X's global
  uint32_t* s_red = tmem_holder + 8;                            // FUSED: [8] warp maxima
  float* s_rtab = reinterpret_cast<float*>(tmem_holder + 16);  // FUSED: [128] g / dec(s)
  // FUSED with a dynamic global and no amax partials: warps 4..11 take
  // max|X| together, meeting at named barrier 3
  const bool x_self_max = FUSED && p.x_global_in == nullptr && p.x_nparts == 0;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit_ns != 0 ? p.wait_limit_ns : kWaitLimitNs;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&tmem_full[b], 1);
      ptx::mbar_init(&tmem_empty[b], 4);
    }
    ptx::mbar_init(drain, 1);
    for (int b = 0; b < C::NSF; ++b) {
      ptx::mbar_init(&sf_full[b], 2);
    }
    ptx::mbar_init(drain_sf, 2);
    if (FUSED) {
      for (int s = 0; s < C::STAGES; ++s) ptx::mbar_init(&xready[s], 1);
      ptx::mbar_init(g_ready, 1);
    }
    *abort_flag = 0u;
    ptx::fence_mbarrier_init();
    ptx::tma_prefetch_desc(&tmW);
    ptx::tma_prefetch_desc(&tmX);
    ptx::tma_prefetch_desc(&tmSFW);
    if (!FUSED) ptx::tma_prefetch_desc(&tmSFX);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_holder, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // The next kernel in the stream may be scheduled on SMs as they free up
  // (it waits for this grid's completion before it reads anything this
  // grid writes): a decode layer's quantizer and GEMM launches then overlap
  // this GEMM's tail.
  ptx::grid_dep_launch();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, pending = 0, pending_parity = 0;
      WorkIter it;
      it.start(p);
      // The first ring's worth of stages needs no empty-slot wait. With
      // early_w their weight halves are requested before the grid-dependency
      // wait, the token halves after it.
      // Every weight byte is read once per call: its lines leave L2 first.
      const uint64_t wpol = ptx::l2_policy_evict_first();
      int npre = 0;
      if (p.early_w) {
        WorkIter w = it;
        for (; npre < C::STAGES && w.sg.valid; ++npre, w.next(p)) {
          uint8_t* st = smem + npre * C::STAGE_BYTES;
          ptx::mbar_arrive_expect_tx(&full[npre], C::TMA_BYTES);
          ptx::tma_load_2d_hint(st, &tmW, &full[npre], w.kt * BK_BYTES, w.sg.wt * BW, wpol);
          ptx::tma_load_3d_hint(st + C::A_BYTES + C::B_BYTES, &tmSFW, &full[npre], 0, w.kt * 4,
                                w.sg.wt, wpol);
        }
      }
      ptx::grid_dep_wait();
      for (int i = 0; i < npre; ++i, it.next(p)) {
        uint8_t* st = smem + i * C::STAGE_BYTES;
        if (FUSED) {
          ptx::tma_load_2d(st + C::XRAW_OFF, &tmX, &full[i], it.kt * BK, 0);
        } else {
          ptx::tma_load_2d(st + C::A_BYTES, &tmX, &full[i], it.kt * BK_BYTES, 0);
          ptx::tma_load_3d(st + C::A_BYTES + C::B_BYTES + C::SFA_BYTES, &tmSFX, &full[i], 0,
                           it.kt * 4, 0);
        }
        pending |= 1u << i;
      }
      stage = static_cast<uint32_t>(npre % C::STAGES);
      phase = static_cast<uint32_t>(npre / C::STAGES);
      bool stall = p.stall_first_stage != 0 && npre == 0;
      for (; it.sg.valid; it.next(p)) {
        if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, kFaultProducer, lim)) {
          break;
        }
        pending &= ~(1u << stage);
        if (stall) {  // self-test: this stage is never filled (nothing in flight for it)
          stall = false;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          continue;
        }
        uint8_t* st = smem + stage * C::STAGE_BYTES;
        ptx::mbar_arrive_expect_tx(&full[stage], C::TMA_BYTES);
        ptx::tma_load_2d_hint(st, &tmW, &full[stage], it.kt * BK_BYTES, it.sg.wt * BW, wpol);
        ptx::tma_load_3d_hint(st + C::A_BYTES + C::B_BYTES, &tmSFW, &full[stage], 0, it.kt * 4,
                              it.sg.wt, wpol);
        if (FUSED) {
          ptx::tma_load_2d(st + C::XRAW_OFF, &tmX, &full[stage], it.kt * BK, 0);
        } else {
          ptx::tma_load_2d(st + C::A_BYTES, &tmX, &full[stage], it.kt * BK_BYTES, 0);
          ptx::tma_load_3d(st + C::A_BYTES + C::B_BYTES + C::SFA_BYTES, &tmSFX, &full[stage], 0,
                           it.kt * 4, 0);
        }
        pending |= 1u << stage;
        pending_parity = (pending_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // Let every issued copy land before the CTA can exit: after an abort
      // (raised here or, later, by another role) nothing else waits for
      // them; without one the MMA thread consumes the same phases, so these
      // waits end as soon as the last copies land.
      for (int s = 0; s < C::STAGES; ++s)
        if (pending & (1u << s)) drain_wait(&full[s], (pending_parity >> s) & 1u);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t smem_base = ptx::smem_u32(smem);
      uint32_t stage = 0, phase = 0, acc_phase = 0, buf = 0;  // acc_phase: bit per buffer
      bool aborted = false;
      SegIter sg;
      for (sg.first(p); sg.valid && !aborted; sg.next(p)) {
        const int k0 = sg.k0, k1 = sg.k1;
        if (!wait_bounded(&tmem_empty[buf], ((acc_phase >> buf) & 1u) ^ 1u, abort_flag, kFaultMma,
                          lim)) {
          aborted = true;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t dacc = tmem + buf * static_cast<uint32_t>(BNT);
        for (int kt = k0; kt < k1; ++kt) {
          // FUSED: the quantized tokens are in the stage once xready is
          // (the token quantizer waited for the stage's TMA data first)
          if (!wait_bounded(FUSED ? &xready[stage] : &full[stage], phase, abort_flag, kFaultMma,
                            lim) ||
              !wait_bounded(&sf_full[stage], phase, abort_flag, kFaultMma, lim)) {
            aborted = true;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sa = smem_base + stage * C::STAGE_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
          const uint32_t tsfa = tmem + C::SF_COL + stage * SF_BUF_COLS;
          const uint32_t tsfb = tsfa + 16u;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t adesc = ptx::smem_desc(sa + 32u * j, 16, 1024, 2);
            const uint64_t bdesc = ptx::smem_desc(sb + 32u * j, 16, 1024, 2);
            ptx::tc_mma_nvf4(dacc, adesc, bdesc, C::IDESC, tsfa + 4u * j, tsfb + C::SFB_COLS * j,
                             (kt != k0 || j != 0) ? 1u : 0u);
          }
          ptx::tc_commit(&empty[stage]);  // frees the stage and its scale buffer
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (aborted) break;
        ptx::tc_commit(&tmem_full[buf]);
        acc_phase ^= 1u << buf;
        buf ^= 1u;
      }
      if (aborted) {
        ptx::tc_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else if (warp < EPI_WARP0) {
    // ----------------------------------------------------- scale-copy warps --
    if (lane == 0) {
      const int part = warp - SF_WARP0;  // 0: weight scales, 1: token scales
      const uint32_t smem_base = ptx::smem_u32(smem);
      uint32_t stage = 0, phase = 0;
      bool aborted = false;
      SegIter sg;
      for (sg.first(p); sg.valid && !aborted; sg.next(p)) {
        for (int kt = sg.k0; kt < sg.k1; ++kt) {
          // the stage's data having landed means its previous MMAs finished
          // (the producer waited for them), so scale buffer `stage` is free;
          // FUSED: the token scales are in the stage once xready is
          if (!wait_bounded(FUSED ? &xready[stage] : &full[stage], phase, abort_flag,
                            kFaultScales, lim)) {
            aborted = true;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t ssfa = smem_base + stage * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES;
          const uint32_t ssfb = ssfa + C::SFA_BYTES;
          const uint32_t tsfa = tmem + C::SF_COL + stage * SF_BUF_COLS;
          const uint32_t tsfb = tsfa + 16u;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (part == 0) {
              ptx::tc_cp_32x128b_warpx4(tsfa + 4u * j, ptx::smem_desc(ssfa + 512u * j, 0, 128, 0));
            } else {
#pragma unroll
              for (int h = 0; h < C::SFB_BLOCKS; ++h)
                ptx::tc_cp_32x128b_warpx4(tsfb + C::SFB_COLS * j + 4u * h,
                                          ptx::smem_desc(ssfb + 2048u * h + 512u * j, 0, 128, 0));
            }
          }
          ptx::tc_commit(&sf_full[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (aborted) {
        ptx::tc_commit(drain_sf);
        drain_wait(drain_sf, 0);
      }
    }
  } else if (warp < XQ_WARP0) {
    // -------------------------------------------------------------- epilogue --
    ptx::grid_dep_wait();  // the globals come from earlier kernels; Y may be in use
    if (x_self_max) {  // this warp's share of max|X| (chunks 128.., the quantizer warps 0..)
      uint32_t m = x_max_part(p.x, p.ldx, p.M, p.K,
                              static_cast<uint32_t>(threadIdx.x - EPI_WARP0 * 32 + XQ_THREADS),
                              XMAX_THREADS);
      m = __reduce_max_sync(0xFFFFFFFFu, m);
      if (lane == 0) s_red[4 + warp - EPI_WARP0] = m;
      asm volatile("bar.sync 3, %0;" ::"n"(XMAX_THREADS) : "memory");
    }
    const int q = warp & 3;  // tensor-memory lane quarter (warps 4..7 -> 0..3)
    bool epi_ok = true;
    float gx;
    if (FUSED) {  // X's global, as the token quantizer warps derived it
      // warp-uniform outcome of every wait: the lanes that saw the phase and
      // a lane that saw another role's abort must not part ways before the
      // warp-wide tensor-memory loads
      epi_ok = __all_sync(0xFFFFFFFFu, wait_bounded(g_ready, 0u, abort_flag, kFaultEpilogue, lim));
      gx = *s_gx;
    } else {
      gx = __ldg(p.a_global);
    }
    const float alpha = 1.0f / (gx * __ldg(p.b_global));
    uint32_t acc_phase = 0, buf = 0;  // acc_phase: bit per accumulator
    const int64_t T = static_cast<int64_t>(p.num_w_tiles) * p.num_k_tiles;
    SegIter sg;
    for (sg.first(p); sg.valid && epi_ok; sg.next(p)) {
      const int wt = sg.wt;
      const bool whole = sg.k0 == 0 && sg.k1 == p.num_k_tiles;  // no other contributor
      int c_first = 0, n_contrib = 1;
      if (!whole) {
        c_first = cta_of(static_cast<int64_t>(wt) * p.num_k_tiles, T, gridDim.x);
        n_contrib = cta_of(static_cast<int64_t>(wt + 1) * p.num_k_tiles - 1, T, gridDim.x) -
                    c_first + 1;
      }
      if (!__all_sync(0xFFFFFFFFu, wait_bounded(&tmem_full[buf], (acc_phase >> buf) & 1u,
                                                abort_flag, kFaultEpilogue, lim)))
        break;
      ptx::tc_fence_after();
      const int nl = q * 32 + lane;            // column within the weight tile
      const int n = wt * BW + nl;              // this thread's output column
      const bool n_ok = n < p.N;
      const uint32_t lane_base =
          tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * static_cast<uint32_t>(BNT);
      // slab of this (tile, contributor): [M][BW]
      float* slab = whole ? nullptr
                          : p.partial + (static_cast<int64_t>(wt) * kMaxContrib +
                                         (static_cast<int>(blockIdx.x) - c_first)) *
                                            p.M * BW;
#pragma unroll
      for (int c0 = 0; c0 < BNT; c0 += 32) {
        uint32_t r[32];
        if (BNT >= 32) {
          ptx::tc_ld_32x32b_x32(lane_base + c0, r);
        } else {
          tc_ld_32x32b_x16(lane_base + c0, r);
        }
        ptx::tc_wait_ld();
        const int cols = BNT < 32 ? BNT : 32;
#pragma unroll
        for (int i = 0; i < cols; ++i) {
          const int m = c0 + i;                 // token
          if (m >= p.M || !n_ok) continue;
          const float v = __uint_as_float(r[i]) * alpha;
          if (!whole) {
            slab[static_cast<int64_t>(m) * BW + nl] = v;
          } else if (p.y_fp32) {
            reinterpret_cast<float*>(p.y)[static_cast<int64_t>(m) * p.ldy + n] = v;
          } else {
            reinterpret_cast<__nv_bfloat16*>(p.y)[static_cast<int64_t>(m) * p.ldy + n] =
                __float2bfloat16_rn(v);
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&tmem_empty[buf]);
      acc_phase ^= 1u << buf;
      buf ^= 1u;
      if (!whole) {
        // count this contributor in for these 32 columns; the last one sums
        // the tile's slabs in contributor order (= k order)
        __threadfence();
        __syncwarp();
        uint32_t last = 0;
        if (lane == 0)
          last = atomicAdd(p.tile_count + wt * 4 + q, 1u) == static_cast<unsigned>(n_contrib - 1);
        last = __shfl_sync(0xFFFFFFFFu, last, 0);
        if (last) {
          __threadfence();
          if (n_ok) {
            const float* col = p.partial + static_cast<int64_t>(wt) * kMaxContrib * p.M * BW + nl;
            const int64_t slab_len = static_cast<int64_t>(p.M) * BW;
            constexpr int T = sum_tokens<BNT, FUSED>();
            for (int m0 = 0; m0 < p.M; m0 += T) {
              float acc[T];
              switch (n_contrib) {
                case 1: sum_slabs<1, T>(col, slab_len, m0, p.M, acc); break;
                case 2: sum_slabs<2, T>(col, slab_len, m0, p.M, acc); break;
                case 3: sum_slabs<3, T>(col, slab_len, m0, p.M, acc); break;
                case 4: sum_slabs<4, T>(col, slab_len, m0, p.M, acc); break;
                case 5: sum_slabs<5, T>(col, slab_len, m0, p.M, acc); break;
                case 6: sum_slabs<6, T>(col, slab_len, m0, p.M, acc); break;
                case 7: sum_slabs<7, T>(col, slab_len, m0, p.M, acc); break;
                case 8: sum_slabs<8, T>(col, slab_len, m0, p.M, acc); break;
                default: sum_slabs<kMaxContrib, T>(col, slab_len, m0, p.M, acc); break;
              }
#pragma unroll
              for (int i = 0; i < T; ++i) {
                if (m0 + i >= p.M) break;
                const int64_t o = static_cast<int64_t>(m0 + i) * p.ldy + n;
                if (p.y_fp32)
                  reinterpret_cast<float*>(p.y)[o] = acc[i];
                else
                  reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(acc[i]);
              }
            }
          }
          if (lane == 0) p.tile_count[wt * 4 + q] = 0u;  // ready for the next call
        }
      }
    }
  } else if (FUSED) {
    // ------------------------------------------------------ token quantizer --
    // nvfp4_quantize's arithmetic on the bf16 token tile each stage receives,
    // written into the stage in the layouts the TMA would have delivered:
    // codes as the 128-byte-swizzled K-major B operand, scales as the stage's
    // four 512-byte atoms. Bit for bit the tokens nvfp4_quantize would write.
    const int t = threadIdx.x - XQ_WARP0 * 32;  // 0..127
    auto xq_sync = [] { asm volatile("bar.sync 2, %0;" ::"n"(XQ_THREADS) : "memory"); };
    // named barrier 2 that also returns whether every thread's predicate held
    auto xq_sync_and = [](bool pred) {
      uint32_t all;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\t"
          "setp.ne.u32 p, %1, 0;\n\t"
          "barrier.cta.red.and.pred q, 2, %2, p;\n\t"
          "selp.u32 %0, 1, 0, q;\n\t}"
          : "=r"(all)
          : "r"(static_cast<uint32_t>(pred)), "n"(XQ_THREADS)
          : "memory");
      return all != 0u;
    };
    // token codes and scales of every stage start at zero (rows >= M stay
    // so); no global memory involved, so this overlaps the previous kernel
    for (int s = 0; s < C::STAGES; ++s) {
      uint4* zc = reinterpret_cast<uint4*>(smem + s * C::STAGE_BYTES + C::A_BYTES);
      for (int i = t; i < C::B_BYTES / 16; i += XQ_THREADS) zc[i] = make_uint4(0u, 0u, 0u, 0u);
      uint4* zs = reinterpret_cast<uint4*>(smem + s * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES +
                                           C::SFA_BYTES);
      for (int i = t; i < C::SFB_BYTES / 16; i += XQ_THREADS) zs[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    ptx::grid_dep_wait();  // X, its static global or the amax partials come from earlier kernels
    if (p.x_global_in != nullptr) {
      if (t == 0) *s_gx = __ldg(p.x_global_in);
    } else {
      uint32_t m = 0;  // FP32 bits of max|X| (non-negative: the bits order as the values)
      int nwarps = 4;
      if (p.x_nparts > 0) {
        for (int i = t; i < p.x_nparts; i += XQ_THREADS)
          m = max(m, __float_as_uint(__ldcg(p.x_partials + i)));
      } else {  // X of at most kSelfAmaxBytes, shared with the epilogue warps
        m = x_max_part(p.x, p.ldx, p.M, p.K, static_cast<uint32_t>(t), XMAX_THREADS);
        nwarps = 8;
      }
      m = __reduce_max_sync(0xFFFFFFFFu, m);
      if ((t & 31) == 0) s_red[t >> 5] = m;
      if (nwarps == 8) {
        asm volatile("bar.sync 3, %0;" ::"n"(XMAX_THREADS) : "memory");
      } else {
        xq_sync();
      }
      if (t == 0) {
        uint32_t mm = 0;
        for (int w = 0; w < nwarps; ++w) mm = max(mm, s_red[w]);
        const float amax = __uint_as_float(mm);
        float g = (amax == 0.0f) ? 1.0f : __fdiv_rn(2688.0f, amax);
        if (!isfinite(g)) g = 1.0f;
        *s_gx = g;
      }
    }
    xq_sync();
    const float g = *s_gx;
    {
      const float ds = ptx::e4m3_value(static_cast<uint32_t>(t));
      s_rtab[t] = (ds == 0.0f) ? 0.0f : __fdiv_rn(g, ds);  // r = 0 keeps only signs
    }
    if (t == 0 && blockIdx.x == 0 && p.x_global_out != nullptr) *p.x_global_out = g;
    xq_sync();
    if (t == 0) ptx::mbar_arrive(g_ready);
    uint32_t stage = 0, phase = 0;
    const int nblk = p.M * 16;  // (token, 16-element block) pairs of one k-tile
    WorkIter it;
    for (it.start(p); it.sg.valid; it.next(p)) {
      // every thread waits; all of them go on only if all saw the data
      const bool landed = wait_bounded(&full[stage], phase, abort_flag, kFaultProducer, lim);
      uint8_t* st = smem + stage * C::STAGE_BYTES;
      const uint16_t* xr = reinterpret_cast<const uint16_t*>(st + C::XRAW_OFF);  // [XR][256]
      const uint32_t codes = ptx::smem_u32(st + C::A_BYTES);
      uint8_t* sfx = st + C::A_BYTES + C::B_BYTES + C::SFA_BYTES;
      const int kcol0 = it.kt * BK;
      for (int i = t; landed && i < nblk; i += XQ_THREADS) {
        const int r = i >> 4, b = i & 15;
        uint32_t c0 = 0u, c1 = 0u, sc = 0u;
        if (kcol0 + 16 * b < p.K) {  // K % 16 == 0: a block is in range or past K
          const uint4 v0 = *reinterpret_cast<const uint4*>(xr + r * BK + 16 * b);
          const uint4 v1 = *reinterpret_cast<const uint4*>(xr + r * BK + 16 * b + 8);
          const uint32_t mb = max(quant::absmax_bits8(v0), quant::absmax_bits8(v1));
          sc = ptx::cvt_e4m3(__fmul_rn(quant::div6_rn(__uint_as_float(mb << 16)), g));
          const float rs = s_rtab[sc];
          float f[8];
          f[0] = __fmul_rn(quant::bf16_lo(v0.x), rs);
          f[1] = __fmul_rn(quant::bf16_hi(v0.x), rs);
          f[2] = __fmul_rn(quant::bf16_lo(v0.y), rs);
          f[3] = __fmul_rn(quant::bf16_hi(v0.y), rs);
          f[4] = __fmul_rn(quant::bf16_lo(v0.z), rs);
          f[5] = __fmul_rn(quant::bf16_hi(v0.z), rs);
          f[6] = __fmul_rn(quant::bf16_lo(v0.w), rs);
          f[7] = __fmul_rn(quant::bf16_hi(v0.w), rs);
          c0 = ptx::cvt_e2m1x8(f);
          f[0] = __fmul_rn(quant::bf16_lo(v1.x), rs);
          f[1] = __fmul_rn(quant::bf16_hi(v1.x), rs);
          f[2] = __fmul_rn(quant::bf16_lo(v1.y), rs);
          f[3] = __fmul_rn(quant::bf16_hi(v1.y), rs);
          f[4] = __fmul_rn(quant::bf16_lo(v1.z), rs);
          f[5] = __fmul_rn(quant::bf16_hi(v1.z), rs);
          f[6] = __fmul_rn(quant::bf16_lo(v1.w), rs);
          f[7] = __fmul_rn(quant::bf16_hi(v1.w), rs);
          c1 = ptx::cvt_e2m1x8(f);
        }
        // codes: bytes [8b, 8b+8) of token row r (128 bytes), 16-byte chunk
        // b/2 at chunk (b/2) ^ (r % 8): the TMA's 128-byte swizzle
        const uint32_t chunk = static_cast<uint32_t>(b >> 1) ^ static_cast<uint32_t>(r & 7);
        ptx::st_shared_v2(codes + static_cast<uint32_t>(r) * 128u + (chunk << 4) +
                              8u * static_cast<uint32_t>(b & 1),
                          c0, c1);
        // scale: atom b/4 (K = 64 step), line r % 32, byte group r / 32, block b % 4
        sfx[(b >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (b & 3)] = static_cast<uint8_t>(sc);
      }
      ptx::fence_proxy_async_smem();  // the MMA and tcgen05.cp read the stage through the async proxy
      if (!xq_sync_and(landed)) break;
      if (t == 0) ptx::mbar_arrive(&xready[stage]);
      if (++stage == C::STAGES) {
        stage = 0;
        phase ^= 1u;
      }
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

// Self-test of the bounded wait every role of this kernel uses: one thread
// waits on an mbarrier that nothing arrives at, with a caller-given limit;
// the wait gives up, records kFaultSelftest in the fault word and the kernel
// returns normally, leaving the context usable.
enum : uint32_t { kFaultSelftest = 256u };

__global__ void __launch_bounds__(32, 1) selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_flag = 0u;
    ptx::fence_mbarrier_init();
    wait_bounded(&bar, 0u, &abort_flag, kFaultSelftest, limit_ns);  // phase 0 never completes
  }
}

}  // namespace skinny
}  // namespace nvfp4
