// gemm_sm100.cuh — W4A4 block-scaled FP4 GEMM on sm_100a tensor cores.
//
//   Y[m][n] = (1 / (g_a * g_b)) * sum_k val(A)[m][k] dec(sfA)[m][k/16]
//                                     * val(B)[n][k] dec(sfB)[n][k/16]
// News article "Qwen3.8-27B最激进4bit量化开源，权重显存暴降2.9倍！" §02: W4A4
// quantizes weights and activations so the GEMM runs on hardware-native 4-bit
// tensor cores; the per-16 E4M3 scales are applied inside the MMA and the two
// FP32 globals in the epilogue.
//
// Design: persistent CTA pairs (clusters of 2, one CTA per SM) over 256x256
// output tiles. The pair issues one M = 256 MMA (tcgen05 cta_group::2): the
// even CTA's tensor memory accumulates tile rows 0-127, the odd CTA's rows
// 128-255, and each CTA stages only its own half of A and half of B, so a
// stage costs each SM 38 KiB of shared memory instead of 54 KiB for a 1-SM
// 128x256 tile.
//   warp 0  TMA producer (both CTAs): A (128 rows x 128 B) and B (128 N rows x
//           128 B) with 128-byte swizzle, this CTA's A scale atoms and all 256
//           B-row scale atoms, into a 5-stage ring. Both CTAs' copies signal
//           the even CTA's barriers, which expect the pair's bytes: the scale
//           atoms (requested first) one barrier, the A and B tiles another.
//   warp 1  allocates 512 tensor-memory columns in both CTAs; in the even CTA
//           one thread issues 4 MMAs (kind::mxf4nvf4.block16, K = 64) per
//           256-element k-tile, then commits to the empty barrier of both
//           CTAs and to the scale buffer's empty barrier.
//   warps 2, 3  (even CTA) copy each stage's scale atoms into that stage's
//           tensor-memory scale buffer (one per ring stage; tcgen05.cp
//           32x128b.warpx4, both CTAs) as soon as the atoms land, 6 of the 12
//           copies each, and commit to the buffer's full barrier. Each tcgen05.cp costs a fixed ~50
//           cycles whatever its size; issued from the MMA thread the 12 copies
//           per k-tile serialise with the 4 MMAs (measured 4302 -> 2803 TF/s),
//           and one copy warp alone issues slower than the MMAs consume.
//           A buffer is reused only when its stage is refilled, which already
//           waited for the stage's MMAs: the copy warps wait for nothing but
//           the data, run ahead of the MMA thread, and their commits (which
//           arrive only after the tensor work queued before them) are
//           complete when the MMA thread needs them. A separate "buffer free"
//           commit from the MMA thread made the copies trail the MMAs and
//           drained the tensor pipe once per k-tile (~15%).
//   warps 4..11  epilogue (both CTAs): two warps per tensor-memory lane
//           quarter drain 128 columns each into registers, release the
//           accumulator (arrive on the even CTA's barrier), then scale by
//           1/(g_a g_b), convert, and write 32-row x 64-byte chunks into a
//           double-buffered swizzled shared-memory tile that a TMA bulk
//           tensor store copies out (full-line writes, ragged edges clipped
//           by the TMA unit). Per-thread 16-byte stores of whole rows would
//           cost one L2 sector write each and steal L2 bandwidth from the
//           operand loads.
// Fused SwiGLU mode (gate_up projection of a gated MLP): the weight rows are
// interleaved in blocks of 128 — gate rows of block b, then up rows of block
// b — so a 256-column tile holds 128 gate and the matching 128 up columns.
// The epilogue then forms h = silu(gate) * up with exactly the roundings of
// the unfused path (gate/up rounded to bf16 as the GEMM stores them, the same
// SwiGLU expression, h rounded to bf16) and quantizes h to NVFP4 with a
// calibrated static global using the quantizer's arithmetic, writing codes
// and swizzled scales of h instead of the 2*ffn-wide bf16 output.
// A second fused mode (dynamic global of h) writes h in bf16 with the same
// TMA-store epilogue as the plain GEMM (128 of the tile's 256 columns) and
// one max|h| per CTA, which the quantizer then reduces to h's global exactly
// as it reduces the amax pass's partials: the output is that of the unfused
// chain (GEMM -> bf16 gate/up -> silu*mul -> dynamic quantization of h).
// Launched with programmatic stream serialisation: barrier set-up and
// tensor-memory allocation overlap the previous kernel in the stream; the
// producer and the epilogue wait for it before touching global memory, except
// that with `early_w` (weights known to be written before that kernel began)
// the first ring's worth of B tiles and scales is requested before the wait.
// Every mbarrier wait is bounded in time; on expiry the kernel records a fault
// word, both CTAs of the pair stop, in-flight copies and MMAs are drained
// (again with a bound) and tensor memory is released before the CTAs exit.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "fault.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "silu_mul.cuh"

namespace nvfp4 {

namespace gemm {

constexpr int BM = 256;                       // tile rows (128 per CTA of the pair)
constexpr int BN = 256;
constexpr int BK = 256;                       // FP4 elements per k-tile
constexpr int BK_BYTES = BK / 2;              // 128 bytes: one swizzle row
constexpr int HALF = 128;                     // rows of A / B per CTA
constexpr int STAGES = 5;
constexpr int A_BYTES = HALF * BK_BYTES;      // 16 KiB
constexpr int B_BYTES = HALF * BK_BYTES;      // 16 KiB
constexpr int SFA_BYTES = HALF * (BK / 16);   // 2 KiB = 4 atoms (this CTA's rows)
constexpr int SFB_BYTES = BN * (BK / 16);     // 4 KiB = 2 row blocks x 4 atoms
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int NUM_EPI_WARPS = 8;
constexpr int SF_WARP0 = 2;                   // warps 2, 3: scale copies
constexpr int NUM_SF_WARPS = 2;
constexpr int EPI_WARP0 = SF_WARP0 + NUM_SF_WARPS;  // warps 4..11
constexpr int NUM_THREADS = 32 * EPI_WARP0 + 32 * NUM_EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;               // [0, 256): FP32 accumulator
constexpr int NSF = STAGES;                   // tensor-memory scale buffers, one per stage
constexpr uint32_t SF_COL = 256;              // NSF x 48 columns: [A 16 | B 32]
constexpr uint32_t SF_BUF_COLS = 48;
static_assert(SF_COL + NSF * SF_BUF_COLS <= TMEM_COLS, "scale buffers exceed tensor memory");
constexpr int EPI_CHUNK_BYTES = 32 * 64;      // 32 rows x 64 bytes, 64-byte swizzle
constexpr int EPI_WARP_BYTES = 2 * EPI_CHUNK_BYTES;
constexpr int EPI_OFF = STAGES * STAGE_BYTES;  // staging tiles after the ring
constexpr int BAR_OFF = EPI_OFF + NUM_EPI_WARPS * EPI_WARP_BYTES;
constexpr int RTAB_OFF = BAR_OFF + 512;      // fused mode: g_h / dec(s) for 128 codes
constexpr size_t SMEM_BYTES = 1024 + static_cast<size_t>(RTAB_OFF) + 512;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait
constexpr uint64_t kDrainLimitNs = 100000000ull;  // 0.1 s for the abort drain

// Instruction descriptor, kind::mxf4nvf4: A/B format E2M1 (1) at bits 7 and
// 10, both K-major, N>>3 at bit 17, scale format UE4M3 (0) at bit 23, M>>4 at
// bit 24 (M = 256 across the pair), scale-factor ids 0, dense K = 64.
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                           (static_cast<uint32_t>(BM >> 4) << 24);

enum : uint32_t { kFaultProducer = 1u, kFaultMma = 2u, kFaultEpilogue = 4u, kFaultScales = 8u };

struct Params {
  int M, N, K;
  int num_m_blk, num_n_blk, num_k_tiles;
  const float* a_global;
  const float* b_global;
  void* y;
  int64_t ldy;
  int y_fp32;
  // Fused SwiGLU modes (h = [M][ffn], ffn = N / 2; y unused):
  //   kFusedQuantStatic  h quantized to NVFP4 with the static h_global
  //   kFusedBf16Amax     h written in bf16 through the tensor map of Y, and
  //                      max|h| over this CTA's tiles to h_partials[CTA]
  int fused;
  const float* h_global;   // static global of h
  uint8_t* h_codes;        // [M][ffn/2]
  uint8_t* h_sf;           // swizzled scales of [M][ffn]
  int64_t h_atoms;         // 512-byte atoms per 128-row block = ffn / 64
  int m_pad;               // rows of the scale buffer = ceil(M/128)*128
  float* h_partials;       // [gridDim.x] per-CTA max|h| (kFusedBf16Amax)
  int early_w;             // B may be read before the previous kernel finishes
  // Failure-detection self-test only (0 in every product call): the
  // producers issue nothing for the first ring stage, so its full barrier
  // never completes and every role's bounded wait runs into its limit.
  int stall_first_stage;
  uint64_t wait_limit_ns;  // per-wait limit; 0 = kWaitLimitNs
  // Split-K (plain mode only; 1 = off): the K range of every tile is cut
  // into `split` slices, one work unit each. A unit stores its FP32 partial
  // tile to `partial`; per epilogue region (32 rows x 128 columns of one
  // CTA) the last slice to count itself in on `tile_count` sums all slices'
  // partials in slice order, writes Y and resets the counter.
  int split;
  float* partial;             // [tiles][split][2 CTAs][8 regions][32 x 128] FP32
  unsigned int* tile_count;   // [tiles][2 CTAs][8 regions], zero before and after
  int raster_n;               // bands of N-tiles (1) or of M-tiles (0)
  int group;                  // tiles per band (>= 1)
};

enum : int { kPlain = 0, kFusedQuantStatic = 1, kFusedBf16Amax = 2 };

// A work unit: one tile's k-tiles [k0, k1) (the whole K range without split).
struct Unit {
  int tile, slice, k0, k1;
};

__device__ __forceinline__ Unit unit_of(int u, const Params& p) {
  Unit w;
  w.tile = u / p.split;
  w.slice = u - w.tile * p.split;
  w.k0 = w.slice * p.num_k_tiles / p.split;
  w.k1 = (w.slice + 1) * p.num_k_tiles / p.split;
  return w;
}

constexpr int kRegionFloats = 32 * 128;  // one epilogue warp's part of a tile
constexpr int kMaxSplitK = 4;            // slices per tile at most (host-checked)
constexpr int kMinSliceKTiles = 16;      // k-tiles per slice at least (host-checked)

// Band rasterization: consecutive tiles walk down a band of `group` tiles of
// one operand (M-tiles when !raster_n, N-tiles when raster_n) and then step
// along the other, so the pairs resident at one time share operand tiles in
// L2 and the band's rows of its operand stay in L2 while the other operand
// streams past once per band. The host sizes the band (about 24 MB of the
// banded operand) and picks the direction with the smaller DRAM read
// traffic. (Fixed 16-tile M bands re-read the 89 MB gate_up weight 8 times.)
__device__ __forceinline__ void tile_coords(int t, const Params& p, int& mb, int& nb) {
  const int nb_band = p.raster_n ? p.num_n_blk : p.num_m_blk;  // tiles along the band's side
  const int nb_walk = p.raster_n ? p.num_m_blk : p.num_n_blk;
  const int per_group = p.group * nb_walk;
  const int group = t / per_group;
  const int first = group * p.group;
  const int gsize = min(nb_band - first, p.group);
  const int r = t - group * per_group;
  const int band = first + r % gsize, walk = r / gsize;
  mb = p.raster_n ? walk : band;
  nb = p.raster_n ? band : walk;
}

struct Abort {
  volatile uint32_t* local;   // this CTA's flag
  uint32_t peer_cluster;      // shared::cluster address of the peer's flag
  uint64_t limit_ns;          // limit of one wait

  __device__ __forceinline__ bool raised() const { return *local != 0u; }
  __device__ __forceinline__ void raise(uint32_t who) const {
    *local = 1u;
    ptx::st_shared_cluster_u32(peer_cluster, 1u);
    atomicOr(&g_fault_word, who);
  }
};

// Bounded wait: true when the phase of parity `parity` completed; false when
// the pair aborted or the time limit passed (then this role aborts the pair).
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, const Abort& ab,
                                             uint32_t who) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (ab.raised()) return false;
    if (ptx::globaltimer_ns() - t0 > ab.limit_ns) {
      ab.raise(who);
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

// Write 64 bytes of this thread's output row into a 32-row x 64-byte staging
// chunk with the 64-byte swizzle (16-byte unit u of row r at u ^ ((r>>1)&3)),
// which the TMA store undoes and which spreads a warp's 32 rows over all
// banks. bf16: 32 accumulator columns; fp32: the 16 starting at `off`.
__device__ __forceinline__ void stage_bf16(uint32_t chunk, int row, const uint32_t (&r)[32],
                                           float alpha) {
  const uint32_t base = chunk + row * 64;
  const int sw = (row >> 1) & 3;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[u * 8 + 2 * e]) * alpha,
                                                      __uint_as_float(r[u * 8 + 2 * e + 1]) * alpha);
      w[e] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    ptx::st_shared_v4(base + ((u ^ sw) << 4), w[0], w[1], w[2], w[3]);
  }
}

__device__ __forceinline__ void stage_f32(uint32_t chunk, int row, const uint32_t (&r)[32],
                                          int off, float alpha) {
  const uint32_t base = chunk + row * 64;
  const int sw = (row >> 1) & 3;
#pragma unroll
  for (int u = 0; u < 4; ++u)
    ptx::st_shared_v4(base + ((u ^ sw) << 4),
                      __float_as_uint(__uint_as_float(r[off + 4 * u + 0]) * alpha),
                      __float_as_uint(__uint_as_float(r[off + 4 * u + 1]) * alpha),
                      __float_as_uint(__uint_as_float(r[off + 4 * u + 2]) * alpha),
                      __float_as_uint(__uint_as_float(r[off + 4 * u + 3]) * alpha));
}

// One 16-column block of h for the fused mode: gate/up accumulators ->
// bf16 (as stored by the plain GEMM) -> SwiGLU -> bf16 h -> NVFP4 codes with
// the quantizer's rounding. Returns the block's E4M3 scale; codes in w[0..1].
__device__ __forceinline__ uint32_t swiglu_quant_block(const uint32_t* g, const uint32_t* u,
                                                       float alpha, float gh, const float* rtab,
                                                       uint32_t& w0, uint32_t& w1) {
  float hv[16];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float gb = __bfloat162float(__float2bfloat16_rn(__uint_as_float(g[i]) * alpha));
    const float ub = __bfloat162float(__float2bfloat16_rn(__uint_as_float(u[i]) * alpha));
    hv[i] = __bfloat162float(__float2bfloat16_rn(act::swiglu(gb, ub)));
    amax = fmaxf(amax, fabsf(hv[i]));
  }
  const uint32_t sc = ptx::cvt_e4m3(__fmul_rn(quant::div6_rn(amax), gh));
  const float r = rtab[sc];
  float f[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(hv[i], r);
  w0 = ptx::cvt_e2m1x8(f);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(hv[8 + i], r);
  w1 = ptx::cvt_e2m1x8(f);
  return sc;
}

// 32 columns of h for the kFusedBf16Amax mode: gate/up accumulators -> bf16
// (as the plain GEMM stores them) -> SwiGLU -> bf16 h, staged like
// stage_bf16; `amax` accumulates max|h| over the values written.
__device__ __forceinline__ void stage_h(uint32_t chunk, int row, const uint32_t (&g)[32],
                                        const uint32_t (&u)[32], float alpha, float& amax) {
  const uint32_t base = chunk + row * 64;
  const int sw = (row >> 1) & 3;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float h[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int c = q * 8 + 2 * e + i;
        const float gb = __bfloat162float(__float2bfloat16_rn(__uint_as_float(g[c]) * alpha));
        const float ub = __bfloat162float(__float2bfloat16_rn(__uint_as_float(u[c]) * alpha));
        h[i] = act::swiglu(gb, ub);
      }
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(h[0], h[1]);
      amax = fmaxf(amax, fmaxf(fabsf(__low2float(b2)), fabsf(__high2float(b2))));
      w[e] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    ptx::st_shared_v4(base + ((q ^ sw) << 4), w[0], w[1], w[2], w[3]);
  }
}

// Split-K: one lane's 32 consecutive columns of a region (8 float4, 32
// float4 apart in the slab layout) summed over the S slices in slice order;
// every slice's loads are issued before the first add (one L2 round trip).
template <int S>
__device__ __forceinline__ void sum_slices(const float4* src, int64_t slice_stride4,
                                           uint32_t (&acc)[32]) {
  float4 v[S][8];
#pragma unroll
  for (int sl = 0; sl < S; ++sl)
#pragma unroll
    for (int c = 0; c < 8; ++c) v[sl][c] = __ldcg(src + 32 * c + sl * slice_stride4);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float4 a = v[0][c];
#pragma unroll
    for (int sl = 1; sl < S; ++sl) {
      a.x += v[sl][c].x;
      a.y += v[sl][c].y;
      a.z += v[sl][c].z;
      a.w += v[sl][c].w;
    }
    acc[4 * c] = __float_as_uint(a.x);
    acc[4 * c + 1] = __float_as_uint(a.y);
    acc[4 * c + 2] = __float_as_uint(a.z);
    acc[4 * c + 3] = __float_as_uint(a.w);
  }
}

// Tensor-memory columns of scale buffer `buf`: A's 16, then B's 32.
__device__ __forceinline__ uint32_t sfa_cols(uint32_t tmem, uint32_t buf) {
  return tmem + SF_COL + buf * SF_BUF_COLS;
}
__device__ __forceinline__ uint32_t sfb_cols(uint32_t tmem, uint32_t buf) {
  return tmem + SF_COL + buf * SF_BUF_COLS + 16u;
}

// Copy half (`part` 0 or 1) of one stage's scale atoms into tensor-memory
// buffer `buf` of both CTAs. Per K = 64 step j, A's 128 rows go to 4 columns
// and B's 256 rows to 8 (row block h -> columns 4h..4h+3). Part 0: the 4 A
// atoms and B row block 0 of steps 0-1; part 1: B row block 0 of steps 2-3
// and row block 1 of all steps.
__device__ __forceinline__ void copy_scales(uint32_t tmem, uint32_t ssfa, uint32_t ssfb,
                                            uint32_t buf, int part) {
  const uint32_t tsfa = sfa_cols(tmem, buf);
  const uint32_t tsfb = sfb_cols(tmem, buf);
  if (part == 0) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      ptx::tc_cp_32x128b_warpx4_pair(tsfa + 4u * j, ptx::smem_desc(ssfa + 512u * j, 0, 128, 0));
#pragma unroll
    for (int j = 0; j < 2; ++j)
      ptx::tc_cp_32x128b_warpx4_pair(tsfb + 8u * j, ptx::smem_desc(ssfb + 512u * j, 0, 128, 0));
  } else {
#pragma unroll
    for (int j = 2; j < 4; ++j)
      ptx::tc_cp_32x128b_warpx4_pair(tsfb + 8u * j, ptx::smem_desc(ssfb + 512u * j, 0, 128, 0));
#pragma unroll
    for (int j = 0; j < 4; ++j)
      ptx::tc_cp_32x128b_warpx4_pair(tsfb + 8u * j + 4u,
                                     ptx::smem_desc(ssfb + 2048u + 512u * j, 0, 128, 0));
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmSFA,
                const __grid_constant__ CUtensorMap tmSFB,
                const __grid_constant__ CUtensorMap tmY, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* tmem_full = empty + STAGES;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* drain = tmem_empty + 1;
  uint64_t* sf_full = drain + 1;
  uint64_t* drain_sf = sf_full + NSF;
  // a stage's scale atoms land on their own barrier, ahead of its A and B
  // tiles: the copy warps move them into tensor memory while the operand
  // tiles are still in flight
  uint64_t* sf_landed = drain_sf + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sf_landed + STAGES);
  volatile uint32_t* abort_flag = tmem_holder + 1;
  uint32_t* h_max = tmem_holder + 2;  // kFusedBf16Amax: max|h| bits over the CTA

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();   // 0 = even CTA (issues the MMAs)
  const bool leader = (rank == 0);
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
      ptx::mbar_init(&sf_landed[s], 1);
    }
    ptx::mbar_init(tmem_full, 1);
    ptx::mbar_init(tmem_empty, 2 * NUM_EPI_WARPS);
    ptx::mbar_init(drain, 1);
    for (int b = 0; b < NSF; ++b) {
      ptx::mbar_init(&sf_full[b], NUM_SF_WARPS);
    }
    ptx::mbar_init(drain_sf, NUM_SF_WARPS);
    *abort_flag = 0u;
    *h_max = 0u;
    ptx::fence_mbarrier_init();
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
    ptx::tma_prefetch_desc(&tmSFA);
    ptx::tma_prefetch_desc(&tmSFB);
    if (p.fused != kFusedQuantStatic) ptx::tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_holder, TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  ptx::tc_fence_after();
  // Every CTA of this grid is resident: the next kernel in the stream may be
  // scheduled on SMs as they free up (it waits for this grid's completion
  // before it reads anything this grid writes).
  ptx::grid_dep_launch();
  const uint32_t tmem = *tmem_holder;
  const Abort ab{abort_flag,
                 ptx::mapa_shared(ptx::smem_u32(const_cast<uint32_t*>(abort_flag)), rank ^ 1u),
                 p.wait_limit_ns != 0 ? p.wait_limit_ns : kWaitLimitNs};
  const int num_tiles = p.num_m_blk * p.num_n_blk;
  const int num_units = num_tiles * p.split;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t pending = 0, pending_parity = 0;  // stages loaded, not yet seen free
      // issue order: (unit, k-tile) pairs of this CTA pair
      struct Item {
        int t, kt, k1, mb, nb;
      };
      auto first = [&](int t) {
        Item it{t, 0, 0, 0, 0};
        if (t < num_units) {
          const Unit w = unit_of(t, p);
          it.kt = w.k0;
          it.k1 = w.k1;
          tile_coords(w.tile, p, it.mb, it.nb);
        }
        return it;
      };
      auto next = [&](Item it) {
        if (++it.kt == it.k1) it = first(it.t + num_pairs);
        return it;
      };
      // the even CTA's barriers count both CTAs' bytes of a stage: scale
      // atoms on sf_landed (requested first), A and B tiles on full
      auto load_b = [&](const Item& it, uint32_t s) {
        uint8_t* st = smem + s * STAGE_BYTES;
        ptx::tma_load_3d_pair(st + A_BYTES + B_BYTES + SFA_BYTES, &tmSFB,
                              ptx::mapa_shared(ptx::smem_u32(&sf_landed[s]), 0), 0, it.kt * 4,
                              it.nb * 2);
        ptx::tma_load_2d_pair(st + A_BYTES, &tmB, ptx::mapa_shared(ptx::smem_u32(&full[s]), 0),
                              it.kt * BK_BYTES, it.nb * BN + static_cast<int>(rank) * HALF);
      };
      auto load_a = [&](const Item& it, uint32_t s) {
        uint8_t* st = smem + s * STAGE_BYTES;
        ptx::tma_load_3d_pair(st + A_BYTES + B_BYTES, &tmSFA,
                              ptx::mapa_shared(ptx::smem_u32(&sf_landed[s]), 0), 0, it.kt * 4,
                              it.mb * 2 + static_cast<int>(rank));
        ptx::tma_load_2d_pair(st, &tmA, ptx::mapa_shared(ptx::smem_u32(&full[s]), 0),
                              it.kt * BK_BYTES, it.mb * BM + static_cast<int>(rank) * HALF);
      };
      // both barriers of a stage are armed by the even CTA for the pair
      auto arm = [&](uint32_t s) {
        if (leader) {
          ptx::mbar_arrive_expect_tx(&sf_landed[s], 2 * (SFA_BYTES + SFB_BYTES));
          ptx::mbar_arrive_expect_tx(&full[s], 2 * (A_BYTES + B_BYTES));
        }
      };
      Item it = first(pair);
      // The ring's first pass needs no empty-slot wait; with early_w its B
      // halves are requested before the grid-dependency wait.
      int npre = 0;
      if (p.early_w) {
        for (Item w = it; npre < STAGES && w.t < num_units; ++npre, w = next(w)) {
          arm(static_cast<uint32_t>(npre));
          load_b(w, static_cast<uint32_t>(npre));
        }
      }
      ptx::grid_dep_wait();
      for (int i = 0; i < npre; ++i, it = next(it)) {
        load_a(it, static_cast<uint32_t>(i));
        pending |= 1u << i;
      }
      stage = static_cast<uint32_t>(npre % STAGES);
      phase = static_cast<uint32_t>(npre / STAGES);
      bool stall = p.stall_first_stage != 0 && npre == 0;
      for (; it.t < num_units; it = next(it)) {
        if (!wait_bounded(&empty[stage], phase ^ 1u, ab, kFaultProducer)) {
          break;
        }
        pending &= ~(1u << stage);
        if (stall) {  // self-test: this stage is never filled (nothing in flight for it)
          stall = false;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          continue;
        }
        arm(stage);
        load_a(it, stage);
        load_b(it, stage);
        pending |= 1u << stage;
        pending_parity = (pending_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (leader) {
        // Let every issued copy of the pair land before the CTAs can exit:
        // after an abort (raised here or, later, by another role) nothing
        // else waits for them. Without one the MMA thread consumes the same
        // phases, so these waits end as soon as the last copies land.
        for (int s = 0; s < STAGES; ++s)
          if (pending & (1u << s)) {
            drain_wait(&sf_landed[s], (pending_parity >> s) & 1u);
            drain_wait(&full[s], (pending_parity >> s) & 1u);
          }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer --
    if (leader && lane == 0) {
      const uint32_t smem_base = ptx::smem_u32(smem);
      uint32_t stage = 0, phase = 0, acc_phase = 0;
      bool aborted = false;
      for (int t = pair; t < num_units && !aborted; t += num_pairs) {
        const Unit w = unit_of(t, p);
        for (int kt = w.k0; kt < w.k1; ++kt) {
          if (!wait_bounded(&full[stage], phase, ab, kFaultMma) ||
              !wait_bounded(&sf_full[stage], phase, ab, kFaultMma)) {
            aborted = true;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sa = smem_base + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          if (kt == w.k0) {
            // the accumulator must have been drained by both epilogues
            if (!wait_bounded(tmem_empty, acc_phase ^ 1u, ab, kFaultMma)) {
              aborted = true;
              break;
            }
            ptx::tc_fence_after();
          }
          const uint32_t tsfa = sfa_cols(tmem, stage);
          const uint32_t tsfb = sfb_cols(tmem, stage);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t adesc = ptx::smem_desc(sa + 32u * j, 16, 1024, 2);
            const uint64_t bdesc = ptx::smem_desc(sb + 32u * j, 16, 1024, 2);
            ptx::tc_mma_nvf4_pair(tmem + ACC_COL, adesc, bdesc, IDESC, tsfa + 4u * j,
                                  tsfb + 8u * j, (kt != w.k0 || j != 0) ? 1u : 0u);
          }
          // frees the stage in both CTAs, and with it the stage's scale buffer
          ptx::tc_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (aborted) break;
        ptx::tc_commit_pair_mc(tmem_full, 0x3);  // accumulators ready in both CTAs
        acc_phase ^= 1u;
      }
      if (aborted) {
        ptx::tc_commit_pair_mc(drain, 0x1);
        drain_wait(drain, 0);
      }
    }
  } else if (warp < EPI_WARP0) {
    // ----------------------------------------------------- scale-copy warps --
    if (leader && lane == 0) {
      const uint32_t smem_base = ptx::smem_u32(smem);
      uint32_t stage = 0, phase = 0;
      bool aborted = false;
      for (int t = pair; t < num_units && !aborted; t += num_pairs) {
        const Unit w = unit_of(t, p);
        for (int kt = w.k0; kt < w.k1; ++kt) {
          // The stage's scale atoms having landed also means the MMAs of its
          // previous use finished (the producer waited for them before
          // reloading it), so scale buffer `stage` is free: no wait on the
          // MMA thread here.
          if (!wait_bounded(&sf_landed[stage], phase, ab, kFaultScales)) {
            aborted = true;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t ssfa = smem_base + stage * STAGE_BYTES + A_BYTES + B_BYTES;
          copy_scales(tmem, ssfa, ssfa + SFA_BYTES, stage, warp - SF_WARP0);
          ptx::tc_commit_pair_mc(&sf_full[stage], 0x1);  // buffer ready when copies land
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (aborted) {
        ptx::tc_commit_pair_mc(drain_sf, 0x1);
        drain_wait(drain_sf, 0);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue --
    ptx::grid_dep_wait();  // globals from earlier kernels; Y / h may still be in use
    float* rtab = reinterpret_cast<float*>(smem + RTAB_OFF);
    if (p.fused == kFusedQuantStatic) {
      // E4M3 code -> g_h / dec(code), as the quantizer tabulates it
      const float gh = __ldg(p.h_global);
      const int t = threadIdx.x - EPI_WARP0 * 32;
      if (t < 128) {
        const float ds = ptx::e4m3_value(static_cast<uint32_t>(t));
        rtab[t] = (ds == 0.0f) ? 0.0f : __fdiv_rn(gh, ds);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(32 * NUM_EPI_WARPS) : "memory");
    }
    const int q = warp & 3;                     // tensor-memory lane quarter
    const int half = (warp - EPI_WARP0) >> 2;   // accumulator columns [128*half, +128)
    const float alpha = 1.0f / (__ldg(p.a_global) * __ldg(p.b_global));
    const uint32_t release = ptx::mapa_shared(ptx::smem_u32(tmem_empty), 0);
    uint8_t* const stage_tiles = smem + EPI_OFF + (warp - EPI_WARP0) * EPI_WARP_BYTES;
    uint32_t nchunk = 0;  // chunks this warp has handed to the TMA (buffer = nchunk & 1)
    // Hand one staged chunk to the TMA once the buffer's previous store has
    // finished reading it.
    auto emit = [&](auto&& fill, int x, int y) {
      uint8_t* buf = stage_tiles + (nchunk & 1u) * EPI_CHUNK_BYTES;
      if (lane == 0) ptx::bulk_wait_group_read<1>();
      __syncwarp();
      fill(ptx::smem_u32(buf));
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        ptx::tma_store_2d(&tmY, buf, x, y);
        ptx::bulk_commit_group();
      }
      ++nchunk;
    };
    uint32_t acc_phase = 0;
    float h_amax = 0.0f;  // kFusedBf16Amax: max|h| over this thread's values
    for (int t = pair; t < num_units; t += num_pairs) {
      const Unit unit = unit_of(t, p);
      int mb, nb;
      tile_coords(unit.tile, p, mb, nb);
      // warp-uniform: no lane may leave while the others go on to the
      // warp-wide tensor-memory loads
      if (!__all_sync(0xFFFFFFFFu, wait_bounded(tmem_full, acc_phase, ab, kFaultEpilogue))) break;
      ptx::tc_fence_after();
      if (p.fused == kFusedBf16Amax) {
        // gate columns [64 half, +64) and the matching up columns (+128) ->
        // 64 bf16 h columns of 32 rows, two TMA-stored chunks
        uint32_t g0[32], g1[32], u0[32], u1[32];
        const uint32_t lb = tmem + (static_cast<uint32_t>(q * 32) << 16) + 64u * half;
        ptx::tc_ld_32x32b_x32(lb + 0u, g0);
        ptx::tc_ld_32x32b_x32(lb + 32u, g1);
        ptx::tc_ld_32x32b_x32(lb + 128u, u0);
        ptx::tc_ld_32x32b_x32(lb + 160u, u1);
        ptx::tc_wait_ld();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(release);
        acc_phase ^= 1u;
        const int row0 = mb * BM + static_cast<int>(rank) * HALF + q * 32;
        if (row0 >= p.M) continue;  // rows past M inside are zero (h = 0) and clipped
        const int hc0 = nb * 128 + 64 * half;
        emit([&](uint32_t b) { stage_h(b, lane, g0, u0, alpha, h_amax); }, hc0, row0);
        emit([&](uint32_t b) { stage_h(b, lane, g1, u1, alpha, h_amax); }, hc0 + 32, row0);
        continue;
      }
      if (p.fused == kFusedQuantStatic) {
        // gate columns [64 half, +64) and the matching up columns (+128)
        uint32_t g0[32], g1[32], u0[32], u1[32];
        const uint32_t lb = tmem + (static_cast<uint32_t>(q * 32) << 16) + 64u * half;
        ptx::tc_ld_32x32b_x32(lb + 0u, g0);
        ptx::tc_ld_32x32b_x32(lb + 32u, g1);
        ptx::tc_ld_32x32b_x32(lb + 128u, u0);
        ptx::tc_ld_32x32b_x32(lb + 160u, u1);
        ptx::tc_wait_ld();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(release);
        acc_phase ^= 1u;
        const int row = mb * BM + static_cast<int>(rank) * HALF + q * 32 + lane;
        if (row >= p.m_pad) continue;  // no scale bytes past the padded rows
        const float gh = __ldg(p.h_global);
        const int hc0 = nb * 128 + 64 * half;  // first h column of this thread
        uint32_t c[8];
        uint32_t sfw = swiglu_quant_block(g0, u0, alpha, gh, rtab, c[0], c[1]);
        sfw |= swiglu_quant_block(g0 + 16, u0 + 16, alpha, gh, rtab, c[2], c[3]) << 8;
        sfw |= swiglu_quant_block(g1, u1, alpha, gh, rtab, c[4], c[5]) << 16;
        sfw |= swiglu_quant_block(g1 + 16, u1 + 16, alpha, gh, rtab, c[6], c[7]) << 24;
        // rows in [M, m_pad) were zero-filled operands: h = 0, scales 0
        if (row < p.M) {
          uint4* dst = reinterpret_cast<uint4*>(p.h_codes + static_cast<int64_t>(row) * (p.N / 4) +
                                                hc0 / 2);
          dst[0] = make_uint4(c[0], c[1], c[2], c[3]);
          dst[1] = make_uint4(c[4], c[5], c[6], c[7]);
        }
        *reinterpret_cast<uint32_t*>(
            p.h_sf + ((row >> 7) * p.h_atoms + (hc0 >> 6)) * 512 + (row & 31) * 16 +
            ((row & 127) >> 5) * 4) = sfw;
        continue;
      }
      uint32_t r0[32], r1[32], r2[32], r3[32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + ACC_COL + half * 128u;
      ptx::tc_ld_32x32b_x32(taddr + 0u, r0);
      ptx::tc_ld_32x32b_x32(taddr + 32u, r1);
      ptx::tc_ld_32x32b_x32(taddr + 64u, r2);
      ptx::tc_ld_32x32b_x32(taddr + 96u, r3);
      ptx::tc_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(release);
      acc_phase ^= 1u;

      const int row0 = mb * BM + static_cast<int>(rank) * HALF + q * 32;  // this warp's rows
      const int col0 = nb * BN + half * 128;
      if (p.split > 1) {
        // rows past M (a tile's padding): no partial, no count, no output
        if (row0 >= p.M) continue;
        // this slice's partial -> its slab; the region's last slice sums all
        // slabs in slice order (whichever slice that is) and writes Y
        const int region = static_cast<int>(rank) * 8 + (warp - EPI_WARP0);
        const int64_t slab_stride = int64_t{16} * kRegionFloats;  // one slice of a tile
        float* const base = p.partial + int64_t{unit.tile} * p.split * slab_stride +
                            int64_t{region} * kRegionFloats;
        float4* mine = reinterpret_cast<float4*>(base + unit.slice * slab_stride) + lane;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          __stcg(mine + 32 * c, make_float4(__uint_as_float(r0[4 * c]), __uint_as_float(r0[4 * c + 1]),
                                            __uint_as_float(r0[4 * c + 2]),
                                            __uint_as_float(r0[4 * c + 3])));
          __stcg(mine + 32 * (8 + c),
                 make_float4(__uint_as_float(r1[4 * c]), __uint_as_float(r1[4 * c + 1]),
                             __uint_as_float(r1[4 * c + 2]), __uint_as_float(r1[4 * c + 3])));
          __stcg(mine + 32 * (16 + c),
                 make_float4(__uint_as_float(r2[4 * c]), __uint_as_float(r2[4 * c + 1]),
                             __uint_as_float(r2[4 * c + 2]), __uint_as_float(r2[4 * c + 3])));
          __stcg(mine + 32 * (24 + c),
                 make_float4(__uint_as_float(r3[4 * c]), __uint_as_float(r3[4 * c + 1]),
                             __uint_as_float(r3[4 * c + 2]), __uint_as_float(r3[4 * c + 3])));
        }
        __threadfence();
        __syncwarp();
        unsigned int* cnt = p.tile_count + unit.tile * 16 + region;
        uint32_t last = 0;
        if (lane == 0) last = atomicAdd(cnt, 1u) == static_cast<unsigned>(p.split - 1);
        last = __shfl_sync(0xFFFFFFFFu, last, 0);
        if (!last) continue;
        __threadfence();
        // 32 columns at a time: all slices' loads first, then the adds
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t acc[32];
          const float4* src = reinterpret_cast<const float4*>(base) + lane + 32 * (8 * cc);
          switch (p.split) {
            case 2: sum_slices<2>(src, slab_stride / 4, acc); break;
            case 3: sum_slices<3>(src, slab_stride / 4, acc); break;
            default: sum_slices<kMaxSplitK>(src, slab_stride / 4, acc); break;
          }
          if (!p.y_fp32) {
            emit([&](uint32_t b) { stage_bf16(b, lane, acc, alpha); }, col0 + 32 * cc, row0);
          } else {
            emit([&](uint32_t b) { stage_f32(b, lane, acc, 0, alpha); }, col0 + 32 * cc, row0);
            emit([&](uint32_t b) { stage_f32(b, lane, acc, 16, alpha); }, col0 + 32 * cc + 16,
                 row0);
          }
        }
        if (lane == 0) *cnt = 0u;  // ready for the next call
        continue;
      }
      if (row0 >= p.M) continue;  // warp-uniform; rows past M inside are clipped by the TMA
      if (!p.y_fp32) {
        emit([&](uint32_t b) { stage_bf16(b, lane, r0, alpha); }, col0 + 0, row0);
        emit([&](uint32_t b) { stage_bf16(b, lane, r1, alpha); }, col0 + 32, row0);
        emit([&](uint32_t b) { stage_bf16(b, lane, r2, alpha); }, col0 + 64, row0);
        emit([&](uint32_t b) { stage_bf16(b, lane, r3, alpha); }, col0 + 96, row0);
      } else {
        emit([&](uint32_t b) { stage_f32(b, lane, r0, 0, alpha); }, col0 + 0, row0);
        emit([&](uint32_t b) { stage_f32(b, lane, r0, 16, alpha); }, col0 + 16, row0);
        emit([&](uint32_t b) { stage_f32(b, lane, r1, 0, alpha); }, col0 + 32, row0);
        emit([&](uint32_t b) { stage_f32(b, lane, r1, 16, alpha); }, col0 + 48, row0);
        emit([&](uint32_t b) { stage_f32(b, lane, r2, 0, alpha); }, col0 + 64, row0);
        emit([&](uint32_t b) { stage_f32(b, lane, r2, 16, alpha); }, col0 + 80, row0);
        emit([&](uint32_t b) { stage_f32(b, lane, r3, 0, alpha); }, col0 + 96, row0);
        emit([&](uint32_t b) { stage_f32(b, lane, r3, 16, alpha); }, col0 + 112, row0);
      }
    }
    if (lane == 0) ptx::bulk_wait_group_all();  // stores done before the CTA can exit
    if (p.fused == kFusedBf16Amax) {
      // one partial max per CTA (order-free, so the global that the
      // quantizer derives from the partials does not depend on timing);
      // every epilogue warp gets here, also after an abort
      const uint32_t wm = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(h_amax));
      if (lane == 0) atomicMax(h_max, wm);
      asm volatile("bar.sync 1, %0;" ::"n"(32 * NUM_EPI_WARPS) : "memory");
      if (threadIdx.x == EPI_WARP0 * 32) p.h_partials[blockIdx.x] = __uint_as_float(*h_max);
    }
  }

  // Neither CTA frees tensor memory or exits while the pair works: the peer
  // may still signal this CTA's barriers (TMA completions, MMA commits,
  // accumulator releases) or write its tensor memory. This barrier is left
  // without a time limit on purpose: every role above reaches it within the
  // sum of its bounded waits and drains, and a CTA that gave up on it and
  // exited could still be addressed by its peer.
  ptx::tc_fence_before();
  __syncwarp();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    ptx::tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace gemm
}  // namespace nvfp4
