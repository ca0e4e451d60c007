// quant.cuh — NVFP4 quantization of a bf16 tensor (weights or activations).
//
// Format: news article "Qwen3.8-27B最激进4bit量化开源，权重显存暴降2.9倍！" §02
// (NVFP4 量化格式): E2M1 values, one E4M3 scale per 16 contiguous elements,
// one FP32 global scale per tensor; W4A4 applies it to activations on the fly.
// Convention (FP32, round-to-nearest-even at every step):
//   g = 2688 / amax;  s = E4M3(amax_b / 6 * g);  code = E2M1(x * (g / dec(s))).
//
// Both kernels wait for the previous kernel in the stream before touching
// global memory, so they may be launched with programmatic stream
// serialisation; each lets the next kernel be scheduled as soon as it starts
// (that kernel in turn waits for this one before it reads what this one
// writes), so a following GEMM's set-up and weight loads can overlap it.
// Two kernels:
//   amax_kernel      one pass over x, one partial max per CTA (no atomics, so
//                    the workspace needs no initialisation);
//   quantize_kernel  every CTA first reduces the partials to g (a few hundred
//                    floats from L2) and tabulates r(s) = g / dec(s) for all
//                    128 E4M3 codes (one IEEE division each, so the per-block
//                    division becomes a shared-memory load with the same
//                    result), then quantizes. A warp task is one (128-row
//                    block, row l in 0..31, 4 consecutive 64-column atoms):
//                    lane (g, j) works on row l + 32g and, per pass, on one
//                    whole 16-element block (two 16-byte loads through L1,
//                    block max without a shuffle); 4 lanes then hold the 4
//                    scales of one 16-byte line of a swizzled atom and OR them
//                    together with two shuffles. Two passes cover the 4 atoms.
//                    (Half a block per lane, the first layout, spent ~25% more
//                    integer work per element; at 32768x17408 this layout
//                    streams at 0.96 of the measured HBM bandwidth.)
// L2 policy: the amax pass reads x with an evict-last hint, so that the
// quantizer's second read of x is served from L2 as far as L2 holds it, and
// the quantizer reads it with an evict-first hint, so that x's lines are the
// first to leave L2 afterwards and the GEMM's operands stay (dynamic
// quantization of 8192x5120: 39.9 -> 35.8 us; the bits are unchanged).
// amax_b / 6 is computed as q = amax_b * RN(1/6), q + RN((amax_b - 6 q) *
// RN(1/6)) with two FMAs; this equals the IEEE quotient for every
// non-negative bf16 value (checked exhaustively with exact rationals in the
// test-suite), which is the only input it ever sees.
#pragma once

#include "ptx.cuh"

namespace nvfp4 {
namespace quant {

constexpr int kAmaxThreads = 1024;
constexpr int kMaxPartials = 4096;            // workspace = 16 KiB
constexpr int kQuantThreads = 256;
constexpr int kAtomsPerTask = 4;
constexpr int64_t kSelfAmaxBytes = 64 * 1024;  // x up to this size: no amax pass
constexpr float kInv6 = 0.16666667163372039794921875f;  // RN(1/6) = 0x3E2AAAAB

// RN(a / 6) for a non-negative bf16 value a (see the header comment).
__device__ __forceinline__ float div6_rn(float a) {
  const float q = __fmul_rn(a, kInv6);
  const float r = __fmaf_rn(-q, 6.0f, a);
  return __fmaf_rn(r, kInv6, q);
}

// L2 cache policies (createpolicy): every line the load touches gets the
// policy's eviction priority.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 16-byte load through L1 with an L2 policy: the two halves of a lane's
// 32-byte block are issued back to back and the second is served from the
// first's line fill.
__device__ __forceinline__ uint4 ldg_l1(const void* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

// 16-byte streaming load (no L1 allocation) with an L2 policy.
__device__ __forceinline__ uint4 ldg_stream(const void* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

// max |x| of 8 bf16 values, as the 15-bit magnitude pattern (sign cleared);
// for non-negative floats the bit pattern orders like the value.
__device__ __forceinline__ uint32_t absmax_bits8(uint4 v) {
  const uint32_t m = 0x7FFF7FFFu;
  const uint32_t w = __vmaxu2(__vmaxu2(v.x & m, v.y & m), __vmaxu2(v.z & m, v.w & m));
  return max(w & 0xFFFFu, w >> 16);
}

__global__ void __launch_bounds__(kAmaxThreads)
    amax_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t k, int64_t ldx,
                float* __restrict__ partials) {
  ptx::grid_dep_launch();  // the next kernel may be scheduled; it waits for this one itself
  ptx::grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t chunks = k >> 3;  // 16-byte chunks per row
  uint32_t m = 0;
  const uint64_t pol = l2_evict_last_policy();  // the quantizer reads x next
  if (ldx == k) {
    // contiguous tensor: one flat stream of 16-byte chunks, 8 loads in flight
    const int64_t total = rows * chunks;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + 7 * nthreads < total; i += 8 * nthreads) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = ldg_stream(x + (i + u * nthreads) * 8, pol);
#pragma unroll
      for (int u = 0; u < 8; ++u) m = max(m, absmax_bits8(v[u]));
    }
    for (; i < total; i += nthreads) m = max(m, absmax_bits8(ldg_stream(x + i * 8, pol)));
  }
  for (int64_t r = (ldx == k) ? rows : warp; r < rows; r += nwarps) {
    const uint16_t* row = x + r * ldx;
    int64_t c = lane;
    for (; c + 96 < chunks; c += 128) {
      const uint4 v0 = ldg_stream(row + c * 8, pol);
      const uint4 v1 = ldg_stream(row + (c + 32) * 8, pol);
      const uint4 v2 = ldg_stream(row + (c + 64) * 8, pol);
      const uint4 v3 = ldg_stream(row + (c + 96) * 8, pol);
      m = max(m, max(max(absmax_bits8(v0), absmax_bits8(v1)),
                     max(absmax_bits8(v2), absmax_bits8(v3))));
    }
    for (; c < chunks; c += 32) m = max(m, absmax_bits8(ldg_stream(row + c * 8, pol)));
  }
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t s_red[32];
  if (lane == 0) s_red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t v = threadIdx.x < (blockDim.x >> 5) ? s_red[threadIdx.x] : 0u;
    v = __reduce_max_sync(0xFFFFFFFFu, v);
    if (threadIdx.x == 0) partials[blockIdx.x] = __uint_as_float(v << 16);
  }
}

struct QuantArgs {
  const uint16_t* x;
  int64_t rows, k, ldx;
  const float* global_in;   // static mode when non-null
  const float* partials;    // dynamic mode: per-CTA maxima of amax_kernel
  int nparts;               // dynamic mode: 0 = no amax pass, every CTA reads x itself
  uint8_t* codes;
  uint8_t* sf;
  float* global_out;
  // 1: scales of the padding rows [rows, 128) of a tensor of fewer than 32
  // rows are not written (a caller-private buffer only the GEMM reads; its
  // padding rows multiply zero-filled codes): a decode step's few tokens
  // then need rows x (k/256) warp tasks instead of 32 x (k/256).
  int skip_pad;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__global__ void __launch_bounds__(kQuantThreads) quantize_kernel(const QuantArgs a) {
  ptx::grid_dep_launch();  // the next kernel may be scheduled; it waits for this one itself
  ptx::grid_dep_wait();    // partials / static global / x come from earlier kernels
  __shared__ float s_g;
  __shared__ float s_rtab[128];
  __shared__ uint32_t s_red[kQuantThreads / 32];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;

  // ---- global scale g (identical in every CTA) -----------------------------
  if (a.global_in != nullptr) {
    if (threadIdx.x == 0) s_g = *a.global_in;
  } else {
    uint32_t m = 0;
    if (a.nparts > 0) {
      for (int i = threadIdx.x; i < a.nparts; i += blockDim.x)
        m = max(m, __float_as_uint(a.partials[i]));  // non-negative: bits order as values
    } else {
      // Small x (the host bounds it by kSelfAmaxBytes): every CTA takes the
      // tensor's max itself from L2, so no amax pass precedes this kernel.
      // Rounds of 8 predicated 16-byte loads per thread, all in flight
      // before the first max: x of at most 64 KiB takes 2 round trips (one
      // dependent load at a time took 9 for a 17408-wide row).
      const uint32_t chunks = static_cast<uint32_t>(a.k >> 3);
      const uint32_t total = static_cast<uint32_t>(a.rows) * chunks;
      const uint32_t nt = blockDim.x;
      for (uint32_t i = threadIdx.x; i < total; i += 8u * nt) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t e = i + u * nt;
          const uint32_t r = e / chunks;
          const uint32_t c = e - r * chunks;
          v[u] = e < total ? __ldg(reinterpret_cast<const uint4*>(
                                 a.x + static_cast<uint64_t>(r) * static_cast<uint64_t>(a.ldx) +
                                 c * 8u))
                           : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) m = max(m, absmax_bits8(v[u]) << 16);  // -> FP32 bits
      }
    }
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (lane == 0) s_red[wib] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t mm = 0;
      for (int w = 0; w < kQuantThreads / 32; ++w) mm = max(mm, s_red[w]);
      const float amax = __uint_as_float(mm);
      float g = (amax == 0.0f) ? 1.0f : __fdiv_rn(2688.0f, amax);
      if (!isfinite(g)) g = 1.0f;
      s_g = g;
    }
  }
  __syncthreads();
  const float g = s_g;
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.global_out = g;
  if (threadIdx.x < 128) {
    const float ds = ptx::e4m3_value(threadIdx.x);
    s_rtab[threadIdx.x] = (ds == 0.0f) ? 0.0f : __fdiv_rn(g, ds);  // r = 0 keeps only signs
  }
  __syncthreads();

  // ---- blocks ----------------------------------------------------------------
  const int64_t n_rb = (a.rows + 127) / 128;
  const int64_t n_ka = (a.k + 63) / 64;  // 512-byte atoms per 128-row block
  const int64_t n_kc = (n_ka + kAtomsPerTask - 1) / kAtomsPerTask;
  const int64_t n_tasks = (a.skip_pad && a.rows < 32) ? a.rows * n_kc : n_rb * 32 * n_kc;
  const int grp = lane >> 3;  // row group: row l + 32*grp
  const int j = lane & 7;     // 16-byte chunk of the row's 128-byte atom slice
  const int64_t half_k = a.k >> 1;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;

  // 32-bit task indexing (the host guarantees n_tasks < 2^31): the 64-bit
  // division and address arithmetic it replaces cost ~15% of the kernel's
  // issue slots, and the smaller register count lets 5 CTAs share an SM
  // instead of 4.
  const uint32_t nkc = static_cast<uint32_t>(n_kc);
  const uint32_t ntask = static_cast<uint32_t>(n_tasks);
  const uint32_t nka = static_cast<uint32_t>(n_ka);
  const uint32_t w0 = static_cast<uint32_t>(warp), nw = static_cast<uint32_t>(nwarps);
  // lane = (row group g = lane >> 3, j = lane & 7): j >> 2 picks one of two
  // adjacent atoms, j & 3 the 16-element block in it, so a lane quantizes one
  // whole block (no shuffle for the block max) and 4 lanes hold one line word
  // of an atom's scales. Two passes cover the task's 4 atoms.
  const uint32_t jb = static_cast<uint32_t>(j & 3), ja = static_cast<uint32_t>(j >> 2);
  const uint32_t k32 = static_cast<uint32_t>(a.k);
  const uint64_t pol = l2_evict_first_policy();  // x is not read again
  for (uint32_t t = w0; t < ntask; t += nw) {
    const uint32_t tl = t / nkc;
    const uint32_t kc = t - tl * nkc;
    const uint32_t l = tl & 31u;
    const uint32_t rb = tl >> 5;
    const uint32_t row = rb * 128u + static_cast<uint32_t>(grp) * 32u + l;
    const bool row_ok = row < static_cast<uint64_t>(a.rows);
    const uint16_t* xrow = a.x + static_cast<uint64_t>(row) * static_cast<uint64_t>(a.ldx);
    uint8_t* crow = a.codes + static_cast<uint64_t>(row) * static_cast<uint64_t>(half_k);
    uint8_t* sfb = a.sf + (static_cast<uint64_t>(rb) * nka) * 512u + l * 16u + grp * 4;
    uint4 v[2][2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t col = (kc * 4u + 2u * u + ja) * 64u + jb * 16u;
      v[u][0] = v[u][1] = make_uint4(0u, 0u, 0u, 0u);
      if (row_ok && col < k32) {
        v[u][0] = ldg_l1(xrow + col, pol);
        v[u][1] = ldg_l1(xrow + col + 8, pol);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t ka = kc * 4u + 2u * u + ja;
      if (kc * 4u + 2u * u >= nka) break;  // warp-uniform: no atom of this pass exists
      const uint32_t col = ka * 64u + jb * 16u;
      const bool ok = row_ok && col < k32;
      const uint32_t mb = max(absmax_bits8(v[u][0]), absmax_bits8(v[u][1]));
      const uint32_t s = ptx::cvt_e4m3(__fmul_rn(div6_rn(__uint_as_float(mb << 16)), g));
      const float r = s_rtab[s];
      uint32_t c[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float f[8];
        f[0] = __fmul_rn(bf16_lo(v[u][h].x), r);
        f[1] = __fmul_rn(bf16_hi(v[u][h].x), r);
        f[2] = __fmul_rn(bf16_lo(v[u][h].y), r);
        f[3] = __fmul_rn(bf16_hi(v[u][h].y), r);
        f[4] = __fmul_rn(bf16_lo(v[u][h].z), r);
        f[5] = __fmul_rn(bf16_hi(v[u][h].z), r);
        f[6] = __fmul_rn(bf16_lo(v[u][h].w), r);
        f[7] = __fmul_rn(bf16_hi(v[u][h].w), r);
        c[h] = ptx::cvt_e2m1x8(f);
      }
      if (ok) *reinterpret_cast<uint2*>(crow + (col >> 1)) = make_uint2(c[0], c[1]);
      // the 4 blocks of this atom line: lanes 4*ja + {0..3}
      uint32_t word = s << (8u * jb);
      word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
      word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
      if (jb == 0 && ka < nka) *reinterpret_cast<uint32_t*>(sfb + ka * 512u) = word;
    }
  }
}

// Calibration step: running_amax = max(running_amax, max of the partials);
// global_out = 2688 / running_amax (1 when that is 0 or not finite). One CTA.
__global__ void __launch_bounds__(256)
    calibrate_kernel(const float* __restrict__ partials, int nparts, float* running_amax,
                     float* global_out) {
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  __shared__ uint32_t s_red[8];
  uint32_t m = 0;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) m = max(m, __float_as_uint(partials[i]));
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 0; w < 8; ++w) m = max(m, s_red[w]);
    const float amax = fmaxf(*running_amax, __uint_as_float(m));
    *running_amax = amax;
    float g = (amax == 0.0f) ? 1.0f : __fdiv_rn(2688.0f, amax);
    if (!isfinite(g)) g = 1.0f;
    *global_out = g;
  }
}

}  // namespace quant
}  // namespace nvfp4
