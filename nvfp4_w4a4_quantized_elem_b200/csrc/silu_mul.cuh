// silu_mul.cuh — the gated-MLP activation between a W4A4 gate_up GEMM and
// the down GEMM: h = bf16_rn(silu(gate) * up), silu(z) = z / (1 + exp(-z)),
// FP32 inside. The pages only state that every linear layer is quantized
// (news article "Qwen3.8-27B最激进4bit量化开源…" §03); the activation between
// the two MLP projections is the model's own and is reproduced plainly here.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace nvfp4 {
namespace act {

constexpr int kThreads = 256;

// silu(g) * u in FP32, shared by the standalone kernel and the fused GEMM
// epilogues so all of them give the same bits. The exponential and the
// division are the hardware's fast forms (__expf, __fdividef: a few FP32 ulp),
// far inside the bf16 rounding of h that follows (h stays within one bf16
// ulp of the FP64 value); in the fused gate_up epilogue the IEEE forms cost
// ~4x the issue slots of this expression, per element of h. Below g = -80,
// 1 + exp(-g) leaves __fdividef's operand range (2^126) and exp(g) is no
// longer a normal number for __expf; there silu(g) = g e^g / (1 + e^g) equals
// g e^g in FP32, taken with the accurate expf.
__device__ __forceinline__ float swiglu(float g, float u) {
  const float s = g < -80.0f ? __fmul_rn(g, expf(g))
                             : __fdividef(g, __fadd_rn(1.0f, __expf(-g)));
  return __fmul_rn(s, u);
}

// h = bf16(silu(gate) * up), gate = y[:, :n], up = y[:, n:2n]; one warp per
// row, 16-byte vectors (8 elements) per lane.
__global__ void __launch_bounds__(kThreads)
    silu_mul_kernel(const uint16_t* __restrict__ y, int64_t m, int64_t n, int64_t ldy,
                    uint16_t* __restrict__ h, int64_t ldh) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t chunks = n >> 3;
  for (int64_t r = warp; r < m; r += nwarps) {
    const uint16_t* yr = y + r * ldy;
    uint16_t* hr = h + r * ldh;
    for (int64_t c = lane; c < chunks; c += 32) {
      const uint4 gv = *reinterpret_cast<const uint4*>(yr + c * 8);
      const uint4 uv = *reinterpret_cast<const uint4*>(yr + n + c * 8);
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
      const uint32_t uw[4] = {uv.x, uv.y, uv.z, uv.w};
      uint32_t ow[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float g0 = __uint_as_float(gw[e] << 16), g1 = __uint_as_float(gw[e] & 0xFFFF0000u);
        const float u0 = __uint_as_float(uw[e] << 16), u1 = __uint_as_float(uw[e] & 0xFFFF0000u);
        const float h0 = swiglu(g0, u0);
        const float h1 = swiglu(g1, u1);
        const __nv_bfloat162 p = __floats2bfloat162_rn(h0, h1);
        ow[e] = *reinterpret_cast<const uint32_t*>(&p);
      }
      *reinterpret_cast<uint4*>(hr + c * 8) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
    }
  }
}

}  // namespace act
}  // namespace nvfp4
