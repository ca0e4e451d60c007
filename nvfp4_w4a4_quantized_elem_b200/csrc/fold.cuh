// fold.cuh — global-scale repair of a fused module group.
//
// News article "Qwen3.8-27B最激进4bit量化开源，权重显存暴降2.9倍！" §03
// (Minima 模型构建): GDN fuses several linear layers (qkv, z, a, b) into one
// GEMM; if the fusion just takes the group's largest global scale without
// rescaling the block scales, the weights are mis-scaled. The repair puts the
// group on one global scale and folds the ratio into the E4M3 block scales.
//   g* = min_i g_i,  r_i = g* / g_i,  s' = E4M3(dec(s) * r_i)  (FP32 RN).
//
// One thread per 32-bit word of the fused swizzled scale buffer: the word is
// one row's 4 block scales inside a 512-byte atom. It finds the module that
// owns the row, reads the same word of that module's own swizzled buffer and
// rescales the 4 bytes. Atoms that straddle two modules are filled from both;
// rows past the group and blocks past k/16 are written as 0.
#pragma once

#include "ptx.cuh"

namespace nvfp4 {
namespace fold {

constexpr int kMaxModules = 16;
constexpr int kThreads = 256;

struct FoldArgs {
  int n;
  int64_t k;
  int64_t n_ka;                         // atoms per 128-row block
  int64_t total_rows;
  int64_t row_start[kMaxModules + 1];   // prefix sums of module rows
  const uint8_t* sf_in[kMaxModules];
  const float* g_in;
  uint8_t* sf_out;
  float* g_out;
};

__global__ void __launch_bounds__(kThreads) fold_kernel(const FoldArgs a) {
  __shared__ float s_ratio[kMaxModules];
  if (threadIdx.x == 0) {
    float gstar = a.g_in[0];
    for (int i = 1; i < a.n; ++i) gstar = fminf(gstar, a.g_in[i]);
    for (int i = 0; i < a.n; ++i) s_ratio[i] = __fdiv_rn(gstar, a.g_in[i]);
    if (blockIdx.x == 0) *a.g_out = gstar;
  }
  __syncthreads();

  const int64_t n_rb = (a.total_rows + 127) / 128;
  const int64_t n_words = n_rb * a.n_ka * 128;
  const int64_t kb = a.k / 16;
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; w < n_words;
       w += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t atom = w >> 7;
    const int li = static_cast<int>(w & 127);
    const int l = li >> 2, grp = li & 3;
    const int64_t rb = atom / a.n_ka, ka = atom % a.n_ka;
    const int64_t row = rb * 128 + grp * 32 + l;
    uint32_t out = 0;
    if (row < a.total_rows) {
      int i = 0;
      while (i + 1 < a.n && row >= a.row_start[i + 1]) ++i;
      const int64_t lr = row - a.row_start[i];
      const int64_t src = ((lr >> 7) * a.n_ka + ka) * 512 + (lr & 31) * 16 + ((lr & 127) >> 5) * 4;
      const uint32_t in = *reinterpret_cast<const uint32_t*>(a.sf_in[i] + src);
      const float ratio = s_ratio[i];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        if (ka * 4 + b >= kb) continue;  // padding block
        const float ds = ptx::e4m3_value((in >> (8 * b)) & 0xFFu);
        out |= ptx::cvt_e4m3(__fmul_rn(ds, ratio)) << (8 * b);
      }
    }
    reinterpret_cast<uint32_t*>(a.sf_out)[w] = out;
  }
}

}  // namespace fold
}  // namespace nvfp4
