/*
 * nvfp4_oracle.c — plain, slow, obviously-correct CPU reference of the NVFP4
 * W4A4 linear-layer path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call this code:
 * only the test-suite, the package smoke check and the benchmark's CPU-baseline
 * leg load it. It shares no source, header, table or helper with the CUDA
 * library; the two meet only at the bytes of their inputs and outputs.
 *
 * What it follows (web pages on arXiv 2609.04098):
 *   - news article "Qwen3.8-27B最激进4bit量化开源，权重显存暴降2.9倍！",
 *     §02 (NVFP4 量化格式): 4-bit E2M1 values, one E4M3 scale per 16 elements,
 *     one FP32 global scale per tensor; weights and activations both (W4A4).
 *   - same article §03 (Minima 模型构建): fused module groups are repaired by
 *     putting the group on one global scale and folding the ratio into the
 *     E4M3 block scales.
 *   - MessageDaily reading of the paper, §一: NVFP4 shares one scale per 16
 *     elements.
 * The pages give no formula for the scales. The convention implemented here
 * (identical to the library's written contract) is:
 *   g = 2688 / amax (FP32; g = 1 when amax == 0 or g is not finite),
 *   s = E4M3(amax_b / 6 * g), code = E2M1(x * (g / dec(s))),
 * each arithmetic step one IEEE FP32 round-to-nearest-even operation, each
 * encoding round-to-nearest with ties to the even code, saturating.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC
 * (contraction off so that no multiply-add is fused: every FP32 step rounds).
 * Parity pins for every function live in tests/ (codec brute force, library
 * casts, closed forms, invariants, exact integer GEMM).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- bf16 ---- */

/* bf16 is the top half of an IEEE binary32: widening is exact. */
float orc_bf16_to_float(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Round a double to the nearest bf16 (8 significant bits, binary32 exponent
 * range), ties to even, by scaling to an integer grid and calling nearbyint.
 * Used only for the silu*mul output, which is compared within one bf16 ulp. */
uint16_t orc_double_to_bf16(double v) {
  double a = fabs(v);
  double q;
  if (a == 0.0) {
    q = 0.0;
  } else {
    int e;
    frexp(a, &e);          /* a in [2^(e-1), 2^e) */
    int E = e - 1;
    if (E < -126) E = -126; /* subnormals share the min-normal spacing */
    double quantum = ldexp(1.0, E - 7);
    q = nearbyint(a / quantum) * quantum;
  }
  float f = (float)q; /* q has <= 8 significant bits: exact (or inf) */
  if (v < 0 || (v == 0 && signbit(v))) f = -f;
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(u >> 16);
}

/* ---------------------------------------------------------------- E2M1 ---- */

/* Magnitudes of the 8 non-negative E2M1 codes (news §02 format; grid
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}). Code = sign*8 + index. */
static const double kE2M1Grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_value(uint8_t code) {
  double m = kE2M1Grid[code & 7];
  return (code & 8) ? -m : m;
}

/* Round v to the E2M1 grid: nearest value, a tie goes to the even code
 * (equivalently: IEEE round-half-even on a 1-mantissa-bit float), and any
 * magnitude >= 6 saturates to 6. The sign bit of v is kept, so -0.0 and small
 * negatives give 0x8. */
uint8_t orc_e2m1_encode(float v) {
  uint8_t sign = signbit(v) ? 8 : 0;
  double a = fabs((double)v);
  double q;
  if (a >= 6.0) {
    q = 6.0;                         /* satfinite */
  } else if (a < 2.0) {
    q = nearbyint(a * 2.0) / 2.0;    /* binades [0,1),[1,2): spacing 0.5 */
  } else if (a < 4.0) {
    q = nearbyint(a);                /* binade [2,4): spacing 1 */
  } else {
    q = 2.0 * nearbyint(a / 2.0);    /* binade [4,8): spacing 2 (6 = max) */
  }
  uint8_t idx = 0;
  for (uint8_t c = 0; c < 8; ++c)
    if (kE2M1Grid[c] == q) idx = c;
  return (uint8_t)(sign | idx);
}

/* ---------------------------------------------------------------- E4M3 ---- */

/* OCP FP8 E4M3 ("E4M3FN"): bias 7, no infinities, 0x7F/0xFF = NaN, largest
 * finite 448, smallest normal 2^-6, subnormal spacing 2^-9. */
double orc_e4m3_value(uint8_t code) {
  int e = (code >> 3) & 0xF;
  int m = code & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  return (code & 0x80) ? -v : v;
}

/* Round v to E4M3: nearest representable value, ties to the even code,
 * magnitudes >= 448 saturate to 448 (never NaN), values below half the
 * smallest subnormal (and exactly half: tie to even code 0) become 0. */
uint8_t orc_e4m3_encode(float v) {
  uint8_t sign = signbit(v) ? 0x80 : 0;
  double a = fabs((double)v);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e);          /* a in [2^(e-1), 2^e) */
  int E = e - 1;
  if (E < -6) E = -6;    /* subnormals use the spacing of the first binade */
  double quantum = ldexp(1.0, E - 3);           /* 3 mantissa bits */
  double q = nearbyint(a / quantum) * quantum;  /* a/quantum is exact */
  if (q == 0.0) return sign;
  int e2;
  frexp(q, &e2);
  int E2 = e2 - 1;
  if (E2 < -6) {                                 /* subnormal: m * 2^-9 */
    int m = (int)(q / ldexp(1.0, -9));
    return (uint8_t)(sign | m);
  }
  int mant = (int)((q / ldexp(1.0, E2) - 1.0) * 8.0);
  return (uint8_t)(sign | ((E2 + 7) << 3) | mant);
}

/* ---------------------------------------------------------- global scale -- */

/* amax over the first k elements of each of `rows` rows of pitch ldx. */
float orc_tensor_amax(const uint16_t* x, int64_t rows, int64_t k, int64_t ldx) {
  float amax = 0.0f;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t j = 0; j < k; ++j) {
      float a = fabsf(orc_bf16_to_float(x[r * ldx + j]));
      if (a > amax) amax = a;
    }
  return amax;
}

/* g = 2688 / amax with one FP32 division (2688 = 448 * 6: the largest E4M3
 * scale times the largest E2M1 value); degenerate tensors get g = 1. */
float orc_global_from_amax(float amax) {
  if (amax == 0.0f) return 1.0f;
  float g = 2688.0f / amax;
  if (!isfinite(g)) return 1.0f;
  return g;
}

/* ------------------------------------------------------------- quantize ---- */

/* Quantize one [rows][k] bf16 tensor with global g. Writes codes [rows][k/2]
 * (element 2j in the low nibble of byte j) and the block scales in plain
 * row-major order sf_rm[rows][k/16] (the swizzle is a separate step). */
void orc_quantize(const uint16_t* x, int64_t rows, int64_t k, int64_t ldx,
                  float g, uint8_t* codes, uint8_t* sf_rm) {
  const int64_t nb = k / 16;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const uint16_t* xb = x + r * ldx + b * 16;
      float xs[16];
      float amax_b = 0.0f;
      for (int i = 0; i < 16; ++i) {
        xs[i] = orc_bf16_to_float(xb[i]);
        float a = fabsf(xs[i]);
        if (a > amax_b) amax_b = a;
      }
      /* block scale: E4M3(amax_b / 6 * g), two FP32 roundings, then encode */
      float t = amax_b / 6.0f;
      float s32 = t * g;
      uint8_t s = orc_e4m3_encode(s32);
      sf_rm[r * nb + b] = s;
      float ds = (float)orc_e4m3_value(s); /* exact */
      uint8_t q[16];
      if (ds == 0.0f) {
        for (int i = 0; i < 16; ++i) q[i] = signbit(xs[i]) ? 8 : 0;
      } else {
        float rcp = g / ds; /* one FP32 division per block */
        for (int i = 0; i < 16; ++i) q[i] = orc_e2m1_encode(xs[i] * rcp);
      }
      uint8_t* cb = codes + r * (k / 2) + b * 8;
      for (int i = 0; i < 8; ++i)
        cb[i] = (uint8_t)(q[2 * i] | (q[2 * i + 1] << 4));
    }
  }
}

/* ------------------------------------------------------------- layout ------ */

/* Byte offset of block (r, c) of a [rows][k] tensor in the 128x4 swizzled
 * scale layout: 512-byte atoms of 128 rows x 4 blocks, atoms ordered by
 * row-block then block-group; inside an atom row r%32 owns 16 bytes holding
 * row groups (r%128)/32 = 0..3, 4 blocks each. */
int64_t orc_sf_offset(int64_t r, int64_t c, int64_t k) {
  int64_t kb4 = ((k / 16 + 3) / 4) * 4;
  return ((r / 128) * (kb4 / 4) + c / 4) * 512 + (r % 32) * 16 +
         ((r % 128) / 32) * 4 + (c % 4);
}

int64_t orc_sf_bytes(int64_t rows, int64_t k) {
  int64_t kb4 = ((k / 16 + 3) / 4) * 4;
  int64_t r128 = ((rows + 127) / 128) * 128;
  return r128 * kb4;
}

void orc_sf_swizzle(const uint8_t* sf_rm, int64_t rows, int64_t k,
                    uint8_t* sf_sw) {
  const int64_t nb = k / 16;
  memset(sf_sw, 0, (size_t)orc_sf_bytes(rows, k));
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < nb; ++c)
      sf_sw[orc_sf_offset(r, c, k)] = sf_rm[r * nb + c];
}

void orc_sf_unswizzle(const uint8_t* sf_sw, int64_t rows, int64_t k,
                      uint8_t* sf_rm) {
  const int64_t nb = k / 16;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < nb; ++c)
      sf_rm[r * nb + c] = sf_sw[orc_sf_offset(r, c, k)];
}

/* ---------------------------------------------------------- dequantize ---- */

/* x_hat = val(code) * dec(s) / g, in FP64 (exact up to the final division).
 * With g == 0 passed in, the division is skipped: out = val * dec(s), which is
 * an exact multiple of 2^-10 (used by the exact-integer GEMM pin). */
void orc_dequantize(const uint8_t* codes, const uint8_t* sf_rm, float g,
                    int64_t rows, int64_t k, double* out) {
  const int64_t nb = k / 16;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t j = 0; j < k; ++j) {
      uint8_t byte = codes[r * (k / 2) + j / 2];
      uint8_t code = (j % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      double v = orc_e2m1_value(code) * orc_e4m3_value(sf_rm[r * nb + j / 16]);
      out[r * k + j] = (g == 0.0f) ? v : v / (double)g;
    }
}

/* ----------------------------------------------------------------- fold ---- */

/* Fused-group repair (news §03): bring n modules with their own globals g_i
 * onto one global g* and fold the ratio into each block scale.
 *   g* = min_i g_i (the module with the largest amax; every ratio <= 1),
 *   r_i = g* / g_i (FP32), s' = E4M3(dec(s) * r_i) (FP32 multiply), codes kept.
 * sf_in[i] / sf_out[i] are row-major [rows_i][k/16]. Returns g*. */
float orc_fold_group(int n, const int64_t* rows, int64_t k,
                     const uint8_t* const* sf_in, const float* g_in,
                     uint8_t* const* sf_out) {
  float gstar = g_in[0];
  for (int i = 1; i < n; ++i)
    if (g_in[i] < gstar) gstar = g_in[i];
  const int64_t nb = k / 16;
  for (int i = 0; i < n; ++i) {
    float ratio = gstar / g_in[i];
    for (int64_t t = 0; t < rows[i] * nb; ++t) {
      float ds = (float)orc_e4m3_value(sf_in[i][t]);
      sf_out[i][t] = orc_e4m3_encode(ds * ratio);
    }
  }
  return gstar;
}

/* ------------------------------------------------------------ silu*mul ---- */

/* h = silu(gate) * up with gate = y[:, 0:n], up = y[:, n:2n], in FP64, then
 * rounded once to bf16. silu(z) = z / (1 + exp(-z)). */
void orc_silu_mul(const uint16_t* y, int64_t m, int64_t n, int64_t ldy,
                  uint16_t* h) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < n; ++j) {
      double gate = orc_bf16_to_float(y[i * ldy + j]);
      double up = orc_bf16_to_float(y[i * ldy + n + j]);
      double s = gate / (1.0 + exp(-gate));
      h[i * n + j] = orc_double_to_bf16(s * up);
    }
}

/* ----------------------------------------------- array forms for Python --- */

void orc_e2m1_encode_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(v[i]);
}

void orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

void orc_e4m3_value_array(const uint8_t* c, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_value(c[i]);
}

void orc_e2m1_value_array(const uint8_t* c, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_value(c[i]);
}
