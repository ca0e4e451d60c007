/*
 * nvfp4.h — C ABI of libnvfp4.so, the NVFP4 W4A4 linear layer for sm_100a.
 *
 * Sources (web pages about "Why Gated DeltaNet Survives 4-Bit Quantization:
 * NVFP4 W4A4 for the Recurrent Half of a Hybrid 27B LLM", arXiv 2609.04098):
 *   [news]     "Qwen3.8-27B最激进4bit量化开源，权重显存暴降2.9倍！", sections 02
 *              (NVFP4 量化格式) and 03 (Minima 模型构建);
 *   [reading]  MessageDaily paper reading "minima-gdn-4bit-quantization",
 *              section 一 (论文背景) and section 4.1;
 *   [abstract] arXiv 2609.04098 abstract (English abstract).
 *
 * FORMAT (news §02; reading §一). A tensor X[rows][k] is stored as
 *   - codes: 4-bit E2M1 values, row-major [rows][k/2] bytes, element 2j of a
 *            row in the LOW nibble of byte j, element 2j+1 in the high nibble.
 *            Code = sign*8 + m, m = 0..7 -> {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 *   - sf:    one unsigned E4M3 block scale per 16 contiguous elements along k,
 *            stored in the 128x4 swizzled layout (below).
 *   - g:     one FP32 global scale per tensor (a device scalar).
 * Dequantized value: val(code) * dec(sf) / g.
 *
 * CONVENTION (the pages name the three scales but give no formula; this is the
 * convention the library fixes, evaluated in IEEE FP32 round-to-nearest-even):
 *   amax = max |x| over the tensor (exact);  g = 2688 / amax  (2688 = 448*6);
 *          g = 1 if amax == 0 or the quotient is not finite.
 *   per 16-element block b:  t = amax_b / 6;  s = E4M3_rne_satfinite(t * g);
 *   per element:  r = g / dec(s);  code = E2M1_rne_satfinite(x * r);
 *                 if dec(s) == 0 every code of the block is a signed zero.
 *   The sign of a code is the sign bit of x * r (so -0.0 and tiny negatives
 *   encode as 0x8).
 *
 * SCALE-FACTOR LAYOUT ("128x4 swizzle"). With kb = k/16 blocks per row,
 *   KB4 = ceil(kb/4)*4 and R128 = ceil(rows/128)*128, the buffer holds
 *   R128*KB4 bytes (nvfp4_sf_bytes). Block (r, c) lives at byte
 *     ((r/128)*(KB4/4) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + (c%4).
 *   Each 512-byte atom covers 128 rows x 4 blocks; bytes for r >= rows or
 *   c >= kb are zero. This is the layout the sm_100 block-scaled tensor-core
 *   instruction consumes after a 32x128b tensor-memory copy.
 *
 * CONVENTIONS OF THE ABI
 *   - Every pointer named "device" is CUDA global memory of the current device.
 *     The caller owns every buffer; the library keeps no per-call state.
 *   - Every compute call is asynchronous on the given stream; argument checks
 *     are synchronous and return a status before anything is launched.
 *   - Global scales stay on the device: no call synchronises with the host.
 *   - NaN / Inf inputs are outside the contract.
 *   - No C++ exception crosses this boundary.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle (cudaStream_t); NULL is the legacy default stream. */
typedef struct CUstream_st* nvfp4_stream_t;

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,  /* null pointer, negative/zero size, bad enum   */
  NVFP4_ERR_UNSUPPORTED = 2,  /* shape outside what the kernels implement     */
  NVFP4_ERR_MISALIGNED = 3,   /* pointer or pitch alignment rule broken       */
  NVFP4_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed          */
  NVFP4_ERR_TIMEOUT = 5       /* a kernel's bounded wait expired (fault word) */
} nvfp4_status;

/* Human-readable name of a status. Never NULL. */
const char* nvfp4_status_string(nvfp4_status s);

/* Bytes of the swizzled scale-factor buffer of a [rows][k] tensor:
 * ceil(rows/128)*128 * ceil(k/64)*4.  Returns 0 if rows < 0, k <= 0 or
 * k % 16 != 0. */
size_t nvfp4_sf_bytes(int64_t rows, int64_t k);

/* Workspace bytes nvfp4_quantize needs in dynamic-global mode (per-CTA
 * partial maxima). Static mode needs none. */
size_t nvfp4_quantize_workspace_bytes(int64_t rows, int64_t k);

/*
 * nvfp4_quantize — activation / weight quantization (news §02: E2M1 values,
 * one E4M3 scale per 16 elements, one FP32 global scale; W4A4 quantizes both
 * weights and activations, reading §4.1 / news §03).
 *
 *   x          device, bf16 [rows][ldx] (only the first k of each row are
 *              read); 16-byte aligned, ldx % 8 == 0, ldx >= k.
 *   rows       >= 0 (0 writes nothing but global_out).
 *   k          > 0, k % 16 == 0.
 *   global_in  device FP32 scalar or NULL. NULL => dynamic mode: amax over x,
 *              g = 2688/amax (two kernels: an amax pass, then the quantizer;
 *              one kernel when rows * k * 2 <= NVFP4_ONE_PASS_MAX_BYTES, in
 *              which every CTA of the quantizer takes the max itself).
 *              Non-NULL => static (calibrated) mode: g = *global_in as given;
 *              block scales may then saturate at 448 and codes at +-6.
 *   codes      device, [rows][k/2] bytes, row pitch k/2; 4-byte aligned.
 *   sf         device, nvfp4_sf_bytes(rows, k) bytes, 16-byte aligned; every
 *              byte is written (padding = 0).
 *   global_out device FP32 scalar: receives g. May equal global_in.
 *   workspace  device scratch of >= nvfp4_quantize_workspace_bytes(rows,k)
 *              bytes, 16-byte aligned (dynamic mode only; may be NULL in
 *              static mode). Contents need no initialisation.
 * Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED (k % 16), CUDA (launch).
 */
#define NVFP4_ONE_PASS_MAX_BYTES 65536
nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t k, int64_t ldx,
                            const float* global_in, uint8_t* codes, uint8_t* sf,
                            float* global_out, void* workspace,
                            size_t workspace_bytes, nvfp4_stream_t stream);

/*
 * nvfp4_quantize_noalloc — nvfp4_quantize for callers that cannot allocate
 * device memory. The paper has no counterpart of this entry point; it exists
 * for integration only. Some callers are handed nothing but their input and
 * output buffers and may not call cudaMalloc themselves: a plugin running
 * inside another framework whose allocator owns all device memory, or a
 * runtime that forbids cudaMalloc after start-up because the call can
 * synchronise the whole device and break its latency budget. This variant
 * takes no workspace: the per-CTA partial maxima of the amax pass live in a
 * file-scope device array of NVFP4_NOALLOC_MAX_PARTIALS floats (4 KiB) that
 * every GPU which loads the library holds until the process exits.
 *
 * Arguments, layouts, results and errors are those of nvfp4_quantize (minus
 * the workspace pair). Additionally:
 *   - NVFP4_ERR_UNSUPPORTED if the amax pass would need more than
 *     NVFP4_NOALLOC_MAX_PARTIALS CTAs. It launches one CTA per 16384
 *     elements (256-thread CTAs) for x of at most 16 MiB, so at most 512,
 *     and for larger x one resident wave of 1024-thread CTAs (SM count x
 *     resident CTAs per SM, from an occupancy query: 296 on a 148-SM B200);
 *     the bound is checked on every call, so a device or build with a
 *     larger wave gets this error, never an overrun.
 *   - The first call in a CUDA context looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture. The library keys the address on the
 *     context's unique id, so after a device reset (which reloads the module,
 *     possibly at another address) the next call looks it up again; that
 *     call, too, should come before any capture. Other calls allocate
 *     nothing and call no allocating routine.
 *   - Every call on a device shares the one array and it keeps the last
 *     call's contents. Nothing in it needs to start at zero: each slot the
 *     quantizer reads is first written by the same call's amax pass. Calls
 *     whose kernels overlap on the GPU (e.g. on two concurrently running
 *     streams of one device) race on the array and may produce wrong scales;
 *     serialise them.
 */
#define NVFP4_NOALLOC_MAX_PARTIALS 1024
nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t k,
                                    int64_t ldx, const float* global_in,
                                    uint8_t* codes, uint8_t* sf,
                                    float* global_out, nvfp4_stream_t stream);

/*
 * nvfp4_calibrate_global — one step of static (calibrated) global-scale
 * calibration: the pages calibrate activation scales offline on a frozen set
 * of 128 samples x 32K tokens (news §03, reading §4.1) and then serve with
 * those fixed scales. Folds one calibration batch into a running maximum and
 * writes the global scale that the running maximum implies:
 *   *running_amax = max(*running_amax, max |x|);
 *   *global_out   = 2688 / *running_amax (1 if that is 0 or not finite).
 * Start with *running_amax = 0; pass *global_out as nvfp4_quantize's
 * global_in (static mode) afterwards.
 *   x, rows, k, ldx, workspace, workspace_bytes: as nvfp4_quantize (dynamic).
 *   running_amax, global_out: device FP32 scalars (4-byte aligned).
 * Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED (k % 16), CUDA.
 */
nvfp4_status nvfp4_calibrate_global(const void* x, int64_t rows, int64_t k,
                                    int64_t ldx, float* running_amax,
                                    float* global_out, void* workspace,
                                    size_t workspace_bytes,
                                    nvfp4_stream_t stream);

/* Workspace bytes nvfp4_gemm can use. It starts with the split GEMMs'
 * reduction counters: 4 * max(4*ceil(n/128), 64*16) bytes rounded up to 256,
 * a region that depends on n only. Then:
 *   m <= 64: ceil(n/128)*9*m*128*4 bytes of FP32 partial slabs. With fewer
 *     128-row weight tiles than SMs, few-token GEMMs deal the (tile,
 *     k-tile) iterations out to every SM in equal contiguous shares
 *     (stream-K) and add the partial tiles in a fixed order.
 *   m > 64 with at most 64 tiles of 256x256 and k >= 8192: tiles*S*256 KiB
 *     of FP32 partial tiles, S = min(4, k/4096): when the tiles cannot
 *     occupy half the CTA pairs, K is cut into up to S slices (split-K, at
 *     least 16 k-tiles of 256 each) and the last slice of each tile region
 *     adds the partials in slice order.
 *   otherwise 0.
 * Passing less (or NULL) is allowed and only disables the split. */
size_t nvfp4_gemm_workspace_bytes(int64_t m, int64_t n, int64_t k);

/*
 * nvfp4_gemm — W4A4 block-scaled GEMM on the 4-bit tensor cores (news §02:
 * "hardware-native 4-bit tensor cores"):
 *   Y[i][j] = (1 / (g_a * g_b)) * sum_k val(A)[i][k]*dec(sfA)[i][k/16]
 *                                      * val(B)[j][k]*dec(sfB)[j][k/16]
 * i.e. Y = dequant(A) @ dequant(B)^T, accumulated in FP32.
 *
 *   a_codes, a_sf, a_global  A = activations, [m][k] NVFP4 as nvfp4_quantize
 *                            writes it; a_global is a device FP32 scalar.
 *   b_codes, b_sf, b_global  B = weights, [n][k] NVFP4 (row j = output j).
 *   y        device, [m][ldy] of bf16 (y_dtype 0) or fp32 (y_dtype 1);
 *            16-byte aligned; ldy >= n; ldy*elem % 16 == 0.
 *   m, n     >= 1.   k: k % 32 == 0 (TMA row pitch k/2 must be a multiple of
 *            16 bytes) and k >= 32.
 *   a_codes, b_codes: 16-byte aligned. a_sf, b_sf: 16-byte aligned.
 *   workspace  device scratch, nvfp4_gemm_workspace_bytes(m,n,k) bytes,
 *              16-byte aligned, or NULL; contents need no initialisation
 *              (the call zeroes the reduction counters itself).
 * m <= 64 runs the few-token kernel (weights on the MMA's 128-row side,
 * tokens as its N); larger m the paired-CTA 256x256-tile kernel. Results do
 * not depend on the run: partial tiles are summed in k order (a workspace
 * too small for the split gives the unsplit kernel's k order instead).
 * The kernel is launched with programmatic stream serialisation; it reads and
 * writes global memory only after the previous kernel in the stream finished.
 * Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED, CUDA.
 */
nvfp4_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_sf,
                        const float* a_global, const uint8_t* b_codes,
                        const uint8_t* b_sf, const float* b_global, void* y,
                        int y_dtype, int64_t ldy, int64_t m, int64_t n,
                        int64_t k, void* workspace, size_t workspace_bytes,
                        nvfp4_stream_t stream);

/* Workspace bytes of nvfp4_linear: the split GEMMs' reduction counters (the
 * n-only region nvfp4_gemm_workspace_bytes starts with, always present) and
 * their partials where nvfp4_gemm would split, then the quantized
 * activations (codes, scales, global) and the amax pass's partial maxima.
 * 0 for invalid sizes. */
size_t nvfp4_linear_workspace_bytes(int64_t m, int64_t n, int64_t k);

/*
 * nvfp4_linear — the W4A4 linear layer in one call (news §02: activations are
 * quantized to NVFP4 on the fly and multiplied with NVFP4 weights on the
 * 4-bit tensor cores): Y = dequant(quantize(X)) @ dequant(W)^T, i.e.
 * nvfp4_quantize of X into the workspace followed by nvfp4_gemm, with
 * identical results. The GEMM is launched to start while the quantizer runs:
 * its set-up and its first weight tiles overlap the quantization. For at
 * most NVFP4_LINEAR_IN_KERNEL_MAX_TOKENS (8) tokens there is no quantizer
 * kernel: the few-token GEMM quantizes
 * each k-tile of X as it lands in shared memory (same arithmetic, same
 * bits), after an amax pass only when the global is dynamic and X exceeds
 * NVFP4_ONE_PASS_MAX_BYTES. This relies on W, w_sf and w_global being
 * written before the call (by work already in the stream or earlier), never
 * by a kernel launched in between.
 *   x         device bf16 [m][ldx], 16-byte aligned, ldx >= k, ldx % 8 == 0.
 *   x_global  NULL: dynamic global scale of X (amax pass, or none for X of at
 *             most NVFP4_ONE_PASS_MAX_BYTES, as in nvfp4_quantize); else a
 *             device FP32 static global (e.g. from nvfp4_calibrate_global).
 *   w_codes, w_sf, w_global  weights [n][k] in NVFP4 (as nvfp4_gemm's B).
 *   y, y_dtype, ldy          as nvfp4_gemm.
 *   m, n >= 1; k % 32 == 0.
 *   workspace  device scratch of nvfp4_linear_workspace_bytes(m,n,k) bytes,
 *              256-byte aligned, owned by the caller, not shared with a call
 *              that may run at the same time, and zero-filled before its
 *              first use: each call leaves the bytes that must start at zero
 *              (the counters at its start) zeroed again (after a kernel
 *              timeout, zero it again). One workspace may serve calls with
 *              the same n and different m (and k) if it is large enough for
 *              each: the counters region depends on n only. For 9 to 31
 *              tokens the scales of the quantized X's padding rows are not
 *              written (only this call's GEMM reads them, against zero
 *              codes); for at most 8 the quantized X is not stored at all.
 * Errors: INVALID_ARG (null pointer, bad size, short workspace), MISALIGNED,
 * UNSUPPORTED (k % 32 != 0, sizes >= 2^31), CUDA.
 */
#define NVFP4_LINEAR_IN_KERNEL_MAX_TOKENS 8
nvfp4_status nvfp4_linear(const void* x, int64_t m, int64_t k, int64_t ldx,
                          const float* x_global, const uint8_t* w_codes,
                          const uint8_t* w_sf, const float* w_global, int64_t n,
                          void* y, int y_dtype, int64_t ldy, void* workspace,
                          size_t workspace_bytes, nvfp4_stream_t stream);

/*
 * nvfp4_gemm_swiglu_quant — gate_up projection of a W4A4 gated MLP with the
 * activation and the next layer's activation quantization fused into the
 * GEMM epilogue. Every linear layer of the recipe is W4A4 (news §03), so the
 * MLP's hidden state h = silu(gate) * up is quantized right away for the down
 * projection; here it never goes to memory in bf16. Computes, bit for bit,
 *   Y  = nvfp4_gemm(A, B) in bf16 (gate and up halves),
 *   h  = nvfp4_silu_mul(Y),
 *   (h_codes, h_sf) = nvfp4_quantize(h, global_in = h_global)   [static]
 * without writing Y or h.
 *   A       activations [m][k] NVFP4 (codes, sf, global) as for nvfp4_gemm.
 *   B       gate_up weights [2*ffn][k] NVFP4 with rows interleaved in blocks
 *           of 128: rows [256b, 256b+128) = gate rows [128b, 128b+128),
 *           rows [256b+128, 256b+256) = up rows [128b, 128b+128).
 *   h_global  device FP32 static global of h (e.g. from
 *           nvfp4_calibrate_global over calibration batches of h).
 *   h_codes device [m][ffn/2] bytes, 16-byte aligned.
 *   h_sf    device nvfp4_sf_bytes(m, ffn) bytes, 16-byte aligned; every byte
 *           is written.
 *   ffn % 128 == 0, k % 32 == 0.
 * Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED, CUDA.
 */
nvfp4_status nvfp4_gemm_swiglu_quant(const uint8_t* a_codes, const uint8_t* a_sf,
                                     const float* a_global,
                                     const uint8_t* b_codes, const uint8_t* b_sf,
                                     const float* b_global, const float* h_global,
                                     uint8_t* h_codes, uint8_t* h_sf, int64_t m,
                                     int64_t ffn, int64_t k,
                                     nvfp4_stream_t stream);

/* Workspace bytes of nvfp4_gemm_swiglu_quant_dynamic: bf16 h [m][ffn]
 * (256-byte padded) and one partial maximum per GEMM CTA. 0 for bad sizes. */
size_t nvfp4_gemm_swiglu_quant_dynamic_workspace_bytes(int64_t m, int64_t ffn);

/*
 * nvfp4_gemm_swiglu_quant_dynamic — as nvfp4_gemm_swiglu_quant, but h is
 * quantized with its own dynamic global (g_h = 2688 / max|h| over the whole
 * [m][ffn] tensor, as nvfp4_quantize derives it), so no calibration is
 * needed: the W4A4 MLP of the recipe (news §03: every linear layer NVFP4)
 * with the activation quantized on the fly like any other. A global over
 * the whole of h is only known once all of h exists, so h is written once in
 * bf16 (to the workspace) by the GEMM epilogue, which also records max|h| per
 * CTA; the quantizer then reduces those maxima to g_h exactly as it reduces
 * an amax pass's and quantizes h (no separate amax pass over h, no bf16
 * gate/up output). Computes, bit for bit,
 *   Y  = nvfp4_gemm(A, B) in bf16 (gate and up halves),
 *   h  = nvfp4_silu_mul(Y),
 *   (h_codes, h_sf, h_global_out) = nvfp4_quantize(h)   [dynamic global]
 * with two launches (GEMM, quantizer) on `stream`.
 *   A, B       as nvfp4_gemm_swiglu_quant (B rows interleaved in blocks of 128).
 *   h_codes    device [m][ffn/2] bytes, 16-byte aligned.
 *   h_sf       device nvfp4_sf_bytes(m, ffn) bytes, 16-byte aligned.
 *   h_global_out  device FP32 scalar: receives g_h.
 *   workspace  device scratch of at least
 *              nvfp4_gemm_swiglu_quant_dynamic_workspace_bytes(m, ffn) bytes,
 *              256-byte aligned, caller-owned, no initialisation needed; after
 *              the call its first m*ffn*2 bytes hold h in bf16 (row-major,
 *              leading dimension ffn).
 *   ffn % 128 == 0, k % 32 == 0.
 * Errors: INVALID_ARG (null pointer, bad size, short workspace), MISALIGNED,
 * UNSUPPORTED (ffn % 128, k % 32, sizes >= 2^31), CUDA.
 */
nvfp4_status nvfp4_gemm_swiglu_quant_dynamic(const uint8_t* a_codes, const uint8_t* a_sf,
                                             const float* a_global, const uint8_t* b_codes,
                                             const uint8_t* b_sf, const float* b_global,
                                             uint8_t* h_codes, uint8_t* h_sf,
                                             float* h_global_out, int64_t m, int64_t ffn,
                                             int64_t k, void* workspace,
                                             size_t workspace_bytes, nvfp4_stream_t stream);

/*
 * nvfp4_fuse_group_scales — global-scale repair of a fused module group
 * (news §03: a serving kernel fuses several GDN linear layers into one GEMM;
 * taking the group's largest global scale without rescaling the block scales
 * distorts the weights, so the group is brought onto one global scale and the
 * ratio folded into the E4M3 block scales; abstract: "global-scale mismatch").
 *
 *   g*   = min_i g_i  (the global of the module with the largest amax, i.e.
 *          the global the concatenated tensor would get; every ratio <= 1 so
 *          no block scale can saturate).
 *   r_i  = g* / g_i (FP32 RN);  s' = E4M3_rne_satfinite(dec(s) * r_i) (FP32 RN
 *          multiply);  codes are unchanged.
 * Out of place: module i's scale factors, as nvfp4_quantize wrote them for its
 * own [rows_i][k] tensor, are rescaled and written into the swizzled layout
 * of the row-concatenated [sum rows_i][k] tensor (modules in argument order;
 * atoms shared by two modules are filled from both; padding = 0). The codes
 * of the concatenated tensor are simply the modules' code rows back to back
 * (quantize module i straight into the fused code buffer at row offset
 * sum_{j<i} rows_j).
 *
 *   n_modules        1..16.
 *   rows_per_module  HOST array [n_modules], each >= 1.
 *   k                > 0, k % 16 == 0 (common to all modules).
 *   sf_modules       HOST array [n_modules] of device pointers, each
 *                    nvfp4_sf_bytes(rows_i, k) bytes, 4-byte aligned.
 *   globals_in       device FP32 [n_modules]: the modules' own g_i.
 *   sf_fused         device, nvfp4_sf_bytes(sum rows_i, k) bytes, 16-byte
 *                    aligned; must not overlap any sf_modules buffer.
 *   global_out       device FP32 scalar: receives g*.
 * Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED, CUDA.
 */
nvfp4_status nvfp4_fuse_group_scales(int n_modules,
                                     const int64_t* rows_per_module, int64_t k,
                                     const uint8_t* const* sf_modules,
                                     const float* globals_in, uint8_t* sf_fused,
                                     float* global_out, nvfp4_stream_t stream);

/*
 * nvfp4_silu_mul — the gated-MLP activation between the gate_up and the down
 * projection of a W4A4 MLP (not specified by the pages, which only state that
 * every linear layer is quantized, news §03): h = bf16_rn(silu(gate) * up),
 * silu(z) = z / (1 + exp(-z)), in FP32.
 *   y   device bf16 [m][ldy]; gate = columns [0, n), up = columns [n, 2n).
 *   h   device bf16 [m][ldh].
 *   n % 8 == 0, ldy % 8 == 0, ldh % 8 == 0, both pointers 16-byte aligned.
 * Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED, CUDA.
 */
nvfp4_status nvfp4_silu_mul(const void* y, int64_t m, int64_t n, int64_t ldy,
                            void* h, int64_t ldh, nvfp4_stream_t stream);

/*
 * nvfp4_selftest_gemm_stall — failure-detection self-test of the GEMM
 * kernels themselves (no counterpart on the pages; it exists so that the
 * time-out and abort path of the kernels that do the work can be run on a
 * GPU without a fault). Runs nvfp4_gemm (bf16 Y, ldy = n) with two changes:
 * every wait of the kernel gives up after `limit_ns` instead of 2 s, and
 * the TMA producers issue nothing for the first ring stage, so that stage's
 * barrier never completes. Every role then runs into its limit (or sees the
 * abort another role raised), in-flight copies and tensor-core work are
 * drained, tensor memory is freed and the kernel returns; nvfp4_read_fault
 * then reports NVFP4_ERR_TIMEOUT with the role bits (paired kernel, m > 64:
 * 1 producer, 2 MMA, 4 epilogue, 8 scale copies; few-token kernel, m <= 64:
 * 16, 32, 64, 128). Y is left undefined, and for m <= 64 the workspace's
 * reduction counters must be zeroed again before it is reused (nvfp4_gemm
 * zeroes them itself; nvfp4_linear does not).
 *   Arguments as nvfp4_gemm (y bf16 [m][n]); limit_ns in [1 us, 10 s].
 * Errors: as nvfp4_gemm; INVALID_ARG for limit_ns out of range.
 */
nvfp4_status nvfp4_selftest_gemm_stall(const uint8_t* a_codes, const uint8_t* a_sf,
                                       const float* a_global, const uint8_t* b_codes,
                                       const uint8_t* b_sf, const float* b_global, void* y,
                                       int64_t m, int64_t n, int64_t k, uint64_t limit_ns,
                                       void* workspace, size_t workspace_bytes,
                                       nvfp4_stream_t stream);

/*
 * nvfp4_read_fault — every mbarrier wait in the GEMM kernel is bounded; on
 * expiry the kernel records a nonzero fault word, stops issuing work and
 * returns instead of hanging. This call synchronises `stream`, copies the
 * fault word to *fault_out (0 = none) and clears it. Returns NVFP4_ERR_TIMEOUT
 * if the word was nonzero, else NVFP4_OK (or NVFP4_ERR_CUDA).
 */
nvfp4_status nvfp4_read_fault(nvfp4_stream_t stream, uint32_t* fault_out);

/*
 * nvfp4_selftest_wait_timeout — a diagnostic with no counterpart on the
 * pages: checks on the GPU that a bounded wait gives up. One thread waits,
 * with the same bounded-wait routine as the few-token GEMM's roles, on an
 * mbarrier that nothing arrives at; after limit_ns nanoseconds (global timer)
 * it records bit 256 in the fault word and the kernel returns. A following
 * nvfp4_read_fault reports NVFP4_ERR_TIMEOUT with that bit set; the context
 * stays usable.
 *   limit_ns  1000 .. 10^10 (1 us .. 10 s).
 * Errors: INVALID_ARG (limit out of range), CUDA.
 */
nvfp4_status nvfp4_selftest_wait_timeout(uint64_t limit_ns, nvfp4_stream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* NVFP4_H_ */
