// nvfp4_api.cu — the C ABI of libnvfp4.so (declared in include/nvfp4.h).
//
// One translation unit: it includes every kernel header, validates arguments
// on the host (returning a status before anything is launched), builds the
// TMA descriptors of the GEMM and launches on the caller's stream. Nothing is
// allocated and no call synchronises with the host except nvfp4_read_fault.
// The quantizer's second kernel and the GEMMs are launched with programmatic
// stream serialisation (each kernel waits on the device for its predecessor
// before touching global memory), so a launch and its set-up overlap the
// previous kernel's tail.
#include "nvfp4.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "fold.cuh"
#include "gemm_sm100.cuh"
#include "gemm_skinny.cuh"
#include "quant.cuh"
#include "silu_mul.cuh"

namespace {

constexpr int kMaxDevices = 64;

// What the library caches per device. Everything here belongs to one CUDA
// context: function attributes, occupancy and symbol addresses are properties
// of the module loaded into that context, and a device reset (or any other
// teardown of the primary context) loads the module again, possibly at other
// addresses. The state is therefore keyed on the context's process-unique id
// (cuCtxGetId) and rebuilt when the current context changes. One context per
// device at a time is assumed (the runtime's primary context, as torch and
// most callers use); threads that drive two contexts of one device at once
// would rebuild each other's state.
struct DeviceState {
  unsigned long long ctx_id = 0;      // context the fields below belong to (0 = none yet)
  int sms = 0;
  bool gemm_smem_set = false;
  unsigned skinny_smem_set = 0;       // bit per token-tile instantiation
  int amax_per_sm = 0;                // resident CTAs per SM of the quantizer's kernels
  int quant_per_sm = 0;
  float* noalloc_partials = nullptr;  // device address of g_noalloc_partials in ctx_id
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

nvfp4_status driver_entry(const char* name, int version, void** fn) {
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, fn, version, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || *fn == nullptr) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

// Unique id of the context current on this thread for device `dev`; binds
// the device's primary context first if the runtime has not done so yet on
// this thread (cudaSetDevice initialises it; the device stays the same).
nvfp4_status current_context_id(int dev, unsigned long long* id) {
  static std::once_flag once;
  std::call_once(once, [] {
    void* a = nullptr;
    void* b = nullptr;
    if (driver_entry("cuCtxGetCurrent", 4000, &a) == NVFP4_OK &&
        driver_entry("cuCtxGetId", 12000, &b) == NVFP4_OK) {
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(a);
      g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(b);
    }
  });
  if (g_ctx_current == nullptr || g_ctx_id == nullptr) return NVFP4_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS) return NVFP4_ERR_CUDA;
  if (ctx == nullptr) {
    if (cudaSetDevice(dev) != cudaSuccess) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return NVFP4_ERR_CUDA;
  }
  return g_ctx_id(ctx, id) == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

nvfp4_status current_device(int* dev, DeviceState** st) {
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  unsigned long long id = 0;
  if (nvfp4_status e = current_context_id(*dev, &id)) return e;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& s = g_dev[*dev];
  if (s.ctx_id != id) {  // first call in this context: nothing cached applies
    s = DeviceState{};
    s.ctx_id = id;
  }
  if (s.sms == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess ||
        sms <= 0) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    s.sms = sms;
  }
  *st = &s;
  return NVFP4_OK;
}

nvfp4_status get_encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_encode == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  *fn = g_encode;
  return NVFP4_OK;
}

nvfp4_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

size_t round_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

// Launch with programmatic stream serialisation (and a cluster shape when
// cluster_x > 1). The kernel must call grid_dep_wait() before any access to
// global memory that earlier work in the stream produces or consumes.
template <typename... KArgs, typename... Args>
nvfp4_status launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                        cudaStream_t s, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  std::memset(attr, 0, sizeof attr);
  unsigned na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cluster_x > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cluster_x;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

constexpr int64_t kSplitMaxTiles = 64;  // paired split-K: at most this many 256x256 tiles

// The reduction counters of both split GEMMs sit at the start of a GEMM or
// linear workspace, in a region whose size depends on n only (few-token
// kernel: 4 per 128 weight rows; paired split-K: 16 per tile, at most
// kSplitMaxTiles tiles). Every call leaves them zero and nothing else is
// ever placed there, so one workspace that is large enough for each call
// may serve calls of different m.
size_t split_counter_bytes(int64_t n) {
  int64_t c = ceil_div(n, 128) * 4;
  if (c < kSplitMaxTiles * 16) c = kSplitMaxTiles * 16;
  return round_up(static_cast<size_t>(c) * sizeof(unsigned int), 256);
}

// Few-token GEMM workspace: the counters, then kMaxContrib FP32 slabs of
// [m][128] per weight tile.
size_t skinny_workspace_bytes(int64_t m, int64_t n) {
  return split_counter_bytes(n) + static_cast<size_t>(ceil_div(n, 128)) *
                                      nvfp4::skinny::kMaxContrib * static_cast<size_t>(m) *
                                      nvfp4::skinny::BW * sizeof(float);
}

// Split-K of the paired kernel (nvfp4::gemm, m > 64): when the 256x256 tiles
// cannot occupy half the CTA pairs, the K range is cut into S slices (at most
// kMaxSplitK, each at least kMinSliceKTiles k-tiles) so that tiles x S units
// occupy the pairs; e.g. 20 tiles of a 256-token 17408 -> 5120 layer run as
// 60 units instead of 20. Workspace: counters (16 per tile), then the FP32
// partial tiles. The workspace bytes depend on the shape only (the largest
// S any device could use); the launch picks S from the SM count.
int64_t paired_tiles(int64_t m, int64_t n) {
  return ceil_div(m, nvfp4::gemm::BM) * ceil_div(n, nvfp4::gemm::BN);
}
int paired_split_cap(int64_t m, int64_t n, int64_t k) {
  using namespace nvfp4::gemm;
  const int64_t kt = ceil_div(k, BK);
  if (m <= 64 || paired_tiles(m, n) > kSplitMaxTiles || kt < 2 * kMinSliceKTiles) return 1;
  return static_cast<int>(kt / kMinSliceKTiles < kMaxSplitK ? kt / kMinSliceKTiles : kMaxSplitK);
}
size_t paired_split_bytes(int64_t m, int64_t n, int split) {
  return split_counter_bytes(n) + static_cast<size_t>(paired_tiles(m, n)) *
                                      static_cast<size_t>(split) * 16 *
                                      nvfp4::gemm::kRegionFloats * sizeof(float);
}
int paired_split(int sms, int64_t m, int64_t n, int64_t k) {
  const int cap = paired_split_cap(m, n, k);
  const int64_t by_pairs = (sms / 2) / paired_tiles(m, n);
  return static_cast<int>(by_pairs < cap ? by_pairs : cap);
}

// Stream-K grid of a few-token GEMM: G CTAs sharing the W x KT iterations,
// at most kMaxSplits per weight tile, shrunk until no tile has more than
// kMaxContrib contributing CTAs (each has a slab slot). 0 = no split: whole
// tiles, when they already occupy more than 3/4 of the SMs — the slab write
// and in-order reduction of split tiles cost ~2 us, more than the extra SMs
// bring then (measured: 136 tiles on 148 SMs, 24.2 -> 26.6 us per decode
// step; 40 tiles, 30.8 -> 28.7 us).
int skinny_stream_k_grid(int sms, int64_t w_tiles, int64_t k_tiles) {
  using namespace nvfp4::skinny;
  if (4 * w_tiles > 3 * static_cast<int64_t>(sms)) return 0;
  const int64_t T = w_tiles * k_tiles;
  int64_t G = sms;
  if (G > T) G = T;
  if (G > w_tiles * kMaxSplits) G = w_tiles * kMaxSplits;
  auto owner = [&](int64_t it, int64_t g) { return ((it + 1) * g - 1) / T; };
  for (; G > w_tiles; --G) {
    int64_t worst = 0;
    for (int64_t w = 0; w < w_tiles; ++w) {
      const int64_t c = owner((w + 1) * k_tiles - 1, G) - owner(w * k_tiles, G) + 1;
      if (c > worst) worst = c;
    }
    if (worst <= kMaxContrib) return static_cast<int>(G);
  }
  return 0;
}

// Resident CTAs per SM of the quantizer's two kernels (occupancy query, once
// per device): their grids are capped at one full wave, since a partial
// second wave of these streaming kernels ran with idle SMs.
nvfp4_status quant_occupancy(DeviceState* st) {
  using namespace nvfp4::quant;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (st->amax_per_sm == 0) {
    int a = 0, q = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&a, amax_kernel, kAmaxThreads, 0) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&q, quantize_kernel, kQuantThreads, 0) !=
            cudaSuccess) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    st->amax_per_sm = a < 1 ? 1 : a;
    st->quant_per_sm = q < 1 ? 1 : q;
  }
  return NVFP4_OK;
}

// CTAs of the amax pass: enough that every thread streams ~8 16-byte chunks
// (the contiguous path is flat over elements, the strided one a warp per
// row), at most one resident wave. Sizing by rows alone starved few-row
// inputs.
int64_t amax_blocks(int64_t rows, int64_t k, int64_t ldx, const DeviceState* st,
                    int threads = nvfp4::quant::kAmaxThreads) {
  using namespace nvfp4::quant;
  const int64_t per_block = (ldx == k) ? static_cast<int64_t>(threads) * 8 * 8
                                       : static_cast<int64_t>(threads / 32);
  const int64_t units = (ldx == k) ? rows * k : rows;
  int64_t blocks = ceil_div(units, per_block);
  const int64_t cap = static_cast<int64_t>(st->sms) * st->amax_per_sm *
                      (kAmaxThreads / threads);
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return blocks;
}

// CTA size of the amax pass: small inputs (a decode step's tokens) run in
// 256-thread CTAs, which fit on an SM next to a running few-token GEMM CTA
// (half an SM), so the pass need not wait for that GEMM's CTAs to exit.
constexpr int64_t kSmallAmaxBytes = int64_t{16} << 20;
int amax_threads(int64_t rows, int64_t k) {
  return rows * k * 2 <= kSmallAmaxBytes ? 256 : nvfp4::quant::kAmaxThreads;
}

// Scratch of nvfp4_quantize_noalloc: the amax pass's per-CTA partial maxima.
// Host code must not use this name as a pointer (it is a host-side stand-in);
// the device address comes from cudaGetSymbolAddress, once per device and
// context (current_device() clears the cached address when the context
// changes, e.g. after a device reset).
static __device__ __align__(256) float g_noalloc_partials[NVFP4_NOALLOC_MAX_PARTIALS];

// First call in the current context: look up the array's device address.
nvfp4_status noalloc_scratch(DeviceState* st, float** out) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (st->noalloc_partials == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_partials) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    st->noalloc_partials = static_cast<float*>(p);
  }
  *out = st->noalloc_partials;
  return NVFP4_OK;
}

// The quantizer kernel over a.rows x a.k (arguments checked, occupancy
// known): one resident wave at most, launched to overlap its predecessor.
nvfp4_status quantizer_launch(const nvfp4::quant::QuantArgs& a, DeviceState* st, cudaStream_t s) {
  using namespace nvfp4::quant;
  const int64_t n_kc = ceil_div(ceil_div(a.k, 64), kAtomsPerTask);
  const int64_t n_tasks =
      (a.skip_pad && a.rows < 32) ? a.rows * n_kc : ceil_div(a.rows, 128) * 32 * n_kc;
  int64_t blocks = ceil_div(n_tasks, kQuantThreads / 32);
  const int64_t cap = static_cast<int64_t>(st->sms) * st->quant_per_sm;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return launch_pdl(quantize_kernel, static_cast<unsigned>(blocks), kQuantThreads, 0, s, 1u, a);
}

// Dynamic or static NVFP4 quantization of x (arguments already checked):
// the amax pass (dynamic only, x above kSelfAmaxBytes) into `partials` (at
// most max_parts CTAs), then the quantizer, launched to overlap the amax
// pass's tail; dynamic x up to kSelfAmaxBytes: the quantizer alone.
nvfp4_status quantize_launch(const void* x, int64_t rows, int64_t k, int64_t ldx,
                             const float* global_in, uint8_t* codes, uint8_t* sf,
                             float* global_out, float* partials, int64_t max_parts,
                             DeviceState* st, cudaStream_t s, bool skip_pad = false) {
  using namespace nvfp4::quant;
  const int64_t n_tasks = ceil_div(rows, 128) * 32 * ceil_div(ceil_div(k, 64), kAtomsPerTask);
  if (n_tasks >= (int64_t{1} << 31)) return NVFP4_ERR_UNSUPPORTED;  // 32-bit task index
  if (nvfp4_status e = quant_occupancy(st)) return e;
  static_assert(kSelfAmaxBytes == NVFP4_ONE_PASS_MAX_BYTES, "one-pass bound of nvfp4.h");
  int nparts = 0;  // dynamic mode with nparts == 0: the quantizer takes the max itself
  if (global_in == nullptr && rows * k * 2 > kSelfAmaxBytes) {
    const int threads = amax_threads(rows, k);
    const int64_t blocks = amax_blocks(rows, k, ldx, st, threads);
    if (blocks > max_parts) return NVFP4_ERR_UNSUPPORTED;
    nparts = static_cast<int>(blocks);
    amax_kernel<<<nparts, threads, 0, s>>>(static_cast<const uint16_t*>(x), rows, k, ldx,
                                           partials);
    if (nvfp4_status e = launch_status()) return e;
  }
  QuantArgs a;
  a.x = static_cast<const uint16_t*>(x);
  a.rows = rows;
  a.k = k;
  a.ldx = ldx;
  a.global_in = global_in;
  a.partials = partials;
  a.nparts = nparts;
  a.codes = codes;
  a.sf = sf;
  a.global_out = global_out;
  a.skip_pad = skip_pad ? 1 : 0;
  return quantizer_launch(a, st, s);
}

}  // namespace

extern "C" {

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
    case NVFP4_ERR_UNSUPPORTED: return "NVFP4_ERR_UNSUPPORTED";
    case NVFP4_ERR_MISALIGNED: return "NVFP4_ERR_MISALIGNED";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
    case NVFP4_ERR_TIMEOUT: return "NVFP4_ERR_TIMEOUT";
  }
  return "NVFP4_ERR_UNKNOWN";
}

size_t nvfp4_sf_bytes(int64_t rows, int64_t k) {
  if (rows < 0 || k <= 0 || k % 16 != 0) return 0;
  return static_cast<size_t>(ceil_div(rows, 128) * 128) * static_cast<size_t>(ceil_div(k, 64) * 4);
}

size_t nvfp4_quantize_workspace_bytes(int64_t rows, int64_t k) {
  (void)rows;
  (void)k;
  return static_cast<size_t>(nvfp4::quant::kMaxPartials) * sizeof(float);
}

nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t k, int64_t ldx,
                            const float* global_in, uint8_t* codes, uint8_t* sf,
                            float* global_out, void* workspace, size_t workspace_bytes,
                            nvfp4_stream_t stream) {
  using namespace nvfp4::quant;
  if (rows < 0 || k <= 0 || global_out == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (k % 16 != 0) return NVFP4_ERR_UNSUPPORTED;
  if (rows > 0 && (x == nullptr || codes == nullptr || sf == nullptr)) return NVFP4_ERR_INVALID_ARG;
  if (ldx < k) return NVFP4_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || !aligned(x, 16) || !aligned(codes, 4) || !aligned(sf, 16) ||
      !aligned(global_out, 4))
    return NVFP4_ERR_MISALIGNED;
  const bool dynamic = (global_in == nullptr);
  if (dynamic) {
    if (workspace == nullptr || workspace_bytes < nvfp4_quantize_workspace_bytes(rows, k))
      return NVFP4_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return NVFP4_ERR_MISALIGNED;
  }
  int dev;
  DeviceState* st;
  if (nvfp4_status e = current_device(&dev, &st)) return e;
  return quantize_launch(x, rows, k, ldx, global_in, codes, sf, global_out,
                         static_cast<float*>(workspace), kMaxPartials, st,
                         reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t k, int64_t ldx,
                                    const float* global_in, uint8_t* codes, uint8_t* sf,
                                    float* global_out, nvfp4_stream_t stream) {
  using namespace nvfp4::quant;
  if (rows < 0 || k <= 0 || global_out == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (k % 16 != 0) return NVFP4_ERR_UNSUPPORTED;
  if (rows > 0 && (x == nullptr || codes == nullptr || sf == nullptr)) return NVFP4_ERR_INVALID_ARG;
  if (ldx < k) return NVFP4_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || !aligned(x, 16) || !aligned(codes, 4) || !aligned(sf, 16) ||
      !aligned(global_out, 4))
    return NVFP4_ERR_MISALIGNED;
  int dev;
  DeviceState* st;
  if (nvfp4_status e = current_device(&dev, &st)) return e;
  float* partials = nullptr;
  if (nvfp4_status e = noalloc_scratch(st, &partials)) return e;
  return quantize_launch(x, rows, k, ldx, global_in, codes, sf, global_out, partials,
                         NVFP4_NOALLOC_MAX_PARTIALS, st, reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_calibrate_global(const void* x, int64_t rows, int64_t k, int64_t ldx,
                                    float* running_amax, float* global_out, void* workspace,
                                    size_t workspace_bytes, nvfp4_stream_t stream) {
  using namespace nvfp4::quant;
  if (rows < 0 || k <= 0 || running_amax == nullptr || global_out == nullptr || ldx < k)
    return NVFP4_ERR_INVALID_ARG;
  if (k % 16 != 0) return NVFP4_ERR_UNSUPPORTED;
  if (rows > 0 && x == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < nvfp4_quantize_workspace_bytes(rows, k))
    return NVFP4_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || !aligned(x, 16) || !aligned(workspace, 16) || !aligned(running_amax, 4) ||
      !aligned(global_out, 4))
    return NVFP4_ERR_MISALIGNED;
  int dev;
  DeviceState* st;
  if (nvfp4_status e = current_device(&dev, &st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (nvfp4_status e = quant_occupancy(st)) return e;
  int64_t blocks = amax_blocks(rows, k, ldx, st);
  if (blocks > kMaxPartials) blocks = kMaxPartials;
  amax_kernel<<<static_cast<unsigned>(blocks), kAmaxThreads, 0, s>>>(
      static_cast<const uint16_t*>(x), rows, k, ldx, static_cast<float*>(workspace));
  if (nvfp4_status e = launch_status()) return e;
  calibrate_kernel<<<1, 256, 0, s>>>(static_cast<const float*>(workspace),
                                     static_cast<int>(blocks), running_amax, global_out);
  return launch_status();
}

size_t nvfp4_gemm_workspace_bytes(int64_t m, int64_t n, int64_t k) {
  if (m < 1 || n < 1 || k < 1) return 0;
  // few-token GEMMs share the work stream-K fashion: counters and FP32 slabs
  if (m <= 64) return skinny_workspace_bytes(m, n);
  // paired kernel with few tiles: split-K counters and FP32 partial tiles
  const int cap = paired_split_cap(m, n, k);
  return cap >= 2 ? paired_split_bytes(m, n, cap) : 0;
}

}  // extern "C"

namespace {

nvfp4_status encode_2d(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, const void* base,
                       uint64_t inner_bytes, uint64_t rows, uint32_t box_rows) {
  cuuint64_t dims[2] = {inner_bytes, rows};
  cuuint64_t strides[1] = {inner_bytes};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Output for TMA stores: [m][ldy] of bf16 / fp32, boxes of 32 rows x 64 bytes
// with the 64-byte swizzle the epilogue's staging tiles use.
nvfp4_status encode_y(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, void* base,
                      int64_t m, int64_t n, int64_t ldy, int y_dtype) {
  const uint64_t esize = y_dtype == 0 ? 2u : 4u;
  cuuint64_t dims[2] = {static_cast<uint64_t>(n), static_cast<uint64_t>(m)};
  cuuint64_t strides[1] = {static_cast<uint64_t>(ldy) * esize};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(64u / esize), 32u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, y_dtype == 0 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                   2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Scale factors as [row blocks][atoms][128 x uint32]: one box = whole atoms.
nvfp4_status encode_sf(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, const void* base,
                       int64_t rows, int64_t k, uint32_t box_row_blocks) {
  const uint64_t n_ka = static_cast<uint64_t>(ceil_div(k, 64));
  const uint64_t n_rb = static_cast<uint64_t>(ceil_div(rows, 128));
  cuuint64_t dims[3] = {128u, n_ka, n_rb};
  cuuint64_t strides[2] = {512u, n_ka * 512u};
  cuuint32_t box[3] = {128u, 4u, box_row_blocks};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

template <int BNT, bool FUSED>
nvfp4_status launch_skinny(DeviceState* st, int bit, const CUtensorMap& tmW, const CUtensorMap& tmX,
                           const CUtensorMap& tmSFW, const CUtensorMap& tmSFX,
                           const nvfp4::skinny::Params& p, int grid, cudaStream_t s) {
  using C = nvfp4::skinny::Cfg<BNT, FUSED>;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!(st->skinny_smem_set & (1u << bit))) {
      if (cudaFuncSetAttribute(nvfp4::skinny::skinny_kernel<BNT, FUSED>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(C::SMEM_BYTES)) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
      }
      st->skinny_smem_set |= 1u << bit;
    }
  }
  return launch_pdl(nvfp4::skinny::skinny_kernel<BNT, FUSED>, static_cast<unsigned>(grid),
                    C::THREADS, C::SMEM_BYTES, s, 1u, tmW, tmX, tmSFW, tmSFX, p);
}

// Tokens quantized inside the few-token GEMM (nvfp4_linear, m <= XR = 8): the
// bf16 X, and where its global comes from (static, amax partials, or the
// kernel's own max over X of at most kSelfAmaxBytes).
struct XFused {
  const void* x;
  int64_t ldx;
  const float* global_in;
  const float* partials;
  int nparts;
  float* global_out;
};

// Few tokens (m <= 64): Y^T = B A^T with the weights on the MMA's 128-row
// side and the tokens as its N; stream-K across all SMs when the weight tiles
// cannot fill the GPU and a workspace (skinny_workspace_bytes) is given.
// The reduction counters at the workspace's start are zeroed here when
// `zero_counters`, else the caller guarantees they are zero (every call
// leaves them so). `early_w`: the weights were written before the previous
// kernel in the stream started, so the kernel may read them before it ends.
nvfp4_status gemm_skinny(PFN_cuTensorMapEncodeTiled_v12000 enc, DeviceState* st,
                         const uint8_t* a_codes, const uint8_t* a_sf, const float* a_global,
                         const uint8_t* b_codes, const uint8_t* b_sf, const float* b_global,
                         void* y, int y_dtype, int64_t ldy, int64_t m, int64_t n, int64_t k,
                         void* workspace, size_t workspace_bytes, bool zero_counters,
                         int early_w, cudaStream_t s, int stall = 0, uint64_t limit_ns = 0,
                         const XFused* xf = nullptr) {
  using namespace nvfp4::skinny;
  const int bnt = m <= 16 ? 16 : m <= 32 ? 32 : 64;  // callers route m <= 64 here
  if (xf != nullptr && m > XR) return NVFP4_ERR_UNSUPPORTED;
  CUtensorMap tmW, tmX, tmSFW, tmSFX;
  if (nvfp4_status e = encode_2d(enc, &tmW, b_codes, static_cast<uint64_t>(k / 2),
                                 static_cast<uint64_t>(n), BW))
    return e;
  if (nvfp4_status e = encode_sf(enc, &tmSFW, b_sf, n, k, 1u)) return e;
  if (xf != nullptr) {
    // bf16 token tiles of [XR][256] (rows past m and columns past k zero-filled)
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(m)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(xf->ldx) * 2u};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(XR)};
    cuuint32_t estr[2] = {1u, 1u};
    if (enc(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(xf->x), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return NVFP4_ERR_CUDA;
    tmSFX = tmSFW;  // not read in this mode
  } else {
    if (nvfp4_status e = encode_2d(enc, &tmX, a_codes, static_cast<uint64_t>(k / 2),
                                   static_cast<uint64_t>(m), static_cast<uint32_t>(bnt)))
      return e;
    if (nvfp4_status e = encode_sf(enc, &tmSFX, a_sf, m, k, 1u)) return e;
  }
  Params p;
  std::memset(&p, 0, sizeof p);
  if (xf != nullptr) {
    p.x = static_cast<const uint16_t*>(xf->x);
    p.ldx = xf->ldx;
    p.x_global_in = xf->global_in;
    p.x_partials = xf->partials;
    p.x_nparts = xf->nparts;
    p.x_global_out = xf->global_out;
  }
  p.M = static_cast<int>(m);
  p.N = static_cast<int>(n);
  p.K = static_cast<int>(k);
  p.num_w_tiles = static_cast<int>(ceil_div(n, BW));
  p.num_k_tiles = static_cast<int>(ceil_div(k, BK));
  p.a_global = a_global;
  p.b_global = b_global;
  p.y = y;
  p.ldy = ldy;
  p.y_fp32 = y_dtype;
  p.partial = nullptr;
  p.tile_count = nullptr;
  p.early_w = early_w;
  p.stream_k = 0;
  p.stall_first_stage = stall;
  p.wait_limit_ns = limit_ns;
  int grid = static_cast<int>(p.num_w_tiles < st->sms ? p.num_w_tiles : st->sms);
  const bool split_ok = workspace != nullptr &&
                        workspace_bytes >= skinny_workspace_bytes(m, n) && aligned(workspace, 16);
  if (split_ok) {
    const int g = skinny_stream_k_grid(st->sms, p.num_w_tiles, p.num_k_tiles);
    if (g > 0) {
      p.stream_k = 1;
      grid = g;
      p.tile_count = static_cast<unsigned int*>(workspace);
      p.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                           split_counter_bytes(n));
      if (zero_counters &&
          cudaMemsetAsync(workspace, 0, split_counter_bytes(n), s) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
      }
    }
  }
  nvfp4_status e;
  if (xf != nullptr) {
    return launch_skinny<16, true>(st, 3, tmW, tmX, tmSFW, tmSFX, p, grid, s);
  }
  switch (bnt) {
    case 16: e = launch_skinny<16, false>(st, 0, tmW, tmX, tmSFW, tmSFX, p, grid, s); break;
    case 32: e = launch_skinny<32, false>(st, 1, tmW, tmX, tmSFW, tmSFX, p, grid, s); break;
    default: e = launch_skinny<64, false>(st, 2, tmW, tmX, tmSFW, tmSFX, p, grid, s); break;
  }
  return e;
}

// The paired-CTA kernel (cta_group::2, 256x256 tiles): M, N, K, tile counts
// and tensor maps filled in here; output / fused fields come in `p`.
// Split-K (plain mode) when `workspace` holds at least paired_split_bytes for
// the S this device uses; its counters are zeroed here when `zero_counters`,
// else the caller guarantees they are zero (every call leaves them so).
nvfp4_status gemm_paired(PFN_cuTensorMapEncodeTiled_v12000 enc, DeviceState* st,
                         const uint8_t* a_codes, const uint8_t* a_sf, const uint8_t* b_codes,
                         const uint8_t* b_sf, int64_t m, int64_t n, int64_t k,
                         nvfp4::gemm::Params p, cudaStream_t stream, int* grid_out = nullptr,
                         void* workspace = nullptr, size_t workspace_bytes = 0,
                         bool zero_counters = true) {
  using namespace nvfp4::gemm;
  CUtensorMap tmA, tmB, tmSFA, tmSFB, tmY;
  std::memset(&tmY, 0, sizeof tmY);
  if (nvfp4_status e = encode_2d(enc, &tmA, a_codes, static_cast<uint64_t>(k / 2),
                                 static_cast<uint64_t>(m), HALF))
    return e;
  if (nvfp4_status e = encode_2d(enc, &tmB, b_codes, static_cast<uint64_t>(k / 2),
                                 static_cast<uint64_t>(n), HALF))
    return e;
  if (nvfp4_status e = encode_sf(enc, &tmSFA, a_sf, m, k, 1u)) return e;
  if (nvfp4_status e = encode_sf(enc, &tmSFB, b_sf, n, k, 2u)) return e;
  if (p.fused == kPlain) {
    if (nvfp4_status e = encode_y(enc, &tmY, p.y, m, n, p.ldy, p.y_fp32)) return e;
  } else if (p.fused == kFusedBf16Amax) {  // bf16 h = [m][n / 2]
    if (nvfp4_status e = encode_y(enc, &tmY, p.y, m, n / 2, p.ldy, 0)) return e;
  }
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!st->gemm_smem_set) {
      if (cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(SMEM_BYTES)) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
      }
      st->gemm_smem_set = true;
    }
  }
  p.M = static_cast<int>(m);
  p.N = static_cast<int>(n);
  p.K = static_cast<int>(k);
  p.num_m_blk = static_cast<int>(ceil_div(m, BM));
  p.num_n_blk = static_cast<int>(ceil_div(n, BN));
  p.num_k_tiles = static_cast<int>(ceil_div(k, BK));
  const int64_t tiles = static_cast<int64_t>(p.num_m_blk) * p.num_n_blk;
  if (tiles >= (int64_t{1} << 31)) return NVFP4_ERR_UNSUPPORTED;
  p.split = 1;
  if (p.fused == kPlain && workspace != nullptr && aligned(workspace, 16)) {
    const int sk = paired_split(st->sms, m, n, k);
    if (sk >= 2 && workspace_bytes >= paired_split_bytes(m, n, sk)) {
      p.split = sk;
      p.tile_count = static_cast<unsigned int*>(workspace);
      p.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                           split_counter_bytes(n));
      if (zero_counters &&
          cudaMemsetAsync(workspace, 0, split_counter_bytes(n), stream) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
      }
    }
  }
  // Band rasterization (tile_coords): the band's tiles of one operand stay
  // in L2 while the other operand streams past once per band. The band is
  // sized to kL2BandBytes, and the direction with the smaller estimated DRAM
  // read traffic (the streamed operand once per band, the banded one once)
  // is chosen. Measured: bands of 48 MB did not stay in L2 (the 32768 x
  // 34816 x 5120 gate_up read 1.38 GB, the down projection 1.21 GB); the
  // h / Y output traffic and the two dies' halves of L2 leave about half of
  // the 126 MB to a band.
  {
    const int64_t kL2BandBytes = int64_t{24} << 20;
    const int64_t a_bytes = m * (k / 2), b_bytes = n * (k / 2);
    const int64_t tile_bytes = int64_t{BM} * (k / 2);  // one M- or N-tile of A or B
    int64_t gm = kL2BandBytes / tile_bytes, gn = gm;
    if (gm < 1) gm = gn = 1;
    if (gm > p.num_m_blk) gm = p.num_m_blk;
    if (gn > p.num_n_blk) gn = p.num_n_blk;
    const int64_t traffic_m = a_bytes + b_bytes * ceil_div(p.num_m_blk, gm);
    const int64_t traffic_n = b_bytes + a_bytes * ceil_div(p.num_n_blk, gn);
    p.raster_n = traffic_n < traffic_m ? 1 : 0;
    p.group = static_cast<int>(p.raster_n ? gn : gm);
  }
  const int64_t units = tiles * p.split;
  // one CTA pair (cluster of 2 SMs) per 256x256 work unit at a time, persistent
  const int64_t max_pairs = st->sms / 2;
  const int pairs = static_cast<int>(units < max_pairs ? units : max_pairs);
  if (grid_out != nullptr) *grid_out = 2 * pairs;
  return launch_pdl(gemm_kernel, static_cast<unsigned>(2 * pairs), NUM_THREADS, SMEM_BYTES,
                    stream, 2u, tmA, tmB, tmSFA, tmSFB, tmY, p);
}

// nvfp4_gemm; `stall` / `limit_ns` only for nvfp4_selftest_gemm_stall.
nvfp4_status gemm_entry(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_global,
                        const uint8_t* b_codes, const uint8_t* b_sf, const float* b_global,
                        void* y, int y_dtype, int64_t ldy, int64_t m, int64_t n, int64_t k,
                        void* workspace, size_t workspace_bytes, nvfp4_stream_t stream,
                        int stall, uint64_t limit_ns) {
  using namespace nvfp4::gemm;
  if (!a_codes || !a_sf || !a_global || !b_codes || !b_sf || !b_global || !y)
    return NVFP4_ERR_INVALID_ARG;
  if (m < 1 || n < 1 || k < 1 || (y_dtype != 0 && y_dtype != 1) || ldy < n)
    return NVFP4_ERR_INVALID_ARG;
  if (k % 32 != 0 || m >= (int64_t{1} << 31) || n >= (int64_t{1} << 31) ||
      k >= (int64_t{1} << 31))
    return NVFP4_ERR_UNSUPPORTED;
  const int64_t esize = y_dtype == 0 ? 2 : 4;
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_sf, 16) || !aligned(b_sf, 16) ||
      !aligned(y, 16) || (ldy * esize) % 16 != 0 || !aligned(a_global, 4) || !aligned(b_global, 4))
    return NVFP4_ERR_MISALIGNED;
  int dev;
  DeviceState* st;
  if (nvfp4_status e = current_device(&dev, &st)) return e;
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (nvfp4_status e = get_encoder(&enc)) return e;
  if (m <= 64)
    return gemm_skinny(enc, st, a_codes, a_sf, a_global, b_codes, b_sf, b_global, y, y_dtype, ldy,
                       m, n, k, workspace, workspace_bytes, true, 0,
                       reinterpret_cast<cudaStream_t>(stream), stall, limit_ns);

  nvfp4::gemm::Params p;
  std::memset(&p, 0, sizeof p);
  p.a_global = a_global;
  p.b_global = b_global;
  p.y = y;
  p.ldy = ldy;
  p.y_fp32 = y_dtype;
  p.stall_first_stage = stall;
  p.wait_limit_ns = limit_ns;
  return gemm_paired(enc, st, a_codes, a_sf, b_codes, b_sf, m, n, k, p,
                     reinterpret_cast<cudaStream_t>(stream), nullptr, workspace, workspace_bytes,
                     true);
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_global,
                        const uint8_t* b_codes, const uint8_t* b_sf, const float* b_global,
                        void* y, int y_dtype, int64_t ldy, int64_t m, int64_t n, int64_t k,
                        void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
  return gemm_entry(a_codes, a_sf, a_global, b_codes, b_sf, b_global, y, y_dtype, ldy, m, n, k,
                    workspace, workspace_bytes, stream, 0, 0);
}

nvfp4_status nvfp4_selftest_gemm_stall(const uint8_t* a_codes, const uint8_t* a_sf,
                                       const float* a_global, const uint8_t* b_codes,
                                       const uint8_t* b_sf, const float* b_global, void* y,
                                       int64_t m, int64_t n, int64_t k, uint64_t limit_ns,
                                       void* workspace, size_t workspace_bytes,
                                       nvfp4_stream_t stream) {
  if (limit_ns < 1000u || limit_ns > 10000000000ull) return NVFP4_ERR_INVALID_ARG;
  return gemm_entry(a_codes, a_sf, a_global, b_codes, b_sf, b_global, y, 0, n, m, n, k,
                    workspace, workspace_bytes, stream, 1, limit_ns);
}

size_t nvfp4_linear_workspace_bytes(int64_t m, int64_t n, int64_t k) {
  if (m < 1 || n < 1 || k < 32 || k % 32 != 0) return 0;
  // the split counters' region always (see split_counter_bytes), then the
  // split GEMMs' partials
  size_t b = round_up(nvfp4_gemm_workspace_bytes(m, n, k), 256);
  if (b < split_counter_bytes(n)) b = split_counter_bytes(n);
  b += round_up(static_cast<size_t>(m) * static_cast<size_t>(k / 2), 256);  // codes
  b += round_up(nvfp4_sf_bytes(m, k), 256);                                // scales
  b += 256;                                                                // global
  b += static_cast<size_t>(nvfp4::quant::kMaxPartials) * sizeof(float);     // amax partials
  return b;
}

nvfp4_status nvfp4_linear(const void* x, int64_t m, int64_t k, int64_t ldx,
                          const float* x_global, const uint8_t* w_codes, const uint8_t* w_sf,
                          const float* w_global, int64_t n, void* y, int y_dtype, int64_t ldy,
                          void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
  if (!x || !w_codes || !w_sf || !w_global || !y || !workspace) return NVFP4_ERR_INVALID_ARG;
  if (m < 1 || n < 1 || k < 1 || (y_dtype != 0 && y_dtype != 1) || ldy < n || ldx < k)
    return NVFP4_ERR_INVALID_ARG;
  if (k % 32 != 0 || m >= (int64_t{1} << 31) || n >= (int64_t{1} << 31) ||
      k >= (int64_t{1} << 31))
    return NVFP4_ERR_UNSUPPORTED;
  const int64_t esize = y_dtype == 0 ? 2 : 4;
  if (ldx % 8 != 0 || !aligned(x, 16) || !aligned(w_codes, 16) || !aligned(w_sf, 16) ||
      !aligned(y, 16) || (ldy * esize) % 16 != 0 || !aligned(w_global, 4) ||
      !aligned(x_global, 4) || !aligned(workspace, 256))
    return NVFP4_ERR_MISALIGNED;
  if (workspace_bytes < nvfp4_linear_workspace_bytes(m, n, k)) return NVFP4_ERR_INVALID_ARG;
  int dev;
  DeviceState* st;
  if (nvfp4_status e = current_device(&dev, &st)) return e;
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (nvfp4_status e = get_encoder(&enc)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // workspace: [counters + slabs (split work)][codes][scales][global][partials]
  uint8_t* w = static_cast<uint8_t*>(workspace);
  size_t split_bytes = round_up(nvfp4_gemm_workspace_bytes(m, n, k), 256);
  if (split_bytes < split_counter_bytes(n)) split_bytes = split_counter_bytes(n);
  uint8_t* a_codes = w + split_bytes;
  uint8_t* a_sf = a_codes + round_up(static_cast<size_t>(m) * static_cast<size_t>(k / 2), 256);
  float* a_global = reinterpret_cast<float*>(a_sf + round_up(nvfp4_sf_bytes(m, k), 256));
  float* partials = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a_global) + 256);
  static_assert(nvfp4::skinny::XR == NVFP4_LINEAR_IN_KERNEL_MAX_TOKENS, "header and kernel agree");
  if (m <= nvfp4::skinny::XR) {
    // A decode step's few tokens are quantized inside the GEMM (bit for bit
    // as nvfp4_quantize): no quantizer kernel sits between the previous
    // layer and this GEMM. A dynamic global over X above kSelfAmaxBytes
    // still takes the amax pass first (its partials are order-free). Every
    // CTA quantizes its k-range of all m tokens, so the redundant work grows
    // with m: measured on graphs of decode steps, 1 and 8 tokens gained
    // 0.6-1.0 us per step, 16 tokens and more lost 1.4-9 us.
    using namespace nvfp4::quant;
    XFused xf{x, ldx, x_global, nullptr, 0, a_global};
    if (x_global == nullptr && m * k * 2 > kSelfAmaxBytes) {
      if (nvfp4_status e = quant_occupancy(st)) return e;
      const int threads = amax_threads(m, k);
      const int64_t blocks = amax_blocks(m, k, ldx, st, threads);
      if (blocks > kMaxPartials) return NVFP4_ERR_UNSUPPORTED;
      amax_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(
          static_cast<const uint16_t*>(x), m, k, ldx, partials);
      if (nvfp4_status e = launch_status()) return e;
      xf.partials = partials;
      xf.nparts = static_cast<int>(blocks);
    }
    return gemm_skinny(enc, st, a_codes, a_sf, a_global, w_codes, w_sf, w_global, y, y_dtype, ldy,
                       m, n, k, w, skinny_workspace_bytes(m, n), false, 1, s, 0, 0, &xf);
  }
  // the quantized X is private to this call: its padding rows' scales are
  // not written (only the GEMM reads them, against zero-filled codes)
  if (nvfp4_status e = quantize_launch(x, m, k, ldx, x_global, a_codes, a_sf, a_global, partials,
                                       nvfp4::quant::kMaxPartials, st, s, true))
    return e;
  if (m <= 64)
    return gemm_skinny(enc, st, a_codes, a_sf, a_global, w_codes, w_sf, w_global, y, y_dtype, ldy,
                       m, n, k, w, skinny_workspace_bytes(m, n), false, 1, s);
  nvfp4::gemm::Params p;
  std::memset(&p, 0, sizeof p);
  p.a_global = a_global;
  p.b_global = w_global;
  p.y = y;
  p.ldy = ldy;
  p.y_fp32 = y_dtype;
  p.early_w = 1;
  return gemm_paired(enc, st, a_codes, a_sf, w_codes, w_sf, m, n, k, p, s, nullptr,
                     split_bytes ? w : nullptr, split_bytes, false);
}

nvfp4_status nvfp4_gemm_swiglu_quant(const uint8_t* a_codes, const uint8_t* a_sf,
                                     const float* a_global, const uint8_t* b_codes,
                                     const uint8_t* b_sf, const float* b_global,
                                     const float* h_global, uint8_t* h_codes, uint8_t* h_sf,
                                     int64_t m, int64_t ffn, int64_t k, nvfp4_stream_t stream) {
  if (!a_codes || !a_sf || !a_global || !b_codes || !b_sf || !b_global || !h_global ||
      !h_codes || !h_sf)
    return NVFP4_ERR_INVALID_ARG;
  if (m < 1 || ffn < 1 || k < 1) return NVFP4_ERR_INVALID_ARG;
  if (ffn % 128 != 0 || k % 32 != 0 || m >= (int64_t{1} << 31) || 2 * ffn >= (int64_t{1} << 31) ||
      k >= (int64_t{1} << 31))
    return NVFP4_ERR_UNSUPPORTED;
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_sf, 16) || !aligned(b_sf, 16) ||
      !aligned(h_codes, 16) || !aligned(h_sf, 16) || !aligned(a_global, 4) ||
      !aligned(b_global, 4) || !aligned(h_global, 4))
    return NVFP4_ERR_MISALIGNED;
  int dev;
  DeviceState* st;
  if (nvfp4_status e = current_device(&dev, &st)) return e;
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (nvfp4_status e = get_encoder(&enc)) return e;
  nvfp4::gemm::Params p;
  std::memset(&p, 0, sizeof p);
  p.a_global = a_global;
  p.b_global = b_global;
  p.fused = nvfp4::gemm::kFusedQuantStatic;
  p.h_global = h_global;
  p.h_codes = h_codes;
  p.h_sf = h_sf;
  p.h_atoms = ffn / 64;
  p.m_pad = static_cast<int>(ceil_div(m, 128) * 128);
  return gemm_paired(enc, st, a_codes, a_sf, b_codes, b_sf, m, 2 * ffn, k, p,
                     reinterpret_cast<cudaStream_t>(stream));
}

size_t nvfp4_gemm_swiglu_quant_dynamic_workspace_bytes(int64_t m, int64_t ffn) {
  if (m < 1 || ffn < 1) return 0;
  return round_up(static_cast<size_t>(m) * static_cast<size_t>(ffn) * 2u, 256) +
         static_cast<size_t>(nvfp4::quant::kMaxPartials) * sizeof(float);
}

nvfp4_status nvfp4_gemm_swiglu_quant_dynamic(const uint8_t* a_codes, const uint8_t* a_sf,
                                             const float* a_global, const uint8_t* b_codes,
                                             const uint8_t* b_sf, const float* b_global,
                                             uint8_t* h_codes, uint8_t* h_sf, float* h_global_out,
                                             int64_t m, int64_t ffn, int64_t k, void* workspace,
                                             size_t workspace_bytes, nvfp4_stream_t stream) {
  if (!a_codes || !a_sf || !a_global || !b_codes || !b_sf || !b_global || !h_codes || !h_sf ||
      !h_global_out || !workspace)
    return NVFP4_ERR_INVALID_ARG;
  if (m < 1 || ffn < 1 || k < 1) return NVFP4_ERR_INVALID_ARG;
  if (ffn % 128 != 0 || k % 32 != 0 || m >= (int64_t{1} << 31) || 2 * ffn >= (int64_t{1} << 31) ||
      k >= (int64_t{1} << 31))
    return NVFP4_ERR_UNSUPPORTED;
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_sf, 16) || !aligned(b_sf, 16) ||
      !aligned(h_codes, 16) || !aligned(h_sf, 16) || !aligned(a_global, 4) ||
      !aligned(b_global, 4) || !aligned(h_global_out, 4) || !aligned(workspace, 256))
    return NVFP4_ERR_MISALIGNED;
  if (workspace_bytes < nvfp4_gemm_swiglu_quant_dynamic_workspace_bytes(m, ffn))
    return NVFP4_ERR_INVALID_ARG;
  using namespace nvfp4::quant;
  // 32-bit task index of the quantizer over h
  if (ceil_div(m, 128) * 32 * ceil_div(ceil_div(ffn, 64), kAtomsPerTask) >= (int64_t{1} << 31))
    return NVFP4_ERR_UNSUPPORTED;
  int dev;
  DeviceState* st;
  if (nvfp4_status e = current_device(&dev, &st)) return e;
  if (nvfp4_status e = quant_occupancy(st)) return e;
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (nvfp4_status e = get_encoder(&enc)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // workspace: [bf16 h, m x ffn][per-CTA max|h|]
  uint16_t* h = static_cast<uint16_t*>(workspace);
  float* partials = reinterpret_cast<float*>(
      static_cast<uint8_t*>(workspace) +
      round_up(static_cast<size_t>(m) * static_cast<size_t>(ffn) * 2u, 256));
  nvfp4::gemm::Params p;
  std::memset(&p, 0, sizeof p);
  p.a_global = a_global;
  p.b_global = b_global;
  p.fused = nvfp4::gemm::kFusedBf16Amax;
  p.y = h;
  p.ldy = ffn;
  p.h_partials = partials;
  int grid = 0;
  if (nvfp4_status e = gemm_paired(enc, st, a_codes, a_sf, b_codes, b_sf, m, 2 * ffn, k, p, s,
                                   &grid))
    return e;
  if (grid > kMaxPartials) return NVFP4_ERR_UNSUPPORTED;  // cannot happen: grid <= SM count
  // the quantizer reduces the GEMM's per-CTA maxima to h's global, as it
  // reduces an amax pass's, and quantizes h (launched to overlap the GEMM's
  // tail; it waits for the GEMM before reading anything)
  QuantArgs a;
  a.x = h;
  a.rows = m;
  a.k = ffn;
  a.ldx = ffn;
  a.global_in = nullptr;
  a.partials = partials;
  a.nparts = grid;
  a.codes = h_codes;
  a.sf = h_sf;
  a.global_out = h_global_out;
  a.skip_pad = 0;
  return quantizer_launch(a, st, s);
}

nvfp4_status nvfp4_fuse_group_scales(int n_modules, const int64_t* rows_per_module, int64_t k,
                                     const uint8_t* const* sf_modules, const float* globals_in,
                                     uint8_t* sf_fused, float* global_out,
                                     nvfp4_stream_t stream) {
  using namespace nvfp4::fold;
  if (n_modules < 1 || n_modules > kMaxModules || !rows_per_module || !sf_modules ||
      !globals_in || !sf_fused || !global_out || k <= 0)
    return NVFP4_ERR_INVALID_ARG;
  if (k % 16 != 0) return NVFP4_ERR_UNSUPPORTED;
  FoldArgs a;
  std::memset(&a, 0, sizeof a);
  a.n = n_modules;
  a.k = k;
  a.n_ka = ceil_div(k, 64);
  int64_t total = 0;
  const uintptr_t out_lo = reinterpret_cast<uintptr_t>(sf_fused);
  for (int i = 0; i < n_modules; ++i) {
    if (rows_per_module[i] < 1 || sf_modules[i] == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(sf_modules[i], 4)) return NVFP4_ERR_MISALIGNED;
    a.row_start[i] = total;
    a.sf_in[i] = sf_modules[i];
    total += rows_per_module[i];
  }
  a.row_start[n_modules] = total;
  a.total_rows = total;
  const size_t out_bytes = nvfp4_sf_bytes(total, k);
  const uintptr_t out_hi = out_lo + out_bytes;
  for (int i = 0; i < n_modules; ++i) {
    const uintptr_t lo = reinterpret_cast<uintptr_t>(sf_modules[i]);
    const uintptr_t hi = lo + nvfp4_sf_bytes(rows_per_module[i], k);
    if (lo < out_hi && out_lo < hi) return NVFP4_ERR_INVALID_ARG;  // in place is not allowed
  }
  const uintptr_t g_lo = reinterpret_cast<uintptr_t>(globals_in);
  const uintptr_t g_out = reinterpret_cast<uintptr_t>(global_out);
  if (g_out + sizeof(float) > g_lo && g_out < g_lo + sizeof(float) * n_modules)
    return NVFP4_ERR_INVALID_ARG;  // g* must not overwrite an input global mid-kernel
  if (!aligned(sf_fused, 16) || !aligned(globals_in, 4) || !aligned(global_out, 4))
    return NVFP4_ERR_MISALIGNED;
  a.g_in = globals_in;
  a.sf_out = sf_fused;
  a.g_out = global_out;
  int dev;
  DeviceState* st;
  if (nvfp4_status e = current_device(&dev, &st)) return e;
  const int64_t words = static_cast<int64_t>(out_bytes / 4);
  int64_t blocks = ceil_div(words, kThreads);
  if (blocks > static_cast<int64_t>(st->sms) * 8) blocks = static_cast<int64_t>(st->sms) * 8;
  if (blocks < 1) blocks = 1;
  fold_kernel<<<static_cast<unsigned>(blocks), kThreads, 0,
                reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return launch_status();
}

nvfp4_status nvfp4_silu_mul(const void* y, int64_t m, int64_t n, int64_t ldy, void* h,
                            int64_t ldh, nvfp4_stream_t stream) {
  using namespace nvfp4::act;
  if (!y || !h || m < 0 || n < 1 || ldy < 2 * n || ldh < n) return NVFP4_ERR_INVALID_ARG;
  if (n % 8 != 0) return NVFP4_ERR_UNSUPPORTED;
  if (ldy % 8 != 0 || ldh % 8 != 0 || !aligned(y, 16) || !aligned(h, 16))
    return NVFP4_ERR_MISALIGNED;
  if (m == 0) return NVFP4_OK;
  int dev;
  DeviceState* st;
  if (nvfp4_status e = current_device(&dev, &st)) return e;
  int64_t blocks = ceil_div(m, kThreads / 32);
  if (blocks > static_cast<int64_t>(st->sms) * 8) blocks = static_cast<int64_t>(st->sms) * 8;
  silu_mul_kernel<<<static_cast<unsigned>(blocks), kThreads, 0,
                    reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(y), m, n, ldy, static_cast<uint16_t*>(h), ldh);
  return launch_status();
}

nvfp4_status nvfp4_selftest_wait_timeout(uint64_t limit_ns, nvfp4_stream_t stream) {
  if (limit_ns < 1000u || limit_ns > 10000000000ull) return NVFP4_ERR_INVALID_ARG;
  nvfp4::skinny::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      limit_ns);
  return launch_status();
}

nvfp4_status nvfp4_read_fault(nvfp4_stream_t stream, uint32_t* fault_out) {
  if (fault_out == nullptr) return NVFP4_ERR_INVALID_ARG;
  unsigned int v = 0;
  const unsigned int zero = 0;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess ||
      cudaMemcpyFromSymbol(&v, nvfp4::g_fault_word, sizeof v) != cudaSuccess ||
      cudaMemcpyToSymbol(nvfp4::g_fault_word, &zero, sizeof zero) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  *fault_out = v;
  return v ? NVFP4_ERR_TIMEOUT : NVFP4_OK;
}

}  // extern "C"
