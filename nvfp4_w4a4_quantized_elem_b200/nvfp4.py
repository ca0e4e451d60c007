"""ctypes binding of libnvfp4.so (C ABI in include/nvfp4.h).

Argument marshalling only: every step of the NVFP4 W4A4 path runs in the CUDA
library. PyTorch supplies device memory (output tensors allocated here for
convenience; callers may pass their own) and the current stream. There is no
CPU fallback: if the library is missing or a call fails, an exception is
raised.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")
# Dynamic quantization of x with rows * k * 2 bytes up to this bound runs
# one kernel (NVFP4_ONE_PASS_MAX_BYTES of nvfp4.h): no amax pass.
ONE_PASS_MAX_BYTES = 65536
# nvfp4_linear quantizes at most this many tokens inside the few-token GEMM
# (NVFP4_LINEAR_IN_KERNEL_MAX_TOKENS of nvfp4.h)
LINEAR_IN_KERNEL_MAX_TOKENS = 8

NVFP4_OK = 0
STATUS_NAMES = {0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_UNSUPPORTED",
                3: "NVFP4_ERR_MISALIGNED", 4: "NVFP4_ERR_CUDA", 5: "NVFP4_ERR_TIMEOUT"}

# every symbol include/nvfp4.h declares
EXPORTS = ("nvfp4_status_string", "nvfp4_sf_bytes", "nvfp4_quantize_workspace_bytes",
           "nvfp4_quantize", "nvfp4_quantize_noalloc", "nvfp4_calibrate_global",
           "nvfp4_gemm_workspace_bytes", "nvfp4_gemm", "nvfp4_linear_workspace_bytes",
           "nvfp4_linear", "nvfp4_gemm_swiglu_quant",
           "nvfp4_gemm_swiglu_quant_dynamic_workspace_bytes", "nvfp4_gemm_swiglu_quant_dynamic",
           "nvfp4_fuse_group_scales", "nvfp4_silu_mul", "nvfp4_read_fault",
           "nvfp4_selftest_wait_timeout", "nvfp4_selftest_gemm_stall")

_lib = None
_lock = threading.Lock()


class NVFP4Error(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libnvfp4.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} not found: build it with "
                "`python -m nvfp4_w4a4_quantized_elem_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I, SZ, U32P = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                               ctypes.c_size_t, ctypes.POINTER(ctypes.c_uint32))
        sigs = {
            "nvfp4_status_string": (ctypes.c_char_p, [I]),
            "nvfp4_sf_bytes": (SZ, [I64, I64]),
            "nvfp4_quantize_workspace_bytes": (SZ, [I64, I64]),
            "nvfp4_quantize": (I, [P, I64, I64, I64, P, P, P, P, P, SZ, P]),
            "nvfp4_quantize_noalloc": (I, [P, I64, I64, I64, P, P, P, P, P]),
            "nvfp4_calibrate_global": (I, [P, I64, I64, I64, P, P, P, SZ, P]),
            "nvfp4_gemm_workspace_bytes": (SZ, [I64, I64, I64]),
            "nvfp4_gemm": (I, [P, P, P, P, P, P, P, I, I64, I64, I64, I64, P, SZ, P]),
            "nvfp4_linear_workspace_bytes": (SZ, [I64, I64, I64]),
            "nvfp4_linear": (I, [P, I64, I64, I64, P, P, P, P, I64, P, I, I64, P, SZ, P]),
            "nvfp4_gemm_swiglu_quant": (I, [P, P, P, P, P, P, P, P, P, I64, I64, I64, P]),
            "nvfp4_gemm_swiglu_quant_dynamic_workspace_bytes": (SZ, [I64, I64]),
            "nvfp4_gemm_swiglu_quant_dynamic": (I, [P, P, P, P, P, P, P, P, P, I64, I64, I64,
                                                    P, SZ, P]),
            "nvfp4_fuse_group_scales": (I, [I, P, I64, P, P, P, P, P]),
            "nvfp4_silu_mul": (I, [P, I64, I64, I64, P, I64, P]),
            "nvfp4_read_fault": (I, [P, U32P]),
            "nvfp4_selftest_wait_timeout": (I, [ctypes.c_uint64, P]),
            "nvfp4_selftest_gemm_stall": (I, [P, P, P, P, P, P, P, I64, I64, I64, ctypes.c_uint64,
                                              P, SZ, P]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
        return L


def _check(status: int, what: str) -> None:
    if status != NVFP4_OK:
        raise NVFP4Error(what, status)


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream: torch.cuda.Stream | None) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _require_cuda(t: torch.Tensor, name: str, dtype: torch.dtype | None = None) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def sf_bytes(rows: int, k: int) -> int:
    return int(lib().nvfp4_sf_bytes(rows, k))


def quantize_workspace_bytes(rows: int, k: int) -> int:
    return int(lib().nvfp4_quantize_workspace_bytes(rows, k))


@dataclass
class NVFP4Tensor:
    """A [rows, k] tensor in NVFP4: packed E2M1 codes, swizzled E4M3 block
    scales and the FP32 global scale (a 1-element device tensor)."""
    codes: torch.Tensor        # uint8 [rows, k // 2]
    sf: torch.Tensor           # uint8 [sf_bytes(rows, k)]
    global_scale: torch.Tensor  # float32 [1]
    rows: int
    k: int

    @staticmethod
    def empty(rows: int, k: int, device="cuda") -> "NVFP4Tensor":
        return NVFP4Tensor(torch.empty((rows, k // 2), dtype=torch.uint8, device=device),
                           torch.empty(sf_bytes(rows, k), dtype=torch.uint8, device=device),
                           torch.empty(1, dtype=torch.float32, device=device), rows, k)


def quantize(x: torch.Tensor, global_scale: torch.Tensor | None = None,
             out: NVFP4Tensor | None = None, workspace: torch.Tensor | None = None,
             stream: torch.cuda.Stream | None = None) -> NVFP4Tensor:
    """nvfp4_quantize: bf16 [rows, k] (rows may be strided) -> NVFP4Tensor.
    ``global_scale`` None => dynamic global (amax pass + quantizer; one
    kernel when x is at most ONE_PASS_MAX_BYTES)."""
    _require_cuda(x, "x", torch.bfloat16)
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit stride along k")
    rows, k = x.shape
    if out is None:
        out = NVFP4Tensor.empty(rows, k, x.device)
    if global_scale is None and workspace is None:
        workspace = torch.empty(quantize_workspace_bytes(rows, k), dtype=torch.uint8,
                                device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().nvfp4_quantize(_ptr(x), rows, k, x.stride(0), _ptr(global_scale),
                              _ptr(out.codes), _ptr(out.sf), _ptr(out.global_scale),
                              _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "nvfp4_quantize")
    return out


def quantize_noalloc(x: torch.Tensor, out: NVFP4Tensor, global_scale: torch.Tensor | None = None,
                     stream: torch.cuda.Stream | None = None) -> NVFP4Tensor:
    """nvfp4_quantize_noalloc: as quantize(), for callers that cannot
    allocate device memory. No workspace: the amax pass uses a fixed device
    array inside the library (shared by every call on the device; calls that
    overlap on the GPU race). The caller supplies the output buffers."""
    _require_cuda(x, "x", torch.bfloat16)
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit stride along k")
    rows, k = x.shape
    st = lib().nvfp4_quantize_noalloc(_ptr(x), rows, k, x.stride(0), _ptr(global_scale),
                                      _ptr(out.codes), _ptr(out.sf), _ptr(out.global_scale),
                                      _stream(stream))
    _check(st, "nvfp4_quantize_noalloc")
    return out


class Calibrator:
    """Static global scale from a stream of calibration batches
    (nvfp4_calibrate_global): observe() each batch, then use .global_scale
    as quantize(..., global_scale=...)."""

    def __init__(self, device="cuda"):
        self.running_amax = torch.zeros(1, dtype=torch.float32, device=device)
        self.global_scale = torch.ones(1, dtype=torch.float32, device=device)
        self._ws = None

    def observe(self, x: torch.Tensor, stream: torch.cuda.Stream | None = None) -> torch.Tensor:
        _require_cuda(x, "x", torch.bfloat16)
        if x.dim() != 2 or x.stride(1) != 1:
            raise ValueError("x must be 2-D with unit stride along k")
        rows, k = x.shape
        need = quantize_workspace_bytes(rows, k)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=x.device)
        st = lib().nvfp4_calibrate_global(_ptr(x), rows, k, x.stride(0), _ptr(self.running_amax),
                                          _ptr(self.global_scale), _ptr(self._ws), self._ws.numel(),
                                          _stream(stream))
        _check(st, "nvfp4_calibrate_global")
        return self.global_scale


def gemm_workspace_bytes(m: int, n: int, k: int) -> int:
    return int(lib().nvfp4_gemm_workspace_bytes(m, n, k))


def gemm(a: NVFP4Tensor, b: NVFP4Tensor, out: torch.Tensor | None = None,
         out_dtype: torch.dtype = torch.bfloat16, workspace: torch.Tensor | None = None,
         stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """nvfp4_gemm: Y[m, n] = dequant(A) @ dequant(B).T (A = activations
    [m, k], B = weights [n, k]); bf16 or fp32 output. ``workspace`` (at least
    gemm_workspace_bytes) lets few-token GEMMs share the work across all SMs
    (stream-K)."""
    if a.k != b.k:
        raise ValueError("k mismatch")
    m, n, k = a.rows, b.rows, a.k
    if out is None:
        out = torch.empty((m, n), dtype=out_dtype, device=a.codes.device)
    if out.dtype not in (torch.bfloat16, torch.float32) or out.stride(1) != 1:
        raise ValueError("out must be bf16/fp32 with unit column stride")
    y_dtype = 0 if out.dtype == torch.bfloat16 else 1
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().nvfp4_gemm(_ptr(a.codes), _ptr(a.sf), _ptr(a.global_scale),
                          _ptr(b.codes), _ptr(b.sf), _ptr(b.global_scale),
                          _ptr(out), y_dtype, out.stride(0), m, n, k, _ptr(workspace), ws_bytes,
                          _stream(stream))
    _check(st, "nvfp4_gemm")
    return out


def interleave_gate_up(w_gate_up: torch.Tensor) -> torch.Tensor:
    """Row order nvfp4_gemm_swiglu_quant expects: [2*ffn, k] with gate rows
    [0, ffn) and up rows [ffn, 2ffn) -> blocks of 128 (gate b, up b, ...).
    Offline weight preparation (a row permutation)."""
    two_ffn = w_gate_up.shape[0]
    ffn = two_ffn // 2
    if two_ffn % 256:
        raise ValueError("ffn must be a multiple of 128")
    idx = torch.arange(two_ffn, device=w_gate_up.device).view(2, ffn // 128, 128)
    return w_gate_up[idx.transpose(0, 1).reshape(-1)]


def gemm_swiglu_quant(a: NVFP4Tensor, b_interleaved: NVFP4Tensor, h_global: torch.Tensor,
                      out: NVFP4Tensor | None = None,
                      stream: torch.cuda.Stream | None = None) -> NVFP4Tensor:
    """nvfp4_gemm_swiglu_quant: NVFP4 h = quantize(silu(gate) * up, h_global)
    straight from the gate_up GEMM (weights row-interleaved, see
    interleave_gate_up)."""
    if a.k != b_interleaved.k:
        raise ValueError("k mismatch")
    m, ffn, k = a.rows, b_interleaved.rows // 2, a.k
    if out is None:
        out = NVFP4Tensor.empty(m, ffn, a.codes.device)
    out.global_scale.copy_(h_global.reshape(1))
    st = lib().nvfp4_gemm_swiglu_quant(_ptr(a.codes), _ptr(a.sf), _ptr(a.global_scale),
                                       _ptr(b_interleaved.codes), _ptr(b_interleaved.sf),
                                       _ptr(b_interleaved.global_scale), _ptr(h_global),
                                       _ptr(out.codes), _ptr(out.sf), m, ffn, k, _stream(stream))
    _check(st, "nvfp4_gemm_swiglu_quant")
    return out


def swiglu_quant_dynamic_workspace(m: int, ffn: int, device="cuda") -> torch.Tensor:
    """Workspace of gemm_swiglu_quant_dynamic (bf16 h + per-CTA maxima)."""
    nb = int(lib().nvfp4_gemm_swiglu_quant_dynamic_workspace_bytes(m, ffn))
    return torch.empty(nb, dtype=torch.uint8, device=device)


def gemm_swiglu_quant_dynamic(a: NVFP4Tensor, b_interleaved: NVFP4Tensor,
                              out: NVFP4Tensor | None = None,
                              workspace: torch.Tensor | None = None,
                              stream: torch.cuda.Stream | None = None) -> NVFP4Tensor:
    """nvfp4_gemm_swiglu_quant_dynamic: NVFP4 h = quantize(silu(gate) * up)
    with h's own dynamic global (weights row-interleaved, see
    interleave_gate_up). ``workspace`` from swiglu_quant_dynamic_workspace()
    (allocated here when None); its first m*ffn*2 bytes hold h in bf16."""
    if a.k != b_interleaved.k:
        raise ValueError("k mismatch")
    m, ffn, k = a.rows, b_interleaved.rows // 2, a.k
    if out is None:
        out = NVFP4Tensor.empty(m, ffn, a.codes.device)
    if workspace is None:
        workspace = swiglu_quant_dynamic_workspace(m, ffn, a.codes.device)
    st = lib().nvfp4_gemm_swiglu_quant_dynamic(
        _ptr(a.codes), _ptr(a.sf), _ptr(a.global_scale), _ptr(b_interleaved.codes),
        _ptr(b_interleaved.sf), _ptr(b_interleaved.global_scale), _ptr(out.codes), _ptr(out.sf),
        _ptr(out.global_scale), m, ffn, k, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "nvfp4_gemm_swiglu_quant_dynamic")
    return out


def fuse_group_scales(modules: list[NVFP4Tensor], sf_out: torch.Tensor | None = None,
                      global_out: torch.Tensor | None = None,
                      stream: torch.cuda.Stream | None = None):
    """nvfp4_fuse_group_scales: fold per-module globals into one (g* = min)
    and write the swizzled scales of the row-concatenated group.
    Returns (sf_fused, global_fused)."""
    n = len(modules)
    k = modules[0].k
    total = sum(m.rows for m in modules)
    dev = modules[0].codes.device
    if sf_out is None:
        sf_out = torch.empty(sf_bytes(total, k), dtype=torch.uint8, device=dev)
    if global_out is None:
        global_out = torch.empty(1, dtype=torch.float32, device=dev)
    globals_in = torch.cat([m.global_scale for m in modules])
    rows = (ctypes.c_int64 * n)(*[m.rows for m in modules])
    ptrs = (ctypes.c_void_p * n)(*[m.sf.data_ptr() for m in modules])
    st = lib().nvfp4_fuse_group_scales(n, ctypes.cast(rows, ctypes.c_void_p), k,
                                       ctypes.cast(ptrs, ctypes.c_void_p), _ptr(globals_in),
                                       _ptr(sf_out), _ptr(global_out), _stream(stream))
    _check(st, "nvfp4_fuse_group_scales")
    return sf_out, global_out


def fuse_group(modules: list[NVFP4Tensor], stream=None) -> NVFP4Tensor:
    """The repaired fused tensor: concatenated codes, folded scales, g*."""
    sf, g = fuse_group_scales(modules, stream=stream)
    codes = torch.cat([m.codes for m in modules], dim=0)
    return NVFP4Tensor(codes, sf, g, codes.shape[0], modules[0].k)


def silu_mul(y: torch.Tensor, out: torch.Tensor | None = None,
             stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """nvfp4_silu_mul: h = silu(y[:, :n]) * y[:, n:] in bf16."""
    _require_cuda(y, "y", torch.bfloat16)
    m, n2 = y.shape
    n = n2 // 2
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=y.device)
    st = lib().nvfp4_silu_mul(_ptr(y), m, n, y.stride(0), _ptr(out), out.stride(0),
                              _stream(stream))
    _check(st, "nvfp4_silu_mul")
    return out


def read_fault(stream: torch.cuda.Stream | None = None) -> int:
    """Synchronise, return and clear the kernels' timeout fault word."""
    v = ctypes.c_uint32(0)
    st = lib().nvfp4_read_fault(_stream(stream), ctypes.byref(v))
    if st not in (NVFP4_OK, 5):
        raise NVFP4Error("nvfp4_read_fault", st)
    return int(v.value)


def selftest_wait_timeout(limit_ns: int = 1_000_000,
                          stream: torch.cuda.Stream | None = None) -> None:
    """nvfp4_selftest_wait_timeout: make one bounded wait give up on the GPU
    (read_fault() then returns 256)."""
    _check(lib().nvfp4_selftest_wait_timeout(limit_ns, _stream(stream)),
           "nvfp4_selftest_wait_timeout")


def selftest_gemm_stall(a: NVFP4Tensor, b: NVFP4Tensor, limit_ns: int = 1_000_000,
                        workspace: torch.Tensor | None = None,
                        stream: torch.cuda.Stream | None = None) -> None:
    """nvfp4_selftest_gemm_stall: run the GEMM kernel for these operands
    with its first ring stage never filled and every wait limited to
    ``limit_ns``; the kernel gives up and returns (read_fault() then returns
    the role bits that timed out)."""
    m, n, k = a.rows, b.rows, a.k
    y = torch.empty((m, n), dtype=torch.bfloat16, device=a.codes.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().nvfp4_selftest_gemm_stall(_ptr(a.codes), _ptr(a.sf), _ptr(a.global_scale),
                                           _ptr(b.codes), _ptr(b.sf), _ptr(b.global_scale),
                                           _ptr(y), m, n, k, limit_ns, _ptr(workspace), ws_bytes,
                                           _stream(stream)),
           "nvfp4_selftest_gemm_stall")


def linear_workspace_bytes(m: int, n: int, k: int) -> int:
    return int(lib().nvfp4_linear_workspace_bytes(m, n, k))


def linear_workspace(m: int, n: int, k: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace for linear() at these sizes (keep it: calls
    leave the bytes that must start at zero zeroed again)."""
    return torch.zeros(linear_workspace_bytes(m, n, k), dtype=torch.uint8, device=device)


def linear(x: torch.Tensor, w: NVFP4Tensor, out: torch.Tensor | None = None,
           out_dtype: torch.dtype = torch.bfloat16, global_scale: torch.Tensor | None = None,
           workspace: torch.Tensor | None = None,
           stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """nvfp4_linear, the W4A4 linear layer in one call: quantize x (dynamic
    global, or the static ``global_scale``) and multiply with the NVFP4
    weights ``w`` [n, k]; the GEMM's launch overlaps the quantization.
    ``workspace`` from linear_workspace() (allocated here when None)."""
    _require_cuda(x, "x", torch.bfloat16)
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit stride along k")
    m, k = x.shape
    if k != w.k:
        raise ValueError("k mismatch")
    n = w.rows
    if out is None:
        out = torch.empty((m, n), dtype=out_dtype, device=x.device)
    if out.dtype not in (torch.bfloat16, torch.float32) or out.stride(1) != 1:
        raise ValueError("out must be bf16/fp32 with unit column stride")
    if workspace is None:
        workspace = linear_workspace(m, n, k, x.device)
    st = lib().nvfp4_linear(_ptr(x), m, k, x.stride(0), _ptr(global_scale), _ptr(w.codes),
                            _ptr(w.sf), _ptr(w.global_scale), n, _ptr(out),
                            0 if out.dtype == torch.bfloat16 else 1, out.stride(0),
                            _ptr(workspace), workspace.numel() * workspace.element_size(),
                            _stream(stream))
    _check(st, "nvfp4_linear")
    return out
