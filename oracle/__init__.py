"""CPU oracle of the NVFP4 W4A4 linear layer — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
/ reference leg may import this package. The product path (the CUDA library
and its Python binding) never touches it, and this package never imports the
product package: the two share no code.

What the oracle computes, and where it comes from (web pages on arXiv
2609.04098 "Why Gated DeltaNet Survives 4-Bit Quantization"):

* news article "Qwen3.8-27B最激进4bit量化开源，权重显存暴降2.9倍！" §02
  (NVFP4 量化格式): E2M1 values, one E4M3 block scale per 16 elements along K,
  one FP32 global scale per tensor; W4A4 quantizes weights and activations.
* same article §03 (Minima 模型构建): a fused module group is put on one
  global scale and the ratio folded into the E4M3 block scales.

Scalar codec, quantizer and fold are plain C (``nvfp4_oracle.c``, one block at
a time, FP32 round-to-nearest-even at every step, no FMA contraction); the
GEMM reference is the FP64 product of the dequantized matrices (numpy float64
matmul, a library primitive), exactly as the format's definition reads:
``Y = dequant(A) @ dequant(B).T``.

Every function is pinned in ``tests/test_oracle_*.py`` by something other than
itself (brute force, library casts, closed forms, invariants, an exact integer
GEMM).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libnvfp4_oracle.so")
_lib = None
_lock = threading.Lock()

# 2688 = 448 (largest E4M3) * 6 (largest E2M1): the global-scale numerator.
GLOBAL_NUMERATOR = 2688.0


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libnvfp4_oracle.so`` (gcc, OpenMP)."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        F = ctypes.c_float
        sig = {
            "orc_bf16_to_float": (F, [ctypes.c_uint16]),
            "orc_double_to_bf16": (ctypes.c_uint16, [ctypes.c_double]),
            "orc_e2m1_encode": (ctypes.c_uint8, [F]),
            "orc_e4m3_encode": (ctypes.c_uint8, [F]),
            "orc_e2m1_value": (ctypes.c_double, [ctypes.c_uint8]),
            "orc_e4m3_value": (ctypes.c_double, [ctypes.c_uint8]),
            "orc_tensor_amax": (F, [P, I64, I64, I64]),
            "orc_global_from_amax": (F, [F]),
            "orc_quantize": (None, [P, I64, I64, I64, F, P, P]),
            "orc_sf_offset": (I64, [I64, I64, I64]),
            "orc_sf_bytes": (I64, [I64, I64]),
            "orc_sf_swizzle": (None, [P, I64, I64, P]),
            "orc_sf_unswizzle": (None, [P, I64, I64, P]),
            "orc_dequantize": (None, [P, P, F, I64, I64, P]),
            "orc_fold_group": (F, [ctypes.c_int, P, I64, P, P, P]),
            "orc_silu_mul": (None, [P, I64, I64, I64, P]),
            "orc_e2m1_encode_array": (None, [P, I64, P]),
            "orc_e4m3_encode_array": (None, [P, I64, P]),
            "orc_e4m3_value_array": (None, [P, I64, P]),
            "orc_e2m1_value_array": (None, [P, I64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    return ctypes.c_void_p(a.ctypes.data)


def _as_bf16_bits(x) -> np.ndarray:
    """Accept a torch bf16 tensor or a numpy uint16 array of bf16 bit patterns."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy input must hold bf16 bit patterns as uint16")
        return x
    import torch  # local: the oracle itself needs only numpy
    if x.dtype != torch.bfloat16:
        raise TypeError("torch input must be bfloat16")
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ codecs --

def e2m1_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    _load().orc_e2m1_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e2m1_value(c: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().orc_e2m1_value_array(_ptr(c), c.size, _ptr(out))
    return out


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    _load().orc_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_value(c: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().orc_e4m3_value_array(_ptr(c), c.size, _ptr(out))
    return out


def double_to_bf16(v: float) -> int:
    return int(_load().orc_double_to_bf16(float(v)))


# ----------------------------------------------------------------- quantize --

@dataclass
class Quantized:
    """An NVFP4 tensor as the oracle produces it."""
    codes: np.ndarray      # uint8 [rows, k/2], element 2j in the low nibble
    sf_rm: np.ndarray      # uint8 [rows, k/16], row-major block scales
    g: np.float32          # FP32 global scale (the encode global)
    rows: int
    k: int

    @property
    def sf_swizzled(self) -> np.ndarray:
        return sf_swizzle(self.sf_rm, self.rows, self.k)


def tensor_amax(x) -> np.float32:
    xb = np.ascontiguousarray(_as_bf16_bits(x))
    rows, k = xb.shape
    return np.float32(_load().orc_tensor_amax(_ptr(xb), rows, k, k))


def global_from_amax(amax) -> np.float32:
    return np.float32(_load().orc_global_from_amax(float(np.float32(amax))))


def quantize(x, global_in=None) -> Quantized:
    """Quantize a 2-D bf16 tensor. ``global_in`` None => dynamic global."""
    xb = np.ascontiguousarray(_as_bf16_bits(x))
    if xb.ndim != 2:
        raise ValueError("expected a 2-D tensor")
    rows, k = xb.shape
    if k % 16:
        raise ValueError("k must be a multiple of 16")
    lib = _load()
    if global_in is None:
        g = np.float32(lib.orc_global_from_amax(lib.orc_tensor_amax(_ptr(xb), rows, k, k)))
    else:
        g = np.float32(global_in)
    codes = np.empty((rows, k // 2), np.uint8)
    sf_rm = np.empty((rows, k // 16), np.uint8)
    lib.orc_quantize(_ptr(xb), rows, k, k, float(g), _ptr(codes), _ptr(sf_rm))
    return Quantized(codes, sf_rm, g, rows, k)


def sf_bytes(rows: int, k: int) -> int:
    return int(_load().orc_sf_bytes(rows, k))


def sf_offset(r: int, c: int, k: int) -> int:
    return int(_load().orc_sf_offset(r, c, k))


def sf_swizzle(sf_rm: np.ndarray, rows: int, k: int) -> np.ndarray:
    sf_rm = np.ascontiguousarray(sf_rm, dtype=np.uint8)
    out = np.empty(sf_bytes(rows, k), np.uint8)
    _load().orc_sf_swizzle(_ptr(sf_rm), rows, k, _ptr(out))
    return out


def sf_unswizzle(sf_sw: np.ndarray, rows: int, k: int) -> np.ndarray:
    sf_sw = np.ascontiguousarray(sf_sw, dtype=np.uint8)
    out = np.empty((rows, k // 16), np.uint8)
    _load().orc_sf_unswizzle(_ptr(sf_sw), rows, k, _ptr(out))
    return out


def dequantize(q: Quantized, scaled: bool = True) -> np.ndarray:
    """FP64 x_hat = val * dec(s) / g (``scaled=False`` omits the / g)."""
    out = np.empty((q.rows, q.k), np.float64)
    codes = np.ascontiguousarray(q.codes)
    sf = np.ascontiguousarray(q.sf_rm)
    _load().orc_dequantize(_ptr(codes), _ptr(sf), float(q.g) if scaled else 0.0,
                           q.rows, q.k, _ptr(out))
    return out


def dequantize_rows(q: Quantized, rows_idx: np.ndarray) -> np.ndarray:
    sub = Quantized(np.ascontiguousarray(q.codes[rows_idx]),
                    np.ascontiguousarray(q.sf_rm[rows_idx]), q.g, len(rows_idx), q.k)
    return dequantize(sub)


# --------------------------------------------------------------------- GEMM --

def gemm(a: Quantized, b: Quantized, a_rows=None) -> np.ndarray:
    """FP64 reference Y = dequant(A) @ dequant(B).T (optionally only the rows
    ``a_rows`` of A). This is the definition of the W4A4 linear layer's output
    before any output rounding."""
    da = dequantize(a) if a_rows is None else dequantize_rows(a, a_rows)
    db = dequantize(b)
    return da @ db.T


# --------------------------------------------------------------------- fold --

def fold_group(mods: list[Quantized]) -> tuple[list[np.ndarray], np.float32]:
    """Repair a fused group: returns the rescaled row-major block scales of
    each module and the shared global g* (= min g_i)."""
    lib = _load()
    n = len(mods)
    k = mods[0].k
    rows = np.array([m.rows for m in mods], np.int64)
    gs = np.array([m.g for m in mods], np.float32)
    ins = [np.ascontiguousarray(m.sf_rm) for m in mods]
    outs = [np.empty_like(a) for a in ins]
    in_ptrs = (ctypes.c_void_p * n)(*[a.ctypes.data for a in ins])
    out_ptrs = (ctypes.c_void_p * n)(*[a.ctypes.data for a in outs])
    gstar = lib.orc_fold_group(n, _ptr(rows), k, ctypes.cast(in_ptrs, ctypes.c_void_p),
                               _ptr(gs), ctypes.cast(out_ptrs, ctypes.c_void_p))
    return outs, np.float32(gstar)


def fuse_group(mods: list[Quantized]) -> Quantized:
    """The fused tensor after repair: codes and folded scales of the modules
    concatenated along rows, one global g*."""
    sfs, gstar = fold_group(mods)
    codes = np.concatenate([m.codes for m in mods], axis=0)
    sf = np.concatenate(sfs, axis=0)
    return Quantized(codes, sf, gstar, codes.shape[0], mods[0].k)


def fuse_group_naive(mods: list[Quantized]) -> Quantized:
    """The faulty fusion the news article §03 describes: the group's largest
    global scale is taken and the block scales are NOT rescaled. Used only to
    show that it distorts the weights."""
    codes = np.concatenate([m.codes for m in mods], axis=0)
    sf = np.concatenate([m.sf_rm for m in mods], axis=0)
    gmax = np.float32(max(float(m.g) for m in mods))
    return Quantized(codes, sf, gmax, codes.shape[0], mods[0].k)


# ----------------------------------------------------------------- silu*mul --

def silu_mul(y) -> np.ndarray:
    """h = bf16(silu(gate) * up), gate = y[:, :n], up = y[:, n:], FP64 inside.
    Returns bf16 bit patterns (uint16)."""
    yb = np.ascontiguousarray(_as_bf16_bits(y))
    m, n2 = yb.shape
    n = n2 // 2
    out = np.empty((m, n), np.uint16)
    _load().orc_silu_mul(_ptr(yb), m, n, n2, _ptr(out))
    return out


# -------------------------------------------------------------- GDN gates --
# Reading of news article §01 (Gated DeltaNet 基础: the gates are parameterized
# in log space; the formula itself was lost from the page) together with the
# abstract's "softplus/exponential and sigmoid parameterizations": per head,
#   g     = -exp(A_log) * softplus(a + dt_bias)   (log-space decay)
#   alpha = exp(g)                                (forget gate)
#   beta  = sigmoid(b)                            (write strength)
# where a, b are the outputs of the a and b projections.

def softplus(z):
    z = np.asarray(z, dtype=np.float64)
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def sigmoid(z):
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def gdn_gates(y_a, y_b, a_log, dt_bias):
    """(g, alpha, beta) in FP64 from projection outputs [tokens, heads]."""
    g = -np.exp(np.asarray(a_log, np.float64)) * softplus(
        np.asarray(y_a, np.float64) + np.asarray(dt_bias, np.float64))
    return g, np.exp(g), sigmoid(y_b)


def rel_fro(approx, exact) -> float:
    approx = np.asarray(approx, np.float64)
    exact = np.asarray(exact, np.float64)
    return float(np.linalg.norm(approx - exact) / np.linalg.norm(exact))


def gate_sensitivity(y_a_ref, y_b_ref, y_a, y_b, a_log, dt_bias) -> dict:
    """Relative Frobenius errors of the projections and of the gates computed
    from them (abstract and paper reading §4.2 (ii): the gate nonlinearities
    compress the W4A4 GEMM error)."""
    g0, al0, be0 = gdn_gates(y_a_ref, y_b_ref, a_log, dt_bias)
    g1, al1, be1 = gdn_gates(y_a, y_b, a_log, dt_bias)
    return {"gemm_a": rel_fro(y_a, y_a_ref), "gemm_b": rel_fro(y_b, y_b_ref),
            "g": rel_fro(g1, g0), "alpha": rel_fro(al1, al0), "beta": rel_fro(be1, be0)}
