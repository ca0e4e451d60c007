"""Helpers shared by the GPU parity tests (not a test module).

Tolerance of the GEMM (written once, used everywhere): relative Frobenius
error <= 1e-3 and per-element |y - ref| <= 2e-2 * ||x_hat_m|| * ||w_hat_n||
(the Cauchy-Schwarz bound on |y_mn|). A bf16 output is compared with the
FP64 reference rounded once to bf16 (bf16 rounding alone is ~1.7e-3 relative
Frobenius on Gaussian outputs, above the 1e-3 limit for a perfect GEMM); the
fp32 output mode is compared with the FP64 reference itself.
"""
from __future__ import annotations

import numpy as np
import torch

REL_FRO = 1e-3
PER_ELEM = 2e-2


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(b: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)


def upload(q, device="cuda"):
    """An oracle-quantized tensor as the library's NVFP4Tensor (inputs flow
    oracle -> CUDA only)."""
    from nvfp4_w4a4_quantized_elem_b200.nvfp4 import NVFP4Tensor
    return NVFP4Tensor(torch.from_numpy(np.ascontiguousarray(q.codes)).to(device),
                       torch.from_numpy(q.sf_swizzled).to(device),
                       torch.tensor([float(q.g)], dtype=torch.float32, device=device),
                       q.rows, q.k)


def assert_quant_equal(gpu, ref, what=""):
    """Bit-exact: codes, the whole swizzled scale buffer (padding included)
    and the global scale."""
    codes = gpu.codes.cpu().numpy()
    sf = gpu.sf.cpu().numpy()
    g = gpu.global_scale.cpu().numpy()[0]
    ref_sf = ref.sf_swizzled
    assert g.view(np.uint32) == np.float32(ref.g).view(np.uint32), f"{what}: g {g} != {ref.g}"
    assert sf.shape == ref_sf.shape
    bad = np.flatnonzero(sf != ref_sf)
    assert bad.size == 0, f"{what}: {bad.size} scale bytes differ, first at {bad[:5]}"
    bad = np.argwhere(codes != ref.codes)
    assert bad.size == 0, f"{what}: {len(bad)} code bytes differ, first at {bad[:5].tolist()}"


def gemm_check(y_gpu: torch.Tensor, y_ref: np.ndarray, row_norm: np.ndarray,
               col_norm: np.ndarray, what=""):
    """Compare a GEMM output with the FP64 reference under the tolerance."""
    y = y_gpu.detach().float().cpu().numpy().astype(np.float64)
    if y_gpu.dtype == torch.bfloat16:
        ref = torch.from_numpy(y_ref).to(torch.bfloat16).double().numpy()
    else:
        ref = y_ref
    err = y - ref
    fro = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)
    bound = PER_ELEM * row_norm[:, None] * col_norm[None, :]
    worst = np.max(np.abs(err) - bound)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    assert fro <= REL_FRO, f"{what}: relative Frobenius error {fro:.3e} > {REL_FRO}"
    assert worst <= 0, f"{what}: per-element bound exceeded by {worst:.3e}"
    return fro


def norms(orc, q, rows=None):
    dq = orc.dequantize(q) if rows is None else orc.dequantize_rows(q, rows)
    return np.linalg.norm(dq, axis=1)


def assert_row_blocks_equal(orc, gpu, x_rows_bf16, blocks, g, what=""):
    """Whole 128-row blocks of a quantized tensor against the oracle: the
    oracle quantizes each block's rows (bf16, taken from the tensor the GPU
    quantized) with the same global g; codes and the block's swizzled scale
    bytes (one 128-row block is n_ka * 512 contiguous bytes) must be equal.
    `x_rows_bf16(r0, r1)` returns rows [r0, r1) on the host."""
    k = gpu.k
    blk = 128 * (-(-k // 64) * 4)
    for rb in blocks:
        r0, r1 = 128 * rb, min(128 * rb + 128, gpu.rows)
        q = orc.quantize(bits(x_rows_bf16(r0, r1)), global_in=np.float32(g))
        codes = gpu.codes[r0:r1].cpu().numpy()
        sf = gpu.sf[rb * blk:(rb + 1) * blk].cpu().numpy()
        bad = np.argwhere(codes != q.codes)
        assert bad.size == 0, f"{what}: block {rb}: {len(bad)} code bytes differ"
        bad = np.flatnonzero(sf != q.sf_swizzled)
        assert bad.size == 0, f"{what}: block {rb}: {bad.size} scale bytes differ"
