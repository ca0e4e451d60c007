"""Pins of the oracle's GEMM reference, fused-group fold and silu*mul.

GEMM: Y = dequant(A) @ dequant(B).T in FP64 (news article "Qwen3.8-27B最激进
4bit量化开源…" §02: W4A4 = both operands NVFP4 on 4-bit tensor cores). Pinned
by (a) an exact integer GEMM — val*dec(s) is a multiple of 2^-10, so scaled by
2^20 every product is an integer and the K=256 sum stays below 2^51 — and
(b) brute force with exact rationals on a tiny shape.

Fold: same article §03 — one global per fused group, ratio folded into the
E4M3 block scales. Pinned by the invariant that every dequantized weight moves
by at most one E4M3 rounding, the module that owns g* is untouched, and the
faulty "largest global, no rescale" fusion distorts module i by |1 - g_i/g_max|.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from nvfp4_w4a4_quantized_elem_b200 import workloads as wl


def bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).numpy().view(np.uint16)


def int_operand(orc, q):
    """val(code)*dec(s)*2^10 as exact int64 (val: multiple of 2^-1, dec: 2^-9)."""
    unscaled = orc.dequantize(q, scaled=False)
    ints = unscaled * 1024.0
    assert np.all(ints == np.round(ints))
    return ints.astype(np.int64)


def test_gemm_exact_integer_tiny(orc):
    cfg = wl.tiny()
    qa, qb = orc.quantize(bits(cfg.x())), orc.quantize(bits(cfg.w()))
    ia, ib = int_operand(orc, qa), int_operand(orc, qb)
    assert np.abs(ia).max() * np.abs(ib).max() * cfg.k < 2 ** 62
    exact = ia @ ib.T                                  # int64, exact
    fp64 = orc.dequantize(qa, scaled=False) @ orc.dequantize(qb, scaled=False).T
    np.testing.assert_array_equal(fp64 * 2.0 ** 20, exact.astype(np.float64))
    # the scaled reference is the same numbers divided by g_a * g_b
    y = orc.gemm(qa, qb)
    ref = exact.astype(np.float64) * 2.0 ** -20 / (float(qa.g) * float(qb.g))
    # FP64 rounding of the 1/g factors only: bounded by ~K ulps of |a|.|b|
    da, db = orc.dequantize(qa), orc.dequantize(qb)
    scale = np.linalg.norm(da, axis=1)[:, None] * np.linalg.norm(db, axis=1)[None, :]
    assert np.all(np.abs(y - ref) <= 1e-13 * scale)


def test_gemm_brute_force_rationals(orc):
    rng = np.random.default_rng(30)
    a = (rng.standard_normal((3, 32)) * 2).astype(np.float32)
    b = (rng.standard_normal((2, 32)) * 0.1).astype(np.float32)
    qa = orc.quantize(bits(torch.from_numpy(a).to(torch.bfloat16)))
    qb = orc.quantize(bits(torch.from_numpy(b).to(torch.bfloat16)))

    def value(q, r, kk):
        byte = int(q.codes[r, kk // 2])
        code = byte & 0xF if kk % 2 == 0 else byte >> 4
        mag = [0, Fraction(1, 2), 1, Fraction(3, 2), 2, 3, 4, 6][code & 7]
        s = int(q.sf_rm[r, kk // 16])
        e, m = s >> 3, s & 7
        ds = Fraction(m, 512) if e == 0 else Fraction(8 + m, 8) * Fraction(2) ** (e - 7)
        v = (-mag if code & 8 else mag) * ds
        return v / Fraction(float(q.g))

    y = orc.gemm(qa, qb)
    for i in range(3):
        for j in range(2):
            exact = sum(value(qa, i, kk) * value(qb, j, kk) for kk in range(32))
            assert abs(y[i, j] - float(exact)) <= 1e-12 * max(1.0, abs(float(exact)))


def test_gemm_row_subset(orc):
    cfg = wl.tiny()
    qa, qb = orc.quantize(bits(cfg.x())), orc.quantize(bits(cfg.w()))
    rows = np.array([0, 5, 63])
    # BLAS may block the two products differently: equal up to FP64 rounding
    np.testing.assert_allclose(orc.gemm(qa, qb, a_rows=rows), orc.gemm(qa, qb)[rows],
                               rtol=0, atol=1e-14)


# ------------------------------------------------------------------- fold --

def small_group():
    g = wl.gdn_fused()
    # same sigmas and seeds as the GDN in_proj group, fewer rows, K = 512
    return [wl.gaussian_bf16(rows, 512, sigma, seed)
            for (_, rows, sigma, seed) in [("qkv", 256, .02, 1), ("z", 128, .02, 2),
                                           ("a", 48, .1, 3), ("b", 48, .005, 4)]], g


def test_fold_invariant(orc):
    ws, _ = small_group()
    mods = [orc.quantize(bits(w)) for w in ws]
    sfs, gstar = orc.fold_group(mods)
    assert gstar == min(m.g for m in mods)
    for m, sf in zip(mods, sfs):
        before = orc.dequantize(m)
        after = orc.dequantize(orc.Quantized(m.codes, sf, gstar, m.rows, m.k))
        ds_after = np.repeat(orc.e4m3_value(sf), 16, axis=1)
        normal = ds_after >= 2.0 ** -6
        diff = np.abs(after - before)
        assert np.all(diff[normal] <= 2.0 ** -4 * np.abs(before[normal]) * (1 + 1e-6))
        # subnormal scales: one step of 2^-10 in dec(s) at most (times |val| <= 6)
        assert np.all(diff[~normal] <= 6 * 2.0 ** -10 / float(gstar) * (1 + 1e-6))
        if m.g == gstar:
            np.testing.assert_array_equal(sf, m.sf_rm)


def test_fold_idempotent_when_globals_equal(orc):
    ws, _ = small_group()
    q = orc.quantize(bits(ws[0]))
    sfs, gstar = orc.fold_group([q, q])
    assert gstar == q.g
    for sf in sfs:
        np.testing.assert_array_equal(sf, q.sf_rm)


def test_naive_fusion_distorts_by_global_ratio(orc):
    """The faulty fusion (largest global, block scales untouched) scales module
    i by g_i / g_max exactly; the repaired fusion stays within one E4M3
    rounding."""
    ws, _ = small_group()
    mods = [orc.quantize(bits(w)) for w in ws]
    naive = orc.fuse_group_naive(mods)
    fixed = orc.fuse_group(mods)
    gmax = max(float(m.g) for m in mods)
    dq_naive, dq_fixed = orc.dequantize(naive), orc.dequantize(fixed)
    r0 = 0
    for m in mods:
        true = orc.dequantize(m)
        sl = slice(r0, r0 + m.rows)
        nz = true != 0
        ratio = dq_naive[sl][nz] / true[nz]
        np.testing.assert_allclose(ratio, float(m.g) / gmax, rtol=1e-12)
        rel_fixed = np.linalg.norm(dq_fixed[sl] - true) / np.linalg.norm(true)
        assert rel_fixed < 2.0 ** -4
        r0 += m.rows
    # the a-gate (sigma 0.1) is shrunk by ~20x when b (sigma 0.005) sets g_max
    g_a, g_b = float(mods[2].g), float(mods[3].g)
    assert 1 - g_a / gmax > 0.9 and gmax == g_b


def test_fused_swizzle_shares_atom_between_modules(orc):
    """a (48 rows) and b (48 rows) after qkv+z (multiple of 128 rows) share one
    128-row atom in the fused layout: rows [0,48) from a, [48,96) from b, the
    rest padding."""
    ws, _ = small_group()
    mods = [orc.quantize(bits(w)) for w in ws]
    fused = orc.fuse_group(mods)
    sw = fused.sf_swizzled
    k = 512
    base = 256 + 128
    sfs, _ = orc.fold_group(mods)
    for r in range(128):
        for c in range(k // 16):
            v = sw[orc.sf_offset(base + r, c, k)]
            if r < 48:
                assert v == sfs[2][r, c]
            elif r < 96:
                assert v == sfs[3][r - 48, c]
            else:
                assert v == 0


# --------------------------------------------------------------- silu*mul --

def test_silu_mul_against_torch_fp64(orc):
    rng = np.random.default_rng(31)
    y = (rng.standard_normal((17, 64)) * 4).astype(np.float32)
    yt = torch.from_numpy(y).to(torch.bfloat16)
    h = orc.silu_mul(bits(yt))
    yd = yt.double()
    ref = (torch.nn.functional.silu(yd[:, :32]) * yd[:, 32:]).to(torch.bfloat16)
    got = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16)
    # both round the FP64 value once to bf16; torch may double-round via FP32
    diff = (got.float() - ref.float()).abs()
    ulp = ref.float().abs() * 2.0 ** -7
    assert torch.all(diff <= ulp + 1e-30)


def test_silu_identities(orc):
    z = np.array([0.0, 30.0, -30.0, 1.0, -1.0], np.float32)
    y = np.concatenate([z, np.ones(5, np.float32)])[None, :]
    h = orc.silu_mul(bits(torch.from_numpy(y).to(torch.bfloat16)))
    hv = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).float().numpy()[0]
    assert hv[0] == 0.0                 # silu(0) = 0
    assert hv[1] == 30.0                # silu(z) -> z for large z
    assert abs(hv[2]) < 1e-10           # silu(-30) ~ -2.8e-12
    # silu(-z) = silu(z) - z
    assert abs((hv[4]) - (hv[3] - 1.0)) <= 2 ** -7
