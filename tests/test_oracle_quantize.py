"""Pins of the oracle's quantizer and scale layout.

Format: news article "Qwen3.8-27B最激进4bit量化开源…" §02 (E2M1 values, one
E4M3 scale per 16 elements, one FP32 global; block scaling confines an
outlier's error to its own 16-element block). Pins:
  * hand-worked blocks (tests/golden/nvfp4_blocks_by_hand.txt);
  * closed form: inputs on the grid times per-block powers of two round-trip
    exactly;
  * homogeneity under 2^q scaling, sign symmetry;
  * outlier locality (bit-exact with a fixed global; bounded by the block's
    own amax with a dynamic global) — mechanism (i) of the abstract;
  * the per-block error bound that follows from the two roundings;
  * the swizzled scale layout is a bijection onto the non-padding bytes and
    matches hand-computed offsets.
"""
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_blocks_by_hand.txt")


def bf16_bits(a) -> np.ndarray:
    t = torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def load_golden():
    cases = []
    for line in open(GOLDEN, encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, g, xs, sf, codes, by = [f.strip() for f in line.split("|")]
        cases.append((name, float(g), [float(v) for v in xs.split()], int(sf, 16),
                      [int(c) for c in codes.split()], bytes.fromhex(by.replace(" ", ""))))
    return cases


@pytest.mark.parametrize("case", load_golden(), ids=lambda c: c[0])
def test_hand_worked_blocks(orc, case):
    name, g, xs, sf, codes, by = case
    x = bf16_bits([xs])
    assert np.all(torch.tensor([xs], dtype=torch.float32).to(torch.bfloat16).float().numpy() == np.float32(xs)), \
        "golden inputs must be exact bf16 values"
    q = orc.quantize(x, global_in=g)
    assert q.sf_rm[0, 0] == sf
    assert bytes(q.codes[0].tolist()) == by
    lo, hi = q.codes[0] & 0xF, q.codes[0] >> 4
    got = np.stack([lo, hi], 1).reshape(-1)
    assert got.tolist() == codes


def test_global_scale_definition(orc):
    x = bf16_bits([[0.5, -3.0, 2.0, 1.0] * 4])
    assert orc.tensor_amax(x) == np.float32(3.0)
    assert orc.global_from_amax(3.0) == np.float32(2688.0) / np.float32(3.0)
    assert orc.global_from_amax(0.0) == np.float32(1.0)            # all-zero tensor
    assert orc.global_from_amax(np.float32(1e-40)) == np.float32(1.0)  # 2688/amax overflows
    q = orc.quantize(bf16_bits(np.zeros((2, 32))))
    assert q.g == np.float32(1.0) and not q.sf_rm.any() and not q.codes.any()


def grid_tensor(rng, rows, k, p, jmax):
    """Grid values times 2^(p-j_block); every block holds +-6*2^(p-j) once."""
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    vals = rng.choice(grid, (rows, k)) * rng.choice([-1, 1], (rows, k))
    j = rng.integers(0, jmax + 1, (rows, k // 16))
    j[0, 0] = 0  # the tensor amax is 6*2^p
    pos = rng.integers(0, 16, (rows, k // 16))
    for r in range(rows):
        for b in range(k // 16):
            vals[r, b * 16 + pos[r, b]] = 6.0 * rng.choice([-1, 1])
    scale = np.repeat(np.exp2(p - j), 16, axis=1)
    return vals * scale, j


@pytest.mark.parametrize("p", [-5, 0, 3])
def test_closed_form_round_trip(orc, p):
    rng = np.random.default_rng(10 + p)
    x, j = grid_tensor(rng, 37, 96, p, jmax=6)
    q = orc.quantize(bf16_bits(x))
    # amax = 6*2^p -> g = 448*2^-p; block scale = 448*2^-j exactly
    assert q.g == np.float32(448.0 * 2.0 ** -p)
    expect_sf = orc.e4m3_encode((448.0 * np.exp2(-j)).astype(np.float32))
    np.testing.assert_array_equal(q.sf_rm, expect_sf)
    np.testing.assert_array_equal(orc.dequantize(q), x)


@pytest.mark.parametrize("qexp", [-7, -1, 1, 6])
def test_homogeneity(orc, qexp):
    rng = np.random.default_rng(20)
    x = rng.standard_normal((19, 160)).astype(np.float32)
    q0 = orc.quantize(bf16_bits(x))
    q1 = orc.quantize(bf16_bits(x * 2.0 ** qexp))
    np.testing.assert_array_equal(q0.codes, q1.codes)
    np.testing.assert_array_equal(q0.sf_rm, q1.sf_rm)
    assert q1.g == np.float32(q0.g * 2.0 ** -qexp)


def test_sign_symmetry(orc):
    rng = np.random.default_rng(21)
    x = rng.standard_normal((23, 128)).astype(np.float32)
    x[0, :5] = 0.0
    q0 = orc.quantize(bf16_bits(x))
    q1 = orc.quantize(bf16_bits(-x))
    np.testing.assert_array_equal(q1.codes, q0.codes ^ 0x88)
    np.testing.assert_array_equal(q1.sf_rm, q0.sf_rm)
    assert q0.g == q1.g


def block_max_err_bound(amax_b):
    # |x - x_hat| <= dec(s)/g <= (1 + 2^-4) * amax_b / 6 for a normal scale
    return (1 + 2.0 ** -4) * amax_b / 6.0 * (1 + 1e-6)


def test_outlier_locality_fixed_global(orc):
    rng = np.random.default_rng(22)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    ch = 37
    x2 = x.copy()
    x2[:, ch] *= 50.0
    g = np.float32(100.0)
    q0, q1 = orc.quantize(bf16_bits(x), g), orc.quantize(bf16_bits(x2), g)
    blk = ch // 16
    other = np.ones(256 // 16, bool)
    other[blk] = False
    np.testing.assert_array_equal(q0.sf_rm[:, other], q1.sf_rm[:, other])
    codes_other = np.ones(128, bool)
    codes_other[blk * 8:(blk + 1) * 8] = False
    np.testing.assert_array_equal(q0.codes[:, codes_other], q1.codes[:, codes_other])
    assert (q0.sf_rm[:, blk] != q1.sf_rm[:, blk]).any()


def test_outlier_locality_dynamic_global(orc):
    """With a dynamic global the outlier moves g, but each other block's error
    stays bounded by that block's own amax; per-tensor scaling (one scale for
    the whole tensor) would not."""
    rng = np.random.default_rng(23)
    x = rng.standard_normal((256, 512)).astype(np.float32)
    chans = [5, 300]
    x[:, chans] *= 50.0
    xb = bf16_bits(x)
    xf = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).double().numpy()
    q = orc.quantize(xb)
    err = np.abs(orc.dequantize(q) - xf)
    amax_b = np.abs(xf).reshape(256, 32, 16).max(axis=2)
    errb = err.reshape(256, 32, 16).max(axis=2)
    ds = orc.e4m3_value(q.sf_rm)
    normal = ds >= 2.0 ** -6
    outlier_blocks = np.zeros(32, bool)
    outlier_blocks[[c // 16 for c in chans]] = True
    mask = normal & ~outlier_blocks[None, :]
    assert mask.mean() > 0.9
    assert np.all(errb[mask] <= block_max_err_bound(amax_b[mask]))
    # contrast: one scale for the whole tensor (E2M1 x amax/6) swamps small values
    s_tensor = np.abs(xf).max() / 6.0
    per_tensor = orc.e2m1_value(orc.e2m1_encode((xf / s_tensor).astype(np.float32))) * s_tensor
    per_tensor_err = np.abs(per_tensor - xf).reshape(256, 32, 16).max(axis=2)
    assert np.median(per_tensor_err[mask]) > 5 * np.median(errb[mask])


def test_block_error_bound_random(orc):
    rng = np.random.default_rng(24)
    x = (rng.standard_normal((128, 512)) * np.exp2(rng.integers(-3, 4, (128, 1)))).astype(np.float32)
    xb = bf16_bits(x)
    xf = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).double().numpy()
    q = orc.quantize(xb)
    errb = np.abs(orc.dequantize(q) - xf).reshape(128, 32, 16).max(axis=2)
    amax_b = np.abs(xf).reshape(128, 32, 16).max(axis=2)
    normal = orc.e4m3_value(q.sf_rm) >= 2.0 ** -6
    assert np.all(errb[normal] <= block_max_err_bound(amax_b[normal]))


def test_static_global_saturates(orc):
    x = bf16_bits(np.full((1, 32), 3.0))
    q = orc.quantize(x, global_in=1e6)       # s = E4M3(0.5e6) saturates
    assert np.all(q.sf_rm == 0x7E)
    assert np.all(q.codes == 0x77)           # 3 * 1e6/448 >> 6 -> code 7


# ------------------------------------------------------------------ layout --

def test_swizzle_hand_offsets(orc):
    # k = 80: 5 blocks per row -> padded to 8 -> 2 atoms per 128-row block
    k = 80
    assert orc.sf_bytes(130, k) == 256 * 8
    cases = {(0, 0): 0, (0, 3): 3, (0, 4): 512, (1, 0): 16, (32, 0): 4,
             (33, 2): 16 + 4 + 2, (96, 1): 12 + 1, (127, 4): 512 + 31 * 16 + 12,
             (128, 0): 1024, (129, 4): 1024 + 512 + 16}
    for (r, c), off in cases.items():
        assert orc.sf_offset(r, c, k) == off, (r, c)


@pytest.mark.parametrize("rows,k", [(1, 16), (130, 80), (256, 512), (48, 5120)])
def test_swizzle_bijection_and_padding(orc, rows, k):
    nb = k // 16
    offs = np.array([[orc.sf_offset(r, c, k) for c in range(nb)] for r in range(rows)])
    total = orc.sf_bytes(rows, k)
    assert len(np.unique(offs)) == rows * nb and offs.min() >= 0 and offs.max() < total
    rng = np.random.default_rng(25)
    sf = rng.integers(1, 256, (rows, nb), dtype=np.uint8)
    sw = orc.sf_swizzle(sf, rows, k)
    pad = np.ones(total, bool)
    pad[offs.reshape(-1)] = False
    assert not sw[pad].any()
    np.testing.assert_array_equal(orc.sf_unswizzle(sw, rows, k), sf)
