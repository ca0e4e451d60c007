"""Pins of the oracle's E2M1 / E4M3 codecs against things other than itself.

Format (news article "Qwen3.8-27B最激进4bit量化开源…" §02): values are 4-bit
E2M1, block scales are E4M3 (OCP FP8 E4M3FN: bias 7, max 448, no infinity).
Pins used here:
  * the grid derived from the E2M1 bit layout (1 sign, 2 exponent bits with
    bias 1, 1 mantissa bit), written independently of the oracle's table;
  * brute-force nearest-grid search (ties -> even code) over every bf16
    value, every tie point +-1 ulp and a random FP32 sweep;
  * torch's float8_e4m3fn decode and its round-to-nearest-even cast.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.filterwarnings("ignore")


def e2m1_grid_from_bits():
    """Value of each 4-bit code from the E2M1 bit layout (bias 1)."""
    vals = []
    for c in range(16):
        s, e, m = c >> 3, (c >> 1) & 3, c & 1
        mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1 + 0.5 * m)
        vals.append(-mag if s else mag)
    return np.array(vals)


def brute_e2m1(v: np.ndarray) -> np.ndarray:
    """Nearest of the 8 magnitudes, ties to the even code, sign from v."""
    grid = np.abs(e2m1_grid_from_bits()[:8])
    # |v| - grid is exact in FP64 while |v| < 2^40; above that every distance
    # would round to the same number, and 2^40 has the same nearest point (6).
    a = np.minimum(np.abs(v.astype(np.float64)), 2.0 ** 40)[:, None]
    d = np.abs(a - grid[None, :])
    best = np.zeros(len(v), np.int64)
    bestd = d[:, 0].copy()
    for c in range(1, 8):
        better = (d[:, c] < bestd) | ((d[:, c] == bestd) & (c % 2 == 0))
        best = np.where(better, c, best)
        bestd = np.where(better, d[:, c], bestd)
    sign = np.signbit(v).astype(np.int64) * 8
    return (best + sign).astype(np.uint8)


def all_finite_bf16_as_f32():
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return f[np.isfinite(f)]


def test_e2m1_grid_matches_bit_layout(orc):
    got = orc.e2m1_value(np.arange(16, dtype=np.uint8))
    np.testing.assert_array_equal(got, e2m1_grid_from_bits())
    # the grid {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}
    assert sorted(set(np.abs(got).tolist())) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e2m1_encode_every_bf16(orc):
    v = all_finite_bf16_as_f32()
    np.testing.assert_array_equal(orc.e2m1_encode(v), brute_e2m1(v))


def test_e2m1_encode_tie_points(orc):
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0], np.float32)
    pts = np.concatenate([mids, np.nextafter(mids, np.float32(0)),
                          np.nextafter(mids, np.float32(100))]).astype(np.float32)
    pts = np.concatenate([pts, -pts])
    np.testing.assert_array_equal(orc.e2m1_encode(pts), brute_e2m1(pts))
    # the stated tie rule, value by value
    expect = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6, 7.0: 7}
    for x, c in expect.items():
        assert orc.e2m1_encode(np.array([x], np.float32))[0] == c
        assert orc.e2m1_encode(np.array([-x], np.float32))[0] == c | 8


def test_e2m1_encode_random_sweep(orc):
    rng = np.random.default_rng(0)
    v = rng.uniform(-8, 8, 1_000_000).astype(np.float32)
    np.testing.assert_array_equal(orc.e2m1_encode(v), brute_e2m1(v))


def test_e2m1_signed_zero_and_saturation(orc):
    v = np.array([0.0, -0.0, -0.1, 1e30, -1e30, np.inf, -np.inf], np.float32)
    np.testing.assert_array_equal(orc.e2m1_encode(v), [0, 8, 8, 7, 15, 7, 15])


# ----------------------------------------------------------------- E4M3 ----

def torch_e4m3_decode(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def torch_e4m3_encode(v: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def test_e4m3_decode_matches_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    finite = (codes & 0x7F) != 0x7F
    ours = orc.e4m3_value(codes)
    ref = torch_e4m3_decode(codes)
    np.testing.assert_array_equal(ours[finite], ref[finite])
    assert np.all(np.isnan(ours[~finite]))


def test_e4m3_range(orc):
    v = orc.e4m3_value(np.arange(128, dtype=np.uint8))
    fin = v[np.isfinite(v)]
    assert fin.max() == 448.0                      # 0x7E
    assert orc.e4m3_value(np.array([0x08], np.uint8))[0] == 2.0 ** -6  # min normal
    assert orc.e4m3_value(np.array([0x01], np.uint8))[0] == 2.0 ** -9  # min subnormal


def test_e4m3_decode_encode_identity(orc):
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = orc.e4m3_value(codes).astype(np.float32)
    np.testing.assert_array_equal(orc.e4m3_encode(vals), codes)


def e4m3_tie_sweep():
    pos = torch_e4m3_decode(np.arange(0x7F, dtype=np.uint8))  # 0 .. 448
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    pts = np.concatenate([pos.astype(np.float32), mids,
                          np.nextafter(mids, np.float32(0)),
                          np.nextafter(mids, np.float32(1000))])
    return np.concatenate([pts, -pts]).astype(np.float32)


def test_e4m3_encode_matches_torch_cast(orc):
    rng = np.random.default_rng(1)
    sweep = np.concatenate([
        e4m3_tie_sweep(),
        rng.uniform(-448, 448, 200_000).astype(np.float32),
        (rng.standard_normal(200_000) * np.exp2(rng.integers(-12, 8, 200_000))).astype(np.float32),
    ])
    sweep = sweep[np.abs(sweep) <= 448]
    np.testing.assert_array_equal(orc.e4m3_encode(sweep), torch_e4m3_encode(sweep))


def test_e4m3_encode_brute_force_nearest(orc):
    pos = orc.e4m3_value(np.arange(0x7F, dtype=np.uint8))  # codes 0..126
    rng = np.random.default_rng(2)
    v = np.concatenate([e4m3_tie_sweep(),
                        rng.uniform(0, 460, 50_000).astype(np.float32)])
    v = np.abs(v)
    d = np.abs(v.astype(np.float64)[:, None] - pos[None, :])
    best = np.argmin(d, axis=1)  # first minimum = lower code
    dmin = d[np.arange(len(v)), best]
    nxt = np.minimum(best + 1, 126)
    tie = d[np.arange(len(v)), nxt] == dmin
    best = np.where(tie & (best % 2 == 1), nxt, best)
    np.testing.assert_array_equal(orc.e4m3_encode(v), best.astype(np.uint8))


def test_e4m3_saturation_and_underflow(orc):
    v = np.array([448, 449, 464, 500, 1e30, np.inf], np.float32)
    assert np.all(orc.e4m3_encode(v) == 0x7E)
    # torch agrees up to 464, then returns NaN: the oracle clamps instead
    np.testing.assert_array_equal(torch_e4m3_encode(np.array([449, 464], np.float32)), [0x7E, 0x7E])
    assert orc.e4m3_encode(np.array([2.0 ** -10], np.float32))[0] == 0x00   # tie -> even 0
    assert orc.e4m3_encode(np.array([3 * 2.0 ** -11], np.float32))[0] == 0x01
    assert orc.e4m3_encode(np.array([2.0 ** -11], np.float32))[0] == 0x00


def test_bf16_rounding_helper(orc):
    rng = np.random.default_rng(3)
    v = (rng.standard_normal(20000) * np.exp2(rng.integers(-30, 30, 20000))).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = np.array([orc.double_to_bf16(float(x)) for x in v], np.uint16)
    np.testing.assert_array_equal(ours, ref)
