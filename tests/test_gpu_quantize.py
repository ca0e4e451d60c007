"""GPU parity of nvfp4_quantize against the oracle: bit-exact codes, swizzled
scale bytes (padding included) and global scale.

Format: news article "Qwen3.8-27B最激进4bit量化开源…" §02 (E2M1 values, one
E4M3 scale per 16 elements, one FP32 global per tensor).
"""
import numpy as np
import pytest
import torch

from parity import assert_quant_equal, bits, from_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    from nvfp4_w4a4_quantized_elem_b200 import build, nvfp4
    build.build()
    assert torch.cuda.is_available()
    return nvfp4


def gaussian(rows, k, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((rows, k), generator=g) * sigma).to(torch.bfloat16)


def check(nv, orc, x_cpu, global_in=None, what=""):
    xg = x_cpu.cuda()
    gin = None if global_in is None else torch.tensor([global_in], dtype=torch.float32, device="cuda")
    out = nv.quantize(xg, global_scale=gin)
    torch.cuda.synchronize()
    ref = orc.quantize(bits(x_cpu), global_in=global_in)
    assert_quant_equal(out, ref, what)
    return out, ref


@pytest.mark.parametrize("rows,k", [(64, 256), (1, 16), (5, 48), (127, 80), (129, 272),
                                    (300, 5120), (2, 17408), (257, 1040)])
def test_quantize_shapes(nv, orc, rows, k):
    check(nv, orc, gaussian(rows, k, seed=rows * 7 + k), what=f"{rows}x{k}")


def test_quantize_strided_rows(nv, orc):
    base = gaussian(70, 256, seed=3)
    xg = base.cuda()[:, :160]          # ldx = 256 > k = 160
    out = nv.quantize(xg)
    ref = orc.quantize(bits(base[:, :160].contiguous()))
    assert_quant_equal(out, ref, "strided")


def test_quantize_every_bf16_value(nv, orc):
    b = np.arange(1 << 16, dtype=np.uint32)
    f = (b << 16).view(np.float32)
    finite = b[np.isfinite(f)].astype(np.uint16)
    rng = np.random.default_rng(0)
    rng.shuffle(finite)
    n = (len(finite) // 256) * 256
    x = from_bits(finite[:n].reshape(-1, 256))
    for gin in (None, 1.0, 3.0e30):
        check(nv, orc, x, gin, what=f"all-bf16 g={gin}")


def test_quantize_every_bf16_as_block_amax(nv, orc):
    """One block per non-negative finite bf16 value v = [v, -v/2, 0, ...]:
    every possible block amax goes through the scale computation, under
    globals that put amax/6*g across the whole E4M3 range."""
    b = np.arange(0, 0x7F80, dtype=np.uint32)
    v = (b << 16).view(np.float32)
    x = np.zeros((len(v), 16), np.float32)
    x[:, 0] = v
    x[:, 1] = -v / 2
    xb = torch.from_numpy(x).to(torch.bfloat16)
    for gin in (1.0, 2.0 ** 100, 2.0 ** -100, 3.0, 1e30):
        check(nv, orc, xb, gin, what=f"block amax sweep g={gin}")


def test_quantize_each_block_scale_path(nv, orc):
    # blocks whose amax spans the whole E4M3 range relative to one global,
    # including subnormal and zero scales (signed-zero codes)
    rng = np.random.default_rng(1)
    mags = np.exp2(rng.uniform(-40, 5, (512, 1)))
    x = torch.from_numpy((rng.standard_normal((512, 64)) * mags).astype(np.float32)).to(torch.bfloat16)
    check(nv, orc, x, what="wide dynamic range")
    check(nv, orc, x, global_in=2.0 ** -10, what="tie to zero scale")
    check(nv, orc, x, global_in=448.0, what="static 448")


def test_quantize_zeros_and_signed_zeros(nv, orc):
    x = torch.zeros((130, 64), dtype=torch.bfloat16)
    x[1::2] = -0.0
    out, _ = check(nv, orc, x, what="zeros")
    assert out.global_scale.item() == 1.0


def test_quantize_golden_blocks_on_gpu(nv, orc):
    from test_oracle_quantize import load_golden
    for name, g, xs, sf, codes, by in load_golden():
        x = torch.tensor([xs], dtype=torch.float32).to(torch.bfloat16)
        out = nv.quantize(x.cuda(), torch.tensor([g], device="cuda"))
        assert bytes(out.codes.cpu().numpy()[0].tolist()) == by, name
        assert out.sf.cpu().numpy()[0] == sf, name


def test_quantize_outlier_config_full(nv, orc):
    """X 8192x5120 ~N(0,1) with 8 channels x50, W 5120x5120 ~N(0,0.02)."""
    from nvfp4_w4a4_quantized_elem_b200 import workloads as wl
    cfg = wl.outlier()
    check(nv, orc, cfg.x(), what="outlier X")
    check(nv, orc, cfg.w(), what="outlier W")


def test_quantize_deterministic_and_reuses_workspace(nv, orc):
    x = gaussian(1000, 512, seed=5).cuda()
    ws = torch.empty(nv.quantize_workspace_bytes(1000, 512), dtype=torch.uint8, device="cuda")
    a = nv.quantize(x, workspace=ws)
    ws.fill_(0xFF)  # garbage in the workspace must not matter
    b = nv.quantize(x, workspace=ws)
    assert torch.equal(a.codes, b.codes) and torch.equal(a.sf, b.sf)
    assert torch.equal(a.global_scale, b.global_scale)


@pytest.mark.parametrize("rows,k", [(2, 16384), (2, 16400), (1, 32768), (3, 16384)])
def test_quantize_one_pass_bound(nv, orc, rows, k):
    """Dynamic quantization on both sides of NVFP4_ONE_PASS_MAX_BYTES (64 KiB
    of x: one kernel that takes the max itself; above it: amax pass, then
    the quantizer). The tensor's largest magnitude sits in the last element,
    so a max that stops short of the end changes g and every scale."""
    x = gaussian(rows, k, seed=rows + k)
    x[-1, -1] = -40.0
    assert (rows * k * 2 <= nv.ONE_PASS_MAX_BYTES) == (rows * k <= 32768)
    out, ref = check(nv, orc, x, what=f"{rows}x{k}")
    assert out.global_scale.item() == np.float32(2688.0) / np.float32(40.0)


@pytest.mark.parametrize("rows", [70, 300])
def test_quantize_dynamic_ignores_row_padding(nv, orc, rows):
    """x with ldx > k and a large value in every row's padding: the global
    comes from the first k columns only, in the one-kernel path (70 rows,
    22 KiB) and behind the amax pass (300 rows, 94 KiB)."""
    base = gaussian(rows, 256, seed=rows)
    base[:, 160:] = 1.0e4
    out = nv.quantize(base.cuda()[:, :160])
    ref = orc.quantize(bits(base[:, :160].contiguous()))
    assert_quant_equal(out, ref, f"padded rows={rows}")
