"""GPU tests of nvfp4_linear, the W4A4 linear layer in one call (news article
"Qwen3.8-27B最激进4bit量化开源…" §02: activations quantized to NVFP4 on the fly,
then the GEMM on the 4-bit tensor cores), and of the few-token GEMM's split-K
reduction.

nvfp4_linear must equal nvfp4_quantize followed by nvfp4_gemm bit for bit (it
runs the same kernels, only launched to overlap), and both agree with the
oracle within the GEMM tolerance (parity.py). Weights come from the oracle.
"""
import numpy as np
import pytest
import torch

from parity import bits, gemm_check, norms, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    from nvfp4_w4a4_quantized_elem_b200 import build, nvfp4
    build.build()
    return nvfp4


def gaussian(rows, k, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((rows, k), generator=g) * sigma).to(torch.bfloat16)


def counter_bytes(n):
    """Split counters at the start of a GEMM / linear workspace (nvfp4.h):
    4 per 128 weight rows, at least 64 x 16 (the paired kernel's split-K),
    4 bytes each, rounded up to 256."""
    return -(-(4 * max(4 * -(-n // 128), 64 * 16)) // 256) * 256


@pytest.mark.parametrize("m", [1, 8, 16, 17, 32, 33, 64, 65, 300])
@pytest.mark.parametrize("static", [False, True])
def test_linear_equals_quantize_then_gemm(nv, orc, m, static):
    """Few-token (m <= 64, K split) and paired (m > 64) GEMMs behind the
    quantizer; the result is the two-call chain's."""
    k, n = 2048, 1000  # 8 weight tiles: few-token calls split K across the GPU
    x = gaussian(m, k, 100 + m)
    qw = orc.quantize(bits(gaussian(n, k, 5, 0.02)))
    W = upload(qw)
    xd = x.cuda()
    g = None
    if static:
        # a static global from a calibration that saw a larger amax
        g = torch.tensor([float(orc.global_from_amax(orc.tensor_amax(bits(x)) * 1.5))],
                         dtype=torch.float32, device="cuda")
    ws = nv.linear_workspace(m, n, k)
    gws = torch.empty(max(16, nv.gemm_workspace_bytes(m, n, k)), dtype=torch.uint8,
                      device="cuda")
    qx = orc.quantize(bits(x), None if g is None else np.float32(g.item()))
    ref = orc.gemm(qx, qw)
    for dt in (torch.bfloat16, torch.float32):
        y = nv.linear(xd, W, out_dtype=dt, global_scale=g, workspace=ws)
        A = nv.quantize(xd, global_scale=g)
        y2 = nv.gemm(A, W, out_dtype=dt, workspace=gws if m <= 64 else None)
        torch.cuda.synchronize()
        assert torch.equal(y, y2), f"m={m} static={static} {dt}: linear != quantize + gemm"
        gemm_check(y, ref, norms(orc, qx), norms(orc, qw), f"linear m={m} static={static} {dt}")
    if m <= 64:
        assert int(ws[:counter_bytes(n)].count_nonzero()) == 0, "split counters not reset"
    assert nv.read_fault() == 0


@pytest.mark.parametrize("m,k", [(8, 4096), (7, 2336), (8, 5120), (2, 65536)])
@pytest.mark.parametrize("static", [False, True])
def test_linear_in_kernel_token_quantization(nv, orc, m, k, static):
    """At most 8 tokens are quantized inside the few-token GEMM. Its dynamic
    global comes from the kernel's own max over X up to 64 KiB of bf16 (8 x
    4096: exactly the bound; 7 x 2336: a ragged last k-tile), from the amax
    pass's partials above that (8 x 5120, 2 x 65536), or from a static
    global; every way equals quantize + GEMM bit for bit, and the oracle
    within the tolerance."""
    n = 640
    x = gaussian(m, k, 31 * m + k)
    qw = orc.quantize(bits(gaussian(n, k, 32, 0.02)))
    W = upload(qw)
    g = None
    if static:
        g = torch.tensor([float(orc.global_from_amax(orc.tensor_amax(bits(x)) * 1.25))],
                         dtype=torch.float32, device="cuda")
    xd = x.cuda()
    y = nv.linear(xd, W, out_dtype=torch.float32, global_scale=g,
                  workspace=nv.linear_workspace(m, n, k))
    gws = torch.empty(nv.gemm_workspace_bytes(m, n, k), dtype=torch.uint8, device="cuda")
    y2 = nv.gemm(nv.quantize(xd, global_scale=g), W, out_dtype=torch.float32, workspace=gws)
    torch.cuda.synchronize()
    assert torch.equal(y, y2), (m, k, static)
    qx = orc.quantize(bits(x), None if g is None else np.float32(g.item()))
    gemm_check(y, orc.gemm(qx, qw), norms(orc, qx), norms(orc, qw), f"in-kernel m={m} k={k}")
    assert nv.read_fault() == 0


@pytest.mark.parametrize("m,k", [(1, 32), (3, 96), (8, 160), (5, 288), (12, 96)])
def test_linear_short_k(nv, orc, m, k):
    """K shorter than one 256-element k-tile, or one k-tile and a ragged
    rest: the token tile's columns past K are zero-filled by the TMA and the
    in-kernel quantizer writes zero codes and scales for their blocks (the
    12-token case runs the separate quantizer for comparison)."""
    n = 384
    x = gaussian(m, k, 7 * m + k)
    qw = orc.quantize(bits(gaussian(n, k, 8, 0.02)))
    W = upload(qw)
    xd = x.cuda()
    y = nv.linear(xd, W, out_dtype=torch.float32, workspace=nv.linear_workspace(m, n, k))
    gws = torch.empty(max(16, nv.gemm_workspace_bytes(m, n, k)), dtype=torch.uint8, device="cuda")
    y2 = nv.gemm(nv.quantize(xd), W, out_dtype=torch.float32, workspace=gws)
    torch.cuda.synchronize()
    assert torch.equal(y, y2), (m, k)
    qx = orc.quantize(bits(x))
    gemm_check(y, orc.gemm(qx, qw), norms(orc, qx), norms(orc, qw), f"short k m={m} k={k}")
    assert nv.read_fault() == 0


@pytest.mark.parametrize("case", ["zeros", "one_outlier", "tiny_and_huge", "zero_rows"])
def test_linear_in_kernel_special_values(nv, orc, case):
    """The in-kernel token quantization on X the quantizer's edge cases are
    made of: all zeros (amax 0, g = 1), one huge outlier among N(0,1) values,
    subnormal-range next to large magnitudes, and all-zero rows among
    ordinary ones. The tokens' quantization equals nvfp4_quantize's bit for
    bit (the same GEMM follows), and the oracle agrees within the tolerance
    wherever the reference output is non-zero."""
    m, k, n = 5, 1024, 256
    x = gaussian(m, k, 77)
    if case == "zeros":
        x = torch.zeros((m, k), dtype=torch.bfloat16)
    elif case == "one_outlier":
        x[2, 517] = 3.0e4
    elif case == "tiny_and_huge":
        x[:, ::2] = x[:, ::2] * 1e-30
        x[:, 1::64] = 6.0e4
    else:
        x[1] = 0.0
        x[3] = 0.0
    x = x.to(torch.bfloat16)
    qw = orc.quantize(bits(gaussian(n, k, 78, 0.02)))
    W = upload(qw)
    xd = x.cuda()
    for g in (None, torch.tensor([float(orc.global_from_amax(max(orc.tensor_amax(bits(x)), 1.0)))],
                                 dtype=torch.float32, device="cuda")):
        y = nv.linear(xd, W, out_dtype=torch.float32, global_scale=g,
                      workspace=nv.linear_workspace(m, n, k))
        gws = torch.empty(max(16, nv.gemm_workspace_bytes(m, n, k)), dtype=torch.uint8,
                          device="cuda")
        y2 = nv.gemm(nv.quantize(xd, global_scale=g), W, out_dtype=torch.float32, workspace=gws)
        torch.cuda.synchronize()
        assert torch.equal(y, y2), (case, g is None)
        qx = orc.quantize(bits(x), None if g is None else np.float32(g.item()))
        ref = orc.gemm(qx, qw)
        if np.linalg.norm(ref) > 0:
            gemm_check(y, ref, norms(orc, qx), norms(orc, qw), f"special {case}")
        else:
            assert float(y.abs().max()) == 0.0
    assert nv.read_fault() == 0


def test_linear_strided_and_ragged_x(nv, orc):
    """x with a row pitch larger than k, and k not a multiple of 256 (the last
    k-tile of every slice is partial): linear equals the chain."""
    for m, k, n in [(3, 2080, 640), (40, 2080, 640), (1, 5152, 1000)]:
        big = gaussian(m, k + 64, 21 + m).cuda()
        x = big[:, :k]
        W = nv.quantize(gaussian(n, k, 22, 0.02).cuda())
        y = nv.linear(x, W)
        gws = torch.empty(max(16, nv.gemm_workspace_bytes(m, n, k)), dtype=torch.uint8,
                          device="cuda")
        y2 = nv.gemm(nv.quantize(x), W, workspace=gws if m <= 64 else None)
        torch.cuda.synchronize()
        assert torch.equal(y, y2), (m, k, n)
    assert nv.read_fault() == 0


@pytest.mark.parametrize("m", [1, 32])
def test_split_k_is_deterministic(nv, m):
    """Decode shape 17408 -> 5120 (40 weight tiles, K in 3 slices): repeated
    calls give identical bits, and the counters are zero afterwards."""
    k, n = 17408, 5120
    x = gaussian(m, k, 9).cuda()
    W = nv.quantize(gaussian(n, k, 10, 0.02).cuda())
    ws = nv.linear_workspace(m, n, k)
    ys = [nv.linear(x, W, workspace=ws).clone() for _ in range(3)]
    gws = torch.empty(nv.gemm_workspace_bytes(m, n, k), dtype=torch.uint8, device="cuda")
    A = nv.quantize(x)
    gs = [nv.gemm(A, W, workspace=gws).clone() for _ in range(3)]
    torch.cuda.synchronize()
    for y in ys[1:] + gs:
        assert torch.equal(y, ys[0])
    assert int(ws[:counter_bytes(n)].count_nonzero()) == 0
    assert int(gws[:counter_bytes(n)].count_nonzero()) == 0
    assert nv.read_fault() == 0


def test_linear_graph_replay(nv):
    """A decode step captured once as a CUDA graph and replayed with new
    activations written into the same input buffer gives the eager result."""
    m, k, n = 1, 5120, 17408
    W = nv.quantize(gaussian(n, k, 3, 0.02).cuda())
    x = gaussian(m, k, 4).cuda()
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    ws = nv.linear_workspace(m, n, k)
    nv.linear(x, W, out=y, workspace=ws)  # first call on the device outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        nv.linear(x, W, out=y, workspace=ws)
    for seed in (4, 5, 6):
        x.copy_(gaussian(m, k, seed).cuda())
        g.replay()
        torch.cuda.synchronize()
        ref = nv.linear(x, W, workspace=nv.linear_workspace(m, n, k))
        torch.cuda.synchronize()
        assert torch.equal(y, ref), f"graph replay differs for input seed {seed}"
    assert nv.read_fault() == 0


def test_linear_decode_full_size_against_oracle(nv, orc):
    """The decode configuration at full size, sampled output columns against
    the oracle (weights from the oracle, activations quantized on the GPU)."""
    from nvfp4_w4a4_quantized_elem_b200 import workloads as wl
    cfg = wl.decode(8, 17408, 5120)
    x = cfg.x()
    qw = orc.quantize(bits(cfg.w()))
    y = nv.linear(x.cuda(), upload(qw))
    torch.cuda.synchronize()
    qx = orc.quantize(bits(x))
    ref = orc.gemm(qx, qw)
    gemm_check(y, ref, norms(orc, qx), norms(orc, qw), "decode 8x17408->5120")
    assert nv.read_fault() == 0


def test_linear_reused_workspace_with_stale_padding(nv, orc):
    """nvfp4_linear leaves the scale bytes of its private quantized X's
    padding rows unwritten for fewer than 32 tokens (only its GEMM reads them,
    against zero-filled codes). A workspace that held a 31-token and then a
    256-token call's data gives a 1-token call the bits of quantize + GEMM,
    and the oracle's result within the tolerance, for both GEMM kernels'
    reuse orders."""
    k, n = 5120, 2048
    qw = orc.quantize(bits(gaussian(n, k, 9, 0.02)))
    W = upload(qw)
    nb = max(nv.linear_workspace_bytes(m, n, k) for m in (1, 31, 256))
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    for m_prev in (31, 256):
        nv.linear(gaussian(m_prev, k, m_prev).cuda(), W, workspace=ws)
    x = gaussian(1, k, 4242)
    y = nv.linear(x.cuda(), W, out_dtype=torch.float32, workspace=ws)
    gws = torch.empty(nv.gemm_workspace_bytes(1, n, k), dtype=torch.uint8, device="cuda")
    y2 = nv.gemm(nv.quantize(x.cuda()), W, out_dtype=torch.float32, workspace=gws)  # same split
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    qx = orc.quantize(bits(x))
    gemm_check(y, orc.gemm(qx, qw), norms(orc, qx), norms(orc, qw), "stale padding")
    assert nv.read_fault() == 0
