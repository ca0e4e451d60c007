"""GPU parity of nvfp4_gemm against the FP64 oracle GEMM of the dequantized
operands (news article "Qwen3.8-27B最激进4bit量化开源…" §02: W4A4 GEMM on the
4-bit tensor cores). Operands are quantized by the oracle and uploaded, so a
GEMM failure cannot hide behind a quantizer failure. Tolerance: parity.py.
"""
import numpy as np
import pytest
import torch

from parity import assert_quant_equal, bits, gemm_check, norms, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    from nvfp4_w4a4_quantized_elem_b200 import build, nvfp4
    build.build()
    return nvfp4


def gaussian(rows, k, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((rows, k), generator=g) * sigma).to(torch.bfloat16)


def run_case(nv, orc, x, w, dtypes=(torch.bfloat16, torch.float32), what="",
             workspaces=(False, True)):
    """Both output dtypes; with and without a GEMM workspace (few-token GEMMs
    split K across CTAs only when one is given)."""
    qa, qb = orc.quantize(bits(x)), orc.quantize(bits(w))
    ref = orc.gemm(qa, qb)
    rn, cn = norms(orc, qa), norms(orc, qb)
    A, B = upload(qa), upload(qb)
    m, n, k = qa.rows, qb.rows, qa.k
    for use_ws in workspaces:
        ws = None
        if use_ws:
            nbytes = nv.gemm_workspace_bytes(m, n, k)
            if nbytes == 0:
                continue
            ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")  # garbage
        for dt in dtypes:
            # the output row pitch must be a multiple of 16 bytes: pad it
            per16 = 16 // torch.tensor([], dtype=dt).element_size()
            ld = -(-n // per16) * per16
            y = nv.gemm(A, B, out=torch.empty((m, ld), dtype=dt, device="cuda")[:, :n],
                        workspace=ws)
            torch.cuda.synchronize()
            gemm_check(y, ref, rn, cn, f"{what} {dt} workspace={use_ws}")
    assert nv.read_fault() == 0


def test_gemm_tiny(nv, orc):
    from nvfp4_w4a4_quantized_elem_b200 import workloads as wl
    cfg = wl.tiny()
    run_case(nv, orc, cfg.x(), cfg.w(), what="tiny")


@pytest.mark.parametrize("m,n,k", [(1, 8, 32), (7, 48, 64), (130, 136, 96), (128, 256, 256),
                                   (300, 520, 288), (129, 257, 1024), (256, 512, 5120),
                                   (513, 1000, 2080)])
def test_gemm_ragged(nv, orc, m, n, k):
    run_case(nv, orc, gaussian(m, k, m + k), gaussian(n, k, n + 2 * k, 0.02), what=f"{m}x{n}x{k}")


def test_gemm_output_pitch(nv, orc):
    x, w = gaussian(100, 256, 1), gaussian(200, 256, 2, 0.02)
    qa, qb = orc.quantize(bits(x)), orc.quantize(bits(w))
    ref = orc.gemm(qa, qb)
    big = torch.full((100, 264), 7.0, dtype=torch.bfloat16, device="cuda")
    y = nv.gemm(upload(qa), upload(qb), out=big[:, :200])
    torch.cuda.synchronize()
    gemm_check(y, ref, norms(orc, qa), norms(orc, qb), "pitched")
    assert torch.all(big[:, 200:] == 7.0)  # nothing written past n


def test_gemm_zero_scales_and_extremes(nv, orc):
    # rows spanning 40 binades (subnormal and zero block scales) and all-zero rows
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((256, 512)) * np.exp2(rng.uniform(-30, 8, (256, 1)))).astype(np.float32)
    x[10] = 0.0
    w = (rng.standard_normal((384, 512)) * 0.02).astype(np.float32)
    run_case(nv, orc, torch.from_numpy(x).to(torch.bfloat16),
             torch.from_numpy(w).to(torch.bfloat16), what="extremes")


def test_gemm_outlier_config_full(nv, orc):
    """X 8192x5120 (8 outlier channels x50) @ W 5120x5120: GPU quantizes X and
    W (checked bit-exact), GPU GEMM vs the full FP64 oracle GEMM."""
    from nvfp4_w4a4_quantized_elem_b200 import workloads as wl
    cfg = wl.outlier()
    x, w = cfg.x(), cfg.w()
    A, B = nv.quantize(x.cuda()), nv.quantize(w.cuda())
    qa, qb = orc.quantize(bits(x)), orc.quantize(bits(w))
    assert_quant_equal(A, qa, "X")
    assert_quant_equal(B, qb, "W")
    y = nv.gemm(A, B)
    torch.cuda.synchronize()
    ref = orc.gemm(qa, qb)
    gemm_check(y, ref, norms(orc, qa), norms(orc, qb), "outlier full")


@pytest.mark.parametrize("m", [1, 8, 32, 128, 256])
@pytest.mark.parametrize("k,n", [(5120, 17408), (17408, 5120)])
def test_gemm_decode_shapes(nv, orc, m, k, n):
    from nvfp4_w4a4_quantized_elem_b200 import workloads as wl
    cfg = wl.decode(m, k, n)
    run_case(nv, orc, cfg.x(), cfg.w(), dtypes=(torch.bfloat16,), what=cfg.name)


@pytest.mark.parametrize("m", [1, 16, 17, 100, 255])
def test_gemm_few_tokens_split_k(nv, orc, m):
    """Few-token path with K split across CTAs (N = 1000: 8 weight tiles,
    so most of the GPU works on K slices) and ragged token counts."""
    run_case(nv, orc, gaussian(m, 2048, 7 * m), gaussian(1000, 2048, 11, 0.02), what=f"split m={m}")


@pytest.mark.parametrize("m,n,k", [(200, 1024, 8192), (300, 512, 12288), (256, 256, 16384),
                                   (65, 2560, 8192)])
def test_gemm_paired_split_k(nv, orc, m, n, k):
    """Paired kernel with K cut into 2-4 slices (few 256x256 tiles, long K):
    within the tolerance in both output dtypes, bit-identical from run to
    run (the last slice of each region sums the partials in slice order,
    whichever slice finishes last), and nvfp4_linear (which takes the same
    split from its workspace) gives the same bits as nvfp4_gemm."""
    x, w = gaussian(m, k, 3 * m + k), gaussian(n, k, 5 * n + k, 0.02)
    assert nv.gemm_workspace_bytes(m, n, k) > 0
    run_case(nv, orc, x, w, what=f"split-K {m}x{n}x{k}", workspaces=(True,))
    qa, qb = orc.quantize(bits(x)), orc.quantize(bits(w))
    A, B = upload(qa), upload(qb)
    ws = torch.zeros(nv.gemm_workspace_bytes(m, n, k), dtype=torch.uint8, device="cuda")
    ys = [nv.gemm(A, B, out_dtype=torch.float32, workspace=ws) for _ in range(3)]
    torch.cuda.synchronize()
    assert all(torch.equal(ys[0], y) for y in ys[1:])
    y_lin = nv.linear(x.cuda(), nv.quantize(w.cuda()), out_dtype=torch.float32)
    y_gemm = nv.gemm(nv.quantize(x.cuda()), nv.quantize(w.cuda()), out_dtype=torch.float32,
                     workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y_lin, y_gemm)
    assert nv.read_fault() == 0
