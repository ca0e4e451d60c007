"""GPU parity of the calibrated static global (nvfp4_calibrate_global) and of
the gate_up GEMM with SwiGLU + NVFP4 quantization of h fused into its epilogue
(nvfp4_gemm_swiglu_quant).

Pages: every linear layer is W4A4 and activation scales are calibrated on a
frozen set (news article "Qwen3.8-27B最激进4bit量化开源…" §03). The fused
kernel must reproduce, bit for bit, the unfused chain GEMM -> silu*mul ->
static quantize (itself checked against the oracle), and its h codes/scales
must equal the oracle's quantization of that chain's bf16 h.
"""
import numpy as np
import pytest
import torch

from parity import assert_quant_equal, assert_row_blocks_equal, bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    from nvfp4_w4a4_quantized_elem_b200 import build, nvfp4
    build.build()
    return nvfp4


def gaussian(rows, k, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((rows, k), generator=g) * sigma).to(torch.bfloat16)


def test_calibrate_global_running_max(nv, orc):
    cal = nv.Calibrator()
    xs = [gaussian(200, 512, s, sigma) for s, sigma in [(1, 1.0), (2, 3.0), (3, 0.5)]]
    for x in xs:
        cal.observe(x.cuda())
    torch.cuda.synchronize()
    amax = max(float(orc.tensor_amax(bits(x))) for x in xs)
    assert cal.running_amax.item() == amax
    g = cal.global_scale.cpu().numpy()[0]
    assert g.view(np.uint32) == orc.global_from_amax(amax).view(np.uint32)
    # static-mode quantization with the calibrated global matches the oracle
    q = nv.quantize(xs[0].cuda(), global_scale=cal.global_scale)
    assert_quant_equal(q, orc.quantize(bits(xs[0]), global_in=g), "static")


def unfused_h(nv, A, Bi, ffn):
    """GEMM with the interleaved weight, columns put back, then silu*mul."""
    y = nv.gemm(A, Bi)
    m = y.shape[0]
    yb = y.view(m, ffn // 128, 2, 128)
    gate = yb[:, :, 0, :].reshape(m, ffn)
    up = yb[:, :, 1, :].reshape(m, ffn)
    return nv.silu_mul(torch.cat([gate, up], dim=1).contiguous())


@pytest.mark.parametrize("m,ffn,k", [(65, 384, 512), (300, 256, 288), (1000, 640, 1024)])
def test_swiglu_quant_equals_unfused_chain(nv, orc, m, ffn, k):
    x = gaussian(m, k, 5 * m)
    w = gaussian(2 * ffn, k, 7 * ffn, 0.02)
    A = nv.quantize(x.cuda())
    Bi = nv.quantize(nv.interleave_gate_up(w.cuda()))
    h = unfused_h(nv, A, Bi, ffn)
    cal = nv.Calibrator()
    gh = cal.observe(h)
    ref = nv.quantize(h, global_scale=gh)
    fused = nv.gemm_swiglu_quant(A, Bi, gh)
    torch.cuda.synchronize()
    assert torch.equal(fused.codes, ref.codes)
    assert torch.equal(fused.sf, ref.sf)
    g = gh.cpu().numpy()[0]
    assert_quant_equal(fused, orc.quantize(bits(h.cpu()), global_in=g), "fused vs oracle")
    assert nv.read_fault() == 0


def test_swiglu_quant_mlp32k_full(nv, orc):
    """The 32K-token MLP: X 32768x5120, gate_up 34816x5120 (interleaved)."""
    from nvfp4_w4a4_quantized_elem_b200 import workloads as wl
    cfg = wl.mlp32k()
    A = nv.quantize(cfg.x().cuda())
    Bi = nv.quantize(nv.interleave_gate_up(cfg.w_gate_up().cuda()))
    h = unfused_h(nv, A, Bi, cfg.ffn)
    gh = nv.Calibrator().observe(h)
    ref = nv.quantize(h, global_scale=gh)
    fused = nv.gemm_swiglu_quant(A, Bi, gh)
    torch.cuda.synchronize()
    assert torch.equal(fused.codes, ref.codes)
    assert torch.equal(fused.sf, ref.sf)
    # whole 128-row blocks (codes and their swizzled scale bytes) vs the oracle
    blocks = np.sort(np.random.default_rng(3).choice(cfg.m // 128, 4, replace=False))
    g = gh.cpu().numpy()[0]
    assert_row_blocks_equal(orc, fused, lambda r0, r1: h[r0:r1].cpu(), blocks, g, "fused h")
    assert nv.read_fault() == 0


@pytest.mark.parametrize("m,ffn,k", [(65, 384, 512), (300, 256, 288), (1000, 640, 1024),
                                     (2048, 1024, 768)])
def test_swiglu_quant_dynamic_equals_unfused_chain(nv, orc, m, ffn, k):
    """Dynamic global of h: the fused GEMM (bf16 h + per-CTA max|h|) followed
    by the quantizer equals GEMM -> silu*mul -> dynamic quantize bit for bit,
    and the oracle's dynamic quantization of the same bf16 h."""
    x = gaussian(m, k, 11 * m)
    w = gaussian(2 * ffn, k, 13 * ffn, 0.02)
    A = nv.quantize(x.cuda())
    Bi = nv.quantize(nv.interleave_gate_up(w.cuda()))
    h = unfused_h(nv, A, Bi, ffn)
    ref = nv.quantize(h)
    ws = nv.swiglu_quant_dynamic_workspace(m, ffn)
    fused = nv.gemm_swiglu_quant_dynamic(A, Bi, workspace=ws)
    torch.cuda.synchronize()
    h_ws = ws[:m * ffn * 2].view(torch.bfloat16).view(m, ffn)
    assert torch.equal(h_ws, h)
    assert torch.equal(fused.codes, ref.codes)
    assert torch.equal(fused.sf, ref.sf)
    assert torch.equal(fused.global_scale, ref.global_scale)
    assert_quant_equal(fused, orc.quantize(bits(h.cpu())), "fused dynamic vs oracle")
    # a second call into the same workspace (stale partials and h) agrees
    fused2 = nv.gemm_swiglu_quant_dynamic(A, Bi, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(fused2.codes, ref.codes) and torch.equal(fused2.sf, ref.sf)
    assert nv.read_fault() == 0


def test_swiglu_quant_dynamic_mlp32k_full(nv, orc):
    """The 32K-token MLP's gate_up with the dynamic global of h: equal to the
    unfused chain bit for bit; g_h equal to the oracle's 2688 / max|h| over
    the whole h; whole 128-row blocks equal to the oracle's quantization."""
    from nvfp4_w4a4_quantized_elem_b200 import workloads as wl
    cfg = wl.mlp32k()
    A = nv.quantize(cfg.x().cuda())
    Bi = nv.quantize(nv.interleave_gate_up(cfg.w_gate_up().cuda()))
    h = unfused_h(nv, A, Bi, cfg.ffn)
    ref = nv.quantize(h)
    fused = nv.gemm_swiglu_quant_dynamic(A, Bi)
    torch.cuda.synchronize()
    assert torch.equal(fused.codes, ref.codes)
    assert torch.equal(fused.sf, ref.sf)
    h_host = h.cpu()
    g = orc.global_from_amax(orc.tensor_amax(bits(h_host)))
    assert fused.global_scale.cpu().numpy()[0].view(np.uint32) == np.float32(g).view(np.uint32)
    blocks = np.sort(np.random.default_rng(4).choice(cfg.m // 128, 4, replace=False))
    assert_row_blocks_equal(orc, fused, lambda r0, r1: h_host[r0:r1], blocks, g, "dynamic h")
    assert nv.read_fault() == 0
