"""GPU parity of the fused-group repair, silu*mul and the two multi-step
workloads (GDN in_proj group, gated MLP at 32K tokens).

Fold: news article "Qwen3.8-27B最激进4bit量化开源…" §03 — a fused GDN
in_proj (qkv, z, a, b) is put on one global scale with the ratio folded into
the E4M3 block scales. Scale bytes and g* are compared bit-exactly; the fused
GEMM under the tolerance of parity.py.
"""
import numpy as np
import pytest
import torch

from parity import assert_quant_equal, bits, from_bits, gemm_check, norms, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    from nvfp4_w4a4_quantized_elem_b200 import build, nvfp4
    build.build()
    return nvfp4


def quantize_group_on_gpu(nv, weights):
    """Quantize each module with its own global straight into its row slice
    of one fused code buffer; returns (per-module NVFP4Tensors, fused codes)."""
    k = weights[0].shape[1]
    total = sum(w.shape[0] for w in weights)
    codes = torch.empty((total, k // 2), dtype=torch.uint8, device="cuda")
    mods, r0 = [], 0
    for w in weights:
        out = nv.NVFP4Tensor(codes[r0:r0 + w.shape[0]],
                             torch.empty(nv.sf_bytes(w.shape[0], k), dtype=torch.uint8, device="cuda"),
                             torch.empty(1, dtype=torch.float32, device="cuda"), w.shape[0], k)
        mods.append(nv.quantize(w.cuda(), out=out))
        r0 += w.shape[0]
    return mods, codes


@pytest.mark.parametrize("rows,k", [((256, 128, 48, 48), 512), ((40, 8, 200), 96),
                                    ((1, 130, 127), 5120)])
def test_fold_small_groups(nv, orc, rows, k):
    ws = [(torch.randn((r, k), generator=torch.Generator().manual_seed(i)) * s).to(torch.bfloat16)
          for i, (r, s) in enumerate(zip(rows, (0.02, 0.1, 0.005, 0.03)))]
    mods, codes = quantize_group_on_gpu(nv, ws)
    ref_mods = [orc.quantize(bits(w)) for w in ws]
    for m, r in zip(mods, ref_mods):
        assert_quant_equal(m, r, "module")
    sf, g = nv.fuse_group_scales(mods)
    fused = nv.NVFP4Tensor(codes, sf, g, sum(rows), k)
    assert_quant_equal(fused, orc.fuse_group(ref_mods), "fused")


def test_gdn_fused_group_full(nv, orc):
    """qkv 8192, z 4096, a 48, b 48 rows (K = 5120), X 8192x5120: fold on the
    GPU, then one fused GEMM N = 12384, checked on 512 sampled rows."""
    from nvfp4_w4a4_quantized_elem_b200 import workloads as wl
    cfg = wl.gdn_fused()
    ws = cfg.weights()
    mods, codes = quantize_group_on_gpu(nv, ws)
    ref_mods = [orc.quantize(bits(w)) for w in ws]
    for m, r in zip(mods, ref_mods):
        assert_quant_equal(m, r, "module")
    sf, g = nv.fuse_group_scales(mods)
    W = nv.NVFP4Tensor(codes, sf, g, cfg.n, cfg.k)
    ref_w = orc.fuse_group(ref_mods)
    assert_quant_equal(W, ref_w, "fused")
    x = cfg.x()
    A = nv.quantize(x.cuda())
    qa = orc.quantize(bits(x))
    assert_quant_equal(A, qa, "X")
    y = nv.gemm(A, W)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(0).choice(cfg.m, 512, replace=False))
    ref = orc.gemm(qa, ref_w, a_rows=rows)
    gemm_check(y[torch.from_numpy(rows).cuda()], ref, norms(orc, qa, rows), norms(orc, ref_w),
               "gdn fused")
    # the a-gate columns [12288, 12336) carry the repaired scale, not the b-gate's
    naive = orc.fuse_group_naive(ref_mods)
    ref_naive = orc.gemm(qa, naive, a_rows=rows[:64])
    ya = y[torch.from_numpy(rows[:64]).cuda(), 12288:12336].float().cpu().numpy()
    err_fixed = np.linalg.norm(ya - ref[:64, 12288:12336]) / np.linalg.norm(ref[:64, 12288:12336])
    err_naive = np.linalg.norm(ref_naive[:, 12288:12336] - ref[:64, 12288:12336]) / \
        np.linalg.norm(ref[:64, 12288:12336])
    assert err_fixed < 1e-2 and err_naive > 0.5


def test_silu_mul_parity(nv, orc):
    g = torch.Generator().manual_seed(9)
    y = (torch.randn((300, 2 * 1040), generator=g) * 3).to(torch.bfloat16)
    h = nv.silu_mul(y.cuda())
    torch.cuda.synchronize()
    ref = from_bits(orc.silu_mul(bits(y))).float()
    got = h.float().cpu()
    ulp = torch.clamp(ref.abs(), min=2.0 ** -126) * 2.0 ** -7
    assert torch.all((got - ref).abs() <= ulp)


def test_silu_mul_extremes(nv, orc):
    """silu*mul over the whole useful range of the gate, bf16 values from
    -128 to 128 (every value the cast gives there, both signs of up): the
    fast exponential and division and the large-negative branch stay within
    one bf16 ulp of the FP64 oracle, zeros and subnormals included."""
    gate = torch.linspace(-128.0, 128.0, 65536).to(torch.bfloat16).unique()
    n = (gate.numel() // 8) * 8
    gate = gate[:n]
    up = torch.tensor([1.0, -3.5, 0.0078125, 200.0], dtype=torch.bfloat16)
    y = torch.cat([gate.repeat(4, 1), up[:, None].expand(4, n)], dim=1).contiguous()
    h = nv.silu_mul(y.cuda())
    torch.cuda.synchronize()
    ref = from_bits(orc.silu_mul(bits(y))).float()
    got = h.float().cpu()
    ulp = torch.clamp(ref.abs(), min=2.0 ** -126) * 2.0 ** -7
    bad = (got - ref).abs() > ulp
    assert not torch.any(bad), (gate.repeat(4, 1)[bad][:5], got[bad][:5], ref[bad][:5])


def test_mlp32k_pipeline_full(nv, orc):
    """X 32768x5120 (5 outlier channels x30) -> gate_up W 34816x5120 ->
    silu*mul -> requantize h (dynamic global) -> down W 5120x17408, all on the
    GPU. Checks: quantized X, W, h bit-exact (h from the GPU's own silu*mul
    output); silu*mul within 1 bf16 ulp; both GEMMs on 1024 sampled rows."""
    from nvfp4_w4a4_quantized_elem_b200 import workloads as wl
    cfg = wl.mlp32k()
    x = cfg.x()
    wgu = cfg.w_gate_up()
    A = nv.quantize(x.cuda())
    Wgu = nv.quantize(wgu.cuda())
    y = nv.gemm(A, Wgu)
    h = nv.silu_mul(y)
    H = nv.quantize(h)
    del wgu
    wd = cfg.w_down()
    Wd = nv.quantize(wd.cuda())
    out = nv.gemm(H, Wd)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(1).choice(cfg.m, 1024, replace=False))
    ridx = torch.from_numpy(rows).cuda()

    qa = orc.quantize(bits(x))
    assert_quant_equal(A, qa, "X")
    qgu = orc.quantize(bits(cfg.w_gate_up()))
    assert_quant_equal(Wgu, qgu, "W gate_up")
    ref_y = orc.gemm(qa, qgu, a_rows=rows)
    gemm_check(y[ridx], ref_y, norms(orc, qa, rows), norms(orc, qgu), "gate_up")
    del qgu

    y_rows = y[ridx].cpu()
    ref_h = from_bits(orc.silu_mul(bits(y_rows))).float()
    ulp = torch.clamp(ref_h.abs(), min=2.0 ** -126) * 2.0 ** -7
    assert torch.all((h[ridx].float().cpu() - ref_h).abs() <= ulp)

    qh = orc.quantize(bits(h.cpu()))
    assert_quant_equal(H, qh, "h")
    qd = orc.quantize(bits(wd))
    assert_quant_equal(Wd, qd, "W down")
    ref_out = orc.gemm(qh, qd, a_rows=rows)
    gemm_check(out[ridx], ref_out, norms(orc, qh, rows), norms(orc, qd), "down")
    assert nv.read_fault() == 0
