"""GPU gate-sensitivity measurement against the same measurement on the
oracle (abstract of arXiv 2609.04098; paper reading §4.2 (ii)): quantization
is bit-exact and the GEMM within tolerance, so every error figure must agree
to a small fraction of itself."""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_quantized_elem_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_gate_sensitivity_matches_oracle(orc):
    from nvfp4_w4a4_quantized_elem_b200 import build, gate_sensitivity, nvfp4
    build.build()
    rows = 512
    gpu = gate_sensitivity.measure(rows=rows)
    cfg = wl.gates()
    x = cfg.x(rows)
    qx = orc.quantize(bits(x))
    xf = x.double().numpy()
    wb = cfg.w_b()
    qb = orc.quantize(bits(wb))
    for r in gpu:
        wa = cfg.w_a(r["sigma_a"])
        qa = orc.quantize(bits(wa))
        y = orc.gemm(qx, orc.fuse_group([qa, qb]))
        ref = orc.gate_sensitivity(xf @ wa.double().numpy().T, xf @ wb.double().numpy().T,
                                   y[:, :48], y[:, 48:], cfg.a_log().numpy(),
                                   cfg.dt_bias().numpy())
        for key in ("gemm_a", "gemm_b", "g", "alpha", "beta"):
            assert r[key] == pytest.approx(ref[key], rel=0.02), (r["sigma_a"], key)
    assert nvfp4.read_fault() == 0
