"""Oracle pins of the GDN gate functions and of the synthetic gate-sensitivity
measurement (abstract of arXiv 2609.04098 and paper reading §4.2 (ii): the
softplus/exp and sigmoid gate parameterizations compress the W4A4 GEMM error;
news article §03: a fused group served with the largest global but unrepaired
block scales distorts the gate projection).

Gate functions are pinned to closed forms and to the derivative bounds that
make them compress (sigmoid' <= 1/4, softplus' <= 1); the measurement to the
order of magnitude the pages report."""
import math

import numpy as np
import pytest
import torch

from nvfp4_w4a4_quantized_elem_b200 import workloads as wl


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_softplus_sigmoid_closed_forms(orc):
    assert orc.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    assert orc.sigmoid(0.0) == 0.5
    z = np.linspace(-40, 40, 8001)
    # softplus(z) - softplus(-z) = z; sigmoid(z) + sigmoid(-z) = 1
    assert np.allclose(orc.softplus(z) - orc.softplus(-z), z, rtol=0, atol=1e-12)
    assert np.allclose(orc.sigmoid(z) + orc.sigmoid(-z), 1.0, rtol=0, atol=1e-15)
    # asymptotes: softplus(z) -> z, softplus(-z) -> exp(-z) for large z
    assert orc.softplus(40.0) == pytest.approx(40.0, rel=1e-15)
    assert orc.softplus(-30.0) == pytest.approx(math.exp(-30.0), rel=1e-12)
    # derivative of softplus is sigmoid (central difference)
    h = 1e-6
    zz = np.linspace(-8, 8, 161)
    d = (orc.softplus(zz + h) - orc.softplus(zz - h)) / (2 * h)
    assert np.allclose(d, orc.sigmoid(zz), atol=1e-8)


def test_gdn_gates_closed_forms(orc):
    a_log = np.log(np.array([1.0, 2.0, 16.0]))
    dt_bias = np.array([-3.0, 0.5, 1.0])
    # a = -dt_bias: softplus(0) = ln 2, so g = -A ln 2 and alpha = 2^-A
    g, alpha, beta = orc.gdn_gates(-dt_bias[None, :], np.zeros((1, 3)), a_log, dt_bias)
    A = np.exp(a_log)
    assert np.allclose(g[0], -A * math.log(2.0), rtol=1e-15)
    assert np.allclose(alpha[0], 2.0 ** -A, rtol=1e-14)
    assert np.all(beta == 0.5)
    assert np.all((alpha > 0) & (alpha < 1))


def test_gate_lipschitz_bounds(orc):
    """|beta(y+e) - beta(y)| <= |e| / 4 and |g(y+e) - g(y)| <= A |e|: the
    gates never amplify an absolute error beyond these slopes."""
    rng = np.random.default_rng(0)
    y = rng.normal(0, 3, (2000, 4))
    e = rng.normal(0, 0.3, (2000, 4))
    a_log = np.log(np.array([1.0, 4.0, 9.0, 16.0]))
    dt = np.array([-2.0, -1.0, 0.0, 1.0])
    g0, _, b0 = orc.gdn_gates(y, y, a_log, dt)
    g1, _, b1 = orc.gdn_gates(y + e, y + e, a_log, dt)
    assert np.all(np.abs(b1 - b0) <= np.abs(e) / 4 + 1e-15)
    assert np.all(np.abs(g1 - g0) <= np.exp(a_log) * np.abs(e) * (1 + 1e-12))


@pytest.fixture(scope="module")
def gate_case(orc):
    cfg = wl.gates()
    x = cfg.x(256)
    qx = orc.quantize(bits(x))
    xf = x.double().numpy()
    wb = cfg.w_b()
    qb = orc.quantize(bits(wb))
    return cfg, qx, xf, wb, qb


@pytest.mark.parametrize("sigma_a", [0.1, 0.005])
def test_sensitivity_measurement(orc, gate_case, sigma_a):
    cfg, qx, xf, wb, qb = gate_case
    wa = cfg.w_a(sigma_a)
    qa = orc.quantize(bits(wa))
    y_a_ref, y_b_ref = xf @ wa.double().numpy().T, xf @ wb.double().numpy().T
    fused = orc.fuse_group([qa, qb])
    y = orc.gemm(qx, fused)
    r = orc.gate_sensitivity(y_a_ref, y_b_ref, y[:, :48], y[:, 48:],
                             cfg.a_log().numpy(), cfg.dt_bias().numpy())
    # NVFP4 W4A4 GEMM error of a Gaussian projection: ~0.13 (the pages: ~11%)
    assert 0.08 < r["gemm_a"] < 0.2 and 0.08 < r["gemm_b"] < 0.2
    # sigmoid on pre-activations of std ~0.36: ~5x compression (the pages: 11% -> 2%)
    assert r["beta"] < r["gemm_b"] / 4
    if sigma_a == 0.005:
        # O(1) pre-activations: the softplus/exp decay compresses too
        assert r["alpha"] < r["gemm_a"] / 4
    else:
        # std ~7 pre-activations: softplus is ~linear, no compression of alpha
        assert r["alpha"] > r["gemm_a"] / 2


def test_unrepaired_fusion_distorts_the_a_gate(orc, gate_case):
    """Serving [a; b] with the largest module global and unchanged block
    scales mis-scales a (whose global is smaller) by their ratio."""
    cfg, qx, xf, wb, qb = gate_case
    wa = cfg.w_a(0.1)
    qa = orc.quantize(bits(wa))
    y_a_ref, y_b_ref = xf @ wa.double().numpy().T, xf @ wb.double().numpy().T
    args = (cfg.a_log().numpy(), cfg.dt_bias().numpy())
    good = orc.gemm(qx, orc.fuse_group([qa, qb]))
    bad = orc.gemm(qx, orc.fuse_group_naive([qa, qb]))
    rg = orc.gate_sensitivity(y_a_ref, y_b_ref, good[:, :48], good[:, 48:], *args)
    rb = orc.gate_sensitivity(y_a_ref, y_b_ref, bad[:, :48], bad[:, 48:], *args)
    assert rb["gemm_a"] > 5 * rg["gemm_a"]
    assert rb["alpha"] > 3 * rg["alpha"]
    assert rb["gemm_b"] == pytest.approx(rg["gemm_b"], rel=0.1)  # b holds the max global
