"""Synthetic gate-sensitivity measurement of the W4A4 path.

The abstract of arXiv 2609.04098 and the paper reading's §4.2 (ii) report that
the GDN gate projections are the least sensitive to NVFP4 W4A4: the softplus /
exponential and sigmoid parameterizations of the gates turn ~11% GEMM error
into ~2% error of the gate values. No trained weights are available, so this
measures the mechanism on seeded synthetic inputs (workloads.Gates): the a and
b projections are quantized and fused into one GEMM exactly as the GDN input
projection group is served (per-module quantization, then the global-scale
repair of nvfp4_fuse_group_scales), multiplied on the GPU in FP32, and
compared with the FP64 product of the unquantized bf16 operands, before and
after the gates:
    g = -exp(A_log) * softplus(a + dt_bias),  alpha = exp(g),  beta = sigmoid(b)
(news article §01 says the gates are parameterized in log space; its formula
did not survive extraction, and this is the Gated DeltaNet form the abstract's
wording describes). Errors are relative Frobenius norms over tokens x heads.

    python -m nvfp4_w4a4_quantized_elem_b200.gate_sensitivity [--rows N]
"""
from __future__ import annotations

import argparse
import json

import torch

from . import nvfp4, workloads

SIGMAS_A = (0.1, 0.02, 0.005)


def _softplus(z: torch.Tensor) -> torch.Tensor:
    return torch.clamp_min(z, 0.0) + torch.log1p(torch.exp(-z.abs()))


def _gates(y_a, y_b, a_log, dt_bias):
    g = -torch.exp(a_log) * _softplus(y_a + dt_bias)
    return g, torch.exp(g), torch.sigmoid(y_b)


def _rel(a: torch.Tensor, b: torch.Tensor) -> float:
    return float(torch.linalg.norm(a - b) / torch.linalg.norm(b))


def measure(rows: int = 8192, sigmas_a=SIGMAS_A, device="cuda") -> list[dict]:
    cfg = workloads.gates()
    x = cfg.x(rows).to(device)
    w_b = cfg.w_b().to(device)
    a_log = cfg.a_log().to(device)
    dt_bias = cfg.dt_bias().to(device)
    X = nvfp4.quantize(x)
    Wb = nvfp4.quantize(w_b)
    xd = x.double()
    y_b_ref = xd @ w_b.double().T
    out = []
    for sa in sigmas_a:
        w_a = cfg.w_a(sa).to(device)
        W = nvfp4.fuse_group([nvfp4.quantize(w_a), Wb])   # the served GEMM: [a; b]
        y = nvfp4.gemm(X, W, out_dtype=torch.float32).double()
        y_a_ref = xd @ w_a.double().T
        h = cfg.heads
        g0, al0, be0 = _gates(y_a_ref, y_b_ref, a_log, dt_bias)
        g1, al1, be1 = _gates(y[:, :h], y[:, h:], a_log, dt_bias)
        out.append({"sigma_a": sa, "rows": rows,
                    "preact_a_std": float(y_a_ref.std()), "preact_b_std": float(y_b_ref.std()),
                    "gemm_a": _rel(y[:, :h], y_a_ref), "gemm_b": _rel(y[:, h:], y_b_ref),
                    "g": _rel(g1, g0), "alpha": _rel(al1, al0), "beta": _rel(be1, be0)})
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--rows", type=int, default=8192)
    args = ap.parse_args()
    for r in measure(args.rows):
        print(json.dumps({k: (round(v, 5) if isinstance(v, float) else v) for k, v in r.items()}))
    if nvfp4.read_fault() != 0:
        raise SystemExit("kernel timeout")


if __name__ == "__main__":
    main()
