"""Seeded synthetic inputs shaped like the projections of a 27B hybrid LLM.

This module only draws random numbers; it holds none of the quantization
arithmetic, so both the CUDA path and the CPU oracle can consume its tensors.
The pages (arXiv 2609.04098 and its write-ups) evaluate a trained 27B hybrid
model on benchmark suites; no weights or data are available, so these seeded
Gaussian tensors stand in for them, with the shapes of the model's linear
layers and the residual-stream outlier channels the abstract describes
(mechanism (i): "extreme outliers" of the residual stream).

Recipe (every tensor): ``torch.Generator().manual_seed(seed)``, FP32
``randn`` times sigma, optional outlier channels multiplied in FP32, then one
round-to-nearest-even cast to bf16. Outlier channels are
``randperm(K, seed=2)[:n_outliers]``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

SEED_X = 0
SEED_W = 1
SEED_OUTLIER = 2


def gaussian_bf16(rows: int, cols: int, sigma: float, seed: int,
                  outlier_channels: torch.Tensor | None = None,
                  outlier_factor: float = 1.0) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    t = torch.randn((rows, cols), generator=g, dtype=torch.float32)
    t.mul_(sigma)
    if outlier_channels is not None and len(outlier_channels):
        t[:, outlier_channels] *= outlier_factor
    return t.to(torch.bfloat16)


def outlier_channels(k: int, n: int, seed: int = SEED_OUTLIER) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    return torch.randperm(k, generator=g)[:n]


@dataclass
class Linear:
    """One W4A4 linear layer problem: X [m, k] activations, W [n, k] weights."""
    name: str
    m: int
    n: int
    k: int
    x_sigma: float = 1.0
    w_sigma: float = 0.02
    n_outliers: int = 0
    outlier_factor: float = 1.0
    x_seed: int = SEED_X
    w_seed: int = SEED_W

    def x(self, rows: int | None = None) -> torch.Tensor:
        ch = outlier_channels(self.k, self.n_outliers) if self.n_outliers else None
        t = gaussian_bf16(self.m, self.k, self.x_sigma, self.x_seed, ch, self.outlier_factor)
        return t if rows is None else t[:rows].contiguous()

    def w(self) -> torch.Tensor:
        return gaussian_bf16(self.n, self.k, self.w_sigma, self.w_seed)

    @property
    def flops(self) -> int:
        return 2 * self.m * self.n * self.k


@dataclass
class FusedGroup:
    """A fused projection group: modules concatenated along the output dim."""
    name: str
    m: int
    k: int
    modules: list = field(default_factory=list)   # (name, rows, sigma, seed)
    x_sigma: float = 1.0

    def x(self) -> torch.Tensor:
        return gaussian_bf16(self.m, self.k, self.x_sigma, SEED_X)

    def weights(self) -> list[torch.Tensor]:
        return [gaussian_bf16(rows, self.k, sigma, seed)
                for (_, rows, sigma, seed) in self.modules]

    @property
    def n(self) -> int:
        return sum(r for (_, r, _, _) in self.modules)

    @property
    def flops(self) -> int:
        return 2 * self.m * self.n * self.k


# --- the five workloads ------------------------------------------------------

def tiny() -> Linear:
    """X 64x256 ~N(0,1), W 256x256 ~N(0,0.02)."""
    return Linear("tiny", m=64, n=256, k=256)


def outlier() -> Linear:
    """Prefill projection 8192 tokens x 5120 -> 5120, X ~N(0,1) with 8 fixed
    random channels x50 (residual-stream outliers), W ~N(0,0.02)."""
    return Linear("outlier", m=8192, n=5120, k=5120, n_outliers=8, outlier_factor=50.0)


def gdn_fused() -> FusedGroup:
    """GDN in_proj group (qkv, z, a, b) at 8192 tokens, K = 5120."""
    return FusedGroup("gdn_fused", m=8192, k=5120, modules=[
        ("qkv", 8192, 0.02, 1), ("z", 4096, 0.02, 2),
        ("a", 48, 0.1, 3), ("b", 48, 0.005, 4)])


@dataclass
class MLP:
    """Gated MLP at 32K prefill tokens: gate_up [2*ffn, d] -> silu*mul -> down."""
    name: str = "mlp32k"
    m: int = 32768
    d: int = 5120
    ffn: int = 17408
    n_outliers: int = 5        # round(0.1% of 5120)
    outlier_factor: float = 30.0

    def x(self, rows: int | None = None) -> torch.Tensor:
        ch = outlier_channels(self.d, self.n_outliers)
        t = gaussian_bf16(self.m, self.d, 1.0, SEED_X, ch, self.outlier_factor)
        return t if rows is None else t[:rows].contiguous()

    def w_gate_up(self) -> torch.Tensor:
        return gaussian_bf16(2 * self.ffn, self.d, 0.02, SEED_W)

    def w_down(self) -> torch.Tensor:
        return gaussian_bf16(self.d, self.ffn, 0.015, SEED_W + 1)

    @property
    def flops(self) -> int:
        return 2 * self.m * (2 * self.ffn) * self.d + 2 * self.m * self.d * self.ffn


def mlp32k() -> MLP:
    return MLP()


DECODE_M = (1, 8, 32, 128, 256)
DECODE_KN = ((5120, 17408), (17408, 5120))


def decode(m: int, k: int, n: int) -> Linear:
    """Decode-shaped skinny GEMM: M tokens, weights [n, k] ~N(0,0.02)."""
    return Linear(f"decode_m{m}_k{k}_n{n}", m=m, n=n, k=k)


@dataclass
class Gates:
    """The GDN gate projections a and b (48 heads each, the gdn_fused group's
    modules: W_a ~N(0,0.1), W_b ~N(0,0.005)) on X ~N(0,1), with per-head gate
    parameters drawn the way Gated DeltaNet layers are initialised:
    A = exp(A_log) ~ U(1, 16) and dt ~ log-uniform on [1e-3, 1e-1] with
    dt_bias = softplus^-1(dt) = log(expm1(dt)). FP64 parameters, seeds 5, 6."""
    name: str = "gates"
    m: int = 8192
    k: int = 5120
    heads: int = 48

    def x(self, rows: int | None = None) -> torch.Tensor:
        t = gaussian_bf16(self.m, self.k, 1.0, SEED_X)
        return t if rows is None else t[:rows].contiguous()

    def w_a(self, sigma: float = 0.1) -> torch.Tensor:
        """sigma 0.1 as in the gdn_fused group; smaller values give the O(1)
        gate pre-activations of a trained layer."""
        return gaussian_bf16(self.heads, self.k, sigma, 3)

    def w_b(self) -> torch.Tensor:
        return gaussian_bf16(self.heads, self.k, 0.005, 4)

    def a_log(self) -> torch.Tensor:
        g = torch.Generator().manual_seed(5)
        return torch.log(1.0 + 15.0 * torch.rand(self.heads, generator=g, dtype=torch.float64))

    def dt_bias(self) -> torch.Tensor:
        g = torch.Generator().manual_seed(6)
        u = torch.rand(self.heads, generator=g, dtype=torch.float64)
        dt = torch.exp(torch.log(torch.tensor(1e-3, dtype=torch.float64)) +
                       u * (torch.log(torch.tensor(1e-1, dtype=torch.float64)) -
                            torch.log(torch.tensor(1e-3, dtype=torch.float64))))
        return torch.log(torch.expm1(dt))


def gates() -> Gates:
    return Gates()
