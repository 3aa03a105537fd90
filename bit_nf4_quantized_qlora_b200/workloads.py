"""Seeded synthetic inputs for the QLoRA linear layer.

This module only draws random numbers: it holds none of the layer's
arithmetic (no quantization, no products).  Tests, the benchmark and the
oracle-side checks all take their inputs from here, so both sides of a parity
check see the same values.  Every tensor is drawn on the CPU from its own
``torch.Generator`` seed in fp32 and, where the layer consumes bf16, cast to
bf16 by torch.

The shapes stand in for the models the QLoRA pages size by hand (7B, 65B and
70B bases; LoRA rank 16 with alpha 32 as in the bitsandbytes/PEFT snippet of
"QLoRA and Quantized Training", 'In code').  Weights are N(0, sigma) like the
zero-centred normal weights NF4 is built for ("A 65B fine-tune on the GPU you
already have", figure 3), optionally with a fraction of 10-sigma outliers.
"""

from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch


def normal(shape: Sequence[int], std: float, seed: int) -> torch.Tensor:
    """fp32 N(0, std) on the CPU from a private generator."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32) * float(std)


def weight(n: int, k: int, std: float, seed: int,
           outlier_frac: float = 0.0, outlier_sigma: float = 10.0) -> torch.Tensor:
    """fp32 W [n x k] ~ N(0, std); a fraction of entries (chosen uniformly
    without replacement from a second seeded stream) is set to
    +-outlier_sigma * std with a random sign."""
    w = normal((n, k), std, seed)
    if outlier_frac > 0.0:
        numel = n * k
        cnt = int(round(outlier_frac * numel))
        g = torch.Generator(device="cpu")
        g.manual_seed(int(seed) * 7919 + 17)
        idx = torch.randperm(numel, generator=g)[:cnt]
        sign = torch.randint(0, 2, (cnt,), generator=g).to(torch.float32) * 2.0 - 1.0
        w.view(-1)[idx] = sign * float(outlier_sigma) * float(std)
    return w


def bf16(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.bfloat16)


@dataclass
class LinearCase:
    """One NF4 + LoRA linear: shapes, LoRA knobs and the seeds of its inputs."""
    name: str
    n: int                      # out features (rows of W)
    k: int                      # in features
    m: int                      # tokens (rows of X)
    r: int                      # LoRA rank
    alpha: float                # LoRA alpha; the scale is alpha / r
    w_std: float = 0.02
    w_seed: int = 1
    x_seed: int = 2
    a_seed: int = 3
    b_seed: int = 4
    dy_seed: int = 5
    lora_std: float = 0.01
    outlier_frac: float = 0.0

    @property
    def scale(self) -> float:
        return float(self.alpha) / float(self.r) if self.r > 0 else 0.0

    def W(self) -> torch.Tensor:
        return weight(self.n, self.k, self.w_std, self.w_seed, self.outlier_frac)

    def X(self, m: Optional[int] = None) -> torch.Tensor:
        return bf16(normal((self.m if m is None else m, self.k), 1.0, self.x_seed))

    def A(self) -> torch.Tensor:
        return bf16(normal((self.r, self.k), self.lora_std, self.a_seed))

    def B(self) -> torch.Tensor:
        return bf16(normal((self.n, self.r), self.lora_std, self.b_seed))

    def dY(self, m: Optional[int] = None) -> torch.Tensor:
        return bf16(normal((self.m if m is None else m, self.n), 1.0, self.dy_seed))

    def with_m(self, m: int) -> "LinearCase":
        c = LinearCase(**{f: getattr(self, f) for f in self.__dataclass_fields__})
        c.m = m
        c.name = f"{self.name}_m{m}"
        return c


# --- the five workloads -----------------------------------------------------

def single_linear() -> LinearCase:
    """W [1024 x 1024], X [16 x 1024], r=16, alpha=32."""
    return LinearCase("single_1024", n=1024, k=1024, m=16, r=16, alpha=32.0,
                      w_seed=1, x_seed=2, a_seed=3, b_seed=4, dy_seed=5)


def attn_proj_7b(m: int = 1) -> LinearCase:
    """7B-shaped attention projection W [4096 x 4096] with 0.1 % outliers at
    10 sigma, decode-sized M in {1, 4, 16}, r=16, alpha=32."""
    return LinearCase(f"attn_proj_4096_m{m}", n=4096, k=4096, m=m, r=16, alpha=32.0,
                      w_seed=11, x_seed=12, a_seed=13, b_seed=14, dy_seed=15,
                      outlier_frac=0.001)


def mlp_7b(which: str, m: int = 4096) -> LinearCase:
    """7B-shaped MLP projections, X [4096 x in], r=64, alpha=16.
    gate/up: W [11008 x 4096]; down: W [4096 x 11008]."""
    if which == "gate":
        return LinearCase(f"mlp_gate_11008x4096_m{m}", n=11008, k=4096, m=m, r=64, alpha=16.0,
                          w_seed=21, x_seed=24, a_seed=26, b_seed=27, dy_seed=28)
    if which == "up":
        return LinearCase(f"mlp_up_11008x4096_m{m}", n=11008, k=4096, m=m, r=64, alpha=16.0,
                          w_seed=22, x_seed=24, a_seed=29, b_seed=30, dy_seed=32)
    if which == "down":
        return LinearCase(f"mlp_down_4096x11008_m{m}", n=4096, k=11008, m=m, r=64, alpha=16.0,
                          w_seed=23, x_seed=25, a_seed=33, b_seed=34, dy_seed=35)
    raise ValueError(which)


def up_proj_70b(m: int = 1) -> LinearCase:
    """70B-shaped MLP up-projection W [28672 x 8192] ~ N(0, 0.015), r=16,
    alpha=32, M swept over {1, 16, 128, 1024, 8192}."""
    return LinearCase(f"up_proj_28672x8192_m{m}", n=28672, k=8192, m=m, r=16, alpha=32.0,
                      w_std=0.015, w_seed=31, x_seed=36, a_seed=37, b_seed=38, dy_seed=39)


M_SWEEP_70B = (1, 16, 128, 1024, 8192)
M_SWEEP_ATTN = (1, 4, 16)


@dataclass
class DecoderLayerCase:
    """Synthetic 7B-shaped decoder layer: hidden 4096, 32 heads of 128,
    SwiGLU MLP 11008, q/k/v/o/gate/up/down all NF4 + LoRA r=64 alpha=16,
    activations [2 x 2048 x 4096]."""
    batch: int = 2
    seq: int = 2048
    hidden: int = 4096
    heads: int = 32
    mlp: int = 11008
    r: int = 64
    alpha: float = 16.0
    x_seed: int = 41
    w_seeds: Sequence[int] = field(default_factory=lambda: (42, 43, 44, 45, 46, 47, 48))
    grad_seed: int = 49
    w_std: float = 0.02

    PROJ = ("q", "k", "v", "o", "gate", "up", "down")

    def proj_shape(self, name: str):
        h, f = self.hidden, self.mlp
        return {"q": (h, h), "k": (h, h), "v": (h, h), "o": (h, h),
                "gate": (f, h), "up": (f, h), "down": (h, f)}[name]

    def W(self, name: str) -> torch.Tensor:
        n, k = self.proj_shape(name)
        return weight(n, k, self.w_std, self.w_seeds[self.PROJ.index(name)])

    def A(self, name: str) -> torch.Tensor:
        n, k = self.proj_shape(name)
        return bf16(normal((self.r, k), 0.01, 100 + self.w_seeds[self.PROJ.index(name)]))

    def B(self, name: str) -> torch.Tensor:
        n, k = self.proj_shape(name)
        return bf16(normal((n, self.r), 0.01, 200 + self.w_seeds[self.PROJ.index(name)]))

    def X(self) -> torch.Tensor:
        return bf16(normal((self.batch, self.seq, self.hidden), 1.0, self.x_seed))

    def grad(self) -> torch.Tensor:
        return bf16(normal((self.batch, self.seq, self.hidden), 1.0, self.grad_seed))
