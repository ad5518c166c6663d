"""Seeded synthetic workloads: shapes and value distributions only.

This module holds no arithmetic of the method.  It is the one piece that both
the CUDA path and the CPU oracle are fed from: tests and bench.py draw inputs
here, then hand the same bits to each side.

All tensors are torch bf16 (bit patterns are what matter).  Every draw uses its
own torch.Generator on the requested device; the same (seed, device) always
yields the same bits.

Workloads (weights of LLaMA-shaped layers stand in for real checkpoints; no
dataset or trained weight is involved):
  pr1      one 1024x1024 weight, N(0, 0.02^2); X 32x1024; r=16, alpha=16
  llama7b  q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008; N(0,0.02^2);
           2048 tokens (4 x 512); r=64, alpha=16
  llama70b 80 layers of q,o 8192x8192; k,v 1024x8192; gate,up 28672x8192;
           down 8192x28672; N(0, 0.015^2) per (layer, matrix) seed; 512 tokens;
           r=64, alpha=16
  decode   28672x8192 and 8192x28672, N(0,0.02^2); M in {1,4,16}; r=16, alpha=16
  robust   4095x11007 Student-t(3) scaled to std 0.02, 0.1% of entries x20;
           4096 tokens; r=8, alpha=32
X and dY are N(0,1); LoRA factors A [K,r] and B [r,N] are N(0, 0.01^2) (B is
not zero so the low-rank path is exercised).
"""
from dataclasses import dataclass, field
import math
import torch

LLAMA7B = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
           ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
LLAMA70B = [("q", 8192, 8192), ("k", 1024, 8192), ("v", 1024, 8192), ("o", 8192, 8192),
            ("gate", 28672, 8192), ("up", 28672, 8192), ("down", 8192, 28672)]
DECODE = [("gate", 28672, 8192), ("down", 8192, 28672)]


@dataclass
class Workload:
    name: str
    mats: list                 # [(name, rows N, cols K)]
    tokens: int                # M
    r: int
    alpha: float
    w_std: float
    w_kind: str = "normal"     # "normal" | "student_t_outliers"
    layers: int = 1
    decode_m: tuple = field(default_factory=tuple)

    @property
    def s(self) -> float:
        return float(self.alpha) / float(self.r)


WORKLOADS = {
    "pr1": Workload("pr1", [("w", 1024, 1024)], 32, 16, 16.0, 0.02),
    "llama7b": Workload("llama7b", LLAMA7B, 2048, 64, 16.0, 0.02),
    "llama70b": Workload("llama70b", LLAMA70B, 512, 64, 16.0, 0.015, layers=80),
    "decode": Workload("decode", DECODE, 16, 16, 16.0, 0.02, decode_m=(1, 4, 16)),
    "robust": Workload("robust", [("w", 4095, 11007)], 4096, 8, 32.0, 0.02,
                       w_kind="student_t_outliers"),
}


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weight(rows, cols, std, seed, device="cpu", kind="normal"):
    """bf16 [rows, cols] weight drawn from the workload's distribution."""
    g = _gen(seed, device)
    if kind == "normal":
        w = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * std
    elif kind == "student_t_outliers":
        # Student-t with 3 degrees of freedom = Z / sqrt(chi2_3 / 3); its
        # variance is 3, so scaling by std/sqrt(3) gives standard deviation std.
        z = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
        c = torch.zeros_like(z)
        for _ in range(3):
            e = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
            c += e * e
        w = z / torch.sqrt(c / 3.0) * (std / math.sqrt(3.0))
        mask = torch.rand(rows, cols, generator=g, device=device) < 0.001
        w = torch.where(mask, w * 20.0, w)
        del z, c
    else:
        raise ValueError(kind)
    return w.to(torch.bfloat16)


def normal(shape, std, seed, device="cpu"):
    g = _gen(seed, device)
    return (torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def layer_inputs(M, N, K, r, seed, device="cpu"):
    """X [M,K], dY [M,N] ~ N(0,1); A [K,r], B [r,N] ~ N(0, 0.01^2)."""
    return dict(
        X=normal((M, K), 1.0, seed * 4 + 1, device),
        dY=normal((M, N), 1.0, seed * 4 + 2, device),
        A=normal((K, r), 0.01, seed * 4 + 3, device),
        B=normal((r, N), 0.01, seed * 4 + 4, device),
    )


def matrix_seed(workload: str, layer: int, index: int, base: int = 0) -> int:
    """Seed of one weight: base + index for single-layer sets, base + 16*layer + index
    for the 80-layer model."""
    if workload == "llama70b":
        return base + 16 * layer + index
    return base + index


def bits(t: torch.Tensor):
    """bf16 torch tensor -> numpy uint16 bit patterns (host copy)."""
    return t.contiguous().view(torch.int16).cpu().numpy().view("uint16")


def from_bits(a, device="cpu"):
    """numpy uint16 bit patterns -> bf16 torch tensor."""
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
