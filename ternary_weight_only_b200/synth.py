"""Seeded synthetic inputs and workload shapes.

This module draws random numbers and names shapes; it holds none of the
method's arithmetic (no packing, no dequantisation, no matmul).  The same
tensors feed the CUDA path and, in the tests, the CPU oracle.

Distributions (one synthetic decoder layer at hidden size 5120, a 5120 ->
151936 output head, and prefill blocks):
  * ternary codes: iid uniform over {-1,0,+1}, or P(0)=0.4, P(+-1)=0.3;
  * 1-bit codes: iid uniform over {-1,+1};
  * group scales: fp32 U[0.005, 0.05] rounded to fp16 (round-to-nearest-even);
  * activations: fp32 N(0,1) rounded to fp16, optionally with each element
    independently multiplied by 20 with probability 0.01 (outliers).
"""
from __future__ import annotations

import torch

GROUP = 128

# One synthetic decoder layer at hidden 5120: (name, K, N) with y = x * W^T.
LAYER_PROJ = [
    ("q", 5120, 6144),
    ("k", 5120, 1024),
    ("v", 5120, 1024),
    ("o", 6144, 5120),
    ("gate", 5120, 17408),
    ("up", 5120, 17408),
    ("down", 17408, 5120),
]
HEAD = ("head", 5120, 151936)
N_LAYERS = 64
# Prefill GEMM blocks: (K, N) pairs at M in {2048, 8192}.
PREFILL = [(5120, 17408), (17408, 5120)]
PREFILL_M = (2048, 8192)
VERIFY_M = (2, 4, 8)


def gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def codes_uniform(N: int, K: int, g: torch.Generator, device="cpu") -> torch.Tensor:
    """int8 [N,K], iid uniform over {-1,0,+1}."""
    return (torch.randint(0, 3, (N, K), generator=g, device=device, dtype=torch.int8) - 1)


def codes_sparse(N: int, K: int, g: torch.Generator, p0: float = 0.4, device="cpu") -> torch.Tensor:
    """int8 [N,K], P(0)=p0 and P(-1)=P(+1)=(1-p0)/2."""
    u = torch.rand((N, K), generator=g, device=device)
    half = (1.0 - p0) / 2.0
    out = torch.zeros((N, K), dtype=torch.int8, device=device)
    out[u < half] = -1
    out[u >= half + p0] = 1
    return out


def codes_sign(N: int, K: int, g: torch.Generator, device="cpu") -> torch.Tensor:
    """int8 [N,K], iid uniform over {-1,+1} (the 1-bit variant)."""
    return (torch.randint(0, 2, (N, K), generator=g, device=device, dtype=torch.int8) * 2 - 1)


def scales_uniform(N: int, K: int, g: torch.Generator, lo: float = 0.005, hi: float = 0.05,
                   device="cpu") -> torch.Tensor:
    """fp16 [N, K/128]: fp32 U[lo,hi] rounded to fp16."""
    G = K // GROUP
    return (torch.rand((N, G), generator=g, device=device) * (hi - lo) + lo).to(torch.float16)


def activations(M: int, K: int, g: torch.Generator, outlier_p: float = 0.0,
                outlier_mult: float = 20.0, device="cpu") -> torch.Tensor:
    """fp16 [M,K]: fp32 N(0,1), optionally x outlier_mult with probability outlier_p."""
    x = torch.randn((M, K), generator=g, device=device)
    if outlier_p > 0:
        mask = torch.rand((M, K), generator=g, device=device) < outlier_p
        x = torch.where(mask, x * outlier_mult, x)
    return x.to(torch.float16)


def case(M: int, K: int, N: int, seed: int, codes: str = "uniform", outlier_p: float = 0.0,
         device="cpu"):
    """(x fp16 [M,K], codes int8 [N,K], scales fp16 [N,K/128]) from one seed."""
    g = gen(seed, device)
    if codes == "uniform":
        c = codes_uniform(N, K, g, device)
    elif codes == "sign":
        c = codes_sign(N, K, g, device)
    else:
        c = codes_sparse(N, K, g, device=device)
    s = scales_uniform(N, K, g, device=device)
    x = activations(M, K, g, outlier_p=outlier_p, device=device)
    return x, c, s


# Named workloads (seeds fixed so every run sees the same bytes).
def tiny_gemv():
    """M=1, K=512, N=256, uniform codes, seed 0."""
    return case(1, 512, 256, seed=0, codes="uniform")


def decode_proj(i: int, M: int = 1):
    """Projection i of the decode layer at M token rows (M>1: 1% outliers x20)."""
    name, K, N = LAYER_PROJ[i]
    if M == 1:
        return case(1, K, N, seed=1000 + i, codes="sparse")
    return case(M, K, N, seed=2000 + 10 * i + M, codes="sparse", outlier_p=0.01)


def prefill(case_idx: int, M: int):
    K, N = PREFILL[case_idx]
    return case(M, K, N, seed=3000 + 10 * case_idx + (0 if M == 2048 else 1), codes="uniform")
