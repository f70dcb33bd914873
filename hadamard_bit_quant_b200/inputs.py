"""Seeded synthetic inputs for the H-BitLinear forward.

This module only draws random numbers. It holds none of the method's
arithmetic (no Hadamard, no scales, no rounding to codes), so both the CUDA
path and the CPU oracle can take their inputs from it without sharing any
computation.

All draws use a CPU ``torch.Generator`` seeded from ``(seed, stream)`` so that
the same bytes come out on every machine. Activations are returned as bf16
(the layer input dtype), weights as fp32 (the latent full-precision weights
that the ternary quantiser reads).

The shapes and value distributions follow the BitNet v2 architecture
walkthrough: model shapes from Table 8 (hidden 4096, GLU 16384 for 7B),
outlier channels that are fixed per channel across tokens (Figure 1 and
Figure 3 describe W_o / W_down inputs with a few channels of very large
magnitude), and the SwiGLU-gated input of W_down.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional, Sequence

import torch

W_STD = 0.02


def _gen(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1_000_003 + int(stream))
    return g


def gaussian_weights(N: int, K: int, seed: int, std: float = W_STD) -> torch.Tensor:
    """Latent weights W (N x K, fp32) drawn from N(0, std^2)."""
    g = _gen(seed, 0)
    return torch.randn(N, K, generator=g, dtype=torch.float32) * std


def outlier_channels(K: int, frac: float, seed: int) -> torch.Tensor:
    """Channel indices (sorted) chosen by a seeded permutation; round(frac*K) of them."""
    n = max(1, int(round(frac * K)))
    g = _gen(seed, 1)
    return torch.sort(torch.randperm(K, generator=g)[:n]).values


def gaussian_with_outliers(M: int, K: int, seed: int, channels: Sequence[int],
                           factor: float, stream: int = 2) -> torch.Tensor:
    """X ~ N(0,1) (M x K) with the given channels multiplied by ``factor`` in every token; bf16."""
    g = _gen(seed, stream)
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    idx = torch.as_tensor(list(channels), dtype=torch.long)
    if idx.numel():
        x[:, idx] *= factor
    return x.to(torch.bfloat16)


def glu_squared_relu(M: int, K: int, seed: int, stream: int = 2) -> torch.Tensor:
    """Heavy-tailed gated input of a down projection: x = max(a,0)^2 * u, a,u ~ N(0,1); bf16.

    About half the entries are exactly zero, the rest are signed with a heavy
    tail (the square of a half-normal times a normal gate).
    """
    g = _gen(seed, stream)
    a = torch.randn(M, K, generator=g, dtype=torch.float32)
    u = torch.randn(M, K, generator=g, dtype=torch.float32)
    return (torch.clamp(a, min=0.0).square() * u).to(torch.bfloat16)


def student_t(M: int, K: int, seed: int, nu: int = 3, stream: int = 2) -> torch.Tensor:
    """Student-t(nu) entries, built as z / sqrt(chi2_nu / nu) from nu+1 normals; bf16."""
    g = _gen(seed, stream)
    z = torch.randn(M, K, generator=g, dtype=torch.float32)
    chi2 = torch.zeros(M, K, dtype=torch.float32)
    for _ in range(nu):
        chi2 += torch.randn(M, K, generator=g, dtype=torch.float32).square()
    return (z / torch.sqrt(chi2 / nu)).to(torch.bfloat16)


@dataclasses.dataclass
class Case:
    """One H-BitLinear call: shapes, mode and how to draw its inputs."""
    name: str
    M: int
    K: int
    N: int
    act_bits: int
    use_hadamard: int
    seed: int
    x_kind: str                     # "outliers" | "glu" | "student_t"
    outlier_factor: float = 0.0
    outlier_list: Optional[List[int]] = None
    outlier_frac: float = 0.0
    x_stream: int = 2

    def make_x(self) -> torch.Tensor:
        if self.x_kind == "outliers":
            ch = (self.outlier_list if self.outlier_list is not None
                  else outlier_channels(self.K, self.outlier_frac, self.seed).tolist())
            return gaussian_with_outliers(self.M, self.K, self.seed, ch,
                                          self.outlier_factor, self.x_stream)
        if self.x_kind == "glu":
            return glu_squared_relu(self.M, self.K, self.seed, self.x_stream)
        if self.x_kind == "student_t":
            return student_t(self.M, self.K, self.seed, 3, self.x_stream)
        raise ValueError(self.x_kind)

    def make_w(self) -> torch.Tensor:
        return gaussian_weights(self.N, self.K, self.seed)

    @property
    def label(self) -> str:
        return (f"{self.name}:M{self.M}_K{self.K}_N{self.N}_a{self.act_bits}"
                f"_h{self.use_hadamard}")


def tiny_case() -> Case:
    """Single H-BitLinear W1.58A4: M=8, K=256, N=256, channels {3,77,128,201} x40, seed 0."""
    return Case("tiny", 8, 256, 256, 4, 1, 0, "outliers", 40.0, [3, 77, 128, 201])


def decode_oproj_cases(Ms: Sequence[int] = (1, 4, 16),
                       acts: Sequence[int] = (8, 4)) -> List[Case]:
    """Decode-shaped o_proj: K=N=4096, 1% of channels x50, seed 1."""
    out = []
    for a in acts:
        for m in Ms:
            out.append(Case("decode_oproj", m, 4096, 4096, a, 1, 1, "outliers", 50.0,
                            None, 0.01, x_stream=100 + m))
    return out


def prefill_down_case(M: int = 4096) -> Case:
    """Prefill down_proj: M=4096, K=16384, N=4096, INT4, H on, GLU-gated input, seed 2."""
    return Case("prefill_down", M, 16384, 4096, 4, 1, 2, "glu")


BLOCK7B_PROJ = (
    # name, N, K, act_bits, use_hadamard
    ("q", 4096, 4096, 8, 0),
    ("k", 4096, 4096, 8, 0),
    ("v", 4096, 4096, 8, 0),
    ("o", 4096, 4096, 4, 1),
    ("up", 16384, 4096, 8, 0),
    ("gate", 16384, 4096, 8, 0),
    ("down", 4096, 16384, 4, 1),
)


def block7b_cases(M: int) -> List[Case]:
    """All projections of one 7B-shaped block (hidden 4096, FFN 16384), seed 3.

    q/k/v/up/gate are plain BitLinear INT8 (no Hadamard); o/down are
    H-BitLinear INT4. Inputs are N(0,1) with 1% of channels x50.
    """
    out = []
    for i, (nm, N, K, a, h) in enumerate(BLOCK7B_PROJ):
        c = Case(f"block7b_{nm}", M, K, N, a, h, 3 * 100 + i, "outliers", 50.0, None, 0.01)
        out.append(c)
    return out


SWEEP_MS = tuple(2 ** i for i in range(15))      # 1 .. 16384
SWEEP_KN = (2048, 4096, 8192, 16384)


def sweep_case(M: int, K: int, N: int, act_bits: int, use_hadamard: int) -> Case:
    """One point of the M x K x N sweep: Student-t(3) activations; seed 4 + point index."""
    idx = (SWEEP_MS.index(M) * 16 + SWEEP_KN.index(K) * 4 + SWEEP_KN.index(N)) * 4 \
        + (act_bits == 8) * 2 + use_hadamard
    return Case("sweep", M, K, N, act_bits, use_hadamard, 4 + idx, "student_t")
