"""Tensor-level helpers over the C ABI: pack a weight matrix, run the forward.

These only allocate outputs with torch and call the binding; the arithmetic
is in libhbl's kernels.
"""
from __future__ import annotations

import torch

from . import hbl


def pack_weights(W: torch.Tensor, stream=None):
    """Ternarise and pack an N x K fp32 CUDA tensor. Returns (Wpk uint8 [N*K/4], wscale fp32 [1])."""
    assert W.is_cuda and W.dtype == torch.float32 and W.dim() == 2 and W.is_contiguous()
    N, K = W.shape
    Wpk = torch.empty(hbl.hbl_packed_bytes(N, K), dtype=torch.uint8, device=W.device)
    wscale = torch.empty(1, dtype=torch.float32, device=W.device)
    hbl.hbl_pack_weights(W, N, K, Wpk, wscale, stream)
    return Wpk, wscale


def unpack_weights(Wpk: torch.Tensor, N: int, K: int, stream=None) -> torch.Tensor:
    T = torch.empty(N, K, dtype=torch.int8, device=Wpk.device)
    hbl.hbl_unpack_weights(Wpk, N, K, T, stream)
    return T


def workspace(M: int, K: int, N: int, device) -> torch.Tensor:
    return torch.empty(max(1, hbl.hbl_workspace_bytes(M, K, N)), dtype=torch.uint8, device=device)


def forward(X: torch.Tensor, Wpk: torch.Tensor, wscale: torch.Tensor, N: int, act_bits: int = 4,
            use_hadamard: int = 1, out: torch.Tensor | None = None, ws: torch.Tensor | None = None,
            stream=None) -> torch.Tensor:
    """Y = H-BitLinear(X) for bf16 X (M x K). Uses ``ws`` (caller workspace) when given."""
    assert X.is_cuda and X.dtype == torch.bfloat16 and X.dim() == 2 and X.is_contiguous()
    M, K = X.shape
    Y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=X.device)
    if ws is None:
        hbl.hbl_forward(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y, stream)
    else:
        hbl.hbl_forward_ws(X, M, K, N, Wpk, wscale, act_bits, use_hadamard, Y, ws, ws.numel(), stream)
    return Y


def hadamard_f32(X: torch.Tensor, stream=None) -> torch.Tensor:
    M, K = X.shape
    Xr = torch.empty(M, K, dtype=torch.float32, device=X.device)
    hbl.hbl_hadamard_f32(X, M, K, Xr, stream)
    return Xr


def quantize(X: torch.Tensor, act_bits: int, use_hadamard: int, stream=None):
    M, K = X.shape
    codes = torch.empty(M, K, dtype=torch.int8, device=X.device)
    scales = torch.empty(M, dtype=torch.float32, device=X.device)
    csum = torch.empty(M, dtype=torch.int32, device=X.device)
    hbl.hbl_quantize(X, M, K, act_bits, use_hadamard, codes, scales, csum, stream)
    return codes, scales, csum


def gemm_codes(codes: torch.Tensor, Wpk: torch.Tensor, N: int, stream=None) -> torch.Tensor:
    M, K = codes.shape
    acc = torch.empty(M, N, dtype=torch.int32, device=codes.device)
    hbl.hbl_gemm_codes(codes, M, K, N, Wpk, acc, stream)
    return acc


class HBitLinear:
    """One H-BitLinear (or plain BitLinear with use_hadamard=0) layer with packed weights."""

    def __init__(self, W: torch.Tensor, act_bits: int = 4, use_hadamard: int = 1):
        self.N, self.K = W.shape
        self.act_bits = act_bits
        self.use_hadamard = use_hadamard
        self.Wpk, self.wscale = pack_weights(W)

    def __call__(self, X: torch.Tensor, out=None, ws=None, stream=None) -> torch.Tensor:
        return forward(X, self.Wpk, self.wscale, self.N, self.act_bits, self.use_hadamard, out, ws, stream)
