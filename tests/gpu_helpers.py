"""Shared plumbing of the GPU parity tests: move seeded inputs to the device,
call the C ABI through the binding, and evaluate the oracle on the same bf16
values (CPU, float64).  Nothing here computes any part of the layer."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import workloads as WL


def f64(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (CPU or CUDA) -> float64 numpy through the oracle's widening."""
    return O.bf16_bits_to_f64(WL.bf16_bits(t.detach().cpu()))


def dev(t: torch.Tensor) -> torch.Tensor:
    return t.to("cuda", non_blocking=False).contiguous()


def run_fwd(L, X, W, A, B, alpha):
    Xd, Wd, Ad, Bd = dev(X), dev(W), dev(A), dev(B)
    Y = torch.full((X.shape[0], W.shape[0]), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.lora_fwd(Xd, Wd, Ad, Bd, Y, alpha)
    assert L.lora_get_device_status() == 0
    return Y


def run_bwd(L, X, W, A, B, dY, alpha):
    M, d_in = X.shape
    d_out, r = B.shape
    Xd, Wd, Ad, Bd, dYd = dev(X), dev(W), dev(A), dev(B), dev(dY)
    nan = float("nan")
    dX = torch.full((M, d_in), nan, dtype=torch.bfloat16, device="cuda")
    dA = torch.full((r, d_in), nan, dtype=torch.bfloat16, device="cuda")
    dB = torch.full((d_out, r), nan, dtype=torch.bfloat16, device="cuda")
    ws_bytes = L.lora_bwd_workspace_size(M, d_in, d_out, r)
    ws = torch.full((max(ws_bytes, 256) // 4,), nan, dtype=torch.float32, device="cuda")
    L.lora_bwd(Xd, Wd, Ad, Bd, dYd, dX, dA, dB, alpha, ws)
    assert L.lora_get_device_status() == 0
    return dX, dA, dB
