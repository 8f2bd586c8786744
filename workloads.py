"""Seeded synthetic workloads for the fused LoRA linear layer.

This module only draws random inputs and names the workload shapes. It holds
none of the layer's arithmetic, so both the fp64 oracle (``oracle/``) and the
GPU path can take their inputs from here without sharing any computation.

Recipe (readings of the workload descriptions, stated once here):

* ``N(0, 1/d)`` means variance ``1/d`` (std ``d**-0.5``), which keeps
  ``X @ W.T`` at unit scale.  ``N(0, 0.02)`` means std ``0.02``, the usual
  LoRA-B / GPT init std.  ``N(0, 1)`` is the standard normal.
* Every tensor is drawn as fp32 from one ``torch.Generator('cpu')`` seeded
  with ``seed``, scaled by its std, and rounded to bf16 (round to nearest
  even, torch's cast).  Draw order: X, W, A, B, dY.
* Tensors are row-major and contiguous, with the nn.Linear / LoRA layout:
  ``X[M, d_in]``, ``W[d_out, d_in]``, ``A[r, d_in]``, ``B[d_out, r]``,
  ``dY[M, d_out]``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """One LoRA layer problem: M tokens, d_in -> d_out, rank r, scale alpha."""

    M: int
    d_in: int
    d_out: int
    r: int
    alpha: float
    name: str = ""

    @property
    def scale(self) -> float:
        return self.alpha / self.r


# The named workloads.  Sizes are those of the fused-LoRA workload list:
# a tiny forward, the attention-projection forward (batch 4 x seq 2048), the
# MLP up-projection forward+backward, the square forward sweep and the
# 36-layer x 7-target adapter merge of a 2560-hidden model.
TINY_FWD = LayerShape(M=256, d_in=512, d_out=512, r=16, alpha=32.0, name="tiny_fwd_256x512x512_r16")
ATTN_PROJ = LayerShape(M=8192, d_in=4096, d_out=4096, r=16, alpha=32.0, name="attn_proj_8192x4096x4096_r16")
MLP_UP = LayerShape(M=16384, d_in=4096, d_out=14336, r=64, alpha=128.0, name="mlp_up_16384x4096x14336_r64")

SWEEP_D = (512, 1024, 2048, 4096, 8192)
SWEEP_M = (128, 512, 2048, 8192, 16384)
SWEEP_R = (8, 16, 32, 64, 128)


def sweep_points() -> List[LayerShape]:
    """The 125-point square sweep, d_in = d_out, alpha = 2r, seed = point index."""
    pts = []
    for d in SWEEP_D:
        for m in SWEEP_M:
            for r in SWEEP_R:
                pts.append(LayerShape(M=m, d_in=d, d_out=d, r=r, alpha=2.0 * r,
                                      name=f"sweep_M{m}_d{d}_r{r}"))
    return pts


# Merge workload: 36 layers x 7 targets of a 2560-hidden model, W is [d_out, d_in].
MERGE_TARGETS = (
    ("q", 2560, 4096),
    ("k", 2560, 1024),
    ("v", 2560, 1024),
    ("o", 4096, 2560),
    ("gate", 2560, 9728),
    ("up", 2560, 9728),
    ("down", 9728, 2560),
)
MERGE_LAYERS = 36
MERGE_R = 32
MERGE_ALPHA = 64.0


def merge_shapes(layers: int = MERGE_LAYERS) -> List[Dict]:
    """(layer, target, d_in, d_out) for every merged matrix, in draw order."""
    out = []
    for layer in range(layers):
        for name, d_in, d_out in MERGE_TARGETS:
            out.append(dict(layer=layer, target=name, d_in=d_in, d_out=d_out))
    return out


def _normal_bf16(gen: torch.Generator, shape, std: float) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def make_layer_inputs(shape: LayerShape, seed: int = 0, with_dy: bool = False,
                      x_std: float = 1.0, w_var_scaled: bool = True,
                      b_std: float = 0.02) -> Dict[str, torch.Tensor]:
    """Draw X, W, A, B (and dY) for one layer as bf16 CPU tensors.

    X ~ N(0, x_std^2), W and A ~ N(0, 1/d_in) (variance), B ~ N(0, b_std^2),
    dY ~ N(0, 1).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    w_std = 1.0 / math.sqrt(shape.d_in) if w_var_scaled else 1.0
    X = _normal_bf16(gen, (shape.M, shape.d_in), x_std)
    W = _normal_bf16(gen, (shape.d_out, shape.d_in), w_std)
    A = _normal_bf16(gen, (shape.r, shape.d_in), w_std)
    B = _normal_bf16(gen, (shape.d_out, shape.r), b_std)
    out = dict(X=X, W=W, A=A, B=B)
    if with_dy:
        out["dY"] = _normal_bf16(gen, (shape.M, shape.d_out), 1.0)
    return out


def make_merge_inputs(d_out: int, d_in: int, r: int, seed: int) -> Dict[str, torch.Tensor]:
    """W ~ N(0, 1/d_in), A ~ N(0, 1/d_in), B ~ N(0, 0.02^2), bf16."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    std = 1.0 / math.sqrt(d_in)
    W = _normal_bf16(gen, (d_out, d_in), std)
    A = _normal_bf16(gen, (r, d_in), std)
    B = _normal_bf16(gen, (d_out, r), 0.02)
    return dict(W=W, A=A, B=B)


def perturb_adapter(A: torch.Tensor, B: torch.Tensor, cycle: int, seed: int = 1000,
                    eps: float = 0.01):
    """A + eps*N(0,1), B + eps*N(0,1), drawn from a generator seeded by cycle.

    Stands for one optimiser step on the adapter between two merge refreshes.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed) + int(cycle))
    dA = torch.randn(A.shape, generator=gen, dtype=torch.float32) * eps
    dB = torch.randn(B.shape, generator=gen, dtype=torch.float32) * eps
    return (A.float() + dA).to(torch.bfloat16), (B.float() + dB).to(torch.bfloat16)


def sample_rows(M: int, seed: int = 0, per_tile: int = 2, tile: int = 128) -> torch.Tensor:
    """Row indices for sampled checks: the first and last row, plus `per_tile`
    seeded rows from every 128-row tile (so every M tile and the ragged tail
    are represented)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed) + 77)
    rows = {0, M - 1}
    for t0 in range(0, M, tile):
        t1 = min(M, t0 + tile)
        for _ in range(per_tile):
            rows.add(int(torch.randint(t0, t1, (1,), generator=gen).item()))
    return torch.tensor(sorted(rows), dtype=torch.int64)


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 array of its bit patterns (no arithmetic)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")
