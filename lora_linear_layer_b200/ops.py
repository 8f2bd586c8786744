"""The fused LoRA layer as PyTorch operators with autograd, and a module.

    Y = X W^T + s (X A^T) B^T,   s = alpha / r   (or an explicit scale)

fastaf 0.1.0, "FWD kernel speedup" / "BWD kernel speedup": the layer and its
backward for a frozen base weight W; section "torch.compile compatibility":
each kernel is a torch.library custom op with a fake implementation, so the
compiler traces through the layer without a graph break (checked with
torch._dynamo.explain).  Here:

* ``torch.ops.lora_b200.lora_linear(X, W, A, B, scale)`` runs
  ``lora_fwd_scaled``;
* ``torch.ops.lora_b200.lora_linear_bwd(X, W, A, B, dY, scale, fp32_grads)``
  runs ``lora_bwd_scaled`` and returns (dX, dA, dB), dA and dB in fp32 when
  ``fp32_grads`` (the unrounded reductions, e.g. for fp32 optimizer states
  or a data-parallel sum before rounding), else bf16;
* ``torch.ops.lora_b200.lora_linear_train(X, W, A, B, scale)`` runs
  ``lora_fwd_save_scaled`` and returns (Y, saved): Y as ``lora_linear`` (bit
  for bit) and the backward's workspace with T = X A^T already in it; its
  backward, ``lora_linear_bwd_saved``, runs ``lora_bwd_scaled`` with
  ``LORA_BWD_T_SAVED`` and so reads X once less (``LoRALinear`` uses this
  pair whenever autograd will need the backward);
* all have fake (meta) implementations, so they trace under FakeTensorMode
  and torch.compile without graph breaks, and ``lora_linear`` and
  ``lora_linear_train`` are differentiable in X, A and B through their
  backward ops.  W is frozen: it gets no gradient.

The scale is passed explicitly, so rsLoRA's alpha / sqrt(r) (unsloth fork
commit log, scripts/benchmarks/qwen3_flex_inference.py: PEFT keeps the
adapter's scaling, alpha / sqrt(r) under rsLoRA, in the module) is as easy
to use as alpha / r.  The operators call the library's explicit-scale entry
points (``lora_fwd_scaled``, ``lora_fwd_save_scaled``, ``lora_bwd_scaled``),
which take s itself (rounded once to fp32) rather than alpha.

Argument marshalling only: all arithmetic runs in the library's kernels.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import torch

from . import (LORA_BWD_FP32_GRADS, LORA_BWD_T_SAVED, lora_bwd_scaled, lora_bwd_workspace_size, lora_fwd_save_scaled,
               lora_fwd_scaled)

_LIB = "lora_b200"


def _check(X: torch.Tensor, W: torch.Tensor, A: torch.Tensor, B: torch.Tensor) -> Tuple[int, int, int, int]:
    if X.dim() != 2 or W.dim() != 2 or A.dim() != 2 or B.dim() != 2:
        raise ValueError("lora_linear takes 2-D X [M, d_in], W [d_out, d_in], A [r, d_in], B [d_out, r]")
    M, d_in = X.shape
    d_out, r = B.shape
    if tuple(W.shape) != (d_out, d_in) or tuple(A.shape) != (r, d_in):
        raise ValueError(f"shape mismatch: X {tuple(X.shape)}, W {tuple(W.shape)}, A {tuple(A.shape)}, "
                         f"B {tuple(B.shape)}")
    return M, d_in, d_out, r


@torch.library.custom_op(f"{_LIB}::lora_linear", mutates_args=())
def lora_linear(X: torch.Tensor, W: torch.Tensor, A: torch.Tensor, B: torch.Tensor, scale: float) -> torch.Tensor:
    """Y = X W^T + scale (X A^T) B^T (bf16, 2-D, contiguous CUDA tensors)."""
    M, d_in, d_out, r = _check(X, W, A, B)
    Y = torch.empty((M, d_out), dtype=X.dtype, device=X.device)
    lora_fwd_scaled(X.contiguous(), W.contiguous(), A.contiguous(), B.contiguous(), Y, scale)
    return Y


@lora_linear.register_fake
def _lora_linear_fake(X, W, A, B, scale):
    M, d_in, d_out, r = _check(X, W, A, B)
    return X.new_empty((M, d_out))


@torch.library.custom_op(f"{_LIB}::lora_linear_bwd", mutates_args=())
def lora_linear_bwd(X: torch.Tensor, W: torch.Tensor, A: torch.Tensor, B: torch.Tensor, dY: torch.Tensor,
                    scale: float, fp32_grads: bool = False) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """(dX, dA, dB) of Y = X W^T + scale (X A^T) B^T for the gradient dY;
    dA and dB in fp32 when fp32_grads, else in the dtype of A and B."""
    M, d_in, d_out, r = _check(X, W, A, B)
    gdt = torch.float32 if fp32_grads else A.dtype
    dX = torch.empty((M, d_in), dtype=X.dtype, device=X.device)
    dA = torch.empty((r, d_in), dtype=gdt, device=A.device)
    dB = torch.empty((d_out, r), dtype=gdt, device=B.device)
    ws = torch.empty(max(lora_bwd_workspace_size(M, d_in, d_out, r), 1), dtype=torch.uint8, device=X.device)
    lora_bwd_scaled(X.contiguous(), W.contiguous(), A.contiguous(), B.contiguous(), dY.contiguous(), dX, dA, dB,
                    scale, ws, LORA_BWD_FP32_GRADS if fp32_grads else 0)
    return dX, dA, dB


@lora_linear_bwd.register_fake
def _lora_linear_bwd_fake(X, W, A, B, dY, scale, fp32_grads=False):
    M, d_in, d_out, r = _check(X, W, A, B)
    gdt = torch.float32 if fp32_grads else A.dtype
    return X.new_empty((M, d_in)), A.new_empty((r, d_in), dtype=gdt), B.new_empty((d_out, r), dtype=gdt)


def _workspace_bytes(M, r: int):
    """Bytes of lora_bwd_workspace_size(M, ., ., r) from its documented
    layout (T and dT as bf16 [M, r_pad], r_pad = r rounded up to 16, each
    padded to 256 bytes); usable on symbolic M, where the library cannot be
    asked.  0 when M == 0."""
    r_pad = (r + 15) // 16 * 16
    return 2 * ((M * r_pad * 2 + 255) // 256 * 256)


@torch.library.custom_op(f"{_LIB}::lora_linear_train", mutates_args=())
def lora_linear_train(X: torch.Tensor, W: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                      scale: float) -> Tuple[torch.Tensor, torch.Tensor]:
    """(Y, saved): Y = X W^T + scale (X A^T) B^T and the backward's
    workspace (uint8) holding T = X A^T for lora_linear_bwd_saved."""
    M, d_in, d_out, r = _check(X, W, A, B)
    nbytes = _workspace_bytes(M, r)
    if nbytes < lora_bwd_workspace_size(M, d_in, d_out, r):
        raise RuntimeError("lora_linear_train: the library needs a larger workspace than its documented layout")
    Y = torch.empty((M, d_out), dtype=X.dtype, device=X.device)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=X.device)
    lora_fwd_save_scaled(X.contiguous(), W.contiguous(), A.contiguous(), B.contiguous(), Y, scale, ws)
    return Y, ws


@lora_linear_train.register_fake
def _lora_linear_train_fake(X, W, A, B, scale):
    M, d_in, d_out, r = _check(X, W, A, B)
    return X.new_empty((M, d_out)), X.new_empty((max(_workspace_bytes(M, r), 1),), dtype=torch.uint8)


@torch.library.custom_op(f"{_LIB}::lora_linear_bwd_saved", mutates_args=("saved",))
def lora_linear_bwd_saved(X: torch.Tensor, W: torch.Tensor, A: torch.Tensor, B: torch.Tensor, dY: torch.Tensor,
                          saved: torch.Tensor, scale: float,
                          fp32_grads: bool = False) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """lora_linear_bwd with T taken from ``saved`` (the workspace that
    lora_linear_train returned for the same X, A); writes dT into ``saved``
    beside T and leaves T as it was."""
    M, d_in, d_out, r = _check(X, W, A, B)
    gdt = torch.float32 if fp32_grads else A.dtype
    dX = torch.empty((M, d_in), dtype=X.dtype, device=X.device)
    dA = torch.empty((r, d_in), dtype=gdt, device=A.device)
    dB = torch.empty((d_out, r), dtype=gdt, device=B.device)
    flags = LORA_BWD_T_SAVED | (LORA_BWD_FP32_GRADS if fp32_grads else 0)
    lora_bwd_scaled(X.contiguous(), W.contiguous(), A.contiguous(), B.contiguous(), dY.contiguous(), dX, dA, dB,
                    scale, saved, flags)
    return dX, dA, dB


@lora_linear_bwd_saved.register_fake
def _lora_linear_bwd_saved_fake(X, W, A, B, dY, saved, scale, fp32_grads=False):
    return _lora_linear_bwd_fake(X, W, A, B, dY, scale, fp32_grads)


def _setup_context_train(ctx, inputs, output):
    X, W, A, B, scale = inputs
    if W.requires_grad:
        raise RuntimeError("lora_linear: the base weight W is frozen and gets no gradient; "
                           "call W.requires_grad_(False)")
    ctx.save_for_backward(X, W, A, B, output[1])
    ctx.scale = scale


def _backward_train(ctx, dY, _d_saved):
    X, W, A, B, saved = ctx.saved_tensors
    dX, dA, dB = torch.ops.lora_b200.lora_linear_bwd_saved(X, W, A, B, dY.contiguous(), saved, ctx.scale)
    return (dX if ctx.needs_input_grad[0] else None, None, dA if ctx.needs_input_grad[2] else None,
            dB if ctx.needs_input_grad[3] else None, None)


lora_linear_train.register_autograd(_backward_train, setup_context=_setup_context_train)


def _setup_context(ctx, inputs, output):
    X, W, A, B, scale = inputs
    if W.requires_grad:
        raise RuntimeError("lora_linear: the base weight W is frozen and gets no gradient; "
                           "call W.requires_grad_(False)")
    ctx.save_for_backward(X, W, A, B)
    ctx.scale = scale


def _backward(ctx, dY):
    X, W, A, B = ctx.saved_tensors
    dX, dA, dB = torch.ops.lora_b200.lora_linear_bwd(X, W, A, B, dY.contiguous(), ctx.scale)
    return (dX if ctx.needs_input_grad[0] else None, None, dA if ctx.needs_input_grad[2] else None,
            dB if ctx.needs_input_grad[3] else None, None)


lora_linear.register_autograd(_backward, setup_context=_setup_context)


class LoRALinear(torch.nn.Module):
    """A linear layer with a frozen base weight and a trainable rank-r adapter:
    y = x W^T + s (x A^T) B^T over the last dimension of x (any leading
    dimensions).  s = alpha / r, or alpha / sqrt(r) with ``rslora=True``.
    A is initialised N(0, 1/d_in) (variance), B to zero (the adapter starts
    as the identity map of the base layer); all parameters are bf16."""

    def __init__(self, d_in: int, d_out: int, r: int, alpha: float, rslora: bool = False,
                 device: Optional[torch.device] = None, generator: Optional[torch.Generator] = None):
        super().__init__()
        self.d_in, self.d_out, self.r, self.alpha = int(d_in), int(d_out), int(r), float(alpha)
        self.scale = self.alpha / (math.sqrt(self.r) if rslora else self.r)
        kw = dict(dtype=torch.bfloat16, device=device)
        self.weight = torch.nn.Parameter(
            (torch.randn(d_out, d_in, generator=generator) * d_in ** -0.5).to(**kw), requires_grad=False)
        self.lora_A = torch.nn.Parameter((torch.randn(r, d_in, generator=generator) * d_in ** -0.5).to(**kw))
        self.lora_B = torch.nn.Parameter(torch.zeros(d_out, r, **kw))

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        x2 = x.reshape(-1, self.d_in)
        if torch.is_grad_enabled() and (x.requires_grad or self.lora_A.requires_grad or self.lora_B.requires_grad):
            # keep T for the backward (it then reads X once less)
            y, _ = torch.ops.lora_b200.lora_linear_train(x2, self.weight, self.lora_A, self.lora_B, self.scale)
        else:
            y = torch.ops.lora_b200.lora_linear(x2, self.weight, self.lora_A, self.lora_B, self.scale)
        return y.reshape(*lead, self.d_out)

    def extra_repr(self) -> str:
        return f"d_in={self.d_in}, d_out={self.d_out}, r={self.r}, scale={self.scale:g}"
