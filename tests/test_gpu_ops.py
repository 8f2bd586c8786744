"""The torch operators and LoRALinear on the GPU: values and gradients
against the fp64 oracle, through autograd, under torch.compile (fullgraph,
eager backend) and with the rsLoRA scale."""
import math

import pytest
import torch

import oracle as O
import workloads as WL
from gpu_helpers import f64
from tolerance import lora_tol_check

pytestmark = pytest.mark.gpu


def _layer(gpu, d_in, d_out, r, alpha, seed, rslora=False):
    from lora_linear_layer_b200 import ops
    g = torch.Generator().manual_seed(seed)
    m = ops.LoRALinear(d_in, d_out, r, alpha, rslora=rslora, device="cuda", generator=g)
    with torch.no_grad():   # a trained-looking adapter (B = 0 would hide the up-projection)
        m.lora_B.copy_((torch.randn(d_out, r, generator=g) * 0.02).to(torch.bfloat16))
    return m


def _oracle(m, x2d, dy2d):
    alpha_eff = m.scale * m.r          # the oracle's s = alpha / r
    X, W, A, B, dY = (f64(t.detach().cpu()) for t in (x2d, m.weight, m.lora_A, m.lora_B, dy2d))
    Y = O.lora_forward(X, W, A, B, alpha_eff)
    dX, dA, dB = O.lora_backward(X, W, A, B, dY, alpha_eff)
    return Y, dX, dA, dB


def _check_all(m, x, y, dy):
    Y, dX, dA, dB = _oracle(m, x.reshape(-1, m.d_in), dy.reshape(-1, m.d_out))
    for got, ref, name in ((y.reshape(-1, m.d_out), Y, "Y"), (x.grad.reshape(-1, m.d_in), dX, "dX"),
                           (m.lora_A.grad, dA, "dA"), (m.lora_B.grad, dB, "dB")):
        ok, info = lora_tol_check(f64(got.detach().cpu()), ref)
        assert ok, (name, info)


@pytest.mark.parametrize("rslora", [False, True])
def test_module_forward_backward_matches_oracle(gpu, rslora):
    m = _layer(gpu, 520, 264, 24, 18.0, seed=1, rslora=rslora)
    x = WL.make_layer_inputs(WL.LayerShape(3 * 100, 520, 264, 24, 18.0), seed=2)["X"].reshape(3, 100, 520)
    x = x.cuda().requires_grad_(True)
    dy = (torch.randn(3, 100, 264, generator=torch.Generator().manual_seed(3))).to(torch.bfloat16).cuda()
    y = m(x)
    y.backward(dy)
    assert m.weight.grad is None
    _check_all(m, x, y, dy)


def test_compiled_fullgraph_equals_eager(gpu):
    m = _layer(gpu, 1024, 512, 16, 32.0, seed=4)
    x0 = WL.make_layer_inputs(WL.LayerShape(256, 1024, 512, 16, 32.0), seed=5)["X"].cuda()
    dy = torch.randn(256, 512, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16).cuda()

    def step(mod, x):
        x = x.clone().requires_grad_(True)
        mod.zero_grad(set_to_none=True)
        y = mod(x)
        y.backward(dy)
        return y.detach(), x.grad, mod.lora_A.grad.clone(), mod.lora_B.grad.clone()

    eager = step(m, x0)
    torch._dynamo.reset()
    cm = torch.compile(m, backend="eager", fullgraph=True)
    comp = step(cm, x0)
    for a, b in zip(eager, comp):
        assert torch.equal(a, b)        # the same kernels on the same inputs
    x = x0.clone().requires_grad_(True)
    m.zero_grad(set_to_none=True)
    y = m(x)
    y.backward(dy)
    _check_all(m, x, y, dy)


def test_opcheck_schema_and_fake(gpu):
    t = WL.make_layer_inputs(WL.LayerShape(130, 256, 136, 8, 6.0), seed=7, with_dy=True)
    X, W, A, B, dY = (t[k].cuda() for k in ("X", "W", "A", "B", "dY"))
    torch.library.opcheck(torch.ops.lora_b200.lora_linear.default, (X, W, A, B, 0.75),
                          test_utils=("test_schema", "test_faketensor"))
    torch.library.opcheck(torch.ops.lora_b200.lora_linear_bwd.default, (X, W, A, B, dY, 0.75),
                          test_utils=("test_schema", "test_faketensor"))


def test_backward_op_fp32_grads(gpu):
    """lora_linear_bwd(..., fp32_grads=True): fp32 dA, dB that round to the
    bf16 op's results bit for bit; dX identical."""
    g = torch.Generator().manual_seed(41)
    M, d_in, d_out, r = 384, 256, 320, 16
    X = torch.randn(M, d_in, generator=g).to(torch.bfloat16).cuda()
    W = (torch.randn(d_out, d_in, generator=g) * d_in ** -0.5).to(torch.bfloat16).cuda()
    A = (torch.randn(r, d_in, generator=g) * d_in ** -0.5).to(torch.bfloat16).cuda()
    B = (torch.randn(d_out, r, generator=g) * 0.02).to(torch.bfloat16).cuda()
    dY = torch.randn(M, d_out, generator=g).to(torch.bfloat16).cuda()
    dX16, dA16, dB16 = torch.ops.lora_b200.lora_linear_bwd(X, W, A, B, dY, 0.75)
    dX, dA, dB = torch.ops.lora_b200.lora_linear_bwd(X, W, A, B, dY, 0.75, True)
    assert dA.dtype == torch.float32 and dB.dtype == torch.float32
    assert torch.equal(dX, dX16)
    assert torch.equal(dA.to(torch.bfloat16), dA16) and torch.equal(dB.to(torch.bfloat16), dB16)


def test_opcheck_saved_t_ops(gpu):
    """Schema (including the declared mutation of ``saved``) and fake
    implementations of lora_linear_train and lora_linear_bwd_saved; Y equals
    lora_linear's bit for bit."""
    t = WL.make_layer_inputs(WL.LayerShape(130, 256, 136, 8, 6.0), seed=7, with_dy=True)
    X, W, A, B, dY = (t[k].cuda() for k in ("X", "W", "A", "B", "dY"))
    torch.library.opcheck(torch.ops.lora_b200.lora_linear_train.default, (X, W, A, B, 0.75),
                          test_utils=("test_schema", "test_faketensor"))
    Y, saved = torch.ops.lora_b200.lora_linear_train(X, W, A, B, 0.75)
    assert torch.equal(Y, torch.ops.lora_b200.lora_linear(X, W, A, B, 0.75))
    torch.library.opcheck(torch.ops.lora_b200.lora_linear_bwd_saved.default, (X, W, A, B, dY, saved, 0.75),
                          test_utils=("test_schema", "test_faketensor"))


def test_saved_t_backward_op_matches_oracle(gpu):
    """Y and (dX, dA, dB) of the training pair against the oracle, with and
    without fp32 gradients."""
    M, d_in, d_out, r, alpha = 777, 520, 1032, 40, 30.0
    t = WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=12, with_dy=True)
    X, W, A, B, dY = (t[k].cuda() for k in ("X", "W", "A", "B", "dY"))
    s = alpha / r
    Y, saved = torch.ops.lora_b200.lora_linear_train(X, W, A, B, s)
    ref = O.lora_backward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), f64(t["dY"]), alpha)
    ok, info = lora_tol_check(f64(Y), O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), alpha))
    assert ok, ("Y", info)
    for fp32 in (False, True):
        got = torch.ops.lora_b200.lora_linear_bwd_saved(X, W, A, B, dY, saved, s, fp32)
        for name, g, want in zip(("dX", "dA", "dB"), got, ref):
            ok, info = lora_tol_check(f64(g.to(torch.bfloat16)), want)
            assert ok, (name, fp32, info)
