"""The torch operators of lora_linear_layer_b200.ops on CPU: registration,
fake (meta) shapes, autograd wiring and a graph-break-free trace.  No GPU:
the real kernels only run in the -m gpu tests."""
import math

import pytest
import torch
from torch._subclasses.fake_tensor import FakeTensorMode

from lora_linear_layer_b200 import ops


def _fake_inputs(M=32, d_in=64, d_out=48, r=8):
    X = torch.empty(M, d_in, dtype=torch.bfloat16, device="cuda")
    W = torch.empty(d_out, d_in, dtype=torch.bfloat16, device="cuda")
    A = torch.empty(r, d_in, dtype=torch.bfloat16, device="cuda")
    B = torch.empty(d_out, r, dtype=torch.bfloat16, device="cuda")
    return X, W, A, B


def test_ops_are_registered():
    assert hasattr(torch.ops.lora_b200, "lora_linear")
    assert hasattr(torch.ops.lora_b200, "lora_linear_bwd")


def test_fake_shapes_forward_and_backward():
    with FakeTensorMode():
        X, W, A, B = _fake_inputs()
        Y = torch.ops.lora_b200.lora_linear(X, W, A, B, 2.0)
        assert Y.shape == (32, 48) and Y.dtype == torch.bfloat16 and Y.device.type == "cuda"
        dX, dA, dB = torch.ops.lora_b200.lora_linear_bwd(X, W, A, B, Y, 2.0)
        assert dX.shape == (32, 64) and dA.shape == (8, 64) and dB.shape == (48, 8)


def test_fake_rejects_mismatched_shapes():
    with FakeTensorMode():
        X, W, A, B = _fake_inputs()
        with pytest.raises(ValueError):
            torch.ops.lora_b200.lora_linear(X, W, A[:, :32], B, 2.0)


def test_autograd_graph_routes_to_the_backward_op():
    """On meta tensors (the fake implementations) the backward of lora_linear
    runs lora_linear_bwd and returns gradients for X, A, B only (W frozen)."""
    X, W, A, B = (t.to("meta") for t in (torch.empty(32, 64), torch.empty(48, 64), torch.empty(8, 64),
                                          torch.empty(48, 8)))
    X, W, A, B = (t.to(torch.bfloat16) for t in (X, W, A, B))
    X.requires_grad_(True)
    A.requires_grad_(True)
    B.requires_grad_(True)
    Y = torch.ops.lora_b200.lora_linear(X, W, A, B, 2.0)
    assert Y.grad_fn is not None
    gX, gA, gB = torch.autograd.grad(Y.sum(), (X, A, B))
    assert gX.shape == X.shape and gA.shape == A.shape and gB.shape == B.shape


def test_trainable_base_weight_is_refused():
    with FakeTensorMode():
        X, W, A, B = _fake_inputs()
        W.requires_grad_(True)
        A.requires_grad_(True)
        with pytest.raises(RuntimeError, match="frozen"):
            torch.ops.lora_b200.lora_linear(X, W, A, B, 2.0)


def test_module_scale_and_init():
    m = ops.LoRALinear(64, 48, 16, 32.0)
    assert m.scale == 2.0
    assert ops.LoRALinear(64, 48, 16, 32.0, rslora=True).scale == 32.0 / math.sqrt(16)
    assert not m.weight.requires_grad and m.lora_A.requires_grad and m.lora_B.requires_grad
    assert torch.count_nonzero(m.lora_B) == 0      # the adapter starts as the identity of the base
    assert m.weight.dtype == torch.bfloat16


def test_dynamo_traces_without_graph_breaks():
    """torch._dynamo.explain over a function that calls the operator (fake
    tensors, so nothing runs on a GPU): one graph, no breaks."""
    import torch._dynamo

    def f(X, W, A, B):
        return torch.ops.lora_b200.lora_linear(X, W, A, B, 2.0) * 2

    with FakeTensorMode():
        args = _fake_inputs()
    torch._dynamo.reset()
    ex = torch._dynamo.explain(f)(*args)
    assert ex.graph_break_count == 0
    assert ex.graph_count == 1


def test_fake_backward_fp32_grads_dtype():
    with FakeTensorMode():
        X, W, A, B = _fake_inputs()
        dY = torch.empty(32, 48, dtype=torch.bfloat16)
        dX, dA, dB = torch.ops.lora_b200.lora_linear_bwd(X, W, A, B, dY, 0.5, True)
        assert dX.dtype == torch.bfloat16 and dA.dtype == torch.float32 and dB.dtype == torch.float32
        dX, dA, dB = torch.ops.lora_b200.lora_linear_bwd(X, W, A, B, dY, 0.5)
        assert dA.dtype == torch.bfloat16 and dB.dtype == torch.bfloat16


def test_train_op_fake_shapes_and_saved_workspace_size(built_lib):
    """lora_linear_train's fake returns Y and the workspace; its byte count
    (from the documented layout) equals the library's
    lora_bwd_workspace_size for several shapes."""
    with FakeTensorMode():
        X, W, A, B = _fake_inputs()
        Y, saved = torch.ops.lora_b200.lora_linear_train(X, W, A, B, 2.0)
        assert Y.shape == (32, 48) and Y.dtype == torch.bfloat16
        assert saved.dtype == torch.uint8 and saved.shape == (built_lib.lora_bwd_workspace_size(32, 64, 48, 8),)
        dX, dA, dB = torch.ops.lora_b200.lora_linear_bwd_saved(X, W, A, B, Y, saved, 2.0)
        assert dX.shape == (32, 64) and dA.shape == (8, 64) and dB.shape == (48, 8)
    for M, r in ((1, 8), (300, 24), (4100, 128), (8192, 16), (0, 64)):
        assert ops._workspace_bytes(M, r) == built_lib.lora_bwd_workspace_size(M, 512, 264, r)


def test_train_op_autograd_routes_to_the_saved_backward():
    """On meta tensors the backward of lora_linear_train runs
    lora_linear_bwd_saved (gradients for X, A, B only)."""
    X, W, A, B = (torch.empty(*s, dtype=torch.bfloat16, device="meta") for s in ((32, 64), (48, 64), (8, 64),
                                                                                   (48, 8)))
    for t in (X, A, B):
        t.requires_grad_(True)
    Y, saved = torch.ops.lora_b200.lora_linear_train(X, W, A, B, 2.0)
    assert Y.grad_fn is not None and not saved.requires_grad
    gX, gA, gB = torch.autograd.grad(Y.sum(), (X, A, B))
    assert gX.shape == X.shape and gA.shape == A.shape and gB.shape == B.shape


def test_module_trains_through_the_saved_t_op():
    """LoRALinear calls lora_linear_train when autograd will need the
    backward and lora_linear otherwise (traced with dynamo on fake tensors:
    one graph, no breaks, the expected operator in it)."""
    import torch._dynamo
    seen = []

    def backend(gm, example_inputs):
        seen.append({str(n.target) for n in gm.graph.nodes if n.op == "call_function"})
        return gm.forward

    with FakeTensorMode():
        m = ops.LoRALinear(64, 48, 8, 16.0, device="cuda")
        x = torch.empty(4, 8, 64, dtype=torch.bfloat16, device="cuda")
    for grad in (True, False):
        torch._dynamo.reset()
        seen.clear()
        with torch.set_grad_enabled(grad):
            ex = torch._dynamo.explain(m)(x)
            assert ex.graph_break_count == 0
            torch.compile(m, backend=backend, fullgraph=True)(x)
        names = {n.rsplit(".default", 1)[0] for n in seen[-1]}
        assert ("lora_b200.lora_linear_train" in names) == grad, names
        assert ("lora_b200.lora_linear" in names) == (not grad), names
