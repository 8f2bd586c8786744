"""GPU parity of lora_bwd (dX, dA, dB) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL
from gpu_helpers import f64, run_bwd
from tolerance import lora_tol_check

pytestmark = pytest.mark.gpu

SHAPES = [
    (256, 512, 512, 16, 32.0),
    (1, 8, 8, 8, 16.0),
    (300, 520, 264, 8, 6.0),
    (129, 64, 136, 24, 18.0),
    (777, 1032, 1000, 40, 30.0),
    (1000, 512, 2056, 64, 128.0),
    (257, 256, 384, 128, 96.0),
    (4100, 1024, 1536, 32, 64.0),   # several M splits with a ragged last one
]


def _check_all(t, alpha, dX, dA, dB, dx_rows=None):
    ref_dX, ref_dA, ref_dB = O.lora_backward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]),
                                             f64(t["dY"]), alpha, dx_rows=dx_rows)
    got_dX = f64(dX.cpu() if dx_rows is None else dX.cpu()[torch.as_tensor(dx_rows)])
    for name, got, ref in (("dX", got_dX, ref_dX), ("dA", f64(dA), ref_dA), ("dB", f64(dB), ref_dB)):
        ok, info = lora_tol_check(got, ref)
        assert ok, (name, info)


@pytest.mark.parametrize("M,d_in,d_out,r,alpha", SHAPES)
def test_bwd_matches_oracle(gpu, M, d_in, d_out, r, alpha):
    sh = WL.LayerShape(M, d_in, d_out, r, alpha)
    t = WL.make_layer_inputs(sh, seed=11 + M, with_dy=True)
    dX, dA, dB = run_bwd(gpu, t["X"], t["W"], t["A"], t["B"], t["dY"], alpha)
    _check_all(t, alpha, dX, dA, dB)


def test_bwd_mlp_up_full_size(gpu):
    """MLP up-projection forward+backward workload at full size: dX on
    sampled rows of every tile, dA and dB in full."""
    sh = WL.MLP_UP
    t = WL.make_layer_inputs(sh, seed=0, with_dy=True)
    dX, dA, dB = run_bwd(gpu, t["X"], t["W"], t["A"], t["B"], t["dY"], sh.alpha)
    rows = WL.sample_rows(sh.M, seed=2, per_tile=1).numpy()
    _check_all(t, sh.alpha, dX, dA, dB, dx_rows=rows)
    assert torch.isfinite(dX.float()).all()


def test_bwd_attn_proj_full_size(gpu):
    sh = WL.ATTN_PROJ
    t = WL.make_layer_inputs(sh, seed=5, with_dy=True)
    dX, dA, dB = run_bwd(gpu, t["X"], t["W"], t["A"], t["B"], t["dY"], sh.alpha)
    rows = WL.sample_rows(sh.M, seed=3, per_tile=1).numpy()
    _check_all(t, sh.alpha, dX, dA, dB, dx_rows=rows)


def test_bwd_zero_B(gpu):
    """B = 0: dT = 0, so dA is exactly zero and dX = dY W."""
    sh = WL.LayerShape(512, 768, 640, 16, 32.0)
    t = WL.make_layer_inputs(sh, seed=21, with_dy=True)
    t["B"] = torch.zeros_like(t["B"])
    dX, dA, dB = run_bwd(gpu, t["X"], t["W"], t["A"], t["B"], t["dY"], sh.alpha)
    assert torch.count_nonzero(dA.float()) == 0
    _check_all(t, sh.alpha, dX, dA, dB)


def test_bwd_bitwise_repeatable(gpu):
    sh = WL.LayerShape(3000, 1024, 2048, 32, 64.0)
    t = WL.make_layer_inputs(sh, seed=8, with_dy=True)
    a = run_bwd(gpu, t["X"], t["W"], t["A"], t["B"], t["dY"], sh.alpha)
    b = run_bwd(gpu, t["X"], t["W"], t["A"], t["B"], t["dY"], sh.alpha)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bwd_empty_batch_zeroes_adapter_grads(gpu):
    d_in, d_out, r = 64, 128, 16
    W = torch.ones((d_out, d_in), dtype=torch.bfloat16, device="cuda")
    A = torch.ones((r, d_in), dtype=torch.bfloat16, device="cuda")
    B = torch.ones((d_out, r), dtype=torch.bfloat16, device="cuda")
    X = torch.empty((0, d_in), dtype=torch.bfloat16, device="cuda")
    dY = torch.empty((0, d_out), dtype=torch.bfloat16, device="cuda")
    dX = torch.empty((0, d_in), dtype=torch.bfloat16, device="cuda")
    dA = torch.full((r, d_in), 7.0, dtype=torch.bfloat16, device="cuda")
    dB = torch.full((d_out, r), 7.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(64, dtype=torch.float32, device="cuda")
    gpu.lora_bwd(X, W, A, B, dY, dX, dA, dB, 32.0, ws)
    assert gpu.lora_get_device_status() == 0
    assert torch.count_nonzero(dA) == 0 and torch.count_nonzero(dB) == 0


@pytest.mark.parametrize("tile", ["256,2", "256,1", "128,2", "128,1"])
@pytest.mark.parametrize("run", ["0", "2"])
@pytest.mark.parametrize("M,d_in,d_out,r,alpha", [(1000, 1544, 1032, 24, 18.0), (777, 2056, 520, 128, 96.0)])
def test_bwd_every_tile_config_and_schedule(gpu, monkeypatch, tile, run, M, d_in, d_out, r, alpha):
    monkeypatch.setenv("LORA_B200_FUSED_TILE", tile)
    monkeypatch.setenv("LORA_B200_FUSED_RUN", run)
    sh = WL.LayerShape(M, d_in, d_out, r, alpha)
    t = WL.make_layer_inputs(sh, seed=13, with_dy=True)
    dX, dA, dB = run_bwd(gpu, t["X"], t["W"], t["A"], t["B"], t["dY"], alpha)
    _check_all(t, alpha, dX, dA, dB)


# (M, d_in, d_out, r): one split per row tile (no cluster reduction), the
# in-cluster reduction with a ragged last split, r = 128, and an empty batch
FP32_SHAPES = [(1, 8, 8, 8), (300, 520, 264, 8), (4100, 1024, 1536, 32), (257, 256, 384, 128), (0, 512, 264, 24)]


@pytest.mark.parametrize("M,d_in,d_out,r", FP32_SHAPES)
def test_bwd_fp32_grads_round_to_the_bf16_results(gpu, M, d_in, d_out, r):
    """lora_bwd_ex with LORA_BWD_FP32_GRADS: dA and dB are the fp32 sums
    lora_bwd rounds, so rounding them (RNE) reproduces lora_bwd's bf16 dA and
    dB bit for bit; dX is unchanged; the fp32 values meet the tolerance."""
    alpha = 2.0 * r
    sh = WL.LayerShape(M, d_in, d_out, r, alpha)
    t = WL.make_layer_inputs(sh, seed=17 + M, with_dy=True)
    dX16, dA16, dB16 = run_bwd(gpu, t["X"], t["W"], t["A"], t["B"], t["dY"], alpha)
    Xd, Wd, Ad, Bd, dYd = (t[k].cuda() for k in ("X", "W", "A", "B", "dY"))
    nan = float("nan")
    dX = torch.full((M, d_in), nan, dtype=torch.bfloat16, device="cuda")
    dA = torch.full((r, d_in), nan, dtype=torch.float32, device="cuda")
    dB = torch.full((d_out, r), nan, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(gpu.lora_bwd_workspace_size(M, d_in, d_out, r), 256), dtype=torch.uint8, device="cuda")
    gpu.lora_bwd_ex(Xd, Wd, Ad, Bd, dYd, dX, dA, dB, alpha, ws, gpu.LORA_BWD_FP32_GRADS)
    assert gpu.lora_get_device_status() == 0
    assert torch.equal(dX, dX16)
    assert torch.equal(dA.to(torch.bfloat16), dA16) and torch.equal(dB.to(torch.bfloat16), dB16)
    if M == 0:
        assert not dA.any() and not dB.any()
        return
    ref_dX, ref_dA, ref_dB = O.lora_backward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]),
                                             f64(t["dY"]), alpha)
    for name, got, ref in (("dA", dA.double().cpu().numpy(), ref_dA), ("dB", dB.double().cpu().numpy(), ref_dB)):
        ok, info = lora_tol_check(got, ref)
        assert ok, (name, info)


@pytest.mark.parametrize("M,d_in,d_out,r", [(300, 520, 264, 8), (4100, 1024, 1536, 32), (257, 256, 384, 128),
                                            (0, 512, 264, 24)])
@pytest.mark.parametrize("fp32", [False, True])
def test_two_call_backward_equals_one_call(gpu, M, d_in, d_out, r, fp32):
    """lora_bwd_grads then lora_bwd_dx on one workspace give lora_bwd_ex's
    dX, dA and dB bit for bit."""
    alpha = 2.0 * r
    sh = WL.LayerShape(M, d_in, d_out, r, alpha)
    t = WL.make_layer_inputs(sh, seed=31 + M, with_dy=True)
    X, W, A, B, dY = (t[k].cuda() for k in ("X", "W", "A", "B", "dY"))
    gdt = torch.float32 if fp32 else torch.bfloat16
    flags = gpu.LORA_BWD_FP32_GRADS if fp32 else 0
    nan = float("nan")

    def outs():
        return (torch.full((M, d_in), nan, dtype=torch.bfloat16, device="cuda"),
                torch.full((r, d_in), nan, dtype=gdt, device="cuda"),
                torch.full((d_out, r), nan, dtype=gdt, device="cuda"))
    ws = torch.full((max(gpu.lora_bwd_workspace_size(M, d_in, d_out, r), 256),), 255, dtype=torch.uint8,
                    device="cuda")
    dX1, dA1, dB1 = outs()
    gpu.lora_bwd_ex(X, W, A, B, dY, dX1, dA1, dB1, alpha, ws, flags)
    ws.fill_(255)
    dX2, dA2, dB2 = outs()
    gpu.lora_bwd_grads(X, A, B, dY, dA2, dB2, alpha, ws, flags)
    gpu.lora_bwd_dx(W, A, dY, dX2, ws)
    assert gpu.lora_get_device_status() == 0
    assert torch.equal(dA1, dA2) and torch.equal(dB1, dB2)
    assert torch.equal(dX1, dX2)
