"""The forward on 224-wide CTA-pair tiles with T folded into the base
product (one N = 256 MMA per K step: the even CTA's 128 rows of W, the odd
CTA's 96 rows of W and 32 rows of A).

Every output element sums the same products in the same order as on the
256-wide pair tile, and T's columns the same products as the separate N = r
MMA there, so Y must equal the 256-wide tile's Y bit for bit, and match the
oracle.  The cases cover the shape class the planner gives the fold, a ragged last
column tile (d_out not a multiple of 224, and tiles wholly past d_out in the
odd CTA's half), ragged M and K, r from 8 to 32 (U rows past r are zero
fill), and T kept for the backward."""
import pytest
import torch

import oracle as O
import workloads as WL
from gpu_helpers import dev, f64, run_fwd
from tolerance import lora_tol_check

pytestmark = pytest.mark.gpu

# (M, d_in, d_out, r, alpha, tile forced or None for the planner's choice)
SHAPES = [
    (512, 8192, 8192, 16, 32.0, None),      # chosen by the planner: 2 x 37 tiles on 74 pairs
    (2048, 8192, 8192, 32, 64.0, "224,2"),  # 8 x 37 tiles, r = 32 fills T's columns
    (512, 4096, 14336, 8, 16.0, "224,2"),   # 2 x 64 tiles, r = 8
    (600, 1032, 712, 24, 12.0, "224,2"),    # ragged M, K, N: 712 = 3 x 224 + 40
    (300, 2048, 248, 16, 32.0, "224,2"),    # the odd CTA's rows all past d_out in the last tile
    (256, 520, 224, 32, 8.0, "224,2"),      # one tile, exactly 224 wide
]


def _env(monkeypatch, tile=None, run=None):
    for k, v in (("LORA_B200_FUSED_TILE", tile), ("LORA_B200_FUSED_RUN", run)):
        if v is None:
            monkeypatch.delenv(k, raising=False)
        else:
            monkeypatch.setenv(k, v)
    monkeypatch.setenv("LORA_B200_SPLITK", "0")


@pytest.mark.parametrize("M,d_in,d_out,r,alpha,tile", SHAPES)
def test_pair_fold_equals_256_tile_and_oracle(gpu, monkeypatch, M, d_in, d_out, r, alpha, tile):
    t = WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=M + d_out + r)
    _env(monkeypatch, tile=tile)
    assert gpu.lora_plan(M, d_in, d_out, r)["fwd_bn"] == 224
    Y = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    _env(monkeypatch, tile="224,2", run="4")     # runs of 4: T computed once per run, reused
    Y_runs = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    _env(monkeypatch, tile="256,2")
    Y_256 = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    assert torch.equal(Y, Y_runs)
    assert torch.equal(Y, Y_256)
    if M * d_out <= 1 << 20:
        ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), alpha)
        ok, info = lora_tol_check(f64(Y.cpu()), ref)
    else:
        rows = WL.sample_rows(M, seed=7, per_tile=1)
        ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), alpha, rows=rows.numpy())
        ok, info = lora_tol_check(f64(Y.cpu()[rows]), ref)
    assert ok, info


def test_pair_fold_saved_t_matches_256_tile(gpu, monkeypatch):
    M, d_in, d_out, r, alpha = 512, 8192, 8192, 16, 32.0
    t = WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=17)
    X, W, A, B = (dev(t[k]) for k in ("X", "W", "A", "B"))
    n_ws = gpu.lora_bwd_workspace_size(M, d_in, d_out, r)
    outs = []
    for tile in (None, "256,2"):
        _env(monkeypatch, tile=tile)
        Y = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
        ws = torch.full((n_ws,), 0xFF, dtype=torch.uint8, device="cuda")
        gpu.lora_fwd_save(X, W, A, B, Y, alpha, ws)
        assert gpu.lora_get_device_status() == 0
        outs.append((Y, ws[: M * 16 * 2].clone()))
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])
    T = outs[0][1].view(torch.bfloat16).view(M, 16)
    ref = f64(t["X"]) @ f64(t["A"]).T
    err = abs(f64(T.cpu()) - ref)
    assert (err <= 2 ** -7 * abs(ref) + 1e-3).all()            # one bf16 rounding of an fp32 sum


def test_pair_fold_zero_adapter_gives_the_base_product(gpu, monkeypatch):
    """B = 0: the T columns and the up-projection add exactly nothing, so Y is
    the 256-wide tile's base product bit for bit."""
    M, d_in, d_out, r, alpha = 512, 4096, 4096, 16, 32.0
    t = WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=23)
    B0 = torch.zeros_like(t["B"])
    _env(monkeypatch, tile="224,2")
    Y = run_fwd(gpu, t["X"], t["W"], t["A"], B0, alpha)
    _env(monkeypatch, tile="256,2")
    Y_256 = run_fwd(gpu, t["X"], t["W"], t["A"], B0, alpha)
    assert torch.equal(Y, Y_256)
