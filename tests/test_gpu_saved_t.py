"""GPU parity of the saved-T path: lora_fwd_save writes T = X A^T into the
backward's workspace beside an unchanged Y, and the backward with
LORA_BWD_T_SAVED uses it instead of recomputing T.

T is checked against the fp64 oracle's down-projection with the bound of a
bf16 rounding of an fp32 sum over d_in products: one bf16 ULP of the exact
value plus (d_in + 2) 2^-23 (|X| |A|^T).  The workspace layout of T (bf16
[M, r_pad] at offset 0, r_pad = r rounded up to 16) is the library's own;
these tests read it to check what the forward wrote."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL
from gpu_helpers import f64
from tolerance import lora_tol_check

pytestmark = pytest.mark.gpu


def _r_pad(r):
    return (r + 15) // 16 * 16


def _inputs(M, d_in, d_out, r, alpha, seed):
    t = WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=seed, with_dy=True)
    return t, {k: t[k].cuda() for k in ("X", "W", "A", "B", "dY")}


def _ws(L, M, d_in, d_out, r):
    # 0xFF bytes: every bf16 in it starts as NaN, so a T row the forward
    # does not write shows up
    return torch.full((max(L.lora_bwd_workspace_size(M, d_in, d_out, r), 256),), 255, dtype=torch.uint8,
                      device="cuda")


def _saved_t(ws, M, r):
    rp = _r_pad(r)
    return ws[: M * rp * 2].view(torch.bfloat16).view(M, rp)


def _check_t(Tg, t, r, rows=None):
    """T rows against the oracle (bound in the module docstring); padding
    columns exactly zero."""
    X, A = f64(t["X"]), f64(t["A"])
    Tg = Tg.cpu()
    if rows is not None:
        Tg = Tg[torch.as_tensor(rows)]
        X = X[rows]
    got = f64(Tg)
    assert np.all(got[:, r:] == 0.0), "T columns past r must be zero"
    ref = O.lora_down(X, A)
    bound = O.ulp_bf16(ref) + (X.shape[1] + 2) * 2.0 ** -23 * (np.abs(X) @ np.abs(A).T)
    err = np.abs(got[:, :r] - ref)
    bad = ~(err <= bound)
    assert not bad.any(), dict(n_bad=int(bad.sum()), worst=float(np.nanmax(err / bound)))


def _fwd_pair(L, d, alpha, ws):
    M, d_out = d["X"].shape[0], d["W"].shape[0]
    Y0 = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
    Y1 = torch.full_like(Y0, float("nan"))
    L.lora_fwd(d["X"], d["W"], d["A"], d["B"], Y0, alpha)
    L.lora_fwd_save(d["X"], d["W"], d["A"], d["B"], Y1, alpha, ws)
    assert L.lora_get_device_status() == 0
    return Y0, Y1


SHAPES = [
    (256, 512, 512, 16, 32.0),      # tiny workload (tiled, 128-wide tiles)
    (1, 8, 8, 8, 16.0),
    (300, 520, 264, 8, 6.0),
    (777, 1032, 1000, 40, 30.0),    # split-contraction forward: T from one more launch
    (1000, 512, 2056, 64, 128.0),
    (257, 256, 384, 128, 96.0),
    (2048, 1024, 4096, 32, 64.0),   # tiled forward, 256-wide tiles, runs of 2
    (4100, 1024, 1536, 32, 64.0),   # ragged last M block
]


@pytest.mark.parametrize("M,d_in,d_out,r,alpha", SHAPES)
def test_fwd_save_keeps_y_and_writes_t(gpu, M, d_in, d_out, r, alpha):
    t, d = _inputs(M, d_in, d_out, r, alpha, seed=40 + M)
    ws = _ws(gpu, M, d_in, d_out, r)
    Y0, Y1 = _fwd_pair(gpu, d, alpha, ws)
    assert torch.equal(Y0, Y1)
    _check_t(_saved_t(ws, M, r), t, r)


@pytest.mark.parametrize("tile", ["256,2", "256,1", "128,2", "128,1"])
@pytest.mark.parametrize("run", ["0", "1", "3"])
@pytest.mark.parametrize("M,d_in,d_out,r,alpha", [(1000, 1032, 1544, 24, 18.0), (777, 520, 2056, 128, 96.0)])
def test_fwd_save_every_tile_config_and_schedule(gpu, monkeypatch, tile, run, M, d_in, d_out, r, alpha):
    """The tile of N index 0 of every M block writes T: checked for every tile
    configuration and schedule (contiguous ranges, runs of 1 and 3; at
    r = 128 a forced 256 x 1 tile falls back to the automatic choice)."""
    monkeypatch.setenv("LORA_B200_FUSED_TILE", tile)
    monkeypatch.setenv("LORA_B200_FUSED_RUN", run)
    t, d = _inputs(M, d_in, d_out, r, alpha, seed=7)
    ws = _ws(gpu, M, d_in, d_out, r)
    Y0, Y1 = _fwd_pair(gpu, d, alpha, ws)
    assert torch.equal(Y0, Y1)
    _check_t(_saved_t(ws, M, r), t, r)


@pytest.mark.parametrize("splitk", ["0", "1"])
def test_fwd_save_both_forward_forms(gpu, monkeypatch, splitk):
    """The same problem through the tiled forward (T from the epilogue) and
    the split-contraction forward (T from one more launch)."""
    monkeypatch.setenv("LORA_B200_SPLITK", splitk)
    M, d_in, d_out, r, alpha = 384, 1344, 1024, 40, 30.0
    t, d = _inputs(M, d_in, d_out, r, alpha, seed=3)
    ws = _ws(gpu, M, d_in, d_out, r)
    Y0, Y1 = _fwd_pair(gpu, d, alpha, ws)
    assert torch.equal(Y0, Y1)
    _check_t(_saved_t(ws, M, r), t, r)


def _bwd(L, d, alpha, ws, flags):
    M, d_in = d["X"].shape
    d_out, r = d["B"].shape
    nan = float("nan")
    gdt = torch.float32 if flags & L.LORA_BWD_FP32_GRADS else torch.bfloat16
    dX = torch.full((M, d_in), nan, dtype=torch.bfloat16, device="cuda")
    dA = torch.full((r, d_in), nan, dtype=gdt, device="cuda")
    dB = torch.full((d_out, r), nan, dtype=gdt, device="cuda")
    L.lora_bwd_ex(d["X"], d["W"], d["A"], d["B"], d["dY"], dX, dA, dB, alpha, ws, flags)
    assert L.lora_get_device_status() == 0
    return dX, dA, dB


@pytest.mark.parametrize("M,d_in,d_out,r,alpha", SHAPES)
def test_bwd_with_saved_t_matches_oracle(gpu, M, d_in, d_out, r, alpha):
    t, d = _inputs(M, d_in, d_out, r, alpha, seed=60 + M)
    ws = _ws(gpu, M, d_in, d_out, r)
    _fwd_pair(gpu, d, alpha, ws)
    dX, dA, dB = _bwd(gpu, d, alpha, ws, gpu.LORA_BWD_T_SAVED)
    ref = O.lora_backward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), f64(t["dY"]), alpha)
    for name, got, want in zip(("dX", "dA", "dB"), (dX, dA, dB), ref):
        ok, info = lora_tol_check(f64(got), want)
        assert ok, (name, info)


@pytest.mark.parametrize("M,d_in,d_out,r", [(300, 520, 264, 8), (4100, 1024, 1536, 32), (257, 256, 384, 128)])
def test_saved_t_backward_two_calls_and_fp32(gpu, M, d_in, d_out, r):
    """With T saved: lora_bwd_grads + lora_bwd_dx give lora_bwd_ex's results
    bit for bit, and the fp32 gradients round to the bf16 ones."""
    alpha = 2.0 * r
    t, d = _inputs(M, d_in, d_out, r, alpha, seed=90 + M)
    ws = _ws(gpu, M, d_in, d_out, r)
    _fwd_pair(gpu, d, alpha, ws)
    T_fwd = _saved_t(ws, M, r).clone()
    flags = gpu.LORA_BWD_T_SAVED
    dX1, dA1, dB1 = _bwd(gpu, d, alpha, ws, flags)
    # the backward leaves the saved T as it found it
    assert torch.equal(_saved_t(ws, M, r), T_fwd)
    dX2 = torch.full_like(dX1, float("nan"))
    dA2 = torch.full_like(dA1, float("nan"))
    dB2 = torch.full_like(dB1, float("nan"))
    gpu.lora_bwd_grads(d["X"], d["A"], d["B"], d["dY"], dA2, dB2, alpha, ws, flags)
    gpu.lora_bwd_dx(d["W"], d["A"], d["dY"], dX2, ws)
    assert gpu.lora_get_device_status() == 0
    assert torch.equal(dX1, dX2) and torch.equal(dA1, dA2) and torch.equal(dB1, dB2)
    _, dA3, dB3 = _bwd(gpu, d, alpha, ws, flags | gpu.LORA_BWD_FP32_GRADS)
    assert torch.equal(dA3.to(torch.bfloat16), dA1) and torch.equal(dB3.to(torch.bfloat16), dB1)


def test_saved_t_attn_proj_full_size(gpu):
    """Attention-projection workload at full size, in the benchmark's launch
    configuration: T on sampled rows of every tile, dX on sampled rows, dA and
    dB in full."""
    sh = WL.ATTN_PROJ
    t = WL.make_layer_inputs(sh, seed=5, with_dy=True)
    d = {k: t[k].cuda() for k in ("X", "W", "A", "B", "dY")}
    ws = _ws(gpu, sh.M, sh.d_in, sh.d_out, sh.r)
    Y0, Y1 = _fwd_pair(gpu, d, sh.alpha, ws)
    assert torch.equal(Y0, Y1)
    rows = WL.sample_rows(sh.M, seed=4, per_tile=1).numpy()
    _check_t(_saved_t(ws, sh.M, sh.r), t, sh.r, rows=rows)
    dX, dA, dB = _bwd(gpu, d, sh.alpha, ws, gpu.LORA_BWD_T_SAVED)
    ref_dX, ref_dA, ref_dB = O.lora_backward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), f64(t["dY"]),
                                             sh.alpha, dx_rows=rows)
    got_dX = f64(dX.cpu()[torch.as_tensor(rows)])
    for name, got, want in (("dX", got_dX, ref_dX), ("dA", f64(dA), ref_dA), ("dB", f64(dB), ref_dB)):
        ok, info = lora_tol_check(got, want)
        assert ok, (name, info)


def test_fwd_save_empty_batch(gpu):
    """M = 0: nothing is written, a NULL (empty) workspace is accepted."""
    d_in, d_out, r = 512, 264, 24
    X = torch.empty((0, d_in), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((d_out, d_in), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((r, d_in), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((d_out, r), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((0, d_out), dtype=torch.bfloat16, device="cuda")
    gpu.lora_fwd_save(X, W, A, B, Y, 48.0, torch.empty(0, dtype=torch.uint8, device="cuda"))
    assert gpu.lora_get_device_status() == 0
