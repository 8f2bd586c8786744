"""GPU parity of the explicit-scale entry points (lora_*_scaled) against the
fp64 oracle, at ranks that are not powers of two with rsLoRA's scale
s = alpha / sqrt(r) (unsloth fork commit log, qwen3_flex_inference.py: under
rsLoRA PEFT keeps alpha / sqrt(r) in the module's scaling).

The oracle takes alpha and uses s = alpha / r in float64; it is given
alpha_eq = s32 * r, where s32 is the scale rounded to fp32 as the C ABI
receives it.  s32 has a 24-bit significand and r < 2^8, so s32 * r and
(s32 * r) / r are exact in float64: the oracle then multiplies by s32
itself.  With scale == fp32(alpha / r) each *_scaled call must give its
alpha form's results bit for bit."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL
from gpu_helpers import dev, f64
from tolerance import lora_tol_check, merge_tol_check

pytestmark = pytest.mark.gpu

# (M, d_in, d_out, r, alpha): r = 24 and 40 are not powers of two, so
# alpha / sqrt(r) is not a dyadic fraction
SHAPES = [(300, 520, 264, 24, 16.0), (1000, 1032, 2056, 40, 32.0), (2048, 1024, 4096, 24, 8.0)]


def _s32(alpha, r):
    return float(np.float32(alpha / math.sqrt(r)))


def _nan(shape, dtype=torch.bfloat16):
    return torch.full(shape, float("nan"), dtype=dtype, device="cuda")


@pytest.mark.parametrize("M,d_in,d_out,r,alpha", SHAPES)
def test_scaled_forward_and_backward_match_oracle(gpu, M, d_in, d_out, r, alpha):
    L = gpu
    s = _s32(alpha, r)
    alpha_eq = s * r
    assert alpha_eq / r == s                                      # exact in float64
    sh = WL.LayerShape(M, d_in, d_out, r, alpha)
    t = WL.make_layer_inputs(sh, seed=M + r, with_dy=True)
    X, W, A, B, dY = (dev(t[k]) for k in ("X", "W", "A", "B", "dY"))
    Xf, Wf, Af, Bf, dYf = (f64(t[k]) for k in ("X", "W", "A", "B", "dY"))

    Y = _nan((M, d_out))
    L.lora_fwd_scaled(X, W, A, B, Y, s)
    ok, info = lora_tol_check(f64(Y), O.lora_forward(Xf, Wf, Af, Bf, alpha_eq))
    assert ok, info
    # the same layer through the alpha form differs (s != alpha / r) ...
    Y_alpha = _nan((M, d_out))
    L.lora_fwd(X, W, A, B, Y_alpha, alpha)
    assert not torch.equal(Y, Y_alpha)
    # ... and lora_fwd_save_scaled gives Y bit for bit
    ws = torch.empty(L.lora_bwd_workspace_size(M, d_in, d_out, r), dtype=torch.uint8, device="cuda")
    Y2 = _nan((M, d_out))
    L.lora_fwd_save_scaled(X, W, A, B, Y2, s, ws)
    assert torch.equal(Y, Y2)

    rdX, rdA, rdB = O.lora_backward(Xf, Wf, Af, Bf, dYf, alpha_eq)
    for flags in (0, L.LORA_BWD_T_SAVED):
        if flags:
            L.lora_fwd_save_scaled(X, W, A, B, Y2, s, ws)
        dX, dA, dB = _nan((M, d_in)), _nan((r, d_in)), _nan((d_out, r))
        L.lora_bwd_scaled(X, W, A, B, dY, dX, dA, dB, s, ws, flags)
        assert L.lora_get_device_status() == 0
        for name, g, ref in (("dX", dX, rdX), ("dA", dA, rdA), ("dB", dB, rdB)):
            ok, info = lora_tol_check(f64(g), ref)
            assert ok, (flags, name, info)
        # the two-call form with the scale given
        dX2, dA2, dB2 = _nan((M, d_in)), _nan((r, d_in)), _nan((d_out, r))
        if flags:
            L.lora_fwd_save_scaled(X, W, A, B, Y2, s, ws)
        L.lora_bwd_grads_scaled(X, A, B, dY, dA2, dB2, s, ws, flags)
        L.lora_bwd_dx(W, A, dY, dX2, ws)
        assert torch.equal(dX, dX2) and torch.equal(dA, dA2) and torch.equal(dB, dB2)


def test_scaled_with_alpha_over_r_is_the_alpha_form_bit_for_bit(gpu):
    L = gpu
    M, d_in, d_out, r, alpha = 777, 1032, 1000, 40, 30.0
    s = float(np.float32(np.float32(alpha) / np.float32(r)))      # what the alpha form computes
    t = WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=3, with_dy=True)
    X, W, A, B, dY = (dev(t[k]) for k in ("X", "W", "A", "B", "dY"))
    Ya, Ys = _nan((M, d_out)), _nan((M, d_out))
    L.lora_fwd(X, W, A, B, Ya, alpha)
    L.lora_fwd_scaled(X, W, A, B, Ys, s)
    assert torch.equal(Ya, Ys)
    ws = torch.empty(L.lora_bwd_workspace_size(M, d_in, d_out, r), dtype=torch.uint8, device="cuda")
    outs = []
    for fn, v in ((L.lora_bwd_ex, alpha), (L.lora_bwd_scaled, s)):
        g = (_nan((M, d_in)), _nan((r, d_in)), _nan((d_out, r)))
        fn(X, W, A, B, dY, *g, v, ws, 0)
        outs.append(g)
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    Wa, Ws = torch.empty_like(W), torch.empty_like(W)
    L.lora_merge(W, A, B, Wa, alpha)
    L.lora_merge_scaled(W, A, B, Ws, s)
    assert torch.equal(Wa, Ws)


@pytest.mark.parametrize("d_out,d_in,r,alpha", [(1000, 520, 24, 16.0), (2560, 9728, 40, 32.0)])
def test_scaled_merge_matches_oracle(gpu, d_out, d_in, r, alpha):
    L = gpu
    s = _s32(alpha, r)
    m = WL.make_merge_inputs(d_out, d_in, r, seed=d_out + r)
    W, A, B = dev(m["W"]), dev(m["A"]), dev(m["B"])
    out = _nan((d_out, d_in))
    L.lora_merge_scaled(W, A, B, out, s)
    Wf, Af, Bf = f64(m["W"]), f64(m["A"]), f64(m["B"])
    exact = O.lora_merge(Wf, Af, Bf, s * r)
    ok, info = merge_tol_check(f64(out), exact, Wf, Af, Bf, s)
    assert ok, info
    assert info["max_ulps_noncancel"] <= 1.0, info
    # the batched form, alone and through a prepared batch, gives the same bits
    out2 = _nan((d_out, d_in))
    L.lora_merge_batched_scaled([(W, A, B, out2)], r, s)
    assert torch.equal(out, out2)
    out3 = _nan((d_out, d_in))
    L.MergeBatch([(W, A, B, out3)], r)(0.0, scale=s)
    assert torch.equal(out, out3)


def test_scaled_grouped_forward_matches_oracle(gpu):
    L = gpu
    r, alpha = 24, 16.0
    s = _s32(alpha, r)
    items, refs = [], []
    for i, (M, d_in, d_out) in enumerate(((256, 2560, 1024), (256, 4096, 2560), (300, 520, 264))):
        t = WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=40 + i)
        X, W, A, B = (dev(t[k]) for k in ("X", "W", "A", "B"))
        items.append((X, W, A, B, _nan((M, d_out))))
        refs.append(O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), s * r))
    L.lora_fwd_batched_scaled(items, s)
    assert L.lora_get_device_status() == 0
    for (X, W, A, B, Y), ref in zip(items, refs):
        ok, info = lora_tol_check(f64(Y), ref)
        assert ok, info
