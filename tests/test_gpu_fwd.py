"""GPU parity of lora_fwd against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL
from gpu_helpers import dev, f64, run_fwd
from tolerance import lora_tol_check

pytestmark = pytest.mark.gpu

# (M, d_in, d_out, r, alpha): several tiles and ragged tails in every
# dimension, every rank-chunk width (16/32/64) and both tile widths.
SHAPES = [
    (256, 512, 512, 16, 32.0),      # tiny forward workload (full check)
    (1, 8, 8, 8, 16.0),             # smallest legal problem
    (300, 520, 264, 8, 6.0),        # r = 8 padded to 16; scale 0.75
    (129, 64, 136, 24, 18.0),       # r = 24 -> 32
    (777, 1032, 1000, 40, 30.0),    # r = 40 -> 48 (64-wide chunk, partly empty)
    (1000, 512, 2056, 64, 128.0),
    (257, 256, 384, 128, 96.0),     # largest rank
    (2048, 1024, 4096, 32, 64.0),   # enough tiles for 256-wide tiles
    (640, 2048, 1544, 16, 12.0),
]


@pytest.mark.parametrize("M,d_in,d_out,r,alpha", SHAPES)
def test_fwd_matches_oracle(gpu, M, d_in, d_out, r, alpha):
    sh = WL.LayerShape(M, d_in, d_out, r, alpha)
    t = WL.make_layer_inputs(sh, seed=M + d_in + r)
    Y = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), alpha)
    ok, info = lora_tol_check(f64(Y), ref)
    assert ok, info


@pytest.mark.parametrize("shape", [WL.ATTN_PROJ, WL.MLP_UP], ids=lambda s: s.name)
def test_fwd_full_size_sampled_rows(gpu, shape):
    """Full-size workloads in the benchmark's launch configuration; every
    128-row tile contributes sampled rows (plus first and last)."""
    t = WL.make_layer_inputs(shape, seed=0)
    Y = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], shape.alpha)
    rows = WL.sample_rows(shape.M, seed=1, per_tile=1)
    ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), shape.alpha, rows=rows.numpy())
    ok, info = lora_tol_check(f64(Y.cpu()[rows]), ref)
    assert ok, info
    assert torch.isfinite(Y.float()).all()


def test_fwd_zero_adapter_gives_base_and_is_bitwise_stable(gpu):
    sh = WL.LayerShape(640, 1024, 768, 16, 32.0)
    t = WL.make_layer_inputs(sh, seed=3)
    zB = torch.zeros_like(t["B"])
    zA = torch.zeros_like(t["A"])
    Y_b0 = run_fwd(gpu, t["X"], t["W"], t["A"], zB, sh.alpha)
    Y_a0 = run_fwd(gpu, t["X"], t["W"], zA, t["B"], sh.alpha)
    # either factor zero => the adapter adds exact zeros to the same base sum
    assert torch.equal(Y_b0, Y_a0)
    ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), np.zeros((768, 16)), sh.alpha)
    ok, info = lora_tol_check(f64(Y_b0), ref)
    assert ok, info


def test_fwd_deterministic(gpu):
    sh = WL.LayerShape(1024, 1024, 2048, 32, 64.0)
    t = WL.make_layer_inputs(sh, seed=9)
    Y1 = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], sh.alpha)
    Y2 = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], sh.alpha)
    assert torch.equal(Y1, Y2)


def test_merged_forward_equals_unmerged(gpu):
    """X W'^T with W' = merge(W, A, B) matches the unmerged forward."""
    sh = WL.LayerShape(512, 1024, 1024, 16, 32.0)
    t = WL.make_layer_inputs(sh, seed=4)
    Wd, Ad, Bd = dev(t["W"]), dev(t["A"]), dev(t["B"])
    Wm = torch.empty_like(Wd)
    gpu.lora_merge(Wd, Ad, Bd, Wm, sh.alpha)
    Y_unmerged = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], sh.alpha)
    Y_merged = run_fwd(gpu, t["X"], Wm.cpu(), t["A"], torch.zeros_like(t["B"]), sh.alpha)
    ok, info = lora_tol_check(f64(Y_merged), f64(Y_unmerged))
    assert ok, info
    ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), sh.alpha)
    ok, info = lora_tol_check(f64(Y_merged), ref)
    assert ok, info


def test_fwd_empty_batch_is_noop(gpu):
    X = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.ones((64, 64), dtype=torch.bfloat16, device="cuda")
    A = torch.ones((16, 64), dtype=torch.bfloat16, device="cuda")
    B = torch.ones((64, 16), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    gpu.lora_fwd(X, W, A, B, Y, 32.0)
    assert gpu.lora_get_device_status() == 0


TILES = ["256,2", "256,1", "128,2", "128,1"]


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("run", ["0", "1", "3"])
@pytest.mark.parametrize("M,d_in,d_out,r,alpha", [(1000, 1032, 1544, 24, 18.0), (777, 520, 2056, 128, 96.0)])
def test_fwd_every_tile_config_and_schedule(gpu, monkeypatch, tile, run, M, d_in, d_out, r, alpha):
    """Every tile configuration (BN, CTA pair or single CTA) and schedule
    (contiguous ranges, runs of 1 and 3 N tiles) against the oracle.  At
    r = 128, 256-wide single-CTA tiles have no room for three stages and the
    override falls back to the automatic choice (tests/test_plan.py)."""
    monkeypatch.setenv("LORA_B200_FUSED_TILE", tile)
    monkeypatch.setenv("LORA_B200_FUSED_RUN", run)
    sh = WL.LayerShape(M, d_in, d_out, r, alpha)
    t = WL.make_layer_inputs(sh, seed=7)
    Y = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), alpha)
    ok, info = lora_tol_check(f64(Y), ref)
    assert ok, info


# Split-K forward (few output tiles): the S CTAs of a cluster share one
# 128 x 128 tile and reduce T and the base through distributed shared memory.
SPLITK_SHAPES = [
    (128, 4096, 4096, 16, 32.0),    # 32 tiles, S = 4
    (100, 1000, 520, 24, 18.0),     # ragged M, N and K; r = 24 -> 32
    (64, 2048, 256, 128, 96.0),     # largest rank: N = 128 + 128 in one MMA
    (200, 3072, 136, 8, 6.0),       # r = 8 -> 16, N tail of 8 columns
    (384, 1344, 1024, 40, 30.0),    # 21 K blocks over 2 splits (11 + 10); 64-wide rank chunk
]


@pytest.mark.parametrize("M,d_in,d_out,r,alpha", SPLITK_SHAPES)
def test_fwd_splitk_matches_oracle_and_fused(gpu, monkeypatch, M, d_in, d_out, r, alpha):
    sh = WL.LayerShape(M, d_in, d_out, r, alpha)
    t = WL.make_layer_inputs(sh, seed=M + d_out + r)
    ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), alpha)
    monkeypatch.setenv("LORA_B200_SPLITK", "1")
    Y1 = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    Y1b = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    assert torch.equal(Y1, Y1b)            # fixed-order reduction: bitwise repeatable
    ok, info = lora_tol_check(f64(Y1), ref)
    assert ok, ("split-K", info)
    monkeypatch.setenv("LORA_B200_SPLITK", "0")
    Y0 = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    ok, info = lora_tol_check(f64(Y0), ref)
    assert ok, ("one CTA per tile", info)
    assert gpu.lora_get_device_status() == 0


def test_fwd_splitk_zero_adapter_gives_base(gpu, monkeypatch):
    """B = 0 and A = 0 both give the base product exactly (split-K path)."""
    monkeypatch.setenv("LORA_B200_SPLITK", "1")
    sh = WL.LayerShape(128, 2048, 512, 16, 32.0)
    t = WL.make_layer_inputs(sh, seed=5)
    Y_b0 = run_fwd(gpu, t["X"], t["W"], t["A"], torch.zeros_like(t["B"]), sh.alpha)
    Y_a0 = run_fwd(gpu, t["X"], t["W"], torch.zeros_like(t["A"]), t["B"], sh.alpha)
    assert torch.equal(Y_b0, Y_a0)
    ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), np.zeros((512, 16)), sh.alpha)
    ok, info = lora_tol_check(f64(Y_b0), ref)
    assert ok, info


def test_fwd_batched_matches_oracle_and_is_repeatable(gpu):
    """One grouped launch over problems of different sizes (an empty one
    included) with a shared rank; every Y against the oracle."""
    r, alpha = 24, 18.0
    # (4096, 512, 2560) has 640 tiles (over four per SM): it takes the lora_fwd path
    shapes = [(300, 520, 264), (1, 64, 136), (0, 256, 128), (700, 1024, 512), (128, 4096, 1024), (64, 2560, 4096),
              (2048, 512, 1280), (4096, 512, 2560)]
    items, hosts = [], []
    for i, (M, d_in, d_out) in enumerate(shapes):
        t = WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=100 + i)
        X, W, A, B = (dev(t[k]) for k in ("X", "W", "A", "B"))
        items.append((X, W, A, B, torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")))
        hosts.append(t)
    gpu.lora_fwd_batched(items, alpha)
    first = [it[4].clone() for it in items]
    gpu.lora_fwd_batched(items, alpha)
    assert gpu.lora_get_device_status() == 0
    for (X, W, A, B, Y), Y1, t in zip(items, first, hosts):
        assert torch.equal(Y, Y1)
        if Y.shape[0] == 0:
            continue
        ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), alpha)
        ok, info = lora_tol_check(f64(Y.cpu()), ref)
        assert ok, (tuple(X.shape), tuple(W.shape), info)


def test_fwd_batched_more_problems_than_one_launch(gpu):
    """45 problems: the call splits them over two launches (40 per launch)."""
    r, alpha = 16, 32.0
    items, hosts = [], []
    for i in range(45):
        M, d_in, d_out = 64 + 8 * (i % 5), 256 + 64 * (i % 3), 128 + 8 * (i % 7)
        t = WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=200 + i)
        X, W, A, B = (dev(t[k]) for k in ("X", "W", "A", "B"))
        items.append((X, W, A, B, torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")))
        hosts.append(t)
    gpu.lora_fwd_batched(items, alpha)
    assert gpu.lora_get_device_status() == 0
    for (X, W, A, B, Y), t in zip(items, hosts):
        ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), alpha)
        ok, info = lora_tol_check(f64(Y.cpu()), ref)
        assert ok, info


@pytest.mark.parametrize("r", [8, 64, 128])
def test_fwd_batched_other_ranks(gpu, r):
    """Grouped launches at the smallest rank, at r = 64 (short contractions
    are not split there) and at r = 128 (base and T in one N = 256 MMA)."""
    alpha = 2.0 * r
    shapes = [(300, 520, 264), (128, 1024, 512), (64, 4096, 1024), (700, 2048, 136)]
    items, hosts = [], []
    for i, (M, d_in, d_out) in enumerate(shapes):
        t = WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=300 + 10 * r + i)
        X, W, A, B = (dev(t[k]) for k in ("X", "W", "A", "B"))
        items.append((X, W, A, B, torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda")))
        hosts.append(t)
    gpu.lora_fwd_batched(items, alpha)
    assert gpu.lora_get_device_status() == 0
    for (X, W, A, B, Y), t in zip(items, hosts):
        ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), alpha)
        ok, info = lora_tol_check(f64(Y.cpu()), ref)
        assert ok, (r, tuple(X.shape), tuple(W.shape), info)
