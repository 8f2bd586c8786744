"""The seeded input recipe (CPU): what the documentation states about the
synthetic inputs holds for the generators in workloads.py.

* one torch CPU generator per seed, fp32 normal draws in the order X, W, A,
  B, dY, each cast to bf16 with round-to-nearest-even;
* X and dY ~ N(0, 1), W and A ~ N(0, 1/d_in) (variance), B ~ N(0, 0.02^2);
* the same seed gives the same bits, and dY is drawn last, so asking for it
  leaves X, W, A, B unchanged;
* sampled rows cover the first and last row and every 128-row tile;
* the merge set is 36 layers x 7 targets, the sweep 5 x 5 x 5 points."""
import math

import torch

import workloads as WL


def _bits_equal(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_draw_order_and_rounding():
    sh = WL.LayerShape(M=37, d_in=40, d_out=24, r=8, alpha=16.0)
    t = WL.make_layer_inputs(sh, seed=123, with_dy=True)
    g = torch.Generator(device="cpu")
    g.manual_seed(123)
    std_w = 1.0 / math.sqrt(sh.d_in)
    want = {}
    for name, shape, std in (("X", (37, 40), 1.0), ("W", (24, 40), std_w), ("A", (8, 40), std_w),
                             ("B", (24, 8), 0.02), ("dY", (37, 24), 1.0)):
        x = torch.randn(*shape, generator=g, dtype=torch.float32)
        want[name] = (x * std if std != 1.0 else x).to(torch.bfloat16)
    for name in want:
        assert t[name].dtype == torch.bfloat16 and t[name].shape == want[name].shape
        assert _bits_equal(t[name], want[name]), name


def test_same_seed_same_bits_and_dy_drawn_last():
    sh = WL.LayerShape(M=64, d_in=128, d_out=96, r=16, alpha=32.0)
    a = WL.make_layer_inputs(sh, seed=5)
    b = WL.make_layer_inputs(sh, seed=5, with_dy=True)
    c = WL.make_layer_inputs(sh, seed=6)
    for k in ("X", "W", "A", "B"):
        assert _bits_equal(a[k], b[k]), k
        assert not torch.equal(a[k], c[k]), k
    assert "dY" not in a and b["dY"].shape == (64, 96)


def test_distributions():
    sh = WL.LayerShape(M=512, d_in=1024, d_out=768, r=64, alpha=128.0)
    t = WL.make_layer_inputs(sh, seed=1, with_dy=True)
    for name, std in (("X", 1.0), ("W", 1.0 / 32.0), ("A", 1.0 / 32.0), ("B", 0.02), ("dY", 1.0)):
        v = t[name].float()
        assert abs(v.mean().item()) < 0.05 * std, name
        assert abs(v.std().item() / std - 1.0) < 0.03, (name, v.std().item())


def test_sample_rows_cover_every_tile():
    for M in (1, 127, 128, 129, 1000, 8192):
        rows = WL.sample_rows(M, seed=3, per_tile=1)
        r = rows.tolist()
        assert r == sorted(set(r)) and r[0] == 0 and r[-1] == M - 1
        assert all(0 <= i < M for i in r)
        for t0 in range(0, M, 128):
            assert any(t0 <= i < t0 + 128 for i in r), (M, t0)
    assert torch.equal(WL.sample_rows(1000, seed=3), WL.sample_rows(1000, seed=3))


def test_workload_sets():
    shapes = WL.merge_shapes()
    assert len(shapes) == 36 * 7 and WL.MERGE_LAYERS == 36
    assert len({(s["target"]) for s in shapes}) == 7
    pts = WL.sweep_points()
    assert len(pts) == 125
    assert {p.r for p in pts} == set(WL.SWEEP_R) and {p.M for p in pts} == set(WL.SWEEP_M)
    assert (WL.ATTN_PROJ.M, WL.ATTN_PROJ.d_in, WL.ATTN_PROJ.d_out, WL.ATTN_PROJ.r) == (8192, 4096, 4096, 16)
    assert (WL.MLP_UP.M, WL.MLP_UP.d_in, WL.MLP_UP.d_out, WL.MLP_UP.r) == (16384, 4096, 14336, 64)


def test_perturbation_is_seeded_by_cycle():
    m = WL.make_merge_inputs(64, 128, 8, seed=9)
    a1, b1 = WL.perturb_adapter(m["A"], m["B"], cycle=1)
    a1b, b1b = WL.perturb_adapter(m["A"], m["B"], cycle=1)
    a2, _ = WL.perturb_adapter(m["A"], m["B"], cycle=2)
    assert _bits_equal(a1, a1b) and _bits_equal(b1, b1b) and not torch.equal(a1, a2)
    d = (a1.float() - m["A"].float()).std().item()
    assert 0.008 < d < 0.012
