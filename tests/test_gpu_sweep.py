"""Forward parity on every point of the square sweep
(d_in = d_out in {512..8192} x M in {128..16384} x r in {8..128},
alpha = 2r, seed = point index), in the launch configuration the library
picks for each shape.  Rows are sampled per 128-row tile (first and last
row included); every column is checked."""
import pytest
import torch

import oracle as O
import workloads as WL
from gpu_helpers import f64, run_fwd
from tolerance import lora_tol_check

pytestmark = pytest.mark.gpu

POINTS = WL.sweep_points()


@pytest.mark.parametrize("idx", range(len(POINTS)), ids=[p.name for p in POINTS])
def test_sweep_point_matches_oracle(gpu, idx):
    sh = POINTS[idx]
    t = WL.make_layer_inputs(sh, seed=idx)
    Y = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], sh.alpha)
    rows = WL.sample_rows(sh.M, seed=idx, per_tile=1).numpy()
    ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), sh.alpha, rows=rows)
    ok, info = lora_tol_check(f64(Y.cpu()[torch.as_tensor(rows)]), ref)
    assert ok, info
