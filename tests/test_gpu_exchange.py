"""The forward's T exchange between clusters (texchange.cuh) and the
schedule it enables (a seeding run per cluster that computes every M
block's T, then single tiles dealt round-robin that copy it).

A cluster that finds an M block's s T published copies it instead of
computing it; the published values are the very ones it would have
computed, so Y must be bit for bit the same with the exchange on or off
(LORA_B200_TX=0) and under the earlier run schedule (LORA_B200_FUSED_RUN),
and must match the oracle.  lora_fwd_save's T must not depend on which
cluster computed it.  Two forwards running at the same time on two streams
each get their own exchange slot."""
import pytest
import torch

import oracle as O
import workloads as WL
from gpu_helpers import dev, f64, run_fwd
from tolerance import lora_tol_check

pytestmark = pytest.mark.gpu

# (M, d_in, d_out, r, alpha, tile override or None)
SHAPES = [
    (8192, 4096, 4096, 16, 32.0, None),      # attention projection: seeding runs of 2 on 74 pairs
    (8192, 4096, 4096, 128, 96.0, None),     # largest rank: T borrows the other accumulator
    (16384, 4096, 4096, 24, 18.0, None),     # 64 M blocks for 74 pairs, r = 24 -> 32
    (8000, 1032, 4104, 40, 30.0, None),      # ragged M, N and K
    (4100, 1024, 6152, 16, 12.0, "128,1"),   # 128-wide single CTAs: T folded into the base product
    (8192, 8192, 8192, 16, 32.0, None),      # four column bands: the tiles after seeding go band by band
]


def _env(monkeypatch, tx=None, run=None, tile=None, seeded_l=None):
    for k, v in (("LORA_B200_TX", tx), ("LORA_B200_FUSED_RUN", run), ("LORA_B200_FUSED_TILE", tile),
                 ("LORA_B200_SEEDED_L", seeded_l)):
        if v is None:
            monkeypatch.delenv(k, raising=False)
        else:
            monkeypatch.setenv(k, v)
    monkeypatch.setenv("LORA_B200_SPLITK", "0")


@pytest.mark.parametrize("M,d_in,d_out,r,alpha,tile", SHAPES)
def test_exchange_gives_identical_y_and_matches_oracle(gpu, monkeypatch, M, d_in, d_out, r, alpha, tile):
    sh = WL.LayerShape(M, d_in, d_out, r, alpha)
    t = WL.make_layer_inputs(sh, seed=M + r)
    _env(monkeypatch, tile=tile)
    plan = gpu.lora_plan(M, d_in, d_out, r)
    assert plan["fwd_tx"] == 1 and plan["fwd_seeded"] == 1
    Y = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    Y_again = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    _env(monkeypatch, tile=tile, tx="0")
    Y_no_tx = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    _env(monkeypatch, tile=tile, run="8")
    Y_runs8 = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    _env(monkeypatch, tile=tile, run="1")                    # every tile starts an M block: mostly copies
    Y_runs1 = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    _env(monkeypatch, tile=tile, seeded_l="1")               # copies start before every T is published
    Y_seed1 = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    _env(monkeypatch, tile=tile, seeded_l="4")
    Y_seed4 = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    for other in (Y_again, Y_no_tx, Y_runs8, Y_runs1, Y_seed1, Y_seed4):
        assert torch.equal(Y, other)
    rows = WL.sample_rows(M, seed=3, per_tile=1)
    ref = O.lora_forward(f64(t["X"]), f64(t["W"]), f64(t["A"]), f64(t["B"]), alpha, rows=rows.numpy())
    ok, info = lora_tol_check(f64(Y.cpu()[rows]), ref)
    assert ok, info


def test_exchange_saved_t_independent_of_who_computed_it(gpu, monkeypatch):
    M, d_in, d_out, r, alpha = 8192, 4096, 4096, 16, 32.0
    t = WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=11)
    X, W, A, B = (dev(t[k]) for k in ("X", "W", "A", "B"))
    n_ws = gpu.lora_bwd_workspace_size(M, d_in, d_out, r)
    outs = []
    for tx in (None, "0"):
        _env(monkeypatch, tx=tx)
        Y = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
        ws = torch.full((n_ws,), 0xFF, dtype=torch.uint8, device="cuda")
        gpu.lora_fwd_save(X, W, A, B, Y, alpha, ws)
        assert gpu.lora_get_device_status() == 0
        outs.append((Y, ws[: M * 16 * 2].clone()))            # the T slot: bf16 [M, 16]
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])
    T = outs[0][1].view(torch.bfloat16).view(M, 16)
    ref = f64(t["X"]) @ f64(t["A"]).T
    err = abs(f64(T.cpu()) - ref)
    assert (err <= 2 ** -7 * abs(ref) + 1e-3).all()            # one bf16 rounding of an fp32 sum


def test_exchange_many_launches_queued_on_one_stream(gpu, monkeypatch):
    """Ten forwards queued back to back on one stream, the host far ahead of
    the GPU, alternating two inputs: each launch finds the stream's slot as
    the previous launch left it (clean), so each output is exact."""
    _env(monkeypatch)
    M, d_in, d_out, r, alpha = 8192, 4096, 4096, 16, 32.0
    ins = [WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=s) for s in (31, 32)]
    dv = [[dev(t[k]) for k in ("X", "W", "A", "B")] for t in ins]
    want = [run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha) for t in ins]
    Ys = [torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(10)]
    torch.cuda.synchronize()
    for k in range(10):
        gpu.lora_fwd(*dv[k % 2], Ys[k], alpha)
    torch.cuda.synchronize()
    assert gpu.lora_get_device_status() == 0
    for k in range(10):
        assert torch.equal(Ys[k], want[k % 2]), k


def test_exchange_two_streams_at_once(gpu, monkeypatch):
    """Two forwards launched on two streams with nothing ordering them: the
    host gives each launch its own exchange slot (or none), never one that
    another running launch holds."""
    _env(monkeypatch)
    M, d_in, d_out, r, alpha = 8192, 4096, 4096, 16, 32.0
    ins = [WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=s) for s in (21, 22)]
    dv = [[dev(t[k]) for k in ("X", "W", "A", "B")] for t in ins]
    want = [run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha) for t in ins]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    for _ in range(5):
        Ys = [torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        torch.cuda.synchronize()
        for i in (0, 1):
            with torch.cuda.stream(streams[i]):
                gpu.lora_fwd(*dv[i], Ys[i], alpha)
        torch.cuda.synchronize()
        assert gpu.lora_get_device_status() == 0
        for i in (0, 1):
            assert torch.equal(Ys[i], want[i]), i


def test_forward_captured_in_a_graph_runs_without_the_exchange_same_bits(gpu, monkeypatch):
    """A forward captured into a CUDA graph gets no exchange slot (a replay
    may run at any time beside the slot's stream) and runs the plain run
    schedule; replayed, it gives the eager forward's Y bit for bit."""
    _env(monkeypatch)
    M, d_in, d_out, r, alpha = 8192, 4096, 4096, 16, 32.0
    t = WL.make_layer_inputs(WL.LayerShape(M, d_in, d_out, r, alpha), seed=41)
    X, W, A, B = (dev(t[k]) for k in ("X", "W", "A", "B"))
    want = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], alpha)
    Y = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        gpu.lora_fwd(X, W, A, B, Y, alpha)          # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    Y.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        gpu.lora_fwd(X, W, A, B, Y, alpha)
    for _ in range(2):
        Y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(Y, want)
    del g
    assert gpu.lora_get_device_status() == 0
