"""lora_bwd_noalloc: the backward for callers that cannot call cudaMalloc.

Such callers (a plugin whose host program owns all device memory, a
service loop that must not allocate after start-up) cannot hand lora_bwd a
workspace; this entry point uses the library's own fixed 32 MiB per-device
scratch array instead.  These tests call it through the C ABI and compare
its results with lora_bwd's (caller workspace) on two calls in a row with
different inputs.  Both entry points run the same kernels with the same
deterministic reductions, so the results must agree bit for bit: anything
the first call leaves in the shared scratch that leaked into the second
would show as a difference, however small.  The first call of each shape is
also checked against the oracle within the parity tolerance (all rows of
the small shape, sampled rows and full dA, dB of the large one).  The r = 64
shape runs before the r = 16 one, so the second shape starts on leftovers
laid out differently.  The file is named to be collected last.
"""
import ctypes

import pytest
import torch

import oracle as O
import workloads as WL
from gpu_helpers import dev, f64, run_bwd
from tolerance import lora_tol_check

SHAPES = [
    (1000, 512, 2056, 64, 128.0),       # ragged tiles, r = 64
    (8192, 4096, 4096, 16, 32.0),       # attention-projection workload
]


@pytest.mark.gpu
@pytest.mark.parametrize("M,d_in,d_out,r,alpha", SHAPES)
def test_noalloc_backward_matches_workspace_backward_twice(gpu, M, d_in, d_out, r, alpha):
    sh = WL.LayerShape(M, d_in, d_out, r, alpha)
    for call, seed in enumerate((101, 202)):
        t = WL.make_layer_inputs(sh, seed=seed, with_dy=True)
        want = run_bwd(gpu, t["X"], t["W"], t["A"], t["B"], t["dY"], alpha)     # caller workspace
        Xd, Wd, Ad, Bd, dYd = (dev(t[k]) for k in ("X", "W", "A", "B", "dY"))
        nan = float("nan")
        got = (torch.full((M, d_in), nan, dtype=torch.bfloat16, device="cuda"),
               torch.full((r, d_in), nan, dtype=torch.bfloat16, device="cuda"),
               torch.full((d_out, r), nan, dtype=torch.bfloat16, device="cuda"))
        gpu.lora_bwd_noalloc(Xd, Wd, Ad, Bd, dYd, *got, alpha)
        assert gpu.lora_get_device_status() == 0
        for name, g, w in zip(("dX", "dA", "dB"), got, want):
            assert torch.equal(g, w), (call, name)
        if call == 0:
            _check_against_oracle(t, got, alpha)


def _check_against_oracle(t, got, alpha):
    M = t["X"].shape[0]
    rows = WL.sample_rows(M, seed=7, per_tile=2).numpy() if M > 2048 else None
    Xf, Wf, Af, Bf, dYf = (f64(t[k]) for k in ("X", "W", "A", "B", "dY"))
    rdX, rdA, rdB = O.lora_backward(Xf, Wf, Af, Bf, dYf, alpha, dx_rows=rows)
    dX, dA, dB = got
    gdX = f64(dX) if rows is None else f64(dX)[rows]
    for name, g, ref in (("dX", gdX, rdX), ("dA", f64(dA), rdA), ("dB", f64(dB), rdB)):
        ok, info = lora_tol_check(g, ref)
        assert ok, (name, info)


def test_noalloc_refuses_shapes_beyond_its_scratch(built_lib):
    """Rejected on the host before any CUDA call (fake pointers are never
    dereferenced), with the workspace status code."""
    L = built_lib
    fake = [0x7f0000001000 + (i << 32) for i in range(8)]
    M, d_in, d_out, r = 1 << 20, 4096, 4096, 128           # needs far more than 32 MiB
    assert L.lora_bwd_workspace_size(M, d_in, d_out, r) > (32 << 20)
    code = L.lib().lora_bwd_noalloc(*[ctypes.c_void_p(p) for p in fake], M, d_in, d_out, r,
                                    ctypes.c_float(256.0), None)
    assert L.STATUS[code] == "LORA_ERR_WORKSPACE"
    code = L.lib().lora_bwd_noalloc(*[ctypes.c_void_p(p) for p in fake], 64, 4096, 4096, 12,
                                    ctypes.c_float(24.0), None)
    assert L.STATUS[code] == "LORA_ERR_RANK"
