"""The host-side launch planning, checked on the CPU through lora_plan (host
only: no GPU, nothing launched) over a sweep of shapes and ranks, with and
without the LORA_B200_* overrides: every configuration must fit the 227 KB
shared-memory opt-in limit, keep a pipeline, cover the output with its
tiles, give the two jobs of a shared backward launch one split count, leave
no split of a contraction empty where the planner sizes the split itself,
and need the documented workspace."""
import itertools
import math

import pytest

SMEM_MAX = 232448
MS = [1, 7, 128, 129, 256, 1000, 2048, 4100, 8192, 16384, 65536]
DS = [8, 64, 136, 520, 1024, 4096, 14336, 16384]
RS = [8, 16, 24, 32, 40, 64, 96, 128]


def _no_empty_split(nk, s):
    return s == 1 or (s - 1) * math.ceil(nk / s) < nk


def _check_plan(p, M, d_in, d_out, r, forced_tile=None, forced_run=None):
    where = (M, d_in, d_out, r, p)
    for k in ("fwd_smem", "bwd1_smem", "bwd2_smem", "dx_smem"):
        assert 0 < p[k] <= SMEM_MAX, (k, where)
    if p["fwd_kind"] == 0:
        assert p["fwd_bn"] in (128, 256) and p["fwd_cg"] in (1, 2) and p["fwd_stages"] >= 2, where
        assert p["fwd_splits"] == 1, where
        assert p["fwd_num_m"] == math.ceil(M / (128 * p["fwd_cg"])), where
        assert p["fwd_num_n"] == math.ceil(d_out / p["fwd_bn"]), where
        if forced_tile:
            assert (p["fwd_bn"], p["fwd_cg"]) == forced_tile, where
        if forced_run is not None:
            assert p["fwd_run_l"] == forced_run, where
        else:
            assert p["fwd_run_l"] == 0 or 1 <= p["fwd_run_l"] <= min(p["fwd_num_n"], 8), where
    else:
        assert p["fwd_kind"] == 1 and forced_tile is None, where
        assert p["fwd_bn"] == 128 and p["fwd_cg"] == 1 and p["fwd_stages"] >= 1, where
        assert 2 <= p["fwd_splits"] <= 8, where
        assert _no_empty_split(math.ceil(d_in / 64), p["fwd_splits"]), where
    # backward launch 1: the dT and T jobs share the launch's split count; the
    # dT-alone form and launch 2 size their own split counts
    assert p["bwd1_splits_dt"] == p["bwd1_splits_t"] and 1 <= p["bwd1_splits_dt"] <= 8, where
    assert 1 <= p["bwd1_saved_splits"] <= 8, where
    assert _no_empty_split(math.ceil(d_out / 64), p["bwd1_saved_splits"]), where
    assert _no_empty_split(math.ceil(max(d_in, d_out) / 64), p["bwd1_splits_dt"]), where
    assert p["bwd2_splits_db"] == p["bwd2_splits_da"] and 1 <= p["bwd2_splits_db"] <= 8, where
    assert _no_empty_split(math.ceil(M / 64), p["bwd2_splits_db"]), where
    assert p["dx_bn"] in (128, 256) and p["dx_cg"] in (1, 2) and p["dx_stages"] >= 2, where
    r_pad = (r + 15) // 16 * 16
    assert p["workspace_bytes"] == 2 * ((M * r_pad * 2 + 255) // 256 * 256), where


@pytest.mark.parametrize("r", RS)
def test_every_plan_fits_and_covers(built_lib, monkeypatch, r):
    for v in ("LORA_B200_FUSED_TILE", "LORA_B200_FUSED_RUN", "LORA_B200_SPLITK"):
        monkeypatch.delenv(v, raising=False)
    for M, d_in, d_out in itertools.product(MS, DS, DS):
        _check_plan(built_lib.lora_plan(M, d_in, d_out, r), M, d_in, d_out, r)


@pytest.mark.parametrize("tile", [(256, 2), (256, 1), (128, 2), (128, 1)])
def test_forced_tiles_fit(built_lib, monkeypatch, tile):
    """Every tile configuration the tests force is launchable for every rank
    (enough shared memory for a pipeline) and is the one used, except 256-wide
    single-CTA tiles at r = 128: they leave room for two stages, the planner
    wants three for 256-wide tiles, and the override falls back to the
    automatic choice for the shape."""
    for v in ("LORA_B200_FUSED_RUN", "LORA_B200_SPLITK"):
        monkeypatch.delenv(v, raising=False)
    for r, M, d in itertools.product(RS, (1, 1000, 8192), (64, 1032, 4096)):
        monkeypatch.delenv("LORA_B200_FUSED_TILE", raising=False)
        auto = built_lib.lora_plan(M, d, d, r)
        monkeypatch.setenv("LORA_B200_FUSED_TILE", f"{tile[0]},{tile[1]}")
        p = built_lib.lora_plan(M, d, d, r)
        if tile == (256, 1) and r == 128:
            _check_plan(p, M, d, d, r)
            assert (p["fwd_bn"], p["fwd_cg"]) == (auto["fwd_bn"], auto["fwd_cg"]) != (256, 1)
        else:
            _check_plan(p, M, d, d, r, forced_tile=tile)


@pytest.mark.parametrize("run", [0, 1, 3, 8])
def test_forced_runs(built_lib, monkeypatch, run):
    monkeypatch.setenv("LORA_B200_FUSED_RUN", str(run))
    monkeypatch.setenv("LORA_B200_SPLITK", "0")
    for r, M, d in itertools.product((16, 128), (1000, 8192), (1544, 4096)):
        _check_plan(built_lib.lora_plan(M, d, d, r), M, d, d, r, forced_run=run)


def test_forced_split_contraction(built_lib, monkeypatch):
    """LORA_B200_SPLITK=1 takes the split-contraction forward wherever it
    gives at least two splits, with no empty split."""
    monkeypatch.setenv("LORA_B200_SPLITK", "1")
    n = 0
    for r, M, d in itertools.product(RS, (1, 100, 384, 1000), (520, 1344, 4096, 8192)):
        p = built_lib.lora_plan(M, d, d, r)
        _check_plan(p, M, d, d, r)
        n += p["fwd_kind"] == 1
    assert n > 30


def test_named_workloads(built_lib, monkeypatch):
    """The launch configurations the benchmark and the documentation name."""
    for v in ("LORA_B200_FUSED_TILE", "LORA_B200_FUSED_RUN", "LORA_B200_SPLITK"):
        monkeypatch.delenv(v, raising=False)
    p = built_lib.lora_plan(8192, 4096, 4096, 16)       # attention projection
    assert (p["fwd_kind"], p["fwd_bn"], p["fwd_cg"], p["fwd_run_l"]) == (0, 256, 2, 8)
    assert (p["dx_bn"], p["dx_cg"]) == (256, 2)
    p = built_lib.lora_plan(16384, 4096, 14336, 64)     # MLP up-projection
    assert (p["fwd_kind"], p["fwd_bn"], p["fwd_cg"], p["fwd_run_l"]) == (0, 256, 2, 7)
    p = built_lib.lora_plan(128, 4096, 4096, 16)        # weight-streaming: split contraction
    assert (p["fwd_kind"], p["fwd_splits"]) == (1, 4)
    assert all(v == 0 for v in built_lib.lora_plan(0, 512, 264, 16).values())


def test_plan_argument_rules(built_lib):
    import ctypes
    L = built_lib
    so = L.lib()
    out = L._Plan()
    assert L.STATUS[so.lora_plan(256, 512, 512, 16, 148, None)] == "LORA_ERR_NULL"
    for args, want in (((256, 512, 512, 12, 148), "LORA_ERR_RANK"), ((256, 516, 512, 16, 148), "LORA_ERR_SHAPE"),
                       ((-1, 512, 512, 16, 148), "LORA_ERR_SHAPE"), ((256, 512, 512, 16, 1), "LORA_ERR_SHAPE"),
                       ((256, 512, 512, 16, 5000), "LORA_ERR_SHAPE"), ((256, 512, 512, 16, 148), "LORA_OK")):
        assert L.STATUS[so.lora_plan(*args, ctypes.byref(out))] == want, args
