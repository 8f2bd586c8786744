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


def schedule_tiles(p, G):
    """Every (m, n) tile the clusters 0..G-1 take under the run schedule of a
    plan (run_l > 0), restated from the kernel's tile schedule.  Runs: runs
    of run_l N tiles of one M block dealt round-robin.  Seeded: cluster c
    first runs run_l tiles of M block c % num_m from N tile
    run_l * (c // num_m); every tile no seeding run covers is then dealt
    round-robin in M-major order."""
    num_m, num_n, L = p["fwd_num_m"], p["fwd_num_n"], p["fwd_run_l"]
    bw = p.get("band_w", num_n)
    out = []
    if p["fwd_seeded"]:
        covered = set()
        for c in range(G):
            n0 = L * (c // num_m)
            run = [(c % num_m, n) for n in range(n0, min(n0 + L, num_n))]
            out.append(run)
            covered.update(run)
        rest = [(m, n) for b0 in range(0, num_n, bw) for m in range(num_m)
                for n in range(b0, min(b0 + bw, num_n)) if (m, n) not in covered]
        for c in range(G):
            out[c] = out[c] + rest[c::G]
        return [t for per in out for t in per]
    rpm = -(-num_n // L)
    for c in range(G):
        for run in range(c, num_m * rpm, G):
            m, n0 = run // rpm, (run % rpm) * L
            out += [(m, n) for n in range(n0, min(n0 + L, num_n))]
    return out


def test_seeded_schedule_covers_every_tile_once_for_any_cluster_count():
    """The kernel learns its cluster count at launch (it may differ from the
    planned one); the seeded schedule must still cover every tile exactly
    once.  The closed-form index map of the kernel (two classes of M block
    by their number of seeding runs) is checked against the plain
    enumeration above."""
    cases = ((32, 16, 2, 16), (32, 16, 4, 16), (64, 16, 2, 16), (5, 9, 3, 9), (1, 3, 2, 3), (7, 40, 2, 40),
             (3, 2, 4, 2), (64, 56, 2, 19), (32, 32, 2, 9), (5, 23, 2, 6), (9, 17, 3, 17))
    for num_m, num_n, L, bw in cases:
        p = dict(fwd_num_m=num_m, fwd_num_n=num_n, fwd_run_l=L, fwd_seeded=1, band_w=bw)
        want = [(m, n) for m in range(num_m) for n in range(num_n)]
        for G in (1, 2, 3, num_m - 1, num_m, num_m + 1, 2 * num_m + 3, 74, 200):
            if G < 1:
                continue
            a_lo, r0 = G // num_m, G % num_m
            if (a_lo + (r0 > 0)) * L > min(bw, num_n):
                continue                                   # the host keeps the seeding in the first band
            assert sorted(schedule_tiles(p, G)) == want, (num_m, num_n, L, bw, G)
            # the kernel's closed form for the round-robin part
            w0 = min(bw, num_n)
            c_hi = w0 - min(w0, (a_lo + 1) * L)
            c_lo = w0 - min(w0, a_lo * L)
            p0 = r0 * c_hi + (num_m - r0) * c_lo
            covered = set()
            for c in range(G):
                n0 = L * (c // num_m)
                covered.update((c % num_m, n) for n in range(n0, min(n0 + L, num_n)))
            rest = [(m, n) for b0 in range(0, num_n, bw) for m in range(num_m)
                    for n in range(b0, min(b0 + bw, num_n)) if (m, n) not in covered]
            assert p0 + num_m * (num_n - w0) == len(rest)
            for i, t in enumerate(rest):
                if i < r0 * c_hi:
                    m, n = i // c_hi, w0 - c_hi + i % c_hi
                elif i < p0:
                    j = i - r0 * c_hi
                    m, n = r0 + j // c_lo, w0 - c_lo + j % c_lo
                else:
                    j = i - p0
                    b = 1 + j // (num_m * bw)
                    jb = j - (b - 1) * num_m * bw
                    wb = min(bw, num_n - b * bw)
                    m, n = jb // wb, b * bw + jb % wb
                assert (m, n) == t, (num_m, num_n, L, bw, G, i)


def _no_empty_split(nk, s):
    return s == 1 or (s - 1) * math.ceil(nk / s) < nk


def _check_plan(p, M, d_in, d_out, r, forced_tile=None, forced_run=None):
    where = (M, d_in, d_out, r, p)
    for k in ("fwd_smem", "bwd1_smem", "bwd2_smem", "dx_smem"):
        assert 0 < p[k] <= SMEM_MAX, (k, where)
    if p["fwd_kind"] == 0:
        assert p["fwd_bn"] in (128, 224, 256) and p["fwd_cg"] in (1, 2) and p["fwd_stages"] >= 2, where
        if p["fwd_bn"] == 224:
            # the pair fold: CTA pairs, T in the base product's last 32 columns, no exchange
            assert p["fwd_cg"] == 2 and r <= 32 and p["fwd_tx"] == 0 and p["fwd_seeded"] == 0, where
            assert p["fwd_stages"] >= 3, where
            if forced_run is None:
                assert p["fwd_run_l"] == 1, where
        assert p["fwd_splits"] == 1, where
        assert p["fwd_num_m"] == math.ceil(M / (128 * p["fwd_cg"])), where
        assert p["fwd_num_n"] == math.ceil(d_out / p["fwd_bn"]), where
        if forced_tile:
            assert (p["fwd_bn"], p["fwd_cg"]) == forced_tile, where
        if forced_run is not None:
            assert p["fwd_run_l"] == forced_run and p["fwd_seeded"] == 0, where
        elif p["fwd_seeded"] == 0:
            assert p["fwd_run_l"] == 0 or 1 <= p["fwd_run_l"] <= min(p["fwd_num_n"], 8), where
        else:
            # seeded: only with the T exchange and a seeding run for every M block
            assert p["fwd_tx"] == 1 and 2 <= p["fwd_run_l"] <= 4, where
            assert p["fwd_num_m"] <= 148 // p["fwd_cg"], where
            if p["fwd_num_m"] * p["fwd_num_n"] <= 4096:
                assert sorted(schedule_tiles(p, 148 // p["fwd_cg"])) == \
                    [(m, n) for m in range(p["fwd_num_m"]) for n in range(p["fwd_num_n"])], where
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
    for v in ("LORA_B200_FUSED_TILE", "LORA_B200_FUSED_RUN", "LORA_B200_SPLITK", "LORA_B200_TX", "LORA_B200_SEEDED_L"):
        monkeypatch.delenv(v, raising=False)
    for M, d_in, d_out in itertools.product(MS, DS, DS):
        _check_plan(built_lib.lora_plan(M, d_in, d_out, r), M, d_in, d_out, r)


@pytest.mark.parametrize("tile", [(256, 2), (256, 1), (128, 2), (128, 1), (224, 2)])
def test_forced_tiles_fit(built_lib, monkeypatch, tile):
    """Every tile configuration the tests force is launchable for every rank
    (enough shared memory for a pipeline) and is the one used, except 256-wide
    single-CTA tiles at r = 128 (they leave room for two stages, the planner
    wants three for 256-wide tiles) and the 224-wide pair fold above r = 32
    (T has 32 columns of the accumulator): there the override falls back to
    the automatic choice for the shape."""
    for v in ("LORA_B200_FUSED_RUN", "LORA_B200_SPLITK", "LORA_B200_TX", "LORA_B200_SEEDED_L"):
        monkeypatch.delenv(v, raising=False)
    for r, M, d in itertools.product(RS, (1, 1000, 8192), (64, 1032, 4096)):
        monkeypatch.delenv("LORA_B200_FUSED_TILE", raising=False)
        auto = built_lib.lora_plan(M, d, d, r)
        monkeypatch.setenv("LORA_B200_FUSED_TILE", f"{tile[0]},{tile[1]}")
        p = built_lib.lora_plan(M, d, d, r)
        if (tile == (256, 1) and r == 128) or (tile == (224, 2) and r > 32):
            _check_plan(p, M, d, d, r)
            assert (p["fwd_bn"], p["fwd_cg"]) == (auto["fwd_bn"], auto["fwd_cg"]) != tile
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
    for v in ("LORA_B200_FUSED_TILE", "LORA_B200_FUSED_RUN", "LORA_B200_SPLITK", "LORA_B200_TX", "LORA_B200_SEEDED_L"):
        monkeypatch.delenv(v, raising=False)
    p = built_lib.lora_plan(8192, 4096, 4096, 16)       # attention projection: seeded, runs of 2
    assert (p["fwd_kind"], p["fwd_bn"], p["fwd_cg"], p["fwd_run_l"], p["fwd_seeded"], p["fwd_tx"]) == \
        (0, 256, 2, 2, 1, 1)
    assert (p["dx_bn"], p["dx_cg"]) == (256, 2)
    p = built_lib.lora_plan(16384, 4096, 14336, 64)     # MLP up-projection
    assert (p["fwd_kind"], p["fwd_bn"], p["fwd_cg"], p["fwd_run_l"], p["fwd_seeded"]) == (0, 256, 2, 2, 1)
    p = built_lib.lora_plan(128, 4096, 4096, 16)        # weight-streaming: split contraction
    assert (p["fwd_kind"], p["fwd_splits"]) == (1, 4)
    # few pair tiles that would each compute T: the 224-wide pair fold (74 tiles
    # for 74 pairs at 512 x 8192^2), at r <= 32 only
    for r in (8, 16, 32):
        p = built_lib.lora_plan(512, 8192, 8192, r)
        assert (p["fwd_kind"], p["fwd_bn"], p["fwd_cg"], p["fwd_run_l"], p["fwd_num_n"]) == (0, 224, 2, 1, 37), r
    assert built_lib.lora_plan(512, 8192, 8192, 64)["fwd_bn"] == 256
    # runs of 2 or 4 with one T each: the 256-wide pair measured as fast or faster
    for M, d_in, d_out in ((1024, 8192, 8192), (2048, 8192, 8192), (512, 4096, 14336), (2048, 4096, 4096)):
        assert built_lib.lora_plan(M, d_in, d_out, 16)["fwd_bn"] == 256, (M, d_in, d_out)
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
