"""bench.py's host-side helpers (CPU): the algorithmic work it divides by,
the source hash that keys the recorded DRAM traffic (comment edits keep it,
code edits change it), the traffic record's format, and when a measurement
idles first."""
import os
import re

import bench
import workloads as WL


def test_algorithmic_flops_match_the_stated_figures():
    sh = WL.ATTN_PROJ
    assert round(bench.flops_fwd(sh.M, sh.d_in, sh.d_out, sh.r) / 1e9, 2) == 277.03
    assert round(bench.flops_bwd(sh.M, sh.d_in, sh.d_out, sh.r) / 1e9, 1) == 279.2
    assert round(bench.flops_merge(sh.d_in, sh.d_out, sh.r) / 1e9, 2) == 0.54
    # forward: the base product plus the down- and up-projections, 2 FLOPs per multiply-add
    M, di, do, r = 3, 5, 7, 2
    assert bench.flops_fwd(M, di, do, r) == 2 * (M * do * di + M * r * di + M * do * r)
    # backward: dX (d_out + r terms per output), dT, dB, dA; the T recompute is not counted
    assert bench.flops_bwd(M, di, do, r) == 2 * (M * di * (do + r) + M * r * do + do * r * M + r * di * M)
    assert bench.step_flops(sh) == (bench.flops_fwd(sh.M, sh.d_in, sh.d_out, sh.r)
                                    + bench.flops_bwd(sh.M, sh.d_in, sh.d_out, sh.r)
                                    + bench.flops_merge(sh.d_in, sh.d_out, sh.r))


def test_source_hash_ignores_comments_only():
    code = "int f(int a) {\n  return a + 1;  // one more\n}\n/* block\n comment */\n"
    same = "// header comment\nint f(int a) {\n    return a + 1;\n}\n"
    other = "int f(int a) {\n  return a + 2;\n}\n"
    assert bench._code_only(code) == bench._code_only(same)
    assert bench._code_only(code) != bench._code_only(other)
    assert re.fullmatch(r"[0-9a-f]{16}", bench.kernel_src_hash())


def test_traffic_record_format():
    path = os.path.join(bench._ROOT, "profiles", "traffic.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    assert rows
    for kernel, workload, h, nbytes in rows:
        assert re.fullmatch(r"[0-9a-f]{16}", h) and int(nbytes) > 0
        # the record is per launch: at least the forward's algorithmic bytes
        if workload == WL.ATTN_PROJ.name:
            sh = WL.ATTN_PROJ
            alg = 2 * (sh.M * sh.d_in + sh.d_out * sh.d_in + sh.M * sh.d_out)
            assert int(nbytes) >= alg
    # lookups: a matching hash returns the bytes, any other hash nothing
    kernel, workload, h, nbytes = rows[0]
    assert bench.recorded_traffic(kernel, workload, h) == float(nbytes)
    assert bench.recorded_traffic(kernel, workload, "0" * 16) is None


def test_peak_follows_the_length_of_the_timed_region():
    peaks = {"bf16_tflops": 1654.6, "bf16_tflops_sustained": 1410.9}
    assert bench.pick_peak(peaks, 0.009) == (1654.6, False)       # 20 short steps: burst
    assert bench.pick_peak(peaks, 0.999) == (1654.6, False)
    assert bench.pick_peak(peaks, 1.0) == (1410.9, True)          # seconds at the power cap: sustained
    assert bench.pick_peak({}, 0.01)[0] == bench.FALLBACK_PEAKS["bf16_tflops"]
    # a short region that nevertheless ran at the power cap takes the sustained figure
    assert bench.pick_peak(peaks, 0.15, {"reasons": ["sw_power_cap"]}) == (1410.9, True)
    assert bench.pick_peak(peaks, 0.15, {"reasons": []}) == (1654.6, False)


def test_clock_normalised_time():
    c = bench._clock_normalised(200.0, {"sm_mhz": 1500.0, "sm_max_mhz": 2000.0})
    assert c["kcycles"] == 300.0 and c["us_at_max_clock"] == 150.0
    assert bench._clock_normalised(200.0, None) is None


def test_measurements_idle_only_after_heavy_work(monkeypatch):
    """_Cooled idles COOL_S before a measurement (before its warm-up) only when
    the measurement before it kept the GPU busy longer than HEAVY_BUSY_S."""
    calls = []

    def fake_time_events(fn, flush, n, warm=3, cool_s=0.0):
        calls.append(cool_s)
        return fn(), 0.0, 0.0          # the "median" in microseconds

    monkeypatch.setattr(bench, "_time_events", fake_time_events)
    c = bench._Cooled()
    light_us = bench.HEAVY_BUSY_S * 1e6 / 20 * 0.5        # 13 calls of it stay under the limit
    heavy_us = bench.HEAVY_BUSY_S * 1e6 / 13 * 2.0        # 13 calls of it exceed the limit
    for us in (light_us, light_us, heavy_us, light_us, heavy_us, heavy_us, light_us):
        c.time(lambda us=us: us, None, 10, warm=3)
    assert calls == [0.0, 0.0, 0.0, bench.COOL_S, 0.0, bench.COOL_S, bench.COOL_S]
