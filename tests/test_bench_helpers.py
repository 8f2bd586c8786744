"""bench.py's host-side helpers (CPU): the algorithmic work it divides by,
the source hash that keys the recorded DRAM traffic (comment edits keep it,
code edits change it), and the traffic record's format."""
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
