#!/usr/bin/env python
"""Benchmark of the fused LoRA layer hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic
input: lora_fwd (Y), lora_bwd (dX, dA, dB; T recomputed) and lora_merge
(W' = W + s B A) on the attention-projection workload X[8192, 4096],
W[4096, 4096], r = 16, alpha = 32 (or, with --workload mlp_up, the MLP
up-projection X[16384, 4096], W[14336, 4096], r = 64, alpha = 128).
With N > 1 GPUs every rank runs the same step on its own batch (data
parallel along M, weak scaling) and the adapter gradients dA, dB are summed
across ranks with one NCCL all-reduce.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line on rank 0.  Metric: TFLOP/s of algorithmic work
(counted below; no recompute, no padding) over device time, max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import time
import threading
import time

_ROOT = os.path.dirname(os.path.abspath(__file__))
if _ROOT not in sys.path:
    sys.path.insert(0, _ROOT)

import workloads as WL  # noqa: E402

METRIC = "fused LoRA fwd/bwd TFLOP/s (bf16) and % of B200 dense peak; µs/call"
UNIT = "TFLOP/s"
# the step's workload: attention projection by default, --workload mlp_up for the MLP up-projection
WORKLOADS = {"attn_proj": WL.ATTN_PROJ, "mlp_up": WL.MLP_UP}
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0   # B200 dense bf16, nominal (context for the measured peaks)
# a kernel timed over less than this many seconds runs cool: its peak is the
# measured burst figure; over longer regions, the sustained (power-capped) one
SUSTAINED_AFTER_S = 1.0
# the sources the forward kernel's DRAM traffic depends on (kernel and launch
# configuration / schedule)
KERNEL_SOURCES = ("lora_linear_layer_b200/csrc/fused.cuh", "lora_linear_layer_b200/csrc/ptx.cuh",
                  "lora_linear_layer_b200/csrc/common.cuh", "lora_linear_layer_b200/csrc/texchange.cuh",
                  "lora_linear_layer_b200/csrc/host_common.cuh", "lora_linear_layer_b200/csrc/host_plan.cuh",
                  "lora_linear_layer_b200/csrc/lora_api.cu")
LAUNCHES_PER_STEP = 5   # fwd 1; bwd: T + dT, dB + dA, dX; merge 1


# ------------------------------------------------------ algorithmic work ----

def flops_fwd(M, d_in, d_out, r):
    return 2.0 * M * (d_in * d_out + r * d_in + r * d_out)


def flops_bwd(M, d_in, d_out, r):
    # dX = dY W + dT A; dT = s dY B; dB = s dY^T T; dA = dT^T X (T recompute not counted)
    return 2.0 * M * (d_out * d_in + r * d_in) + 2.0 * M * d_out * r * 2 + 2.0 * M * r * d_in


def flops_merge(d_in, d_out, r):
    return 2.0 * r * d_out * d_in


def step_flops(sh):
    return (flops_fwd(sh.M, sh.d_in, sh.d_out, sh.r) + flops_bwd(sh.M, sh.d_in, sh.d_out, sh.r)
            + flops_merge(sh.d_in, sh.d_out, sh.r))


# ---------------------------------------------------------------- peaks ----

def load_peaks():
    p = os.path.join(_ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def pick_peak(peaks, timed_s, clocks=None):
    """(peak TFLOP/s, sustained?) for a kernel timed over `timed_s` seconds:
    the measured burst figure for a short region in which the part stays
    cool, the sustained power-capped one from SUSTAINED_AFTER_S on or when
    the clock record shows the power cap (sw_power_cap) during the region."""
    capped = bool(clocks) and "sw_power_cap" in (clocks.get("reasons") or [])
    long_run = timed_s >= SUSTAINED_AFTER_S or capped
    key = "bf16_tflops_sustained" if long_run else "bf16_tflops"
    return float(peaks.get(key, FALLBACK_PEAKS[key])), long_run


def _code_only(text):
    """C++ source with comments and blank space removed, so that the hash
    below changes with the code, not with its comments (no '//' or '/*'
    appears inside a string literal in these files)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(" ".join(line.split()) for line in text.splitlines() if line.strip())


def kernel_src_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(_ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload, src_hash):
    """Per-launch DRAM bytes from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(_ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload \
                    and parts[2] == src_hash:
                return float(parts[3])
    return None


# --------------------------------------------------------------- clocks ----

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 100):
        self.gpu_index = gpu_index
        self.period_ms = period_ms
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=5)
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                continue
            for name, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ reference ----

def oracle_step_sample(t, sh, rows):
    """One sampled step of the fp64 oracle: forward and backward on the first
    `rows` rows of the batch, merge of the full weight."""
    import oracle as O
    X = t["X"][:rows]
    dY = t["dY"][:rows]
    f = lambda x: O.bf16_bits_to_f64(WL.bf16_bits(x))  # noqa: E731
    Xf, Wf, Af, Bf, dYf = f(X), f(t["W"]), f(t["A"]), f(t["B"]), f(dY)
    O.lora_forward(Xf, Wf, Af, Bf, sh.alpha)
    O.lora_backward(Xf, Wf, Af, Bf, dYf, sh.alpha)
    O.lora_merge(Wf, Af, Bf, sh.alpha)
    return (flops_fwd(rows, sh.d_in, sh.d_out, sh.r) + flops_bwd(rows, sh.d_in, sh.d_out, sh.r)
            + flops_merge(sh.d_in, sh.d_out, sh.r))


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline(sh, budget_s=12.0, rows=512):
    """Time the oracle as it stands on a bounded sample of the workload."""
    t = WL.make_layer_inputs(WL.LayerShape(rows, sh.d_in, sh.d_out, sh.r, sh.alpha), seed=0, with_dy=True)
    flops, n = 0.0, 0
    t0 = time.perf_counter()
    while True:
        flops += oracle_step_sample(t, sh, rows)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} sampled steps: fwd+bwd on {rows} of {sh.M} rows, merge of the full "
                      f"{sh.d_out}x{sh.d_in} weight, fp64 numpy/BLAS; {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    sh = WORKLOADS[args.workload]
    rows = 512
    t = WL.make_layer_inputs(WL.LayerShape(rows, sh.d_in, sh.d_out, sh.r, sh.alpha), seed=0, with_dy=True)
    for _ in range(max(args.warmup, 0)):
        oracle_step_sample(t, sh, rows)
    times, flops = [], 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        flops += oracle_step_sample(t, sh, rows)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = flops / total / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": sh.name, "M": sh.M, "d_in": sh.d_in, "d_out": sh.d_out, "r": sh.r,
                   "alpha": sh.alpha, "sample_rows": rows, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: fp64 oracle fwd+bwd on {rows} of {sh.M} rows + full merge"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ ours ----

def run_ours(args):
    import torch
    import torch.distributed as dist

    import lora_linear_layer_b200 as L
    from lora_linear_layer_b200 import dp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    L.lib()

    sh = WORKLOADS[args.workload]
    M, d_in, d_out, r, alpha = sh.M, sh.d_in, sh.d_out, sh.r, sh.alpha
    host = WL.make_layer_inputs(sh, seed=rank, with_dy=True)
    X, W, A, B, dY = (host[k].cuda() for k in ("X", "W", "A", "B", "dY"))
    Y = torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")
    dX = torch.empty((M, d_in), dtype=torch.bfloat16, device="cuda")
    # with several ranks the adapter gradients stay fp32 until they are summed
    # (lora_bwd_ex with LORA_BWD_FP32_GRADS), so the exchange adds unrounded
    # partials; on one GPU they are the layer's bf16 outputs
    gdt = torch.float32 if world > 1 else torch.bfloat16
    dA = torch.empty((r, d_in), dtype=gdt, device="cuda")
    dB = torch.empty((d_out, r), dtype=gdt, device="cuda")
    Wm = torch.empty_like(W)
    ws = torch.empty(L.lora_bwd_workspace_size(M, d_in, d_out, r), dtype=torch.uint8, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    # --saved-t: the forward keeps T for the backward (one pass over X less)
    bwd_flags = L.LORA_BWD_T_SAVED if args.saved_t else 0

    def step(ev_f0=None, ev_f1=None, Xb=None, dYb=None):
        Xb = X if Xb is None else Xb
        dYb = dY if dYb is None else dYb
        if ev_f0 is not None:
            ev_f0.record(stream)
        if args.saved_t:
            L.lora_fwd_save(Xb, W, A, B, Y, alpha, ws, stream)     # Y, and T into the workspace
        else:
            L.lora_fwd(Xb, W, A, B, Y, alpha, stream)
        if ev_f1 is not None:
            ev_f1.record(stream)
        if world > 1:
            # dA and dB first; their exchange (NCCL, fp32) overlaps the dX step
            L.lora_bwd_grads(Xb, A, B, dYb, dA, dB, alpha, ws, L.LORA_BWD_FP32_GRADS | bwd_flags, stream)
            works = dp.allreduce_adapter_grads(dA, dB, async_op=True)
            L.lora_bwd_dx(W, A, dYb, dX, ws, stream)
            for w in works:
                w.wait()
        else:
            L.lora_bwd_ex(Xb, W, A, B, dYb, dX, dA, dB, alpha, ws, bwd_flags, stream)
        L.lora_merge(W, A, B, Wm, alpha, stream)

    warm = max(3, args.warmup)
    for _ in range(warm):
        step()
    torch.cuda.synchronize()
    if L.lora_get_device_status() != 0:
        raise SystemExit("device status not OK after warm-up")

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(local, period_ms=25) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    for i in range(K):
        flush.zero_()                       # evict L2 (outside the timed pairs)
        s0, s1, f0, f1 = ev[i]
        s0.record(stream)
        step(f0, f1)
        s1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    if L.lora_get_device_status() != 0:
        raise SystemExit("device status not OK after the timed region")
    step_ms = [s0.elapsed_time(s1) for (s0, s1, _, _) in ev]
    fwd_ms = [f0.elapsed_time(f1) for (_, _, f0, f1) in ev]
    total_ms = sum(step_ms)
    fwd_avg_ms = sum(fwd_ms) / K
    total_ms, fwd_avg_ms = dp.max_over_ranks([total_ms, fwd_avg_ms], device="cuda")

    # ---------------- end to end through the C ABI with host buffers -------
    e2e = None
    if not args.no_e2e:
        # per-step inputs: the batch X and its upstream gradient dY; the frozen
        # base weight W and the adapter A, B are parameters that stay resident
        pin = {k: host[k].pin_memory() for k in ("X", "dY")}
        out_dA = torch.empty_like(dA, device="cpu").pin_memory()
        out_dB = torch.empty_like(dB, device="cpu").pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in pin.values())
        d2h = out_dA.numel() * out_dA.element_size() + out_dB.numel() * out_dB.element_size()
        Ke = max(3, min(K, args.e2e_steps))

        # Two device buffers per input: while step i computes on one, a copy
        # stream brings batch i + 1 into the other (as a training loop
        # prefetches its data).  Every step's copies are inside the timed
        # region; the step waits for its own batch, and a buffer is refilled
        # only after the step that read it.
        copy_s = torch.cuda.Stream()
        Xs, dYs = [X, torch.empty_like(X)], [dY, torch.empty_like(dY)]
        copied = [torch.cuda.Event(), torch.cuda.Event()]
        freed = [torch.cuda.Event(), torch.cuda.Event()]

        def issue_copy(i):
            b = i % 2
            if i >= 2:
                copy_s.wait_event(freed[b])
            with torch.cuda.stream(copy_s):
                Xs[b].copy_(pin["X"], non_blocking=True)
                dYs[b].copy_(pin["dY"], non_blocking=True)
                copied[b].record(copy_s)

        def e2e_run(n, start_event=None):
            if start_event is not None:
                copy_s.wait_event(start_event)
            issue_copy(0)
            for i in range(n):
                b = i % 2
                if i + 1 < n:
                    issue_copy(i + 1)
                stream.wait_event(copied[b])
                step(Xb=Xs[b], dYb=dYs[b])
                freed[b].record(stream)
                out_dA.copy_(dA, non_blocking=True)
                out_dB.copy_(dB, non_blocking=True)

        e2e_run(2)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_run(Ke, start_event=e0)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = dp.max_over_ranks([e0.elapsed_time(e1)], device="cuda")[0]
        e2e = {"value": step_flops(sh) * Ke * world / (e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": Ke,
               "what": "every step copies its batch X and upstream gradient dY from pinned host memory "
                       "(W, A, B are resident parameters) and reads the gradients dA, dB back; the copy "
                       "of batch i+1 overlaps the compute of step i (two device buffers)"}

    if world > 1:
        dist.barrier()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    peaks, peak_src = load_peaks()
    value = step_flops(sh) * K * world / (total_ms * 1e-3) / 1e12
    fwd_flops = flops_fwd(M, d_in, d_out, r)
    achieved = fwd_flops / (fwd_avg_ms * 1e-3) / 1e12
    peak_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sust = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    timed_s = total_ms * 1e-3
    peak, long_run = pick_peak(peaks, timed_s, clocks)
    src_hash = kernel_src_hash()
    traffic = recorded_traffic("fused_lora_kernel_fwd", sh.name, src_hash)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": warm,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded normal inputs, bf16)",
        "config": {"workload": sh.name, "M": M, "d_in": d_in, "d_out": d_out, "r": r, "alpha": alpha,
                   "global_batch_tokens": M * world, "step": ("lora_fwd_save + lora_bwd_ex (T saved) + lora_merge" if args.saved_t
                            else "lora_fwd + lora_bwd + lora_merge"),
                   "l2": "flushed between steps (256 MB write outside the timed pairs); inputs > L2",
                   "parallelism": f"dp{world}" if world > 1 else "single GPU"},
        "breakdown": {"fwd_us": 1e3 * fwd_avg_ms, "fwd_tflops": achieved,
                      "rest_of_step_us": 1e3 * (total_ms / K - fwd_avg_ms)},
        "roofline": {"kernel": "fused_lora_kernel (forward)", "bound": "tensor", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                     "peak_kind": (f"bf16_tflops_sustained ({peak_src}): the timed region lasts {timed_s:.2f} s "
                                   "and/or the clock record shows the power cap (sw_power_cap)") if long_run else
                                  (f"bf16_tflops burst ({peak_src}): the timed region lasts only {timed_s:.3f} s "
                                   f"(< {SUSTAINED_AFTER_S:.0f} s), so the part runs cool as in the burst measurement"),
                     "peak_burst": peak_burst, "frac_burst": achieved / peak_burst,
                     "peak_sustained": peak_sust, "frac_sustained": achieved / peak_sust,
                     "peak_datasheet": DATASHEET_BF16_TFLOPS, "frac_datasheet": achieved / DATASHEET_BF16_TFLOPS,
                     "timed_region_s": timed_s,
                     "clock_normalised": _clock_normalised(1e3 * fwd_avg_ms, clocks),
                     "algorithmic_flops_per_launch": fwd_flops, "src_hash": src_hash},
        "gpu_launches": LAUNCHES_PER_STEP * K,
        "clocks": clocks,
        "e2e": e2e,
    }
    if world == 1 and not args.no_configs:
        line["configs"] = run_configs(args, peaks, peak_src)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(sh, budget_s=args.cpu_budget)
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------- extra modes ----

# After a burst of heavy work the part holds a lower SM clock for 0.1-0.2 s
# (measured: the 512 x 8192^2 forward took 63.5 us cool, 89 us right after
# 65 calls of 16384 x 8192^2 with the clock at about 1.3 GHz, 72.6 us 50 ms
# later and 62.5-63.5 us after 0.2 s).  A measurement that follows heavy
# work in the same process idles COOL_S first, then warms up, so that it is
# taken on a part in the state the burst peak was measured in, whatever ran
# before it.  (Idling before every measurement instead slowed the short ones:
# the tiny forward's calls, timed right after an idle, took 20 us against
# 12.3 us.)
COOL_S = 0.25
HEAVY_BUSY_S = 0.002       # work that kept the GPU busy longer than this heats what follows


def _time_events(fn, flush, n, warm=3, cool_s=0.0):
    import torch
    if cool_s > 0:
        torch.cuda.synchronize()
        time.sleep(cool_s)
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(n):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    ts.sort()
    return ts[len(ts) // 2], ts[max(0, len(ts) // 10)], ts[min(len(ts) - 1, (9 * len(ts)) // 10)]


def _clock_normalised(us, clocks):
    """A time scaled to the part's top SM clock (time x median MHz / max MHz)
    and expressed in SM cycles, so that runs on parts at different clocks
    compare."""
    if not clocks or not clocks.get("sm_mhz"):
        return None
    mhz, mx = float(clocks["sm_mhz"]), float(clocks.get("sm_max_mhz") or clocks["sm_mhz"])
    return {"us": us, "sm_mhz_median": mhz, "kcycles": us * mhz / 1e3, "us_at_max_clock": us * mhz / mx}


def _dev_inputs(sh, seed, with_dy=False):
    """Seeded device-side inputs of the workload recipe's distributions, for
    timing only (the parity tests use the host recipe bit for bit): X, dY
    N(0, 1); W, A N(0, 1/d_in) (variance); B N(0, 0.02^2)."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(int(seed))
    bf = torch.bfloat16
    X = torch.randn(sh.M, sh.d_in, generator=g, device="cuda").to(bf)
    W = (torch.randn(sh.d_out, sh.d_in, generator=g, device="cuda") * sh.d_in ** -0.5).to(bf)
    A = (torch.randn(sh.r, sh.d_in, generator=g, device="cuda") * sh.d_in ** -0.5).to(bf)
    B = (torch.randn(sh.d_out, sh.r, generator=g, device="cuda") * 0.02).to(bf)
    dY = torch.randn(sh.M, sh.d_out, generator=g, device="cuda").to(bf) if with_dy else None
    return X, W, A, B, dY


class _Cooled:
    """Times measurements one after another, each after a COOL_S idle when
    the one before it kept the GPU busy longer than HEAVY_BUSY_S."""

    def __init__(self):
        self.busy_s = 0.0

    def time(self, fn, flush, n, warm=3):
        res = _time_events(fn, flush, n, warm=warm, cool_s=COOL_S if self.busy_s > HEAVY_BUSY_S else 0.0)
        self.busy_s = res[0] * 1e-6 * (n + warm)
        return res


def measure_sweep(L, flush, P, BW, n=5, warm=2, name_filter=""):
    """lora_fwd on every point of the square sweep: us/call (median, p10,
    p90), TFLOP/s, GB/s of the minimum bytes and the fraction of the binding
    roof (tensor at the burst bf16 peak, or HBM at the copy bandwidth)."""
    import torch
    out = []
    cooled = _Cooled()
    for idx, sh in enumerate(WL.sweep_points()):
        if name_filter and name_filter not in sh.name:
            continue
        X, W, A, B, _ = _dev_inputs(sh, seed=idx)
        Y = torch.empty((sh.M, sh.d_out), dtype=torch.bfloat16, device="cuda")
        med, p10, p90 = cooled.time(lambda: L.lora_fwd(X, W, A, B, Y, sh.alpha), flush, n, warm=warm)
        F = flops_fwd(sh.M, sh.d_in, sh.d_out, sh.r)
        by = 2.0 * (sh.M * sh.d_in + sh.d_out * sh.d_in + sh.r * (sh.d_in + sh.d_out) + sh.M * sh.d_out)
        t_roof = max(F / P, by / BW)
        out.append({"point": sh.name, "M": sh.M, "d": sh.d_in, "r": sh.r, "us_median": med, "us_p10": p10,
                    "us_p90": p90, "tflops": F / med / 1e6, "gbs_min_bytes": by / med / 1e3,
                    "bound": "tensor" if F / P >= by / BW else "hbm", "roof_frac": t_roof * 1e6 / med})
        del X, W, A, B, Y
    return out


def run_sweep(args):
    """--sweep: one JSON line per sweep point."""
    import torch
    import lora_linear_layer_b200 as L
    peaks, src = load_peaks()
    P = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * 1e12
    BW = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])) * 1e9
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    for row in measure_sweep(L, flush, P, BW, n=args.steps, warm=3, name_filter=args.sweep_filter):
        row["peaks"] = f"bf16 burst and HBM copy ({src})"
        print(json.dumps(row), flush=True)
    return 0


def _graph_replay_us(fn, flush, n, calls=1):
    """Median device time of one CUDA-graph replay of `calls` back-to-back
    calls of fn (captured after warm-up), L2 flushed before each replay."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(calls):
            fn()
    med, p10, p90 = _time_events(g.replay, flush, n)
    del g
    return med / calls, p10 / calls, p90 / calls


def measure_tiny(L, flush, n):
    """The tiny forward (X[256,512], W[512,512], r = 16): launch-bound, so
    per call as eager (through the Python binding), CUDA-graph replay of one
    call, and graph replay of 20 back-to-back calls."""
    import torch
    sh = WL.TINY_FWD
    t = WL.make_layer_inputs(sh, seed=0)
    X, W, A, B = (t[k].cuda() for k in ("X", "W", "A", "B"))
    Y = torch.empty((sh.M, sh.d_out), dtype=torch.bfloat16, device="cuda")
    fn = lambda: L.lora_fwd(X, W, A, B, Y, sh.alpha)  # noqa: E731
    eager = _time_events(fn, flush, n)
    g1 = _graph_replay_us(fn, flush, n)
    g20 = _graph_replay_us(fn, flush, n, calls=20)
    F = flops_fwd(sh.M, sh.d_in, sh.d_out, sh.r)
    return {"workload": sh.name, "us_per_call_eager": eager[0], "us_per_call_graph": g1[0],
            "us_per_call_graph_x20": g20[0], "tflops_graph_x20": F / g20[0] / 1e6,
            "p10_p90_eager": [eager[1], eager[2]], "l2": "flushed before each timed call or replay"}


def run_tiny(args):
    import torch
    import lora_linear_layer_b200 as L
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    print(json.dumps(measure_tiny(L, flush, args.steps)), flush=True)
    return 0


def measure_merge(L, flush, n, BW):
    """The 36-layer x 7-target adapter refresh (r = 32): one batched
    restore-and-merge from the pristine copies per cycle, eager through the
    binding, through a prepared MergeBatch, and as CUDA-graph replay."""
    import torch
    r, alpha = WL.MERGE_R, WL.MERGE_ALPHA
    gen = torch.Generator(device="cuda")
    gen.manual_seed(0)
    items, nbytes = [], 0.0
    for s in WL.merge_shapes():
        d_out, d_in = s["d_out"], s["d_in"]
        W = (torch.randn(d_out, d_in, generator=gen, device="cuda") * d_in ** -0.5).to(torch.bfloat16)
        A = (torch.randn(r, d_in, generator=gen, device="cuda") * d_in ** -0.5).to(torch.bfloat16)
        B = (torch.randn(d_out, r, generator=gen, device="cuda") * 0.02).to(torch.bfloat16)
        items.append((W, A, B, torch.empty_like(W)))
        nbytes += 4.0 * d_out * d_in + 2.0 * r * (d_in + d_out)
    batch = L.MergeBatch(items, r)          # descriptors built once, as in a refresh loop
    med, p10, p90 = _time_events(lambda: batch(alpha), flush, n)
    py_med = _time_events(lambda: L.lora_merge_batched(items, r, alpha), flush, n)[0]
    g_med = _graph_replay_us(lambda: batch(alpha), flush, n)[0]
    out = {"workload": "merge 36 layers x 7 targets, hidden 2560, r=32", "matrices": len(items),
           "ms_per_cycle": med / 1e3, "ms_p10": p10 / 1e3, "ms_p90": p90 / 1e3,
           "gbs": nbytes / med / 1e3, "hbm_frac": nbytes / med / 1e3 / (BW / 1e9),
           "eager": "one lora_merge_batched C call per cycle on a descriptor array built once (MergeBatch)",
           "ms_per_cycle_graph": g_med / 1e3, "gbs_graph": nbytes / g_med / 1e3,
           "hbm_frac_graph": nbytes / g_med / 1e3 / (BW / 1e9), "eager_over_graph": med / g_med,
           "ms_per_cycle_python_descriptors": py_med / 1e3,
           "python_descriptors": "the binding's lora_merge_batched, which checks the 1008 tensors and builds "
                                 "the descriptor array in Python on every call",
           "bytes_per_cycle": nbytes, "inputs": "seeded torch.randn on the device (timing only; parity in tests)"}
    del items, batch
    return out


def run_merge(args):
    import torch
    import lora_linear_layer_b200 as L
    peaks, src = load_peaks()
    BW = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])) * 1e9
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    row = measure_merge(L, flush, args.steps, BW)
    row["peak"] = f"HBM copy {BW/1e9:.0f} GB/s ({src})"
    print(json.dumps(row), flush=True)
    return 0


def measure_step(L, sh, flush, steps, warm, P):
    """One full step (lora_fwd + lora_bwd + lora_merge) of a workload,
    events around the forward, the backward and the merge."""
    import torch
    X, W, A, B, dY = _dev_inputs(sh, seed=0, with_dy=True)
    Y = torch.empty((sh.M, sh.d_out), dtype=torch.bfloat16, device="cuda")
    dX, dA, dB, Wm = torch.empty_like(X), torch.empty_like(A), torch.empty_like(B), torch.empty_like(W)
    ws = torch.empty(L.lora_bwd_workspace_size(sh.M, sh.d_in, sh.d_out, sh.r), dtype=torch.uint8, device="cuda")

    def step(ev=None):
        if ev:
            ev[0].record()
        L.lora_fwd(X, W, A, B, Y, sh.alpha)
        if ev:
            ev[1].record()
        L.lora_bwd(X, W, A, B, dY, dX, dA, dB, sh.alpha, ws)
        if ev:
            ev[2].record()
        L.lora_merge(W, A, B, Wm, sh.alpha)
        if ev:
            ev[3].record()

    for _ in range(warm):
        step()
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        step(ev)
        evs.append(ev)
    torch.cuda.synchronize()
    f_us = [1e3 * e[0].elapsed_time(e[1]) for e in evs]
    b_us = [1e3 * e[1].elapsed_time(e[2]) for e in evs]
    s_us = [1e3 * e[0].elapsed_time(e[3]) for e in evs]
    fm, bm, sm = statistics.median(f_us), statistics.median(b_us), statistics.median(s_us)
    Ff, Fb = flops_fwd(sh.M, sh.d_in, sh.d_out, sh.r), flops_bwd(sh.M, sh.d_in, sh.d_out, sh.r)
    out = {"workload": sh.name, "steps": steps, "step_ms": sm / 1e3, "step_tflops": step_flops(sh) / sm / 1e6,
           "fwd_us": fm, "fwd_tflops": Ff / fm / 1e6, "fwd_frac_burst": Ff / fm / 1e6 / (P / 1e12),
           "bwd_us": bm, "bwd_tflops": Fb / bm / 1e6, "bwd_frac_burst": Fb / bm / 1e6 / (P / 1e12),
           "l2": "flushed before each step", "inputs": "seeded torch.randn on the device"}
    del X, W, A, B, dY, Y, dX, dA, dB, Wm, ws
    return out


def measure_vs_unfused(L, sh, flush, n):
    """The pages' speedup metric on one workload: unfused PyTorch (cuBLAS,
    the six-launch forward and its autograd backward with W frozen) against
    lora_fwd / lora_bwd, median device time, L2 flushed before every call."""
    import torch
    X, W, A, B, dY = _dev_inputs(sh, seed=0, with_dy=True)
    s = sh.alpha / sh.r
    Y = torch.empty((sh.M, sh.d_out), dtype=torch.bfloat16, device="cuda")
    dX, dA, dB = torch.empty_like(X), torch.empty_like(A), torch.empty_like(B)
    ws = torch.empty(L.lora_bwd_workspace_size(sh.M, sh.d_in, sh.d_out, sh.r), dtype=torch.uint8, device="cuda")
    Xg, Ag, Bg = (v.clone().requires_grad_(True) for v in (X, A, B))

    def torch_fwd():
        return X @ W.t() + (X @ A.t()) @ B.t() * s

    def torch_fwd_bwd():
        y = Xg @ W.t() + (Xg @ Ag.t()) @ Bg.t() * s
        return torch.autograd.grad(y, (Xg, Ag, Bg), dY)

    # the arms run one after another, the unfused ones heavier: each follows
    # an idle when the arm before it was heavy
    ct = _Cooled().time
    tf = ct(torch_fwd, flush, n)[0]
    of = ct(lambda: L.lora_fwd(X, W, A, B, Y, sh.alpha), flush, n)[0]
    tfb = ct(torch_fwd_bwd, flush, n)[0]
    tfg = ct(lambda: Xg @ W.t() + (Xg @ Ag.t()) @ Bg.t() * s, flush, n)[0]
    tb = max(tfb - tfg, 1e-3)          # the unfused backward alone
    ob = ct(lambda: L.lora_bwd(X, W, A, B, dY, dX, dA, dB, sh.alpha, ws), flush, n)[0]
    out = {"workload": sh.name, "torch_fwd_us": tf, "ours_fwd_us": of, "fwd_speedup": tf / of,
           "torch_bwd_us": tb, "ours_bwd_us": ob, "bwd_speedup": tb / ob}
    del X, W, A, B, dY, Y, dX, dA, dB, ws, Xg, Ag, Bg
    return out


def run_configs(args, peaks, peak_src):
    """The other workloads, timed in the same run, each with its own clock
    record: the tiny forward per call (eager and graph), the MLP
    up-projection step with its forward / backward split, the 252-matrix
    merge refresh, the 125-point forward sweep (summary, and every M = 128
    point), and the unfused-PyTorch comparison on the two large layers."""
    import torch
    import lora_linear_layer_b200 as L
    P = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * 1e12
    BW = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])) * 1e9
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    out = {"peaks": f"bf16 burst {P/1e12:.1f} TFLOP/s and HBM copy {BW/1e9:.0f} GB/s ({peak_src})"}
    dev = torch.cuda.current_device()

    def clocked(name, fn):
        smp = ClockSampler(dev, period_ms=50)
        smp.start()
        time.sleep(0.2)
        t0 = time.perf_counter()
        res = fn()
        res["wall_s"] = time.perf_counter() - t0
        res["clocks"] = smp.stop()
        out[name] = res
        torch.cuda.empty_cache()

    clocked("tiny_fwd", lambda: measure_tiny(L, flush, 20))
    clocked("mlp_up_step", lambda: measure_step(L, WL.MLP_UP, flush, 10, 3, P))

    def sweep():
        rows = measure_sweep(L, flush, P, BW, n=5, warm=2)
        fr = [x["roof_frac"] for x in rows]
        m128 = [{"d": x["d"], "r": x["r"], "us": round(x["us_median"], 2), "frac": round(x["roof_frac"], 3),
                 "bound": x["bound"]} for x in rows if x["M"] == 128]
        worst = min(rows, key=lambda x: x["roof_frac"])
        return {"points": len(rows), "median_roof_frac": statistics.median(fr), "min_roof_frac": min(fr),
                "max_roof_frac": max(fr), "worst_point": worst["point"],
                "median_roof_frac_tensor": statistics.median([x["roof_frac"] for x in rows
                                                              if x["bound"] == "tensor"]),
                "median_roof_frac_hbm": statistics.median([x["roof_frac"] for x in rows if x["bound"] == "hbm"]),
                "m128": m128, "timing": "median of 5 calls, L2 flushed before each; a point that follows one "
                                            "that kept the GPU busy over 2 ms idles 0.25 s before its warm-up"}

    clocked("sweep", sweep)
    clocked("merge_refresh", lambda: measure_merge(L, flush, 5, BW))
    clocked("vs_unfused_torch", lambda: {"attn_proj": measure_vs_unfused(L, WL.ATTN_PROJ, flush, 10),
                                         "mlp_up": measure_vs_unfused(L, WL.MLP_UP, flush, 5)})
    del flush
    torch.cuda.empty_cache()
    return out


def compare_shapes():
    """The pages' benchmark grid (fastaf 0.1.0, "FWD kernel speedup": batch
    {1, 4, 16} x seq {256, 1024} x d_model {512, 1024, 2048} x rank {8, 16},
    alpha = 2r, square layers), then the attention-projection and MLP
    up-projection workloads."""
    out = []
    for b in (1, 4, 16):
        for seq in (256, 1024):
            for d in (512, 1024, 2048):
                for r in (8, 16):
                    out.append(WL.LayerShape(b * seq, d, d, r, 2.0 * r, name=f"b{b}_s{seq}_d{d}_r{r}"))
    return out + [WL.ATTN_PROJ, WL.MLP_UP]


def run_compare(args):
    """Unfused PyTorch LoRA (cuBLAS matmuls, the pages' six-launch forward and
    its autograd backward with W frozen) against lora_fwd / lora_bwd: median
    device time of each, L2 flushed before every call, and the speedup.  The
    unfused backward reuses the X A^T its forward kept; the same holds for
    lora_bwd_ex with LORA_BWD_T_SAVED after lora_fwd_save, reported beside
    lora_bwd (which recomputes T)."""
    import torch
    import lora_linear_layer_b200 as L
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    cooled = _Cooled()
    for sh in compare_shapes():
        if args.sweep_filter and args.sweep_filter not in sh.name:
            continue
        t = WL.make_layer_inputs(sh, seed=0, with_dy=True)
        X, W, A, B, dY = (t[k].cuda() for k in ("X", "W", "A", "B", "dY"))
        s = sh.alpha / sh.r
        Y = torch.empty((sh.M, sh.d_out), dtype=torch.bfloat16, device="cuda")
        dX = torch.empty_like(X)
        dA = torch.empty_like(A)
        dB = torch.empty_like(B)
        ws = torch.empty(max(1, L.lora_bwd_workspace_size(sh.M, sh.d_in, sh.d_out, sh.r)), dtype=torch.uint8,
                         device="cuda")
        Xg, Ag, Bg = (v.clone().requires_grad_(True) for v in (X, A, B))

        def torch_fwd():
            return X @ W.t() + (X @ A.t()) @ B.t() * s

        def torch_bwd():
            y = Xg @ W.t() + (Xg @ Ag.t()) @ Bg.t() * s
            return torch.autograd.grad(y, (Xg, Ag, Bg), dY)

        n = max(5, min(args.steps, 50))
        ct = cooled.time       # an idle before an arm that follows a heavy one (the unfused arms are heavier)
        tf = ct(torch_fwd, flush, n)[0]
        of = ct(lambda: L.lora_fwd(X, W, A, B, Y, sh.alpha), flush, n)[0]
        # the unfused backward includes its forward (autograd needs the graph); time the
        # forward alone and subtract it
        tfb = ct(torch_bwd, flush, n)[0]
        ob = ct(lambda: L.lora_bwd(X, W, A, B, dY, dX, dA, dB, sh.alpha, ws), flush, n)[0]
        L.lora_fwd_save(X, W, A, B, Y, sh.alpha, ws)       # T into the workspace, kept by the backward
        obs = ct(lambda: L.lora_bwd_ex(X, W, A, B, dY, dX, dA, dB, sh.alpha, ws, L.LORA_BWD_T_SAVED), flush, n)[0]
        tb = max(tfb - ct(lambda: Xg @ W.t() + (Xg @ Ag.t()) @ Bg.t() * s, flush, n)[0], 1e-3)
        print(json.dumps({"point": sh.name, "M": sh.M, "d_in": sh.d_in, "d_out": sh.d_out, "r": sh.r,
                          "torch_fwd_us": tf, "ours_fwd_us": of, "fwd_speedup": tf / of,
                          "torch_bwd_us": tb, "ours_bwd_us": ob, "bwd_speedup": tb / ob,
                          "ours_bwd_saved_t_us": obs, "bwd_saved_t_speedup": tb / obs,
                          "torch": "unfused: X@W.T + (X@A.T)@B.T*s, autograd backward (W frozen)",
                          "l2": "flushed before every call"}), flush=True)
        del X, W, A, B, dY, Y, dX, dA, dB, ws, Xg, Ag, Bg
    return 0


def run_grouped(args):
    """The seven LoRA targets of one layer of the merge model (hidden 2560:
    q, k, v, o, gate, up, down; r = 16) as independent forwards on a batch of
    M tokens: seven lora_fwd calls against one lora_fwd_batched call, eager
    and as CUDA-graph replay, L2 flushed before each timed call or replay."""
    import torch
    import lora_linear_layer_b200 as L
    r, alpha = 16, 32.0
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    for M in (256, 1024, 2048):
        items = []
        F = 0.0
        for i, s in enumerate(WL.merge_shapes(layers=1)):
            t = WL.make_layer_inputs(WL.LayerShape(M, s["d_in"], s["d_out"], r, alpha), seed=i)
            X, W, A, B = (t[k].cuda() for k in ("X", "W", "A", "B"))
            items.append((X, W, A, B, torch.empty((M, s["d_out"]), dtype=torch.bfloat16, device="cuda")))
            F += flops_fwd(M, s["d_in"], s["d_out"], r)

        def separate():
            for (X, W, A, B, Y) in items:
                L.lora_fwd(X, W, A, B, Y, alpha)

        def grouped():
            L.lora_fwd_batched(items, alpha)

        sep = _time_events(separate, flush, args.steps)[0]
        grp = _time_events(grouped, flush, args.steps)[0]
        sep_g = _graph_replay_us(separate, flush, args.steps)[0]
        grp_g = _graph_replay_us(grouped, flush, args.steps)[0]
        print(json.dumps({"workload": f"7 LoRA targets of one hidden-2560 layer, M={M}, r={r}", "problems": len(items),
                          "separate_us": sep, "grouped_us": grp, "separate_graph_us": sep_g,
                          "grouped_graph_us": grp_g, "grouped_tflops_graph": F / grp_g / 1e6,
                          "l2": "flushed before each timed call or replay"}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=tuple(WORKLOADS), default="attn_proj",
                    help="attn_proj: X[8192,4096] W[4096,4096] r=16 (default); "
                         "mlp_up: X[16384,4096] W[14336,4096] r=64")
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload block (tiny, MLP step, merge refresh, sweep summary, unfused comparison)")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--sweep", action="store_true", help="time lora_fwd on every sweep point (one line each)")
    ap.add_argument("--sweep-filter", default="", help="only sweep points whose name contains this")
    ap.add_argument("--saved-t", action="store_true",
                    help="the step keeps T from the forward: lora_fwd_save + lora_bwd_ex with LORA_BWD_T_SAVED")
    ap.add_argument("--merge", action="store_true", help="time the 252-matrix batched merge refresh")
    ap.add_argument("--tiny", action="store_true", help="time the tiny forward (eager and CUDA-graph replay)")
    ap.add_argument("--grouped", action="store_true",
                    help="seven small forwards: separate lora_fwd calls vs one lora_fwd_batched")
    ap.add_argument("--compare", action="store_true",
                    help="unfused PyTorch LoRA vs lora_fwd / lora_bwd on the pages' grid (speedup)")
    args = ap.parse_args()
    if args.sweep:
        return run_sweep(args)
    if args.merge:
        return run_merge(args)
    if args.tiny:
        return run_tiny(args)
    if args.compare:
        return run_compare(args)
    if args.grouped:
        return run_grouped(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
