#!/usr/bin/env python
"""Benchmark of the HARP rotation hot path on B200.

One step = one harp_apply (forward) over a batch of the d=4096, schedule
(8,8,8,8) workload: 65,536 bf16 rows per GPU (Student-t nu=3 entries, 8 outlier
channels x50, theta ~ N(0, 0.05)), inputs already resident in HBM.  The batch is
512 MiB in and 512 MiB out, larger than L2 (126 MB), so no flush is needed
between steps.  With N GPUs (one process per GPU, launched by torchrun) every rank
rotates its own 65,536-row shard (weak scaling, no data-path collective).

Prints one JSON line (rank 0).  `--impl reference` times the float64 CPU oracle on
a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from structured_rotations_b200.shard import max_over_ranks, weak_shard  # noqa: E402

METRIC = "HARP rotation rows/s and HBM GB/s (fraction of B200 roofline), d=4096/5120/8192"
UNIT = "rows/s"
FALLBACK_HBM_GBS = 6650.0
WORKLOAD_TEXT = {
    "d4096": "d=4096 schedule (8,8,8,8), 65536 rows/GPU bf16 Student-t(3) with 8 outlier channels x50, "
          "theta~N(0,0.05), forward",
    "d5120_64k": "d=5120 schedule (8,8,8,5,2), 65536 rows/GPU bf16 N(0,1) with 1% entries x20, forward",
    "two_sided": "two-sided T_U^T W T_V: W 28672x8192 bf16 N(0,0.02^2) with 16 outlier columns x30, "
          "U (8,8,8,8,7), V (8,8,8,8,2), theta~N(0,0.05)",
    "d8192_int8": "d=8192 schedule (8,8,8,8,2), int8 theta + per-stage scale, 65536 rows/GPU bf16 N(0,1), forward",
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="d4096", choices=["d4096", "d5120_64k", "d8192_int8"])
    ap.add_argument("--no-extra", action="store_true", help="skip the d=5120 / d=8192 side measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quant-rows", type=int, default=0,
                    help="time only the fused rotate-then-quantize pass (harp_apply_quant) on this many d=4096 "
                         "rows and print its line (for profiling that kernel alone)")
    ap.add_argument("--grad-rows", type=int, default=0,
                    help="time only the calibration backward (harp_grad_theta) on this many d=4096 rows and "
                         "print its line (for profiling that kernel alone)")
    ap.add_argument("--two-sided-cols", type=int, default=0,
                    help="time only the two-sided rotation T_U^T W T_V of the two-sided workload with W cut to "
                         "this many columns (8^k, 2 * 8^k or 4 * 8^k; V = (8,...,8, 2 or 4), the workload's own "
                         "schedule at 8192) and print one JSON line")
    ap.add_argument("--decode-rows", type=int, default=0,
                    help="time only decode-shaped calls (this many rows of the d=8192 int8 workload, forward) "
                         "and print their line (for profiling that call alone)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--rows", type=int, default=0, help="rows per GPU (default: the workload's; "
                    "smaller values are for profiling captures, not bench lines)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------- clocks ---

class ClockSampler:
    """SM clock and clock-event reasons sampled during the timed region: NVML polled
    every 5 ms from a thread, or `nvidia-smi -lms 100` when NVML is not importable.
    Read-only queries; no GPU setting is touched."""
    REASONS = ((0x8, "hw_slowdown"), (0x40, "hw_thermal_slowdown"), (0x20, "sw_thermal_slowdown"),
               (0x4, "sw_power_cap"), (0x80, "hw_power_brake_slowdown"))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.thread = None
        self.samples = []
        self.stop_flag = False
        self.nvml = None
        self.handle = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        try:
            self.nvml, self.handle = self._nvml_handle()
            self.max_mhz = self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
            import threading

            def loop():
                while not self.stop_flag:
                    try:
                        sm = self.nvml.nvmlDeviceGetClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
                        rs = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                        self.samples.append((sm, rs))
                    except Exception:
                        pass
                    time.sleep(0.005)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.nvml = None
        fd, self.path = tempfile.mkstemp(prefix="harp_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
            if not self.samples:
                return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "source": "nvml"}
            reasons = set()
            for _, rs in self.samples:
                for bit, name in self.REASONS:
                    if rs & bit:
                        reasons.add(name)
            return {"sm_mhz": statistics.median(sm for sm, _ in self.samples), "sm_max_mhz": self.max_mhz,
                    "reasons": sorted(reasons), "samples": len(self.samples), "source": "nvml, 5 ms"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    rows.append({"sm": float(parts[1]), "max": float(parts[2]), "util": float(parts[4]),
                                 "hw": parts[6], "hwt": parts[7], "swt": parts[8], "pcap": parts[9]})
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": "nvidia-smi"}
        load = [r for r in rows if r["util"] >= 50] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(load), "source": "nvidia-smi, 100 ms"}


# --------------------------------------------------------------- profiles ---

def kernel_sources():
    d = os.path.join(ROOT, "structured_rotations_b200", "csrc")
    return {f: os.path.join(d, f) for f in os.listdir(d)}


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if its kernel source
    hash still matches the source being benchmarked; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_src = re.search(r"^source_file:\s*(\S+)", text, re.M)
    m_sha = re.search(r"^source_sha256:\s*([0-9a-f]{64})", text, re.M)
    m_b = re.search(r"^dram_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    if not (m_src and m_sha and m_b):
        return None
    src = kernel_sources().get(m_src.group(1))
    if not src:
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    return float(m_b.group(1)) if sha == m_sha.group(1) else None


# ------------------------------------------------------------- workloads ---

def make_plan(name, H, W, O_theta_count=None):
    w = W.get(name)
    n = H.theta_count(w.schedule)
    theta = W.draw_theta(n, w.theta_sigma, w.theta_seed)
    if w.theta_kind == "i8":
        counts = [(w.d // b) * (1 if b == 2 else b * (b - 1) // 2) for b in w.schedule]
        codes, scales = W.quantize_theta_int8(theta, counts)
        return H.Plan(w.d, w.schedule, codes=codes, scales=scales, sign_seed=w.sign_seed).materialize()
    return H.Plan(w.d, w.schedule, theta=theta, sign_seed=w.sign_seed).materialize()


def to_device_bf16(enc, torch, device):
    import numpy as np
    return torch.from_numpy(enc.view(np.int16)).view(torch.bfloat16).to(device)


# ------------------------------------------------------------- reference ---

def run_reference(args):
    import numpy as np
    import workloads as W
    from oracle import harp_oracle as O

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = W.get(args.workload)
    theta = W.draw_theta(O.theta_count(w.schedule), w.theta_sigma, w.theta_seed)
    if w.theta_kind == "i8":
        codes, scales = W.quantize_theta_int8(theta, O.stage_theta_counts(w.schedule))
        plan = O.make_plan(w.d, w.schedule, codes=codes, scales=scales, sign_seed=w.sign_seed)
    else:
        plan = O.make_plan(w.d, w.schedule, theta, sign_seed=w.sign_seed)
    tr = O.Transform(plan)
    sample = 256
    x = W.draw_rows(w, 0, sample)
    for _ in range(args.warmup):
        tr.forward(x)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        tr.forward(x)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = sample * args.steps / total
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "rows_per_step": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "host_cores": host_threads()[0], "thread_env": host_threads()[1],
                         "sample": f"{sample} rows of the workload per step (float64 scipy CSR stages, one core "
                                   f"of {host_threads()[0]})"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


def host_threads():
    """The host's usable cores and the BLAS / OpenMP thread settings, recorded beside the
    oracle's timing (its scipy CSR stage products run on one core)."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    env = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    return cores, {k: v for k, v in env.items() if v is not None}


def cpu_baseline(args, W):
    from oracle import harp_oracle as O
    w = W.get(args.workload)
    theta = W.draw_theta(O.theta_count(w.schedule), w.theta_sigma, w.theta_seed)
    tr = O.Transform(O.make_plan(w.d, w.schedule, theta, sign_seed=w.sign_seed))
    chunk = 512
    x = W.draw_rows(w, 0, chunk)
    rows, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < args.cpu_seconds:
        tr.forward(x)
        rows += chunk
    dt = time.perf_counter() - t0
    host_cores, blas_env = host_threads()
    return {"value": rows / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
            "host_cores": host_cores, "thread_env": blas_env,
            "sample": f"{rows} rows of the workload ({chunk}-row chunks, float64 scipy CSR stages, "
                      f"one core of {host_cores}) in {dt:.1f} s"}


# ------------------------------------------------------------------ ours ---

def time_apply(plan, x, y, steps, warmup, torch, dist=None, direction="forward"):
    """Warm up, then time exactly `steps` applies between a barrier and a sync on
    both sides.  Returns (elapsed_ms, mean kernel ms, launches)."""
    import structured_rotations_b200 as H
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        plan.apply(x, y, direction=direction)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for a, b in ev:
        a.record(stream)
        plan.apply(x, y, direction=direction)
        b.record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    elapsed = t0.elapsed_time(t1)
    kern = statistics.mean(a.elapsed_time(b) for a, b in ev)
    return elapsed, kern, steps, H.last_kernel()


def time_calls(plan, x, y, calls, warmup, torch, direction):
    """Per-call cost of small launches, three ways (microseconds): on the device, with the
    stream held back by a sleep kernel so that all `calls` launches are queued before the
    first runs (launch gaps included, host time excluded); on the host, the time the public
    call takes to return while the device is busy; and the wall time per call of `calls`
    back-to-back calls followed by one synchronize."""
    import structured_rotations_b200 as H
    for _ in range(warmup):
        plan.apply(x, y, direction=direction)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(int(2e8))          # about 0.1 s at the B200's clock: longer than the submissions
    e0.record(stream)
    t0 = time.perf_counter()
    for _ in range(calls):
        plan.apply(x, y, direction=direction)
    host_us = (time.perf_counter() - t0) * 1e6 / calls
    e1.record(stream)
    torch.cuda.synchronize()
    dev_us = e0.elapsed_time(e1) * 1e3 / calls
    t0 = time.perf_counter()
    for _ in range(calls):
        plan.apply(x, y, direction=direction)
    torch.cuda.synchronize()
    wall_us = (time.perf_counter() - t0) * 1e6 / calls
    return dev_us, host_us, wall_us, H.last_kernel()


def end_to_end(args, plan, enc, x, y, torch, dist, device, world, rows):
    """The same metric through the public host-buffer call (harp_apply_host): every step
    copies this rank's rows from pinned host memory to the GPU, rotates them and copies
    them back, chunk by chunk on overlapping streams; host wall clock around the
    synchronous call, max over ranks."""
    import numpy as np
    xh = torch.from_numpy(enc.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    for _ in range(2):
        plan.apply_host(xh, yh)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.e2e_steps):
        plan.apply_host(xh, yh)
    e2e_s = time.perf_counter() - t0
    e2e_s = max_over_ranks(e2e_s, dist, device)
    e2e = {"value": world * rows * args.e2e_steps / e2e_s, "unit": UNIT,
           "h2d_bytes_per_step": int(xh.numel() * 2), "d2h_bytes_per_step": int(yh.numel() * 2),
           "path": "harp_apply_host: pinned host rows -> GPU -> pinned host rows, 32 MiB chunks on 3 streams"}
    del xh, yh
    return e2e


SIDE = (("d4096", "inverse"), ("d5120_64k", "forward"), ("d5120_64k", "inverse"), ("d8192_int8", "forward"),
        ("d8192_int8", "inverse"))


def side_measurements(args, H, W, torch, device, peak):
    """The other configurations' rows/s and GB/s (device-timed, one line each): every
    direction the workloads list, and the two-sided weight rotation."""
    out = []
    cache = {}
    for name, direction in SIDE:
        ww = W.get(name)
        if name not in cache:
            cache.clear()
            e2 = W.draw_encoded(ww, 0, ww.rows)
            cache[name] = (make_plan(name, H, W), to_device_bf16(e2, torch, device))
        p2, x2 = cache[name]
        y2 = torch.empty_like(x2)
        st = max(3, args.steps // 4)
        el, km, _, kn = time_apply(p2, x2, y2, st, max(3, args.warmup // 2), torch, direction=direction)
        b2 = 2 * ww.rows * ww.d * 2
        out.append({"workload": WORKLOAD_TEXT[name].replace("forward", direction), "rows_per_s": ww.rows * st / (el / 1e3),
                    "hbm_gbs": b2 / (km / 1e3) / 1e9, "hbm_frac": b2 / (km / 1e3) / 1e9 / peak,
                    "kernel": kn, "kernel_ms": km,
                    "traffic": recorded_traffic(kn, name) if direction == "forward" else None})
        del y2
    cache.clear()
    # decode-shaped batches of the d = 8192 int8 workload: cost of one call
    wd = W.get("d8192_int8")
    pd_ = make_plan("d8192_int8", H, W)
    for rows_d in (1, 16, 256):
        xd = to_device_bf16(W.draw_encoded(wd, 0, rows_d), torch, device)
        yd = torch.empty_like(xd)
        for direction in ("forward", "inverse"):
            dev_us, host_us, wall_us, kn = time_calls(pd_, xd, yd, 200, 20, torch, direction)
            coef = 4 * wd.d * sum(wd.schedule)      # the plan's fp32 blocks, read once per call
            rb = 4 * rows_d * wd.d
            out.append({"workload": f"d=8192 schedule (8,8,8,8,2), int8 theta, {rows_d} bf16 rows (decode-shaped), "
                                    f"{direction}", "rows_per_s": rows_d / (wall_us / 1e6),
                        "us_per_call": wall_us, "device_us_per_call": dev_us, "host_us_per_call": host_us,
                        "kernel": kn, "row_bytes": rb, "coefficient_bytes": coef,
                        "row_hbm_frac": rb / (dev_us / 1e6) / 1e9 / peak,
                        "hbm_frac": (rb + coef) / (dev_us / 1e6) / 1e9 / peak})
        del xd, yd
    del pd_
    ts, pv, wo = two_sided_measurement(args, H, W, torch, device, peak, keep=True)
    out.append(ts)
    out.append(fit_measurement(H, W, torch, device, peak, pv, wo, W.get("two_sided")))
    del pv, wo
    out.append(quant_measurement(args, H, W, torch, device, peak))
    out.append(compose_measurement(args, H, W, torch, device, peak))
    out.append(moment_measurement(args, H, W, torch, device, peak))
    return out


def moment_measurement(args, H, W, torch, device, peak, steps=20):
    """The moment check that picks the number of composed passes (harp_moment_check) on the
    d = 4096 workload's rows: one read of the rows (2 d bytes each), per-row moments and pass
    counts written (28 bytes each)."""
    w = W.get("d4096")
    x = to_device_bf16(W.draw_encoded(w, 0, w.rows), torch, device)
    m = torch.empty(w.rows, 3, dtype=torch.float64, device=device)
    k = torch.empty(w.rows, dtype=torch.int32, device=device)
    tau1, tau2 = 4.0 / w.d, 40.0 / w.d
    for _ in range(3):
        H.moment_check(x, tau1, tau2, m, k)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        H.moment_check(x, tau1, tau2, m, k)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    byt = w.rows * (2 * w.d + 28)
    counts = torch.bincount(k, minlength=4).cpu().tolist()
    return {"workload": f"moment check (passes for tau = 4/d, 40/d): d=4096, {w.rows} bf16 rows", "kernel_ms": ms,
            "rows_per_s": w.rows / (ms / 1e3), "hbm_gbs": byt / (ms / 1e3) / 1e9,
            "hbm_frac": byt / (ms / 1e3) / 1e9 / peak, "kernel": "moment_check_kernel",
            "rows_needing_1_2_3_passes": counts[1:4]}


def fit_measurement(H, W, torch, device, peak, pv, w_rot, w4, q=128, steps=10):
    """The fit's evaluation terms on the two-sided workload's shapes: the Hessian proxy of
    the V side (8192 x 8192, fp32) rotated to H' = T_V^T H T_V by the two-sided rotation,
    then R_bd's off-block energy of H' (harp_off_block_energy, q = 128) and L_diag of the
    rotated bf16 weight W' (28672 x 8192) weighted by diag(H') (harp_l_diag, qblock 128).
    The two reductions read their matrix once: algorithmic bytes 4 n^2 and 2 n_out n_in."""
    import numpy as np
    n = w4.n_in
    hdev = torch.from_numpy(W.draw_hessian(n, 4000 + w4.index).astype(np.float32)).to(device)
    hrot = torch.empty_like(hdev)
    ws = torch.empty(H.workspace_bytes(n, n), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    rot_ms = timed(lambda: H.apply_two_sided(pv, pv, hdev, hrot, ws))
    e = torch.empty(2, dtype=torch.float64, device=device)
    rbd_ms = timed(lambda: H.off_block_energy(hrot, q, e))
    ld = torch.empty(1, dtype=torch.float64, device=device)
    ldiag_ms = timed(lambda: H.l_diag(w_rot, hrot, q, ld))
    ev = e.cpu().numpy()
    b_rbd, b_ld = 4 * n * n, 2 * w_rot.numel()
    del hdev, hrot, ws
    return {"workload": f"fit terms on the two-sided shapes: H' = T_V^T H T_V ({n}x{n} fp32 Hessian proxy), "
                        f"R_bd at q={q}, L_diag of W' ({w4.n_out}x{n} bf16) at qblock {q}",
            "rotate_hessian_ms": rot_ms, "r_bd": float(ev[0] / ev[1]), "l_diag": float(ld.cpu().numpy()[0]),
            "off_block_energy_ms": rbd_ms, "off_block_energy_hbm_gbs": b_rbd / (rbd_ms / 1e3) / 1e9,
            "off_block_energy_hbm_frac": b_rbd / (rbd_ms / 1e3) / 1e9 / peak,
            "l_diag_ms": ldiag_ms, "l_diag_hbm_gbs": b_ld / (ldiag_ms / 1e3) / 1e9,
            "l_diag_hbm_frac": b_ld / (ldiag_ms / 1e3) / 1e9 / peak,
            "kernel": "off_block_energy_kernel, l_diag_kernel"}


def compose_measurement(args, H, W, torch, device, peak):
    """Two rotations composed (harp_plan_compose) on the d = 4096 workload's rows: the C2
    plan, then a second (8,8,8,8) plan (theta seed + 1, sign seed + 1), in one pass; beside
    it the same two plans as two separate passes with a bf16 intermediate."""
    w = W.get("d4096")
    p1 = make_plan("d4096", H, W)
    th2 = W.draw_theta(H.theta_count(w.schedule), w.theta_sigma, w.theta_seed + 1)
    p2 = H.Plan(w.d, w.schedule, theta=th2, sign_seed=w.sign_seed + 1).materialize()
    comp = H.Plan.compose([p1, p2])
    x = to_device_bf16(W.draw_encoded(w, 0, w.rows), torch, device)
    y = torch.empty_like(x)
    st = max(3, args.steps // 4)
    el, km, _, kn = time_apply(comp, x, y, st, 3, torch)
    mid = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    for _ in range(3):
        p1.apply(x, mid)
        p2.apply(mid, y)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(st):
        p1.apply(x, mid)
        p2.apply(mid, y)
    e1.record(stream)
    torch.cuda.synchronize()
    two = e0.elapsed_time(e1) / st
    byt = 2 * w.rows * w.d * 2
    return {"workload": "two rotations composed: d=4096 (8,8,8,8) x 2, 65536 bf16 rows, one pass",
            "kernel_ms": km, "rows_per_s": w.rows / (km / 1e3), "hbm_gbs": byt / (km / 1e3) / 1e9,
            "hbm_frac": byt / (km / 1e3) / 1e9 / peak, "kernel": kn,
            "two_passes_ms": two, "two_passes_kernels": "harp_fast_d4096_fwd_kernel x 2 (bf16 between)"}



def two_sided_v_schedule(n_in, w4):
    """V's schedule for a two-sided case with n_in columns: the workload's own at its n_in (or
    when n_in is 0), else radix 8 stages and one radix 2 or 4 (n_in = 8^k, 2 8^k or 4 8^k)."""
    if not n_in or n_in == w4.n_in:
        return tuple(w4.schedule)
    k = 0
    while 8 ** (k + 1) <= n_in:
        k += 1
    r = n_in // 8 ** k
    if k < 1 or r * 8 ** k != n_in or r not in (1, 2, 4):
        raise SystemExit(f"--two-sided-cols must be 8^k, 2 * 8^k or 4 * 8^k, got {n_in}")
    return (8,) * k + ((r,) if r > 1 else ())


def two_sided_measurement(args, H, W, torch, device, peak, n_in=None, keep=False):
    """The two-sided weight rotation W_out = T_U^T W T_V on the two-sided workload (V on the
    rows, d = n_in; U on the columns, d = n_out); n_in cuts W to fewer columns, with V's
    schedule the workload's (8,8,8,8,2) shortened to match (a smaller case for profiles).
    Algorithmic HBM bytes: two passes, each reading and writing W once.  keep: also return
    plan V and the rotated weight (the fit terms' line uses them)."""
    import numpy as np
    w4 = W.get("two_sided")
    v_sched = two_sided_v_schedule(n_in, w4)
    n_in = int(np.prod(v_sched))
    th_v = W.draw_theta(H.theta_count(v_sched), w4.theta_sigma, w4.theta_seed)
    th_u = W.draw_theta(H.theta_count(w4.u_schedule), w4.theta_sigma, w4.theta_seed + 7)
    pv = H.Plan(n_in, v_sched, theta=th_v, sign_seed=w4.sign_seed).materialize()
    pu = H.Plan(w4.n_out, w4.u_schedule, theta=th_u, sign_seed=w4.sign_seed + 11).materialize()
    wt = to_device_bf16(W.draw_encoded(w4, 0, w4.n_out, n_in), torch, device)
    wo = torch.empty_like(wt)
    ws = torch.empty(H.workspace_bytes(w4.n_out, n_in), dtype=torch.uint8, device=device)
    for _ in range(2):
        H.apply_two_sided(pu, pv, wt, wo, ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    st = 3
    e0.record(stream)
    for _ in range(st):
        H.apply_two_sided(pu, pv, wt, wo, ws)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / st
    b4 = 2 * (2 * w4.n_out * n_in * 2)        # two passes, each reading and writing W once
    text = WORKLOAD_TEXT["two_sided"] if n_in == w4.n_in else \
        f"two-sided T_U^T W T_V: W {w4.n_out}x{n_in} bf16, U {tuple(w4.u_schedule)}, V {v_sched}"
    res = {"workload": text, "ms": ms, "hbm_gbs": b4 / (ms / 1e3) / 1e9, "hbm_frac": b4 / (ms / 1e3) / 1e9 / peak,
           "kernel": "harp_apply_two_sided: harp_tiled_kernel (rows) + 2 x harp_cols_kernel (columns)"}
    del wt, ws
    return (res, pv, wo) if keep else res

def quant_measurement(args, H, W, torch, device, peak, qblock=128, rows=None):
    """The fused rotate-then-quantize pass (harp_apply_quant) on the d = 4096 workload:
    bf16 rows in, int8 codes and one fp32 scale per 128 coordinates out; algorithmic HBM
    bytes 2 d + d + 4 d / qblock per row."""
    w = W.get("d4096", rows)
    plan = make_plan("d4096", H, W)
    x = to_device_bf16(W.draw_encoded(w, 0, w.rows), torch, device)
    q = torch.empty(w.rows, w.d, dtype=torch.int8, device=device)
    sc = torch.empty(w.rows, w.d // qblock, dtype=torch.float32, device=device)
    for _ in range(3):
        plan.apply_quant(x, qblock, q=q, scales=sc)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    st = max(3, args.steps // 4)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(st)]
    for a, b in ev:
        a.record(stream)
        plan.apply_quant(x, qblock, q=q, scales=sc)
        b.record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    byt = w.rows * (2 * w.d + w.d + 4 * (w.d // qblock))
    kn = H.last_kernel()
    return {"workload": f"rotate + int8 quantize (qblock {qblock}): d=4096 schedule (8,8,8,8), {w.rows} bf16 rows "
                        f"-> int8 codes + fp32 scales, forward",
            "kernel_ms": ms, "rows_per_s": w.rows / (ms / 1e3), "hbm_gbs": byt / (ms / 1e3) / 1e9,
            "hbm_frac": byt / (ms / 1e3) / 1e9 / peak, "kernel": kn + " (int8 epilogue)",
            "traffic": recorded_traffic(kn, "quant_d4096") if rows is None else None}


def grad_roofline(res, clocks, device, torch):
    """The FMA roofline of a grad_measurement line at the sampled median SM clock (the
    maximum clock if none was sampled)."""
    mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    alu_peak = sms * 128 * mhz * 1e6
    res["roofline"] = {"bound": "alu", "achieved": res["fma_per_s"] / 1e12, "peak": alu_peak / 1e12,
                       "unit": "TFMA/s", "frac": res["fma_per_s"] / alu_peak,
                       "peak_source": f"{sms} SMs x 128 FP32 lanes x {mhz} MHz (median sampled SM clock)"}
    return res


def grad_measurement(H, W, torch, device, peak, rows=None, steps=10):
    """The calibration backward dL/dtheta (harp_grad_theta) on the d = 4096 workload: rows
    x and upstream gradients g (bf16, N(0, 1)), device-timed over `steps` calls (each
    call: accumulator reset, the block-gradient kernel, the theta kernel).  Its roof is
    the FP32 FMA rate: 4 d sum(b) FMA per row (the forward chain once, the backward
    chain's two transposed products and the outer product) against 148 SMs x 128 FMA
    lanes at the sampled SM clock; it reads 4 d bytes per row from HBM."""
    w = W.get("d4096")
    rows = rows or w.rows
    plan = make_plan("d4096", H, W)
    x = to_device_bf16(W.draw_encoded(w, 0, rows), torch, device)
    g = to_device_bf16(W.draw_upstream(w, 0, rows), torch, device)
    out = torch.empty(H.theta_count(w.schedule), dtype=torch.float32, device=device)
    ws = torch.empty(int(H.lib().harp_grad_workspace_bytes(plan.handle)), dtype=torch.uint8, device=device)
    for _ in range(3):
        plan.grad_theta(x, g, out, ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        plan.grad_theta(x, g, out, ws)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    fma = 4 * w.d * sum(w.schedule) * rows
    byt = 4 * rows * w.d
    return {"workload": f"calibration backward dL/dtheta, d=4096 schedule (8,8,8,8), {rows} bf16 rows x and "
                        f"upstream gradients g (N(0,1)), theta~N(0,0.05)",
            "ms": ms, "rows_per_s": rows / (ms / 1e3), "hbm_gbs": byt / (ms / 1e3) / 1e9,
            "hbm_frac": byt / (ms / 1e3) / 1e9 / peak, "fma_per_row": 4 * w.d * sum(w.schedule),
            "fma_per_s": fma / (ms / 1e3),
            "kernel": "harp_grad_blocks_kernel + harp_grad_theta_kernel", "steps": steps,
            "traffic": (recorded_traffic("harp_grad_blocks_kernel", "d4096") if rows == w.rows else None)}


def run_ours(args):
    import numpy as np
    import torch
    import structured_rotations_b200 as H
    import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        log(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=device)
        dist = tdist

    if args.decode_rows:
        wd = W.get("d8192_int8")
        pd_ = make_plan("d8192_int8", H, W)
        xd = to_device_bf16(W.draw_encoded(wd, 0, args.decode_rows), torch, device)
        yd = torch.empty_like(xd)
        dev_us, host_us, wall_us, kn = time_calls(pd_, xd, yd, max(1, args.steps), max(3, args.warmup), torch,
                                                  "forward")
        pd_.device_status()
        print(json.dumps({"workload": f"d=8192 schedule (8,8,8,8,2), int8 theta, {args.decode_rows} bf16 rows, "
                                      "forward", "device_us_per_call": dev_us, "host_us_per_call": host_us,
                          "us_per_call": wall_us, "kernel": kn}))
        return 0
    if args.two_sided_cols:
        print(json.dumps(two_sided_measurement(args, H, W, torch, device, peaks()[0], args.two_sided_cols)))
        return 0
    if args.quant_rows:
        peak, _ = peaks()
        print(json.dumps(quant_measurement(args, H, W, torch, device, peak, rows=args.quant_rows)))
        return 0
    if args.grad_rows:
        peak, _ = peaks()
        sampler = ClockSampler(local)
        sampler.start()
        res = grad_measurement(H, W, torch, device, peak, args.grad_rows, args.steps)
        clocks = sampler.stop()
        print(json.dumps(grad_roofline(res, clocks, device, torch)))
        return 0

    w = W.get(args.workload, args.rows or None)
    rows, d = w.rows, w.d
    plan = make_plan(args.workload, H, W)
    t = time.time()
    row0, rows = weak_shard(rows, rank)              # this rank's block of the global batch
    enc = W.draw_encoded(w, row0, rows)
    log(f"rank {rank}: generated {rows}x{d} input in {time.time() - t:.1f}s")
    x = to_device_bf16(enc, torch, device)
    y = torch.empty_like(x)

    sampler = ClockSampler(local)
    sampler.start()
    elapsed, kern_ms, launches, kname = time_apply(plan, x, y, args.steps, args.warmup, torch, dist)
    clocks = sampler.stop()

    elapsed = max_over_ranks(elapsed, dist, device)
    step_ms = elapsed / args.steps
    value = world * rows * args.steps / (elapsed / 1e3)
    bytes_per_launch = 2 * rows * d * 2
    peak, peak_kind = peaks()
    achieved = bytes_per_launch / (kern_ms / 1e3) / 1e9
    traffic = recorded_traffic(kname, args.workload)

    # end to end through the public API: pinned host rows in, pinned host rows out
    e2e = end_to_end(args, plan, enc, x, y, torch, dist, device, world, rows) if args.e2e_steps > 0 else None

    also = []
    if not args.no_extra and rank == 0 and world == 1:
        also = side_measurements(args, H, W, torch, device, peak)
        also.append(grad_roofline(grad_measurement(H, W, torch, device, peak), clocks, device, torch))

    cpu = None
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        cpu = cpu_baseline(args, W)

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "d": d, "schedule": list(w.schedule),
                   "rows_per_gpu": rows, "io_dtype": "bf16", "parallelism": f"row shards x{world}",
                   "l2": "inputs 512 MiB per step > 126 MB L2; no flush"},
        "hbm_gbs": achieved, "hbm_frac": achieved / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_kind} copy bandwidth", "kernel": kname,
                     "algorithmic_bytes_per_launch": bytes_per_launch, "kernel_ms": kern_ms},
        "clocks": clocks, "gpu_launches": launches, "e2e": e2e,
        "cpu_baseline": cpu, "also": also,
    }
    print(json.dumps(out), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
