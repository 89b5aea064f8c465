"""Benchmark of the W4 g64 quantized linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload qkv] [--impl ours|reference]

One step = one qlinear_forward call (y = x . W^T) on the workload's seeded
synthetic inputs, which are resident in HBM when the timed region starts.
Between timed steps a 512 MiB buffer is written to flush the 126 MB L2, so no
step starts with its operands cached.  Each step is timed on the launching
stream with CUDA events; the main kernel is timed alone through the
library's profile-event hook.  Under torchrun every rank runs an independent
replica (the layer needs no exchange for data-parallel tokens), the slowest
rank's time is reported, and `value` counts the work of all ranks.

--impl reference times the CPU oracle (numpy, float64) on a bounded row
sample of the same workload; it is the deliberately slow baseline of this
build, not a tuned CPU implementation.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from group_wise_affine_qlinear_b200 import synthetic as S  # noqa: E402

METRIC = "W4g64 qmatmul TFLOP/s (large-M tensor-core path)"
FLUSH_BYTES = 512 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="qkv", choices=sorted(S.WORKLOADS))
    ap.add_argument("--M", type=int, default=0, help="override the token count (0 = the workload's)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("bf16_tflops", 1590.0), d.get("hbm_gbs", 6650.0), "measured"
    return 1590.0, 6650.0, "fallback"


def kernel_source_hash() -> str:
    import hashlib
    d = os.path.join(ROOT, "group_wise_affine_qlinear_b200", "csrc")
    src = open(os.path.join(d, "ql_tc_fused.cuh"), "rb").read() + open(os.path.join(d, "ql_ptx.cuh"), "rb").read()
    return hashlib.sha256(src).hexdigest()[:12]


def recorded_traffic(path: str, key: str):
    """DRAM bytes per launch from the last ncu capture, if it was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    h = kernel_source_hash()
    for ln in open(p):
        f = ln.split()
        if len(f) == 4 and f[0] == path and f[1] == key and f[2] == h:
            return int(f[3])
    return None


# ---------------------------------------------------------------------------- CPU oracle timing

def oracle_rate(w: S.Workload, M: int, seconds: float, x_bits=None, weights=None):
    """Time the oracle on whole 64-row chunks of the workload until `seconds` pass (at least one chunk)."""
    from oracle import qlinear_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count() or 1
    codes, s, b = weights if weights is not None else w.w()
    x = x_bits if x_bits is not None else w.x(min(M, 512))
    rows_done = 0
    t0 = time.perf_counter()
    chunk = 0
    while True:
        r0 = (chunk * 64) % x.shape[0]
        rows = np.arange(r0, min(r0 + 64, x.shape[0]))
        O.forward_rows(x, codes, s, b, rows)
        rows_done += rows.size
        chunk += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    flops = 2.0 * rows_done * w.K * w.N
    return flops / dt / 1e12, cores, rows_done, dt


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

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
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- reference arm

def run_reference(a, rank, world):
    if rank != 0:
        return
    w = S.WORKLOADS[a.workload]
    M = a.M or w.M
    x = w.x(min(M, 512))
    weights = w.w()
    per = []
    for i in range(a.warmup + a.steps):
        rate, cores, rows, dt = oracle_rate(w, M, 0.0, x, weights)     # one 64-row chunk per step
        if i >= a.warmup:
            per.append((rate, rows, dt))
    rate = sum(r[1] for r in per) * 2.0 * w.K * w.N / sum(r[2] for r in per) / 1e12
    ms = 1e3 * 2.0 * M * w.K * w.N / (rate * 1e12)
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": "TFLOP/s", "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name} M={M} K={w.K} N={w.N}", "sample": "64 rows per step"},
        "cpu_baseline": {"value": rate, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"64 of {M} rows per step (rows are independent), full N and K"},
        "e2e": {"value": rate, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- our arm

def main():
    a = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        return run_reference(a, rank, world)

    import torch
    import torch.distributed as dist
    import group_wise_affine_qlinear_b200 as ql

    torch.cuda.set_device(local)
    pg = False
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
        pg = True

    def barrier():
        if pg:
            dist.barrier()
        torch.cuda.synchronize()

    w = S.WORKLOADS[a.workload]
    M = a.M or w.M
    K, N = w.K, w.N
    x_np = w.x(M)
    codes_np, s_np, b_np = w.w()
    dev = torch.device("cuda", local)
    x = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).to(dev)
    codes = torch.from_numpy(codes_np.view(np.int32)).to(dev)
    sc = torch.from_numpy(s_np).to(dev)
    bi = torch.from_numpy(b_np).to(dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws_bytes = ql.workspace_size(M, K, N)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    x_host = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()

    def step():
        ql.forward(x, codes, sc, bi, out=y, workspace=ws)

    for _ in range(a.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    dispatch = ql.last_dispatch()
    launches_per_step = int(dispatch.split("launches=")[1].split()[0]) if "launches=" in dispatch else 1

    # ---- device-timed steps (inputs resident; L2 flushed between steps)
    K_ = a.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K_)]
    evm = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K_)]
    for e0, e1 in evm:            # create the handles so the library can record them
        e0.record()
        e1.record()
    clocks = ClockSampler(local)
    barrier()
    clocks.start()
    for i in range(K_):
        flush.fill_(i & 0xFF)
        ql.set_profile_events(*evm[i])
        ev[i][0].record()
        step()
        ev[i][1].record()
    ql.set_profile_events(None, None)
    barrier()
    clk = clocks.stop()
    step_ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    main_ms = [e0.elapsed_time(e1) for e0, e1 in evm]
    assert ql.device_status() == 0, "a kernel reported an error"

    # ---- end to end: pinned host x -> device, forward, y -> pinned host, per step
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K_)]
    barrier()
    for i in range(K_):
        flush.fill_(i & 0xFF)
        ev2[i][0].record()
        x.copy_(x_host, non_blocking=True)
        step()
        y_host.copy_(y, non_blocking=True)
        ev2[i][1].record()
    barrier()
    e2e_ms = [e0.elapsed_time(e1) for e0, e1 in ev2]

    mean_step = sum(step_ms) / K_
    mean_main = sum(main_ms) / K_
    mean_e2e = sum(e2e_ms) / K_
    if pg:
        t = torch.tensor([mean_step, mean_main, mean_e2e], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        mean_step, mean_main, mean_e2e = t.tolist()

    flops = 2.0 * M * K * N
    value = world * flops / (mean_step * 1e-3) / 1e12
    e2e_value = world * flops / (mean_e2e * 1e-3) / 1e12
    peak_tf, peak_gbs, peak_kind = peaks()
    main_tf = flops / (mean_main * 1e-3) / 1e12
    traffic = recorded_traffic(dispatch.split()[0], f"{w.name}:M={M}")

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K_, "warmup": a.warmup,
        "ms_per_step": mean_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 MMA, fp32 accumulate (bf16 in/out)", "data": "synthetic",
        "config": {"workload": f"{w.name} M={M} K={K} N={N}", "seed": w.seed, "l2": "flushed between steps (512 MiB write)",
                   "parallelism": f"replicas x{world}", "dispatch": dispatch,
                   "weight_GBps": (w.weight_bytes) / (mean_step * 1e-3) / 1e9},
        "roofline": {"bound": "tensor", "achieved": main_tf, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": main_tf / peak_tf, "traffic": traffic,
                     "kernel": dispatch.split()[0].replace("path=", ""), "kernel_ms": mean_main,
                     "peak_kind": f"{peak_kind} bf16 dense burst (f16 has the same tcgen05 rate)"},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2},
        "gpu_launches": launches_per_step * K_,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        rate, cores, rows, dt = oracle_rate(w, M, a.cpu_seconds, x_np[: min(M, 512)], (codes_np, s_np, b_np))
        line["cpu_baseline"] = {"value": rate, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": f"{rows} rows x full K x full N of {w.name} in {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
