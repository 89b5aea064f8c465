"""Benchmark of the W4 g64 quantized linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload qkv] [--impl ours|reference]

One step = one qlinear_forward call (y = x . W^T) on the workload's seeded
synthetic inputs, which are resident in HBM when the timed region starts.
Between timed steps a 512 MiB buffer is written to flush the 126 MB L2 and a
256 MiB buffer is read so the flush's dirty lines are written back first: no
step starts with its operands cached, and none pays for the flush.  Each step is timed on the launching
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
SPEC_TFLOPS, SPEC_GBPS = 2250.0, 8000.0     # B200 spec sheet: dense bf16 tensor rate, HBM3e bandwidth
FLUSH_BYTES = 512 << 20
CLEAN_BYTES = 256 << 20
L2_NOTE = ("flushed between steps: 512 MiB written, then 256 MiB of another buffer read, so the flush's "
           "dirty lines are back in HBM before the step starts")


class L2Flush:
    """Evicts every operand from the 126 MB L2 between timed steps.

    fill_() writes 512 MiB (the flush) and, unless dirty=True, then reads 256 MiB of a second buffer: the
    read evicts the flush's own dirty lines, whose write-back would otherwise run inside the next timed
    step and be charged to it (a memory-only streaming kernel on 123 MB measured 31 us after the write
    alone against 27.6 us after write + read on a B200).  dirty=True keeps the write alone, for context.
    """

    def __init__(self, torch, dev, dirty: bool = False):
        self.torch = torch
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = None if dirty else torch.ones(CLEAN_BYTES // 4, dtype=torch.int32, device=dev)

    def fill_(self, v: int):
        self.w.fill_(v)
        if self.r is not None:
            self.sink = self.torch.amax(self.r)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="qkv", choices=sorted(S.WORKLOADS))
    ap.add_argument("--M", type=int, default=0, help="override the token count (0 = the workload's)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", type=int, default=0, help="force a kernel path (0 = dispatcher's choice)")
    ap.add_argument("--split", type=int, default=0, help="force the split-K factor (0 = dispatcher's choice)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-small-m", action="store_true", help="skip the small-M weight-streaming measurements")
    ap.add_argument("--no-pack", action="store_true", help="skip the quantizer (qlinear_pack) measurement")
    ap.add_argument("--no-swiglu", action="store_true",
                    help="skip the fused SwiGLU pair on the MLP at the pages' width (I = 12288)")
    ap.add_argument("--no-split", action="store_true",
                    help="skip the text projection at M = 512 on the fused path with and without split-K")
    ap.add_argument("--no-comparators", action="store_true",
                    help="skip the cuBLAS context measurements (dense bf16 and dequant-then-matmul)")
    ap.add_argument("--no-w8", action="store_true",
                    help="skip the 8-bit conditioning projection (text_proj_w8) at M = 1, 8, 32")
    ap.add_argument("--no-large", action="store_true",
                    help="skip the other M >= 4608 workloads (the MLP pair, the 2048^2 canvas)")
    ap.add_argument("--no-dispatch", action="store_true",
                    help="skip the dispatcher-versus-forced-configurations sweep on the text projection")
    ap.add_argument("--no-noalloc", action="store_true", help="skip the allocation-free entry's measurement")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("bf16_tflops", 1590.0), d.get("hbm_gbs", 6650.0), "measured"
    return 1590.0, 6650.0, "fallback"


def kernel_source_hash() -> str:
    """First 12 hex digits of the sha256 over every CUDA source of the library, in name order: a recorded
    ncu traffic figure is used only while the kernels it was taken on are unchanged."""
    import hashlib
    d = os.path.join(ROOT, "group_wise_affine_qlinear_b200", "csrc")
    names = sorted(f for f in os.listdir(d) if f.endswith((".cu", ".cuh", ".h")))
    src = b"".join(f.encode() + b"\0" + open(os.path.join(d, f), "rb").read() for f in names)
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


# ---------------------------------------------------------------------------- quantizer timing

PACK_ROWS, PACK_K = 4608, 4608


def pack_inputs():
    """DiT-shaped dense weight N(0, 0.02^2) and E[x^2] of 512 synthetic activation rows (fp32)."""
    w = S.dense_weight(2, 0, PACK_ROWS, PACK_K, 0.02)
    xb = S.activations(2, 0, 512, PACK_K)
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return w, (xf * xf).mean(axis=0).astype(np.float32)


def pack_measure(ql, torch, dev, flush, runs=3):
    """Device time of qlinear_pack on a 4608 x 4608 weight: importance-weighted fit and RTN."""
    w, imp = pack_inputs()
    wd = torch.from_numpy(w).to(dev)
    impd = torch.from_numpy(imp).to(dev)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        ms = []
        for i in range(runs):
            flush.fill_(i & 0xFF)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        return sum(ms) / runs

    fit_ms = timed(lambda: ql.pack(wd, imatrix=impd))
    rtn_ms = timed(lambda: ql.pack(wd))
    assert ql.device_status() == 0, "qlinear_pack reported an error"
    groups = PACK_ROWS * PACK_K // 64
    rtn_bytes = PACK_ROWS * PACK_K * 4 + PACK_ROWS * PACK_K // 2 + groups * 4
    return {"workload": f"dense N(0, 0.02^2) {PACK_ROWS} x {PACK_K}, imatrix = E[x^2] of 512 synthetic rows",
            "groups": groups, "fit_ms": fit_ms, "fit_groups_per_s": groups / (fit_ms * 1e-3),
            "rtn_ms": rtn_ms, "rtn_GBps": rtn_bytes / (rtn_ms * 1e-3) / 1e9}


def swiglu_measure(ql, torch, dev, flush, peak_tf, steps=10):
    """Device time of the fused SwiGLU pair on the MLP at the pages' width (4608 tokens, K 4608, I 12288)."""
    w = S.WORKLOADS["mlp_gate_up_12288"]
    x = torch.from_numpy(w.x().view(np.int16)).view(torch.bfloat16).to(dev)
    gate, up = w.w_pair()
    dev3 = lambda c, s, b: (torch.from_numpy(c.view(np.int32)).to(dev), torch.from_numpy(s).to(dev),  # noqa: E731
                            torch.from_numpy(b).to(dev))
    gd, ud = dev3(*gate), dev3(*up)
    h = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(ql.swiglu_workspace_size(w.M, w.K, w.N), dtype=torch.uint8, device=dev)
    step = lambda: ql.swiglu(x, gd, ud, out=h, workspace=ws)  # noqa: E731
    for _ in range(3):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    assert ql.device_status() == 0, "the SwiGLU pair reported an error in warm-up"
    dispatch = ql.last_dispatch()
    call_ms, main_ms = [], []
    for i in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.fill_(i & 0xFF)
        e0.record()
        step()
        e1.record()
        flush.fill_(i & 0xFF)
        m0.record()
        m1.record()
        ql.set_profile_events(m0, m1)
        step()
        ql.set_profile_events(None, None)
        torch.cuda.synchronize()
        call_ms.append(e0.elapsed_time(e1))
        main_ms.append(m0.elapsed_time(m1))
    assert ql.device_status() == 0, "the SwiGLU pair reported an error"
    flops = 2.0 * w.M * w.K * 2 * w.N
    call, main = sum(call_ms) / steps, sum(main_ms) / steps
    return {"workload": f"{w.name} M={w.M} K={w.K} I={w.N} (gate + up)", "dispatch": dispatch,
            "step_ms": call, "kernel_ms": main, "TFLOPs": flops / (call * 1e-3) / 1e12,
            "kernel_TFLOPs": flops / (main * 1e-3) / 1e12, "kernel_frac": flops / (main * 1e-3) / 1e12 / peak_tf,
            "traffic": recorded_traffic(dispatch.split()[0], f"{w.name}:M={w.M}")}


def comparators(ql, torch, dev, flush, steps=10):
    """Context, not targets: the same layers through cuBLAS (torch.matmul) on this machine.

    dense: a bf16 copy of W (made once by qlinear_dequant) times x, the unquantized layer's GEMM;
    dequant_then_matmul: qlinear_dequant to bf16 every step, then the same GEMM, the way a packed
    layer runs when it only has a library GEMM.  L2 is flushed before every step.
    """
    out = {}
    for name, Ms in (("qkv", None), ("text_proj", 32)):
        w = S.WORKLOADS[name]
        M = Ms or w.M
        x = torch.from_numpy(w.x(M).view(np.int16)).view(torch.bfloat16).to(dev)
        c, s, b = w.w()
        cd = torch.from_numpy(c.view(np.int32)).to(dev)
        sd, bd = torch.from_numpy(s).to(dev), torch.from_numpy(b).to(dev)
        wb = ql.dequant(cd, sd, bd, out_dtype=torch.bfloat16)
        wtmp = torch.empty_like(wb)
        y = torch.empty((M, w.N), dtype=torch.bfloat16, device=dev)

        def dense():
            torch.matmul(x, wb.t(), out=y)

        def deq_mm():
            torch.matmul(x, ql.dequant(cd, sd, bd, out_dtype=torch.bfloat16, out=wtmp).t(), out=y)

        res = {}
        for key, fn in (("dense_bf16_matmul", dense), ("dequant_then_matmul", deq_mm)):
            for _ in range(3):
                flush.fill_(1)
                fn()
            torch.cuda.synchronize()
            ms = []
            for i in range(steps):
                flush.fill_(i & 0xFF)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                ms.append(e0.elapsed_time(e1))
            mean = sum(ms) / steps
            res[key] = {"ms": mean, "TFLOPs": 2.0 * M * w.K * w.N / (mean * 1e-3) / 1e12}
        out[f"{name} M={M} K={w.K} N={w.N}"] = res
        del wb, wtmp, x, y, cd, sd, bd
        torch.cuda.empty_cache()
    return out


def split_measure(ql, torch, dev, flush, peak_tf, steps=10):
    """The text projection at M = 512 (54 output tiles on 148 SMs) on the fused path, whole and split 8 ways."""
    w = S.WORKLOADS["text_proj"]
    M = 512
    flops = 2.0 * M * w.K * w.N
    out = {"workload": f"{w.name} M={M} K={w.K} N={w.N}"}
    for split in (1, 8):
        c = Case(ql, torch, w, M, 3, dev, flush, split)          # 3 = the fused tensor-core path
        c.warm(3)
        assert ql.device_status() == 0, "the fused path reported an error in warm-up"
        st, mn = c.timed(steps)
        assert ql.device_status() == 0, "the fused path reported an error"
        out[f"split{split}"] = {"dispatch": c.dispatch, "step_us": st * 1e3, "kernel_us": mn * 1e3,
                                "TFLOPs": flops / (st * 1e-3) / 1e12,
                                "kernel_frac": flops / (mn * 1e-3) / 1e12 / peak_tf,
                                "traffic": recorded_traffic(c.dispatch.split()[0], f"{w.name}:M={M}:split={split}")}
        del c
    torch.cuda.synchronize()
    return out


def fitted_weights(ql, torch, dev, w, x_bits, codes, scales, biases):
    """Device copies of the workload's packed weight with its first w.fitted_rows rows replaced by the
    importance-weighted fit (qlinear_pack with an imatrix, byte-identical to the oracle's fit) of dense
    N(0, 0.02^2) floats, the importance being E[x^2] of the workload's own activations."""
    R = w.fitted_rows
    dense = S.dense_weight(w.seed, w.widx, R, w.K, 0.02)
    xf = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    imp = (xf * xf).mean(axis=0).astype(np.float32)
    cf, sf, bf = ql.pack(torch.from_numpy(dense).to(dev), imatrix=torch.from_numpy(imp).to(dev))
    codes[:R].copy_(cf)
    scales[:R].copy_(sf)
    biases[:R].copy_(bf)
    torch.cuda.synchronize()
    assert ql.device_status() == 0, "qlinear_pack reported an error"


def large_m_measure(ql, torch, dev, flush, peak_tf, steps=5):
    """The other M >= 4608 workloads, each through the dispatcher: the MLP pair (up/gate N = 2 x 18432 with
    its first 4608 rows fitted, down K = 18432) and the 2048^2 canvas (M = 33792, N = 4608 and 13824)."""
    out = {}
    for name in ("mlp_up_gate", "mlp_down", "canvas2048_n4608", "canvas2048_n13824"):
        w = S.WORKLOADS[name]
        c = Case(ql, torch, w, w.M, 0, dev, flush)
        if w.fitted_rows:
            fitted_weights(ql, torch, dev, w, c.x_np, c.codes, c.sc, c.bi)
        c.warm(3)
        assert ql.device_status() == 0, f"{name}: a kernel reported an error in warm-up"
        st, mn = c.timed(steps)
        assert ql.device_status() == 0, f"{name}: a kernel reported an error"
        flops = 2.0 * w.M * w.K * w.N
        out[name] = {"workload": f"{w.name} M={w.M} K={w.K} N={w.N}" + (f" ({w.fitted_rows} rows fitted)"
                                                                          if w.fitted_rows else ""),
                     "dispatch": c.dispatch, "step_ms": st, "kernel_ms": mn,
                     "TFLOPs": flops / (st * 1e-3) / 1e12, "kernel_TFLOPs": flops / (mn * 1e-3) / 1e12,
                     "frac": flops / (st * 1e-3) / 1e12 / peak_tf,
                     "frac_of_spec": flops / (st * 1e-3) / 1e12 / SPEC_TFLOPS,
                     "kernel_frac": flops / (mn * 1e-3) / 1e12 / peak_tf}
        del c
        torch.cuda.empty_cache()
    return out


def dispatch_measure(ql, torch, dev, flush, steps=10):
    """The dispatcher against every forced configuration on the text projection for 33 <= M <= 512: the
    automatic choice's whole-call time beside the best forced one (weight streaming up to 64 tokens, the
    fused kernel with split-K 1, 2, 4, 5, 8)."""
    w = S.WORKLOADS["text_proj"]
    out = []
    base = None
    for M in (33, 48, 64, 65, 128, 256, 512):
        c = Case(ql, torch, w, M, 0, dev, flush, weights=base)
        base = (c.codes, c.sc, c.bi, c.codes_np, c.s_np, c.b_np)
        c.warm(2)
        auto_us = c.timed(steps)[0] * 1e3
        auto = c.dispatch
        forced = {}
        for path, split in ([(2, 0)] if M <= 64 else []) + [(3, 1), (3, 2), (3, 4), (3, 5), (3, 8)]:
            c.set_config(path, split)
            c.warm(2)
            forced[f"path{path}_split{split}"] = c.timed(steps)[0] * 1e3
        best = min(forced, key=forced.get)
        out.append({"M": M, "auto_us": auto_us, "auto_dispatch": auto, "best_forced": best,
                    "best_forced_us": forced[best], "auto_over_best": auto_us / forced[best], "forced_us": forced})
        del c
    torch.cuda.empty_cache()
    return out


def noalloc_measure(ql, torch, dev, flush, steps=10):
    """The allocation-free entry (CUDA-core split-K path, scratch inside the library) on the text projection."""
    w = S.WORKLOADS["text_proj"]
    out = []
    base = None
    for M in (1, 8, 32, 64):
        c = Case(ql, torch, w, M, 0, dev, flush, weights=base)
        base = (c.codes, c.sc, c.bi, c.codes_np, c.s_np, c.b_np)
        c.fwd = lambda x, cd, s, b, out, workspace, path, split_k: ql.forward_noalloc(x, cd, s, b, out=out)
        c.warm(2)
        st, _ = c.timed(steps)
        out.append({"M": M, "step_us": st * 1e3, "weight_GBps": w.weight_bytes / (st * 1e-3) / 1e9})
        del c
    assert ql.device_status() == 0, "the allocation-free entry reported an error"
    return out


def guarded(fn):
    """Run an extra measurement; an error is recorded in the line instead of costing it."""
    try:
        return fn()
    except Exception as exc:            # noqa: BLE001
        return {"error": f"{type(exc).__name__}: {exc}"[:200]}


def oracle_fit_rate(rows=4):
    """CPU oracle's importance-weighted fit on the first rows of the same weight: groups per second."""
    from oracle import qlinear_oracle as O
    w, imp = pack_inputs()
    t0 = time.perf_counter()
    O.pack_imatrix(w[:rows], imp.astype(np.float64))
    dt = time.perf_counter() - t0
    return rows * PACK_K // 64 / dt, f"{rows} rows of the same weight in {dt:.1f} s"


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
        (O.forward8_rows if w.bits == 8 else O.forward_rows)(x, codes, s, b, rows)
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
    rows_per_step = per[0][1]
    rate = sum(r[1] for r in per) * 2.0 * w.K * w.N / sum(r[2] for r in per) / 1e12
    ms = 1e3 * sum(r[2] for r in per) / len(per)          # measured wall time of one step (its row sample)
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": "TFLOP/s", "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name} M={M} K={w.K} N={w.N}", "seed": w.seed,
                   "sample": f"each step computes {rows_per_step} of the {M} rows (rows are independent), "
                             f"full K and N; ms_per_step is that step's measured time"},
        "cpu_baseline": {"value": rate, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows_per_step} of {M} rows per step (rows are independent), full N and K"},
        "e2e": {"value": rate, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- multi-rank reduction

def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings over the default process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(work_per_rank: float, slowest_ms: float, world: int) -> float:
    """Throughput of all ranks together: every rank does work_per_rank (weak scaling); the slowest sets the time."""
    return world * work_per_rank / (slowest_ms * 1e-3)


# ---------------------------------------------------------------------------- our arm

class Case:
    """Device-resident inputs of one workload and timed qlinear_forward steps on them."""

    def __init__(self, ql, torch, w, M, path, dev, flush, split=0, weights=None):
        import numpy as np
        self.ql, self.torch, self.w, self.M, self.path, self.flush = ql, torch, w, M, path, flush
        self.split, self.dev = split, dev
        self.K, self.N = w.K, w.N
        self.x_np = w.x(M)
        self.x = torch.from_numpy(self.x_np.view(np.int16)).view(torch.bfloat16).to(dev)
        if weights is None:
            self.codes_np, self.s_np, self.b_np = w.w()
            self.codes = torch.from_numpy(self.codes_np.view(np.int32)).to(dev)
            self.sc = torch.from_numpy(self.s_np).to(dev)
            self.bi = torch.from_numpy(self.b_np).to(dev)
        else:                       # device weights of the same workload from another case
            self.codes, self.sc, self.bi, self.codes_np, self.s_np, self.b_np = weights
        self.y = torch.empty((M, self.N), dtype=torch.bfloat16, device=dev)
        self.ws = None
        self.set_config(path, split)
        self.fwd = ql.forward8 if w.bits == 8 else ql.forward

    def set_config(self, path, split):
        self.path, self.split = path, split
        ws_bytes = self.ql.workspace_size(self.M, self.K, self.N, path, split, bits=self.w.bits)
        if self.ws is None or self.ws.numel() < ws_bytes:
            self.ws = None
            self.ws = self.torch.empty(max(ws_bytes, 16), dtype=self.torch.uint8, device=self.dev)

    def step(self):
        self.fwd(self.x, self.codes, self.sc, self.bi, out=self.y, workspace=self.ws, path=self.path,
                 split_k=self.split)

    def warm(self, n):
        for _ in range(n):
            self.flush.fill_(1)
            self.step()
        self.torch.cuda.synchronize()
        self.dispatch = self.ql.last_dispatch()
        self.launches = int(self.dispatch.split("launches=")[1].split()[0]) if "launches=" in self.dispatch else 1

    def timed_warm(self, steps):
        """Mean device time of back-to-back calls with no L2 flush between them (inputs may stay in L2)."""
        torch = self.torch
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        self.step()
        e0.record()
        for _ in range(steps):
            self.step()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    def timed(self, steps):
        """Per-step device time of the whole call and of its main kernel (L2 flushed before every step).

        Two passes: the whole call is timed with nothing recorded inside it (an event between two
        launches would serialise kernels that otherwise overlap under programmatic dependent
        launch); the main kernel is timed in a second pass by events the library records around it.
        """
        torch, ql = self.torch, self.ql
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        evm = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            self.flush.fill_(i & 0xFF)
            ev[i][0].record()
            self.step()
            ev[i][1].record()
        for e0, e1 in evm:            # create the handles so the library can record them
            e0.record()
            e1.record()
        for i in range(steps):
            self.flush.fill_(i & 0xFF)
            ql.set_profile_events(*evm[i])
            self.step()
        ql.set_profile_events(None, None)
        torch.cuda.synchronize()
        step_ms = [a.elapsed_time(b) for a, b in ev]
        main_ms = [a.elapsed_time(b) for a, b in evm]
        return sum(step_ms) / steps, sum(main_ms) / steps

    def timed_graph(self, steps):
        """Per-step device time of the same call replayed from a CUDA graph, L2 flushed before every step.

        A serving loop captures a decode-sized layer once and replays it: the kernels then start without
        the host launching each of them.  The capture records the call's launches (programmatic dependent
        launch edges included) with this case's buffers.
        """
        torch = self.torch
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.step()
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.step()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            self.flush.fill_(i & 0xFF)
            ev[i][0].record()
            g.replay()
            ev[i][1].record()
        torch.cuda.synchronize()
        ms = [e0.elapsed_time(e1) for e0, e1 in ev]
        del g
        return sum(ms) / steps

    def algorithmic_bytes(self):
        """Bytes a weight-streaming pass must move: packed W + x + y."""
        return self.w.weight_bytes * self.N // self.w.N + self.M * self.K * 2 + self.M * self.N * 2


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

    dev = torch.device("cuda", local)
    flush = L2Flush(torch, dev)
    w = S.WORKLOADS[a.workload]
    M = a.M or w.M
    K, N = w.K, w.N
    case = Case(ql, torch, w, M, a.path, dev, flush, a.split)
    case.warm(a.warmup)

    # ---- device-timed steps (inputs resident; L2 flushed between steps)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)                     # let the sampler start before the timed region
    barrier()
    mean_step, mean_main = case.timed(a.steps)
    barrier()
    clk = clocks.stop()
    assert ql.device_status() == 0, "a kernel reported an error"
    warm_ms = case.timed_warm(a.steps)     # context: the same call without the L2 flush

    # ---- end to end: every step copies its x from pinned host memory, runs the layer through the
    # public API and copies its y back to pinned host memory.  No L2 flush runs inside this loop: a
    # step's x, packed W and y together exceed the 126 MB L2 for the large-M workloads.  Steps are pipelined the way a serving
    # loop would run them: copies in, compute and copies out on three streams, with device x and y
    # double-buffered, so a step's copies overlap its neighbours' work (PCIe is full duplex).  The
    # per-step figure is the device time of the whole loop divided by the number of steps.
    x_host = torch.from_numpy(case.x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    xb = [case.x, torch.empty_like(case.x)]
    yb = [case.y, torch.empty_like(case.y)]
    s_c = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done = [ev() for _ in range(a.steps)]
    comp_done = [ev() for _ in range(a.steps)]
    out_done = [ev() for _ in range(a.steps)]
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    t_begin.record(s_c)
    s_in.wait_event(t_begin)
    s_out.wait_event(t_begin)
    for i in range(a.steps):
        b = i & 1
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[i - 2])       # step i-2's forward has read this x buffer
            xb[b].copy_(x_host, non_blocking=True)
            in_done[i].record(s_in)
        s_c.wait_event(in_done[i])
        if i >= 2:
            s_c.wait_event(out_done[i - 2])             # step i-2's y buffer has been copied out
        case.fwd(xb[b], case.codes, case.sc, case.bi, out=yb[b], workspace=case.ws, path=case.path,
                 split_k=case.split)
        comp_done[i].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[i])
            y_host.copy_(yb[b], non_blocking=True)
            out_done[i].record(s_out)
    s_c.wait_event(out_done[a.steps - 1])
    t_end.record(s_c)
    barrier()
    mean_e2e = t_begin.elapsed_time(t_end) / a.steps

    # ---- the small-M half of the metric: weight streaming on the 53248 -> 4608 text projection
    dirty = L2Flush(torch, dev, dirty=True)

    def small_m(name):
        out = []
        tp = S.WORKLOADS[name]
        for Ms in (1, 8, 32):
            c = Case(ql, torch, tp, Ms, 0, dev, flush)
            c.warm(3)
            st, mn = c.timed(max(10, a.steps))
            sg = c.timed_graph(max(10, a.steps))
            c.flush = dirty
            st_d, _ = c.timed(max(10, a.steps))
            out.append({"M": Ms, "dispatch": c.dispatch, "step_us": st * 1e3, "kernel_us": mn * 1e3,
                        "weight_GBps": tp.weight_bytes / (st * 1e-3) / 1e9,
                        "algorithmic_GBps": c.algorithmic_bytes() / (st * 1e-3) / 1e9,
                        "graph_step_us": sg * 1e3, "graph_weight_GBps": tp.weight_bytes / (sg * 1e-3) / 1e9,
                        "step_us_dirty_l2": st_d * 1e3,
                        "traffic": recorded_traffic(c.dispatch.split()[0], f"{name}:M={Ms}")})
            del c
        torch.cuda.synchronize()
        return out

    small = [] if a.no_small_m else small_m("text_proj")
    small_w8 = [] if a.no_w8 else small_m("text_proj_w8")

    # ---- the quantizer: importance-weighted fit and RTN pack of a DiT-shaped weight
    pack = None if a.no_pack else pack_measure(ql, torch, dev, flush)
    large = guarded(lambda: large_m_measure(ql, torch, dev, flush, peaks()[0])) if world == 1 and not a.no_large else None
    disp = guarded(lambda: dispatch_measure(ql, torch, dev, flush)) if world == 1 and not a.no_dispatch else None
    noalloc = guarded(lambda: noalloc_measure(ql, torch, dev, flush)) if world == 1 and not a.no_noalloc else None
    # Extras, one GPU only (their errors are recorded, never raised; with several ranks every rank would
    # have to take the same collective steps afterwards).
    single = world == 1
    swiglu = guarded(lambda: swiglu_measure(ql, torch, dev, flush, peaks()[0])) if single and not a.no_swiglu else None
    split = guarded(lambda: split_measure(ql, torch, dev, flush, peaks()[0])) if single and not a.no_split else None
    comp = guarded(lambda: comparators(ql, torch, dev, flush)) if single and not a.no_comparators else None

    mean_step, mean_main, mean_e2e, warm_ms = max_over_ranks([mean_step, mean_main, mean_e2e, warm_ms], dev)

    flops = 2.0 * M * K * N
    value = whole_job_rate(flops, mean_step, world) / 1e12
    e2e_value = whole_job_rate(flops, mean_e2e, world) / 1e12
    peak_tf, peak_gbs, peak_kind = peaks()
    dispatch = case.dispatch
    kernel = dispatch.split()[0].replace("path=", "")
    traffic = recorded_traffic(dispatch.split()[0], f"{w.name}:M={M}")
    if kernel == "tc_fused":
        main_rate = flops / (mean_main * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": main_rate, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": main_rate / peak_tf, "traffic": traffic, "kernel": "fused_gemm_kernel",
                "kernel_ms": mean_main,
                "peak_kind": f"{peak_kind} bf16 dense burst (f16 has the same tcgen05 rate)",
                "algorithmic": "2*M*N*K FLOPs per launch"}
    else:
        main_rate = case.algorithmic_bytes() / (mean_main * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": main_rate, "peak": peak_gbs, "unit": "GB/s",
                "frac": main_rate / peak_gbs, "traffic": traffic, "kernel": kernel, "kernel_ms": mean_main,
                "peak_kind": f"{peak_kind} HBM copy bandwidth",
                "algorithmic": f"packed W ({w.bits / 8 + 0.0625:g} B/weight) + x + y bytes per launch"}
    for sm in small + small_w8:
        sm["frac_hbm_weight"] = sm["weight_GBps"] / peak_gbs
        sm["frac_hbm_weight_spec"] = sm["weight_GBps"] / SPEC_GBPS
    roof["spec_peak"] = SPEC_TFLOPS if roof["bound"] == "tensor" else SPEC_GBPS
    roof["frac_of_spec"] = roof["achieved"] / roof["spec_peak"]

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": mean_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 MMA, fp32 accumulate (bf16 in/out)", "data": "synthetic",
        "config": {"workload": f"{w.name} M={M} K={K} N={N}", "seed": w.seed,
                   "inputs_sha256": S.digest(case.x_np, case.codes_np, case.s_np, case.b_np),
                   "l2": L2_NOTE, "parallelism": f"replicas x{world}",
                   "dispatch": dispatch, "weight_GBps": w.weight_bytes / (mean_step * 1e-3) / 1e9,
                   "l2_warm": {"ms_per_step": warm_ms, "value": whole_job_rate(flops, warm_ms, world) / 1e12,
                               "note": "same call back to back, no flush between steps (context)"}},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
                "l2": "no flush inside the loop; per-step x + packed W + y bytes: "
                      f"{(M * K * 2 + w.weight_bytes + M * N * 2) / 1e6:.1f} MB"},
        "gpu_launches": case.launches * a.steps,
        "clocks": clk,
        "small_m": small,
    }
    if small_w8:
        line["small_m_w8"] = small_w8
    if swiglu is not None:
        line["swiglu"] = swiglu
    if split is not None:
        line["split_m512"] = split
    if comp is not None:
        line["comparators"] = comp
    if pack is not None:
        line["pack"] = pack
    if large is not None:
        line["large_m"] = large
    if disp is not None:
        line["dispatch"] = disp
    if noalloc is not None:
        line["noalloc"] = noalloc
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        rate, cores, rows, dt = oracle_rate(w, M, a.cpu_seconds, case.x_np[: min(M, 512)],
                                            (case.codes_np, case.s_np, case.b_np))
        line["cpu_baseline"] = {"value": rate, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": f"{rows} rows x full K x full N of {w.name} in {dt:.1f} s"}
        if pack is not None:
            pack["oracle_fit_groups_per_s"], pack["oracle_fit_sample"] = oracle_fit_rate()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
