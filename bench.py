#!/usr/bin/env python
"""Benchmark of the IF4 hot path on B200.

One step = one pass of the whole quantization path over one tensor that is
already resident in HBM:
    tensor amax (A1) -> tensor scale (A2) -> IF4 quantize (A3-A6)
    -> IF4 dequantize to bf16 (A7) -> NVFP4 quantize with the same scale (A9)
Default workload: the LLM weight matrix, bf16 4096 x 4096, Student-t(3)
scaled to std 0.02, groups of 16 along K.  The IF4 x IF4 linear has its own
workload and is reported under "linear" when its entry point is built.

value = elements / step time (Gelem/s), max over ranks; with N GPUs every
rank quantizes its own tensor (independent problems, weak scaling, no data
collective).  L2: the step rotates over buffer sets whose total exceeds twice
the 126 MB L2, so no step reads what the previous one left in L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "IF4 quantize Gelem/s & HBM GB/s vs ~8 TB/s peak (1 B200); MSE vs NVFP4"
UNIT = "Gelem/s"
WORKLOAD = "weight_bf16_4096x4096"
L2_BYTES = 126e6


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=WORKLOAD)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--no-linear", action="store_true")
    p.add_argument("--kernel-only", default=None,
                   choices=["amax", "if4_quantize", "if4_dequantize", "nvfp4_quantize", "gemm"],
                   help="launch only this kernel, warmup+steps times (for ncu captures)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def make_input(name, seed=0):
    from adaptive_block_scaled_b200 import workloads
    w = workloads.WORKLOADS[name]
    return w.make(seed)


# ------------------------------------------------------------- clocks ----

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while it runs,
    read through a pipe by a thread."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def _drain(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._drain, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self):
        rows = []
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), max=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if "Active" in r[key] and "Not" not in r[key]:
                    reasons.add(name)
        busy = [r["sm"] for r in rows if r["power"] > 250.0] or [r["sm"] for r in rows]
        return {"sm_mhz": statistics.median(busy),
                "sm_max_mhz": max(r["max"] for r in rows),
                "samples": len(rows), "samples_under_load": len(busy),
                "power_w_max": max(r["power"] for r in rows),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------- distributed --

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local) if args.impl == "ours" else None
        backend = "nccl" if args.impl == "ours" else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(value, world):
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64,
                     device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------- CPU oracle --

def cpu_oracle_step(x_np):
    import oracle
    q = oracle.quantize_tensor(x_np)
    oracle.dequantize(q["codes"], q["scales"], q["ts"])
    n = oracle.quantize(x_np, q["ts"], mode=oracle.MODE_NVFP4)
    return q, n


def cpu_baseline(x_cpu, seconds):
    """The oracle as it stands (C, OpenMP over rows, all host cores) on a
    bounded row sample of the same workload; elements/s of the whole step."""
    import oracle
    x_np = x_cpu.float().numpy()
    rows = x_np.shape[0]
    sample_rows = max(1, min(rows, 256))
    t0 = time.perf_counter()
    cpu_oracle_step(x_np[:sample_rows])
    dt = time.perf_counter() - t0
    per_row = dt / sample_rows
    sample_rows = int(max(1, min(rows, seconds / max(per_row, 1e-9))))
    sample = np.ascontiguousarray(x_np[:sample_rows])
    reps, elapsed, near = 0, 0.0, 0
    while elapsed < seconds or reps == 0:
        t0 = time.perf_counter()
        q, _ = cpu_oracle_step(sample)
        elapsed += time.perf_counter() - t0
        reps += 1
        near = int(q["near"].sum())
        if reps >= 50:
            break
    elems = sample.size * reps
    return {"value": elems / elapsed / 1e9, "unit": UNIT, "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": f"first {sample_rows} of {rows} rows of {WORKLOAD}, {reps} passes of "
                      f"amax+scale+IF4 quantize+dequantize+NVFP4 quantize ({elapsed:.1f} s)",
            "near_ties_in_sample": near}


def run_reference(args):
    rank, world, _ = dist_setup(args)
    if rank != 0:
        return
    import oracle
    x = make_input(args.workload)
    x_np = x.float().numpy()
    rows = x_np.shape[0]
    probe = np.ascontiguousarray(x_np[:128])
    t0 = time.perf_counter()
    cpu_oracle_step(probe)
    per_row = (time.perf_counter() - t0) / 128
    budget = 150.0 / max(1, args.steps + args.warmup)
    sample_rows = int(max(16, min(rows, budget / max(per_row, 1e-9))))
    sample = np.ascontiguousarray(x_np[:sample_rows])
    for _ in range(args.warmup):
        cpu_oracle_step(sample)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        cpu_oracle_step(sample)
        times.append(time.perf_counter() - t0)
    step = sum(times) / len(times)
    value = sample.size / step / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": args.workload, "rows_sampled": sample_rows,
                       "cols": int(x_np.shape[1]), "l2": "host CPU"},
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle",
                             "cores": oracle.max_threads(),
                             "sample": f"first {sample_rows} rows of {args.workload} per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------- our kernels --

class Step:
    """Buffers and launches of one pass of the path; R rotating sets."""

    def __init__(self, x_cpu, sets):
        from adaptive_block_scaled_b200 import binding as b
        self.b = b
        self.rows, self.cols = x_cpu.shape
        dev = torch.device("cuda")
        self.sets = []
        for _ in range(sets):
            s = dict(
                x=x_cpu.to(dev),
                amax=torch.empty(1, dtype=torch.float32, device=dev),
                ts=torch.empty(1, dtype=torch.float32, device=dev),
                codes=torch.empty((self.rows, self.cols // 2), dtype=torch.uint8, device=dev),
                scales=torch.empty((self.rows, self.cols // 16), dtype=torch.uint8, device=dev),
                y=torch.empty((self.rows, self.cols), dtype=torch.bfloat16, device=dev),
                ncodes=torch.empty((self.rows, self.cols // 2), dtype=torch.uint8, device=dev),
                nscales=torch.empty((self.rows, self.cols // 16), dtype=torch.uint8, device=dev),
            )
            self.sets.append(s)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.kernels = ["amax", "scale", "if4_quantize", "if4_dequantize", "nvfp4_quantize"]
        self.launches_per_step = 5

    def bytes_per_set(self):
        s = self.sets[0]
        return sum(t.numel() * t.element_size() for t in s.values())

    def run(self, i, events=None):
        b, s = self.b, self.sets[i % len(self.sets)]
        ev = events if events is not None else [None] * 6
        if ev[0] is not None:
            ev[0].record()
        b.if4_tensor_amax(s["x"], s["amax"], self.err)
        if ev[1] is not None:
            ev[1].record()
        b.if4_tensor_scale(s["amax"], s["ts"])
        if ev[2] is not None:
            ev[2].record()
        b.if4_quantize(s["x"], s["codes"], s["scales"], s["ts"], b.TS_GIVEN, self.err)
        if ev[3] is not None:
            ev[3].record()
        b.if4_dequantize(s["codes"], s["scales"], s["ts"], s["y"])
        if ev[4] is not None:
            ev[4].record()
        b.nvfp4_quantize(s["x"], s["ncodes"], s["nscales"], s["ts"], b.TS_GIVEN, self.err)
        if ev[5] is not None:
            ev[5].record()


def measure_e2e(x_cpu, steps, warmup):
    """Same step through the C ABI from pinned host memory: H2D of the input,
    the five kernels, D2H of every result (IF4 codes, scales, scale, bf16
    dequantized tensor, NVFP4 codes and scales), inside the timed region."""
    from adaptive_block_scaled_b200 import binding as b
    rows, cols = x_cpu.shape
    dev = torch.device("cuda")
    h_x = x_cpu.contiguous().pin_memory()
    outs = dict(codes=((rows, cols // 2), torch.uint8), scales=((rows, cols // 16), torch.uint8),
                ts=((1,), torch.float32), y=((rows, cols), torch.bfloat16),
                ncodes=((rows, cols // 2), torch.uint8), nscales=((rows, cols // 16), torch.uint8))
    d = {k: torch.empty(sh, dtype=dt, device=dev) for k, (sh, dt) in outs.items()}
    h = {k: torch.empty(sh, dtype=dt, pin_memory=True) for k, (sh, dt) in outs.items()}
    d_x = torch.empty_like(h_x, device=dev)
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def step():
        d_x.copy_(h_x, non_blocking=True)
        b.if4_tensor_amax(d_x, amax, err)
        b.if4_tensor_scale(amax, d["ts"])
        b.if4_quantize(d_x, d["codes"], d["scales"], d["ts"], b.TS_GIVEN, err)
        b.if4_dequantize(d["codes"], d["scales"], d["ts"], d["y"])
        b.nvfp4_quantize(d_x, d["ncodes"], d["nscales"], d["ts"], b.TS_GIVEN, err)
        for k in h:
            h[k].copy_(d[k], non_blocking=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = h_x.numel() * h_x.element_size()
    d2h = sum(t.numel() * t.element_size() for t in h.values())
    return {"value": rows * cols / (ms * 1e-3) / 1e9, "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


def quality_report(x_cpu, step):
    """MSE of IF4 and NVFP4 against the input (x domain, float64 on the host)
    from the GPU outputs of set 0, and the INT4 group fraction."""
    from adaptive_block_scaled_b200 import binding as b
    s = step.sets[0]
    y_if4 = s["y"].float().cpu().numpy().astype(np.float64)
    y_nv = b.dequantize(s["ncodes"], s["nscales"], s["ts"], dtype=torch.float32).cpu().numpy()
    x = x_cpu.float().numpy().astype(np.float64)
    mse_if4 = float(np.mean((x - y_if4) ** 2))
    mse_nv = float(np.mean((x - y_nv.astype(np.float64)) ** 2))
    sc = s["scales"].cpu().numpy()
    return {"mse_if4": mse_if4, "mse_nvfp4": mse_nv,
            "mse_reduction_pct": 100.0 * (1.0 - mse_if4 / mse_nv) if mse_nv > 0 else 0.0,
            "int4_group_fraction": float(np.mean(sc >> 7)),
            "note": "IF4 MSE measured on the bf16 dequantized output; NVFP4 on fp32 dequant"}


def linear_report(pk, steps=20, warmup=3):
    """IF4 x IF4 linear on its own workload (A 8192x4096 activations, B
    4096x4096 weights, both IF4 along K): decode A, decode B, tcgen05 GEMM,
    each timed with CUDA events; cuBLAS fp16 on the same decoded operands is
    timed beside it for context.  Inputs stay resident; the operands (100 MB
    of fp16 after decode) are re-read from HBM/L2 every launch."""
    from adaptive_block_scaled_b200 import binding as b
    M, N, K = 8192, 4096, 4096
    a, bw = make_input("linear_8192x4096x4096")
    dev = torch.device("cuda")
    aq = b.quantize(a.to(dev))
    bq = b.quantize(bw.to(dev))
    ws = torch.empty(b.if4_linear_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
    wa = ws[: M * K * 2].view(torch.float16).view(M, K)
    off = ((M * K * 2 + 255) // 256) * 256
    wb = ws[off: off + N * K * 2].view(torch.float16).view(N, K)
    c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def run(ev=None):
        if ev: ev[0].record()
        b.if4_decode_f16(aq[0], aq[1], wa)
        if ev: ev[1].record()
        b.if4_decode_f16(bq[0], bq[1], wb)
        if ev: ev[2].record()
        b.if4_gemm_f16(wa, wb, aq[2], bq[2], c, err)
        if ev: ev[3].record()

    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        run(evs[i])
    torch.cuda.synchronize()
    t = [sum(e[k].elapsed_time(e[k + 1]) for e in evs) / steps for k in range(3)]
    ref = torch.empty((M, N), dtype=torch.float16, device=dev)
    for _ in range(warmup):
        torch.matmul(wa, wb.t(), out=ref)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps):
        torch.matmul(wa, wb.t(), out=ref)
    e1.record()
    torch.cuda.synchronize()
    t_cublas = e0.elapsed_time(e1) / steps
    flops = 2.0 * M * N * K
    gemm_tf = flops / (t[2] * 1e-3) / 1e12
    total = sum(t)
    return {"workload": "linear_8192x4096x4096", "err": int(err.item()),
            "decode_a_ms": t[0], "decode_b_ms": t[1], "gemm_ms": t[2], "linear_ms": total,
            "gemm_tflops": gemm_tf, "linear_tflops": flops / (total * 1e-3) / 1e12,
            "cublas_f16_ms": t_cublas, "cublas_f16_tflops": flops / (t_cublas * 1e-3) / 1e12,
            "roofline": {"bound": "tensor", "achieved": gemm_tf, "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": gemm_tf / pk["bf16_tflops"],
                         "peak_source": f"{pk['source']} bf16_tflops (burst); fp16 dense rate = bf16"}}


def run_ours(args):
    rank, world, local = dist_setup(args)
    torch.cuda.set_device(local)
    pk = peaks()
    x_cpu = make_input(args.workload, seed=rank)
    n_elem = x_cpu.numel()
    in_bytes = n_elem * x_cpu.element_size()

    step = Step(x_cpu, sets=1)
    per_set = step.bytes_per_set()
    sets = max(2, int(np.ceil(2 * L2_BYTES / per_set)) + 1)
    step = Step(x_cpu, sets=sets)

    for i in range(args.warmup):
        step.run(i)
    torch.cuda.synchronize()
    if int(step.err.item()) != 0:
        raise RuntimeError(f"device error flag {int(step.err.item())} during warm-up")

    n_ev = 6
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record()
        for i in range(args.steps):
            step.run(args.warmup + i, events[i])
        stop.record()
        torch.cuda.synchronize()
    barrier(world)
    ms_local = start.elapsed_time(stop) / args.steps
    ms = max_over_ranks(ms_local, world)
    kern_ms = {}
    for k, name in enumerate(step.kernels):
        kern_ms[name] = sum(events[i][k].elapsed_time(events[i][k + 1]) for i in range(args.steps)) / args.steps

    value = world * n_elem / (ms * 1e-3) / 1e9
    q_bytes = in_bytes + n_elem // 2 + n_elem // 16
    kernels = {
        "amax": {"ms": kern_ms["amax"], "bytes": in_bytes},
        "scale": {"ms": kern_ms["scale"], "bytes": 8},
        "if4_quantize": {"ms": kern_ms["if4_quantize"], "bytes": q_bytes},
        "if4_dequantize": {"ms": kern_ms["if4_dequantize"], "bytes": n_elem // 2 + n_elem // 16 + 2 * n_elem},
        "nvfp4_quantize": {"ms": kern_ms["nvfp4_quantize"], "bytes": q_bytes},
    }
    for k, v in kernels.items():
        v["gbs"] = v["bytes"] / (v["ms"] * 1e-3) / 1e9
        v["frac_of_measured_hbm"] = v["gbs"] / pk["hbm_gbs"]
        v["frac_of_8tbs"] = v["gbs"] / 8000.0
    kernels["if4_quantize"]["gelems"] = n_elem / (kern_ms["if4_quantize"] * 1e-3) / 1e9

    top = kernels["if4_quantize"]
    roofline = {"bound": "hbm", "kernel": "if4_quantize (A3-A6, ts given)",
                "achieved": top["gbs"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": top["gbs"] / pk["hbm_gbs"],
                "peak_source": f"{pk['source']} hbm_gbs (copy bandwidth, read+write)",
                "algorithmic_bytes_per_launch": q_bytes,
                "traffic": None}
    traffic_file = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(traffic_file):
        tr = json.load(open(traffic_file)).get(args.workload, {}).get("if4_quantize")
        if tr:
            roofline["traffic"] = tr

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": args.workload, "rows": int(x_cpu.shape[0]),
                       "cols": int(x_cpu.shape[1]), "input_dtype": str(x_cpu.dtype).replace("torch.", ""),
                       "group": 16, "parallelism": f"independent tensors x{world}",
                       "l2": f"rotating {sets} buffer sets, {sets * per_set / 1e6:.0f} MB > 2x126 MB L2",
                       "step": "amax, scale, IF4 quantize, IF4 dequantize (bf16), NVFP4 quantize"},
            "gpu_launches": step.launches_per_step * args.steps,
            "kernels": kernels, "roofline": roofline}
    if rank == 0:
        line["clocks"] = clk.summary()
        line["quality"] = quality_report(x_cpu, step)
        line["e2e"] = measure_e2e(x_cpu, max(5, args.steps // 5), 2)
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(x_cpu, args.cpu_seconds)
        if not args.no_linear and hasattr(step.b.lib, "if4_linear"):
            line["linear"] = linear_report(pk)
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_kernel_only(args):
    """Only the chosen kernel, on the chosen workload: the command ncu wraps."""
    from adaptive_block_scaled_b200 import binding as b
    if args.kernel_only == "gemm":
        M, N, K = 8192, 4096, 4096
        a, bw = make_input("linear_8192x4096x4096")
        dev = torch.device("cuda")
        aq, bq = b.quantize(a.to(dev)), b.quantize(bw.to(dev))
        wa, wb = b.decode_f16(aq[0], aq[1]), b.decode_f16(bq[0], bq[1])
        c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        for _ in range(args.warmup + args.steps):
            b.if4_gemm_f16(wa, wb, aq[2], bq[2], c, err)
        torch.cuda.synchronize()
        print(json.dumps({"kernel_only": "gemm", "launches": args.warmup + args.steps,
                          "err": int(err.item())}))
        return
    x_cpu = make_input(args.workload)
    step = Step(x_cpu, sets=1)
    s = step.sets[0]
    b.if4_tensor_amax(s["x"], s["amax"], step.err)
    b.if4_tensor_scale(s["amax"], s["ts"])
    b.if4_quantize(s["x"], s["codes"], s["scales"], s["ts"], b.TS_GIVEN, step.err)
    torch.cuda.synchronize()
    calls = {
        "amax": lambda: b.if4_tensor_amax(s["x"], s["amax"], step.err),
        "if4_quantize": lambda: b.if4_quantize(s["x"], s["codes"], s["scales"], s["ts"],
                                               b.TS_GIVEN, step.err),
        "if4_dequantize": lambda: b.if4_dequantize(s["codes"], s["scales"], s["ts"], s["y"]),
        "nvfp4_quantize": lambda: b.nvfp4_quantize(s["x"], s["ncodes"], s["nscales"], s["ts"],
                                                   b.TS_GIVEN, step.err),
    }
    for _ in range(args.warmup + args.steps):
        calls[args.kernel_only]()
    torch.cuda.synchronize()
    print(json.dumps({"kernel_only": args.kernel_only, "workload": args.workload,
                      "launches": args.warmup + args.steps, "err": int(step.err.item())}))


def main():
    args = parse()
    if args.kernel_only:
        run_kernel_only(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
