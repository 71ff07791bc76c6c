#!/usr/bin/env python
"""Benchmark of the IF4 hot path on B200.

One step = one pass of the whole quantization path over one tensor that is
already resident in HBM, as one launch (if4_quantize_fused_dequant):
    tensor amax -> tensor scale -> IF4 quantize (block scale, FP4 and INT4
    candidates, choice) and NVFP4 quantize with the same tensor scale ->
    the IF4 codes dequantized to bf16
The same step as two launches (single-launch quantizer, then the
dequantizer) and as five is timed beside it.  Default workload: the
activation tensor, bf16 8192 tokens x 8192 hidden, N(0, 1) with 1 % of the
channels (fixed by the seed) scaled by 20, groups of 16 along the hidden
dimension: the largest of the quantizer workloads (67 M elements, with the
gradient tensor) and the one whose outlier groups put the most groups near
an FP4/INT4 tie.  The other quantizer workloads (the 256 x 1024 float32
tensor, the 4096 x 4096 weight, the 16384 x 4096 Hadamard-transformed
gradient) get their own kernel tables and, like the headline, a parity and
quality block: every group's codes and scale byte against the CPU oracle
(mismatches counted), the oracle's near ties counted, and the MSE of IF4 and
its comparators.  The IF4 x IF4 linear has its own workload and is reported
under "linear".

value = elements / step time (Gelem/s), max over ranks; with N GPUs every
rank quantizes its own tensor (independent problems, weak scaling, no data
collective).  L2: the step rotates over buffer sets whose inputs total more
than three times the 126 MB L2, so no step reads what the previous one left
in L2.

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
WORKLOAD = "activation_bf16_8192x8192"
# the quantizer workloads: each gets a parity and quality block
QUANT_WORKLOADS = ("small_fp32_256x1024", "weight_bf16_4096x4096", "activation_bf16_8192x8192",
                   "gradient_bf16_16384x4096")
L2_BYTES = 126e6
RHT_SIGNS = 0x6A3C          # one fixed random-sign vector for the transform


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
    p.add_argument("--no-large", action="store_true",
                   help="skip the per-kernel tables of the other quantizer workloads")
    p.add_argument("--no-quality", action="store_true",
                   help="skip the per-workload parity and quality block")
    p.add_argument("--kernel-only", default=None,
                   choices=["amax", "if4_quantize", "if4_dequantize", "nvfp4_quantize", "gemm",
                            "linear_fused", "linear_quantized",
                            "nvint4_quantize", "nvfp4_4over6_quantize", "if4_quantize_rht",
                            "if4_decode_f16", "fused_quantize", "fused_quantize_rht",
                            "fused_quantize_dequant", "if6_quantize", "if3_quantize",
                            "if6_dequantize", "if3_dequantize"],
                   help="launch only this kernel, warmup+steps times (for ncu captures)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def b_lib():
    from adaptive_block_scaled_b200 import binding
    return binding.lib


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

def cpu_oracle_step(x_np, threads=0):
    """One step of the path on the oracle: tensor amax and scale, IF4
    quantize, dequantize, NVFP4 quantize with the same tensor scale.
    threads = 0: every host core (OpenMP over rows)."""
    import oracle
    q = oracle.quantize_tensor(x_np, threads=threads)
    oracle.dequantize(q["codes"], q["scales"], q["ts"], threads=threads)
    n = oracle.quantize(x_np, q["ts"], mode=oracle.MODE_NVFP4, threads=threads)
    return q, n


def oracle_rate(x_np, seconds, threads):
    """Elements/s of the oracle's step on the first rows of x_np, as many
    rows as take about `seconds` (sized by a probe of 64 rows)."""
    rows = x_np.shape[0]
    probe = np.ascontiguousarray(x_np[:min(rows, 64)])
    t0 = time.perf_counter()
    cpu_oracle_step(probe, threads)
    per_row = (time.perf_counter() - t0) / probe.shape[0]
    sample_rows = int(max(1, min(rows, seconds / max(per_row, 1e-9))))
    sample = np.ascontiguousarray(x_np[:sample_rows])
    t0 = time.perf_counter()
    q, _ = cpu_oracle_step(sample, threads)
    dt = time.perf_counter() - t0
    return sample.size / dt / 1e9, sample_rows, dt, int(q["near"].sum())


def cpu_baseline(x_cpu, seconds, workload):
    """The oracle as it stands (C, OpenMP over rows) timed on a bounded row
    sample of the same workload, on every host core and on one core;
    elements/s of the whole step."""
    import oracle
    x_np = x_cpu.float().numpy()
    rows = x_np.shape[0]
    cores = oracle.max_threads()
    v_all, r_all, t_all, near = oracle_rate(x_np, seconds, 0)
    v_one, r_one, t_one, _ = oracle_rate(x_np, seconds, 1)
    what = "amax+scale+IF4 quantize+dequantize+NVFP4 quantize"
    return {"value": v_all, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"first {r_all} of {rows} rows of {workload}, one pass of {what} "
                      f"({t_all:.1f} s, {cores} threads)",
            "near_ties_in_sample": near,
            "one_core": {"value": v_one, "unit": UNIT, "cores": 1,
                         "sample": f"first {r_one} of {rows} rows of {workload}, one pass of "
                                   f"{what} ({t_one:.1f} s, 1 thread)"}}


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
    sample_desc = (f"first {sample_rows} of {rows} rows of {args.workload} per step "
                   f"(amax+scale+IF4 quantize+dequantize+NVFP4 quantize)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": bench_config(args.workload, x, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle",
                             "cores": oracle.max_threads(), "sample": sample_desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def bench_config(workload, x_cpu, world):
    """The `config` object of the JSON line; the same for both arms."""
    rows, cols = x_cpu.shape
    return {"workload": workload, "rows": int(rows), "cols": int(cols),
            "input_dtype": str(x_cpu.dtype).replace("torch.", ""), "group": 16,
            "parallelism": f"independent tensors x{world}",
            "l2": "inputs larger than L2: rotating buffer sets whose inputs total more than "
                  "3x the 126 MB L2",
            "step": "amax, scale, IF4 quantize, NVFP4 quantize and the IF4 round trip "
                    "(codes decoded to bf16)"}


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
                sync=torch.zeros(64, dtype=torch.int32, device=dev),
                ts_rht=torch.empty(1, dtype=torch.float32, device=dev),
                codes6=torch.empty((self.rows, self.cols * 6 // 8), dtype=torch.uint8, device=dev),
                codes3=torch.empty((self.rows, self.cols * 3 // 8), dtype=torch.uint8, device=dev),
                scales6=torch.empty((self.rows, self.cols // 16), dtype=torch.uint8, device=dev),
                scales3=torch.empty((self.rows, self.cols // 16), dtype=torch.uint8, device=dev),
                ts6=torch.empty(1, dtype=torch.float32, device=dev),
                ts3=torch.empty(1, dtype=torch.float32, device=dev),
            )
            self.sets.append(s)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.kernels = ["fused_quantize_dequant", "fused_quantize", "amax", "scale",
                        "if4_quantize", "if4_dequantize", "nvfp4_quantize"]
        self.launches_per_step = 1

    def init_widths(self):
        """IF6 / IF3 tensor scales, codes and scales of every set (computed
        once; their timed quantizers then take the tensor scale as given)."""
        b = self.b
        for s in self.sets:
            for bits in (6, 3):
                b.ifw_quantize(s["x"], bits, b.W_ADAPTIVE, s["codes%d" % bits],
                               s["scales%d" % bits], s["ts%d" % bits], b.TS_COMPUTE, self.err)

    def bytes_per_set(self):
        s = self.sets[0]
        return sum(t.numel() * t.element_size() for t in s.values())

    EXTRA = ["nvint4_quantize", "nvfp4_4over6_quantize", "if4_quantize_rht", "if4_decode_f16",
             "fused_quantize_rht", "if6_quantize", "if6_dequantize", "if3_quantize",
             "if3_dequantize"]

    def run_one(self, name, i):
        b, s = self.b, self.sets[i % len(self.sets)]
        if name == "nvint4_quantize":
            b.nvint4_quantize(s["x"], s["ncodes"], s["nscales"], s["ts"], b.TS_GIVEN, self.err)
            return
        if name == "nvfp4_4over6_quantize":
            b.nvfp4_4over6_quantize(s["x"], s["ncodes"], s["nscales"], s["ts"], b.TS_GIVEN, self.err)
            return
        if name == "if4_quantize_rht":
            b.if4_quantize_rht(s["x"], RHT_SIGNS, s["ncodes"], s["nscales"], s["ts"], b.TS_GIVEN,
                               self.err)
            return
        if name == "fused_quantize_rht":
            # its own tensor scale: the transformed tensor's must not replace
            # the one the step and the quality report use
            b.if4_quantize_fused(s["x"], s["codes"], s["scales"], s["ncodes"], s["nscales"],
                                 s["ts_rht"], s["sync"], self.err, signs=RHT_SIGNS)
            return
        if name in ("if6_quantize", "if3_quantize"):
            bits = 6 if name == "if6_quantize" else 3
            # the width's own tensor scale, computed once before timing
            b.ifw_quantize(s["x"], bits, b.W_ADAPTIVE, s["codes%d" % bits], s["scales%d" % bits],
                           s["ts%d" % bits], b.TS_GIVEN, self.err)
            return
        if name in ("if6_dequantize", "if3_dequantize"):
            bits = 6 if name == "if6_dequantize" else 3
            b.ifw_dequantize(s["codes%d" % bits], s["scales%d" % bits], s["ts%d" % bits], bits,
                             s["y"])
            return
        if name == "if4_decode_f16":
            b.if4_decode_f16(s["codes"], s["scales"], s["y"].view(torch.float16))
            return
        if name == "fused_quantize_dequant":
            b.if4_quantize_fused_dequant(s["x"], s["codes"], s["scales"], s["ncodes"],
                                         s["nscales"], s["ts"], s["sync"], s["y"], self.err)
            return
        if name == "fused_quantize":
            b.if4_quantize_fused(s["x"], s["codes"], s["scales"], s["ncodes"], s["nscales"],
                                 s["ts"], s["sync"], self.err)
        elif name == "amax":
            b.if4_tensor_amax(s["x"], s["amax"], self.err)
        elif name == "scale":
            b.if4_tensor_scale(s["amax"], s["ts"])
        elif name == "if4_quantize":
            b.if4_quantize(s["x"], s["codes"], s["scales"], s["ts"], b.TS_GIVEN, self.err)
        elif name == "if4_dequantize":
            b.if4_dequantize(s["codes"], s["scales"], s["ts"], s["y"])
        elif name == "nvfp4_quantize":
            b.nvfp4_quantize(s["x"], s["ncodes"], s["nscales"], s["ts"], b.TS_GIVEN, self.err)
        else:
            raise ValueError(name)

    def run(self, i, events=None):
        """One step on buffer set i, one launch: tensor amax, tensor scale,
        IF4 codes, the NVFP4 comparator and the IF4 round trip (the codes
        decoded to bf16 in the same launch).  events: optional pair recorded
        right before and right after the launch."""
        b, s = self.b, self.sets[i % len(self.sets)]
        if events is not None:
            events[0].record()
        b.if4_quantize_fused_dequant(s["x"], s["codes"], s["scales"], s["ncodes"], s["nscales"],
                                     s["ts"], s["sync"], s["y"], self.err)
        if events is not None:
            events[1].record()

    def run_two_streams(self, n, streams):
        """n steps with the shared single launch (share 2): consecutive steps
        on alternating streams, each on its own buffer set, so one step's
        amax pass runs beside the other's encode pass; the current stream
        forks to both and joins them."""
        b = self.b
        cur = torch.cuda.current_stream()
        for st in streams:
            st.wait_stream(cur)
        for i in range(n):
            s = self.sets[i % len(self.sets)]
            with torch.cuda.stream(streams[i % 2]):
                b.if4_quantize_fused_dequant_shared(s["x"], s["codes"], s["scales"], s["ncodes"],
                                                    s["nscales"], s["ts"], s["sync"], s["y"], 2,
                                                    self.err)
        for st in streams:
            cur.wait_stream(st)

    def run_two_launch(self, i):
        """The same step as two launches: the single-launch quantizer, then
        the IF4 dequantizer reading the codes back."""
        b, s = self.b, self.sets[i % len(self.sets)]
        b.if4_quantize_fused(s["x"], s["codes"], s["scales"], s["ncodes"], s["nscales"], s["ts"],
                             s["sync"], self.err)
        b.if4_dequantize(s["codes"], s["scales"], s["ts"], s["y"])

    def run_unfused(self, i, events=None, side=None):
        """The same step as five launches.  With a side stream, the NVFP4 quantizer
        (which needs only ts) runs on it beside IF4 quantize -> dequantize:
        the two quantizers read the same input at about the same time."""
        b, s = self.b, self.sets[i % len(self.sets)]
        ev = events if events is not None else [None] * 6
        if ev[0] is not None:
            ev[0].record()
        b.if4_tensor_amax(s["x"], s["amax"], self.err)
        if ev[1] is not None:
            ev[1].record()
        b.if4_tensor_scale(s["amax"], s["ts"])
        if side is not None:
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                b.nvfp4_quantize(s["x"], s["ncodes"], s["nscales"], s["ts"], b.TS_GIVEN, self.err)
        if ev[2] is not None:
            ev[2].record()
        b.if4_quantize(s["x"], s["codes"], s["scales"], s["ts"], b.TS_GIVEN, self.err)
        if ev[3] is not None:
            ev[3].record()
        b.if4_dequantize(s["codes"], s["scales"], s["ts"], s["y"])
        if ev[4] is not None:
            ev[4].record()
        if side is None:
            b.nvfp4_quantize(s["x"], s["ncodes"], s["nscales"], s["ts"], b.TS_GIVEN, self.err)
        else:
            torch.cuda.current_stream().wait_stream(side)
        if ev[5] is not None:
            ev[5].record()


def upload_graph(g):
    """Upload an instantiated CUDA graph to the device (cuGraphUpload on the
    current stream) before its first replay.  The upload is a one-time setup
    cost: left to the first replay it adds about 90 us to it, 1.8 us per step
    of a 50-step timed graph.  Returns whether the upload was made."""
    import ctypes
    try:
        exec_handle = g.raw_cuda_graph_exec()
        lib = ctypes.CDLL("libcuda.so.1")
        rc = lib.cuGraphUpload(ctypes.c_void_p(int(exec_handle)),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        return rc == 0
    except (AttributeError, OSError, RuntimeError, TypeError, ValueError):
        return False


def kernel_times(step, names, reps, min_launches=32):
    """Per-kernel times: one CUDA graph per kernel launching it on every
    buffer set in turn, as many passes over the sets as make at least
    `min_launches` launches (so that the gap at a graph boundary, where
    programmatic dependent launch cannot overlap two launches, is a small
    share), replayed `reps` times between two events on the replay stream;
    mean time per launch (ms)."""
    out = {}
    sets = len(step.sets)
    n = sets * max(1, -(-min_launches // sets))
    if any(k.startswith(("if6", "if3")) for k in names):
        step.init_widths()
    for name in names:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                step.run_one(name, i % sets)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        out[name] = e0.elapsed_time(e1) / (reps * n)
        del g
    return out


def quantizer_in_sequence(step, steps, sleep_cycles=int(4e7)):
    """Launch durations of the step's dominant kernel, the single-launch
    quantizer, inside the step sequence: the K steps launched on the stream
    (not as a graph: an event-record node in a graph adds microseconds of its
    own) with a timing event recorded right before and right after each
    quantizer launch.  The stream is first held by a sleep of about 20 ms
    so that the host has enqueued every step before the first one runs, and
    no launch waits for the host.  Each quantizer launch then starts after
    the previous dequantizer has finished (the event sits between them), so
    these durations include the launch's own ramp.  Returns (mean, median)
    over the K launches, in ms, or (None, None) when torch offers no sleep
    kernel to hold the stream with."""
    hold = getattr(torch.cuda, "_sleep", None)
    if hold is None:                          # no way to hold the stream: no bound
        return None, None
    before = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    after = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for rep in range(2):                      # the first pass warms up
        torch.cuda.synchronize()
        hold(sleep_cycles)
        for i in range(steps):
            step.run(i, events=(before[i], after[i]))
        torch.cuda.synchronize()
    t = np.array([b.elapsed_time(a) for b, a in zip(before, after)])
    return float(t.mean()), float(np.median(t))


def kernel_table(ms, n_elem, in_bytes, pk):
    q_bytes = in_bytes + n_elem // 2 + n_elem // 16
    w_bytes = {w: n_elem * w // 8 + n_elem // 16 for w in (6, 3)}     # IF6 / IF3 codes + scales
    dq_bytes = n_elem // 2 + n_elem // 16 + 2 * n_elem
    # the single-launch quantizer: x once, IF4 and NVFP4 codes and scales
    fused_bytes = in_bytes + 2 * (n_elem // 2 + n_elem // 16)
    nbytes = {"fused_quantize_dequant": fused_bytes + 2 * n_elem,
              "fused_quantize": fused_bytes, "fused_quantize_rht": fused_bytes,
              "amax": in_bytes, "scale": 8,
              "if4_quantize": q_bytes, "if4_dequantize": dq_bytes,
              "nvfp4_quantize": q_bytes, "nvint4_quantize": q_bytes,
              "nvfp4_4over6_quantize": q_bytes, "if4_quantize_rht": q_bytes,
              "if4_decode_f16": dq_bytes,
              "if6_quantize": in_bytes + w_bytes[6], "if3_quantize": in_bytes + w_bytes[3],
              "if6_dequantize": w_bytes[6] + 2 * n_elem, "if3_dequantize": w_bytes[3] + 2 * n_elem}
    table = {}
    for k, t in ms.items():
        b = nbytes[k]
        gbs = b / (t * 1e-3) / 1e9
        table[k] = {"ms": t, "bytes": b, "gbs": gbs, "frac_of_measured_hbm": gbs / pk["hbm_gbs"],
                    "frac_of_8tbs": gbs / 8000.0, "gelems": n_elem / (t * 1e-3) / 1e9}
    return table


def other_workloads(pk, headline):
    """Per-kernel tables of the other bf16 quantizer workloads (the weight,
    activation and gradient tensors, whichever is not the headline)."""
    out = {}
    for wname in ("weight_bf16_4096x4096", "activation_bf16_8192x8192",
                  "gradient_bf16_16384x4096"):
        if wname == headline:
            continue
        x_cpu = make_input(wname)
        n_elem, in_bytes = x_cpu.numel(), x_cpu.numel() * x_cpu.element_size()
        sets = max(4, int(np.ceil(3 * L2_BYTES / in_bytes)) + 1)
        step = Step(x_cpu, sets=sets)
        for i in range(sets):
            step.run(i)
        torch.cuda.synchronize()
        ms = kernel_times(step, step.kernels + Step.EXTRA, 10)
        out[wname] = kernel_table(ms, n_elem, in_bytes, pk)
        del step
        torch.cuda.empty_cache()
    return out


def _group_mismatches(codes_gpu, scales_gpu, codes_ref, scales_ref):
    """Groups whose 8 code bytes or scale byte differ."""
    c = codes_gpu.reshape(-1, 8) != codes_ref.reshape(-1, 8)
    s = scales_gpu.reshape(-1) != scales_ref.reshape(-1)
    return int(np.count_nonzero(c.any(axis=1) | s))


def parity_quality(name, x_cpu=None):
    """Parity and quality of one quantizer workload, outside any timed
    region: the library's IF4 quantizer (tensor scale computed) and its
    comparators (NVFP4, NVINT4, 4/6 under that tensor scale) against the CPU
    oracle on the same input, group by group (code bytes and scale byte);
    the oracle's near ties (candidate errors within 1e-6 relative, or a zero
    block scale), counted; the dequantized IF4 values against the oracle's,
    element by element; the MSE of each format in the x domain (float64, from
    the library's dequantized output) and the IF4 INT4-group fraction; the
    same for IF6 and IF3 (each with its own tensor scale) and their FP-only
    formats."""
    import oracle
    from adaptive_block_scaled_b200 import binding as b
    if x_cpu is None:
        x_cpu = make_input(name)
    x_np = np.ascontiguousarray(x_cpu.float().numpy())
    x64 = x_np.astype(np.float64)
    dev = torch.device("cuda")
    xd = x_cpu.to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ref = oracle.quantize_tensor(x_np)
    c, sc, ts = b.quantize(xd, "if4", err_flag=err)
    y = b.dequantize(c, sc, ts, dtype=torch.float32).cpu().numpy()
    c_np, sc_np = c.cpu().numpy(), sc.cpu().numpy()
    y_ref = oracle.dequantize(ref["codes"], ref["scales"], ref["ts"])
    out = {"groups": int(sc_np.size),
           "near_ties": int(ref["near"].sum()),
           "ts_bit_identical": bool(np.float32(ts.item()) == ref["ts"]),
           "mismatched_groups": {"if4": _group_mismatches(c_np, sc_np, ref["codes"],
                                                          ref["scales"])},
           "dequantize_mismatched_elements": int(np.count_nonzero(
               y.view(np.uint32) != y_ref.view(np.uint32))),
           "int4_group_fraction": float(np.mean(sc_np >> 7)),
           "mse_if4": float(np.mean((x64 - y) ** 2))}
    for mode, omode in (("nvfp4", oracle.MODE_NVFP4), ("nvint4", oracle.MODE_NVINT4),
                        ("4over6", oracle.MODE_4OVER6)):
        cm, scm, _ = b.quantize(xd, mode, ts=ts.clone(), err_flag=err)
        rm = oracle.quantize(x_np, ref["ts"], mode=omode)
        out["mismatched_groups"][mode] = _group_mismatches(cm.cpu().numpy(), scm.cpu().numpy(),
                                                           rm["codes"], rm["scales"])
        ym = b.dequantize(cm, scm, ts, dtype=torch.float32).cpu().numpy()
        out["mse_" + mode] = float(np.mean((x64 - ym) ** 2))
    # the same adaptive choice at 6 and 3 bits (IF6, IF3) and their FP-only
    # formats, each against the oracle
    for bits in (6, 3):
        name = "if%d" % bits
        rw = oracle.quantize_tensor_w(x_np, bits, oracle.W_IF)
        cw, sw, tw = b.quantize_w(xd, bits, b.W_ADAPTIVE, err_flag=err)
        cw_np, sw_np = cw.cpu().numpy(), sw.cpu().numpy()
        bad = (cw_np.reshape(sw_np.size, -1) != rw["codes"].reshape(sw_np.size, -1)).any(axis=1)
        out["mismatched_groups"][name] = int(np.count_nonzero(bad | (sw_np.reshape(-1) !=
                                                                     rw["scales"].reshape(-1))))
        out["near_ties_" + name] = int(rw["near"].sum())
        out["ts_bit_identical_" + name] = bool(np.float32(tw.item()) == rw["ts"])
        yw = b.dequantize_w(cw, sw, tw, bits, dtype=torch.float32).cpu().numpy()
        out["mse_" + name] = float(np.mean((x64 - yw) ** 2))
        out["int_group_fraction_" + name] = float(np.mean(sw_np >> 7))
        fw = oracle.quantize_w(x_np, rw["ts"], bits, oracle.W_FP)
        cf, sf, _ = b.quantize_w(xd, bits, b.W_FP_ONLY, ts=tw.clone(), err_flag=err)
        cf_np, sf_np = cf.cpu().numpy(), sf.cpu().numpy()
        badf = (cf_np.reshape(sf_np.size, -1) != fw["codes"].reshape(sf_np.size, -1)).any(axis=1)
        out["mismatched_groups"]["fp%d" % bits] = int(np.count_nonzero(
            badf | (sf_np.reshape(-1) != fw["scales"].reshape(-1))))
        yf = b.dequantize_w(cf, sf, tw, bits, dtype=torch.float32).cpu().numpy()
        out["mse_fp%d" % bits] = float(np.mean((x64 - yf) ** 2))
    torch.cuda.synchronize()
    out["device_error_flag"] = int(err.item())
    nv = out["mse_nvfp4"]
    out["mse_reduction_vs_nvfp4_pct"] = 100.0 * (1.0 - out["mse_if4"] / nv) if nv > 0 else 0.0
    return out


def step_outputs_vs_oracle(x_cpu, s):
    """The timed step's own outputs (buffer set s: IF4 codes and scales,
    tensor scale, NVFP4 codes and scales, bf16 round trip) against the
    oracle on the same input."""
    import oracle
    x_np = np.ascontiguousarray(x_cpu.float().numpy())
    ref = oracle.quantize_tensor(x_np)
    nref = oracle.quantize(x_np, ref["ts"], mode=oracle.MODE_NVFP4)
    y_ref = torch.from_numpy(oracle.dequantize(ref["codes"], ref["scales"], ref["ts"]))
    y_ref = y_ref.to(torch.bfloat16).view(torch.int16).numpy()
    return {"groups": int(ref["scales"].size),
            "near_ties": int(ref["near"].sum()),
            "ts_bit_identical": bool(np.float32(s["ts"].item()) == ref["ts"]),
            "if4_mismatched_groups": _group_mismatches(s["codes"].cpu().numpy(),
                                                       s["scales"].cpu().numpy(),
                                                       ref["codes"], ref["scales"]),
            "nvfp4_mismatched_groups": _group_mismatches(s["ncodes"].cpu().numpy(),
                                                         s["nscales"].cpu().numpy(),
                                                         nref["codes"], nref["scales"]),
            "y_mismatched_elements": int(np.count_nonzero(
                s["y"].cpu().view(torch.int16).numpy() != y_ref))}


def measure_e2e(x_cpu, steps, warmup):
    """The same step through the C ABI from pinned host memory: per step, the
    H2D copy of the input, the step's launch, and the D2H copy of every result
    (IF4 codes, scales and tensor scale, the bf16 dequantized tensor, NVFP4
    codes and scales), all inside the timed region.  Consecutive steps
    alternate between two streams with their own buffers, so one step's
    upload overlaps the previous step's download (PCIe is full duplex)."""
    from adaptive_block_scaled_b200 import binding as b
    rows, cols = x_cpu.shape
    dev = torch.device("cuda")
    h_x = x_cpu.contiguous().pin_memory()
    outs = dict(codes=((rows, cols // 2), torch.uint8), scales=((rows, cols // 16), torch.uint8),
                ts=((1,), torch.float32), y=((rows, cols), torch.bfloat16),
                ncodes=((rows, cols // 2), torch.uint8), nscales=((rows, cols // 16), torch.uint8))
    lanes = []
    for _ in range(2):
        lanes.append(dict(
            stream=torch.cuda.Stream(),
            x=torch.empty_like(h_x, device=dev),
            sync=torch.zeros(64, dtype=torch.int32, device=dev),
            d={k: torch.empty(sh, dtype=dt, device=dev) for k, (sh, dt) in outs.items()},
            h={k: torch.empty(sh, dtype=dt, pin_memory=True) for k, (sh, dt) in outs.items()}))
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(i):
        L = lanes[i % 2]
        with torch.cuda.stream(L["stream"]):
            d = L["d"]
            L["x"].copy_(h_x, non_blocking=True)
            b.if4_quantize_fused_dequant(L["x"], d["codes"], d["scales"], d["ncodes"],
                                         d["nscales"], d["ts"], L["sync"], d["y"], err)
            for k in L["h"]:
                L["h"][k].copy_(d[k], non_blocking=True)

    cur = torch.cuda.current_stream()
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for L in lanes:
        L["stream"].wait_stream(cur)
    for i in range(steps):
        step(i)
    for L in lanes:
        cur.wait_stream(L["stream"])
    e1.record(cur)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = h_x.numel() * h_x.element_size()
    d2h = sum(t.numel() * t.element_size() for t in lanes[0]["h"].values())
    return {"value": rows * cols / (ms * 1e-3) / 1e9, "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "how": "C ABI calls from Python, two streams alternating steps"}


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
    # the same linear with its output quantized to IF4 in the epilogue (no
    # bf16 C), against the bf16 linear followed by a separate IF4 quantize
    c_ts = torch.ones(1, dtype=torch.float32, device=dev)
    b.if4_tensor_amax(c, c_ts)
    b.if4_tensor_scale(c_ts, c_ts)
    c_codes = torch.empty((M, N // 2), dtype=torch.uint8, device=dev)
    c_scales = torch.empty((M, N // 16), dtype=torch.uint8, device=dev)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    t_q = timed(lambda: b.if4_linear_quantized(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], ws,
                                               c_codes, c_scales, c_ts, err_flag=err))
    t_sep = timed(lambda: (b.if4_linear(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], ws, c, err),
                           b.if4_quantize(c, c_codes, c_scales, c_ts, b.TS_GIVEN, err)))
    # the public entry point as one call: both operands' decode in one
    # launch, then the GEMM
    t_call = timed(lambda: b.if4_linear(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], ws, c, err))
    # the decoders inside the GEMM (no workspace): the same C
    t_fused = timed(lambda: b.if4_linear_fused(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], c, err))
    flops = 2.0 * M * N * K
    gemm_tf = flops / (t[2] * 1e-3) / 1e12
    total = sum(t)
    return {"workload": "linear_8192x4096x4096", "err": int(err.item()),
            "decode_a_ms": t[0], "decode_b_ms": t[1], "gemm_ms": t[2], "linear_ms": total,
            "gemm_tflops": gemm_tf, "linear_tflops": flops / (total * 1e-3) / 1e12,
            "cublas_f16_ms": t_cublas, "cublas_f16_tflops": flops / (t_cublas * 1e-3) / 1e12,
            "linear_call_ms": t_call, "linear_call_tflops": flops / (t_call * 1e-3) / 1e12,
            "linear_if4_out_ms": t_q, "linear_then_quantize_ms": t_sep,
            "linear_fused_decode_ms": t_fused,
            "linear_fused_decode_tflops": flops / (t_fused * 1e-3) / 1e12,
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
    # enough rotating sets that even the lightest kernel (amax: 2 B/element)
    # cycles through more than three times the 126 MB L2 before reusing one
    sets = max(4, int(np.ceil(3 * L2_BYTES / in_bytes)) + 1)
    step = Step(x_cpu, sets=sets)

    for i in range(args.warmup):
        step.run(i)
    torch.cuda.synchronize()
    if int(step.err.item()) != 0:
        raise RuntimeError(f"device error flag {int(step.err.item())} during warm-up")

    # The timed steps are captured as one CUDA graph (each step on the next
    # buffer set in turn), so neither host launch overhead nor the gaps
    # between graph launches pace the GPU; the warm-up steps are a graph of
    # their own, replayed first.
    uploaded = []

    def capture(fn, n, **kw):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                fn(i, **kw)
        uploaded.append(upload_graph(g))
        return g

    warm = capture(step.run, max(args.warmup, sets))
    timed = capture(step.run, args.steps)
    warm.replay()
    torch.cuda.synchronize()

    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record()
        timed.replay()
        stop.record()
        torch.cuda.synchronize()
    barrier(world)
    ms_local = start.elapsed_time(stop) / args.steps
    ms = max_over_ranks(ms_local, world)
    del warm

    # the same step as five launches (NVFP4 on a parallel graph branch), for
    # comparison
    side = torch.cuda.Stream()
    # the same step as two launches (quantizer, then dequantizer)
    twarm = capture(step.run_two_launch, sets)
    ttimed = capture(step.run_two_launch, args.steps)
    twarm.replay()
    torch.cuda.synchronize()
    start.record()
    ttimed.replay()
    stop.record()
    torch.cuda.synchronize()
    ms_two_launch = start.elapsed_time(stop) / args.steps
    del twarm, ttimed
    uwarm = capture(step.run_unfused, sets, side=side)
    utimed = capture(step.run_unfused, args.steps, side=side)
    uwarm.replay()
    torch.cuda.synchronize()
    start.record()
    utimed.replay()
    stop.record()
    torch.cuda.synchronize()
    ms_unfused = start.elapsed_time(stop) / args.steps
    del uwarm, utimed

    # the same steps on two streams with the shared launch (share 2):
    # independent steps overlapping, one's amax pass beside the other's encode
    pair = [torch.cuda.Stream(), torch.cuda.Stream()]
    pwarm = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pwarm):
        step.run_two_streams(max(args.warmup, sets), pair)
    ptimed = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ptimed):
        step.run_two_streams(args.steps, pair)
    uploaded.append(upload_graph(ptimed))
    pwarm.replay()
    torch.cuda.synchronize()
    start.record()
    ptimed.replay()
    stop.record()
    torch.cuda.synchronize()
    ms_two_streams = start.elapsed_time(stop) / args.steps
    del pwarm, ptimed

    kern_ms = kernel_times(step, step.kernels, 5)
    seq_mean, seq_median = quantizer_in_sequence(step, args.steps)
    if int(step.err.item()) != 0:
        raise RuntimeError(f"device error flag {int(step.err.item())}")
    graphs_keep = timed

    value = world * n_elem / (ms * 1e-3) / 1e9
    kernels = kernel_table(kern_ms, n_elem, in_bytes, pk)
    extra = kernel_table(kernel_times(step, Step.EXTRA, 5), n_elem, in_bytes, pk)

    def roof(name, label):
        k = kernels[name]
        r = {"bound": "hbm", "kernel": label, "achieved": k["gbs"], "peak": pk["hbm_gbs"],
             "unit": "GB/s", "frac": k["gbs"] / pk["hbm_gbs"],
             "peak_source": f"{pk['source']} hbm_gbs (copy bandwidth, read+write; of {pk['source']})",
             "algorithmic_bytes_per_launch": k["bytes"], "traffic": None,
             "timing": "CUDA events around a graph of at least 32 back-to-back launches over "
                       "the buffer sets, on the launching stream; mean per launch"}
        traffic_file = os.path.join(ROOT, "profiles", "traffic.json")
        if os.path.exists(traffic_file):
            tr = json.load(open(traffic_file)).get(args.workload, {}).get(name)
            if tr:
                r["traffic"] = tr
        return r

    # the dominant kernel of the step is the single-launch quantizer; the
    # IF4 quantizer alone (tensor scale given) is reported beside it
    roofline = roof("fused_quantize_dequant",
                    "if4_quantize_fused_dequant (amax + scale + IF4 + NVFP4 + bf16 round trip)")
    # the same kernel inside the step (the step is this one launch): the
    # timed step itself, and events around each launch of the steps run again
    roofline["in_step"] = {
        "step_us": ms * 1e3,
        "frac_at_step": kernels["fused_quantize_dequant"]["bytes"] / (ms * 1e-3) / 1e9
        / pk["hbm_gbs"],
        "event_us_mean": None if seq_mean is None else seq_mean * 1e3,
        "event_us_median": None if seq_median is None else seq_median * 1e3,
        "event_note": "events on the stream around each launch of the timed steps run again "
                      "eagerly; includes the launch latency the events expose"}
    roofline_if4 = roof("if4_quantize", "if4_quantize (tensor scale given)")

    config = bench_config(args.workload, x_cpu, world)
    config.update({"buffer_sets": sets,
                   "l2_detail": f"rotating {sets} buffer sets, {sets * per_set / 1e6:.0f} MB "
                                f"(inputs {sets * in_bytes / 1e6:.0f} MB > 3x126 MB L2)",
                   "launch": "the timed steps as one CUDA graph, uploaded to the device before "
                             "its timed replay; per-kernel times from one graph per kernel of at "
                             "least 32 launches over all sets",
                   "graph_uploaded": bool(uploaded) and all(uploaded)})
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": config,
            "gpu_launches": step.launches_per_step * args.steps,
            "ms_per_step_two_launch": ms_two_launch,
            "ms_per_step_unfused": ms_unfused,
            "two_streams_shared": {
                "ms_per_step": ms_two_streams,
                "value": world * n_elem / (ms_two_streams * 1e-3) / 1e9, "unit": UNIT,
                "gbs": kernels["fused_quantize_dequant"]["bytes"] / (ms_two_streams * 1e-3) / 1e9,
                "frac_of_measured_hbm": kernels["fused_quantize_dequant"]["bytes"]
                / (ms_two_streams * 1e-3) / 1e9 / pk["hbm_gbs"],
                "how": "the same K steps as one CUDA graph, consecutive steps alternating "
                       "between two streams, each step one if4_quantize_fused_dequant_shared "
                       "launch with share 2 (half the resident blocks per SM), so one "
                       "step's amax pass overlaps the other's encode pass"},
            "kernels": kernels, "kernels_outside_step": extra, "roofline": roofline,
            "roofline_if4_quantize": roofline_if4}
    if rank == 0:
        line["clocks"] = clk.summary()
        # the step's own outputs (buffer set 0, last written by the timed
        # steps or the per-kernel graphs that ran the same launch) against
        # the oracle: rerun the step on set 0 so it holds the step's results
        step.run(0)
        torch.cuda.synchronize()
        line["step_outputs_vs_oracle"] = step_outputs_vs_oracle(x_cpu, step.sets[0])
        line["e2e"] = measure_e2e(x_cpu, max(5, args.steps // 5), 2)
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(x_cpu, args.cpu_seconds, args.workload)
    del step, graphs_keep
    torch.cuda.empty_cache()
    if rank == 0:
        # parity and quality of every quantizer workload (the headline's own
        # tensor included), outside the timed region: N = 1 only
        if world == 1 and not args.no_quality:
            line["quality"] = {w: parity_quality(w, x_cpu if w == args.workload else None)
                               for w in QUANT_WORKLOADS}
        # single-GPU reports: only at N = 1, so that with N > 1 the other
        # ranks do not wait long at the final barrier
        if not args.no_linear and world == 1 and hasattr(b_lib(), "if4_linear"):
            line["linear"] = linear_report(pk)
        if not args.no_large and world == 1:
            line["other_workloads"] = other_workloads(pk, args.workload)
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_kernel_only(args):
    """Only the chosen kernel, on the chosen workload: the command ncu wraps."""
    from adaptive_block_scaled_b200 import binding as b
    if args.kernel_only in ("gemm", "linear_fused", "linear_quantized"):
        M, N, K = 8192, 4096, 4096
        a, bw = make_input("linear_8192x4096x4096")
        dev = torch.device("cuda")
        aq, bq = b.quantize(a.to(dev)), b.quantize(bw.to(dev))
        wa, wb = b.decode_f16(aq[0], aq[1]), b.decode_f16(bq[0], bq[1])
        c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        if args.kernel_only == "linear_quantized":
            # the output's tensor scale from one plain linear first
            ws = torch.empty(b.if4_linear_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
            b.if4_linear(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], ws, c, err)
            c_ts = torch.ones(1, dtype=torch.float32, device=dev)
            b.if4_tensor_amax(c, c_ts)
            b.if4_tensor_scale(c_ts, c_ts)
            c_codes = torch.empty((M, N // 2), dtype=torch.uint8, device=dev)
            c_scales = torch.empty((M, N // 16), dtype=torch.uint8, device=dev)
        for _ in range(args.warmup + args.steps):
            if args.kernel_only == "gemm":
                b.if4_gemm_f16(wa, wb, aq[2], bq[2], c, err)
            elif args.kernel_only == "linear_quantized":
                b.if4_linear_quantized(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], ws, c_codes,
                                       c_scales, c_ts, err_flag=err)
            else:
                b.if4_linear_fused(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], c, err)
        torch.cuda.synchronize()
        print(json.dumps({"kernel_only": args.kernel_only, "launches": args.warmup + args.steps,
                          "err": int(err.item())}))
        if int(err.item()) != 0:
            sys.exit(1)
        return
    x_cpu = make_input(args.workload)
    step = Step(x_cpu, sets=1)
    if args.kernel_only.startswith(("if6", "if3")):
        step.init_widths()
    s = step.sets[0]
    b.if4_tensor_amax(s["x"], s["amax"], step.err)
    b.if4_tensor_scale(s["amax"], s["ts"])
    b.if4_quantize(s["x"], s["codes"], s["scales"], s["ts"], b.TS_GIVEN, step.err)
    torch.cuda.synchronize()
    calls = {name: (lambda name=name: step.run_one(name, 0))
             for name in Step.EXTRA + ["fused_quantize", "fused_quantize_dequant"]}
    calls.update({
        "amax": lambda: b.if4_tensor_amax(s["x"], s["amax"], step.err),
        "if4_quantize": lambda: b.if4_quantize(s["x"], s["codes"], s["scales"], s["ts"],
                                               b.TS_GIVEN, step.err),
        "if4_dequantize": lambda: b.if4_dequantize(s["codes"], s["scales"], s["ts"], s["y"]),
        "nvfp4_quantize": lambda: b.nvfp4_quantize(s["x"], s["ncodes"], s["nscales"], s["ts"],
                                                   b.TS_GIVEN, step.err),
    })
    for _ in range(args.warmup + args.steps):
        calls[args.kernel_only]()
    torch.cuda.synchronize()
    print(json.dumps({"kernel_only": args.kernel_only, "workload": args.workload,
                      "launches": args.warmup + args.steps, "err": int(step.err.item())}))
    if int(step.err.item()) != 0:
        sys.exit(1)


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
