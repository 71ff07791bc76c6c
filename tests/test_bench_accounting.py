"""The benchmark's algorithmic bytes per element, on which every reported
bandwidth and roofline fraction rests: each kernel's count is the bytes the
operation must move at least (inputs read once, outputs written once)."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


@pytest.mark.parametrize("elem_bytes", [2, 4])
def test_algorithmic_bytes_per_element(elem_bytes):
    n = 4096 * 4096
    names = ["fused_quantize_dequant", "fused_quantize", "amax", "if4_quantize",
             "if4_dequantize", "nvfp4_quantize", "if4_decode_f16", "nvint4_quantize",
             "nvfp4_4over6_quantize", "if4_quantize_rht", "fused_quantize_rht", "if6_quantize",
             "if3_quantize", "if6_dequantize", "if3_dequantize"]
    t = bench.kernel_table({k: 1.0 for k in names}, n, n * elem_bytes, {"hbm_gbs": 6552.0})
    codes = 0.5 + 1 / 16                        # 4-bit codes + one scale byte per 16
    want = {
        "amax": elem_bytes,                                 # x once
        "if4_quantize": elem_bytes + codes,                 # x, IF4 codes and scales
        "nvfp4_quantize": elem_bytes + codes,
        "fused_quantize": elem_bytes + 2 * codes,           # x once, IF4 and NVFP4
        "fused_quantize_dequant": elem_bytes + 2 * codes + 2,   # ... and the bf16 y
        "if4_dequantize": codes + 2,                        # codes in, bf16 out
        "if4_decode_f16": codes + 2,                        # codes in, fp16 out
        "nvint4_quantize": elem_bytes + codes,
        "nvfp4_4over6_quantize": elem_bytes + codes,
        "if4_quantize_rht": elem_bytes + codes,             # the transform is in registers
        "fused_quantize_rht": elem_bytes + 2 * codes,
        "if6_quantize": elem_bytes + 6 / 8 + 1 / 16,        # 6-bit codes, one scale per 16
        "if3_quantize": elem_bytes + 3 / 8 + 1 / 16,
        "if6_dequantize": 6 / 8 + 1 / 16 + 2,               # bf16 out
        "if3_dequantize": 3 / 8 + 1 / 16 + 2,
    }
    for k, per_elem in want.items():
        assert t[k]["bytes"] == pytest.approx(per_elem * n, rel=0, abs=0.5), k
        # 1 ms per launch: GB/s is bytes / 1e6
        assert t[k]["gbs"] == pytest.approx(t[k]["bytes"] / 1e6)


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference (the oracle, on the host cores) prints one
    JSON line with the contract's keys, its cpu_baseline and e2e describing
    that run."""
    import json
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         timeout=600, cwd=root, check=True).stdout
    line = json.loads(out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 0
    assert line["config"]["workload"] == bench.WORKLOAD
    # the same config object as the GPU arm's (its extra keys aside)
    x = bench.make_input(bench.WORKLOAD)
    assert line["config"] == bench.bench_config(bench.WORKLOAD, x, 1)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == line["value"]
    assert line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_clock_summary_reads_reasons_and_the_clock_under_load():
    """The nvidia-smi samples the bench takes during the timed region: the
    median SM clock of the samples under load, the maximum clock, and every
    throttle reason seen active ("Not Active" is not a reason; malformed
    lines are skipped)."""
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1965, 1965, 120.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n",
        "0, 1965, 1965, 612.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "0, 1890, 1965, 655.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "0, 1950, 1965, 640.0, 0x0000000000000008, Active, Not Active, Not Active, Not Active\n",
        "garbage line\n",
        "0, [N/A], 1965, 600.0, 0x0, Not Active, Not Active, Not Active, Not Active\n",
    ]
    s = c.summary()
    assert s["samples"] == 4 and s["samples_under_load"] == 3
    assert s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0
    assert s["power_w_max"] == 655.1
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]
    c.lines = []
    assert c.summary() is None


def test_cpu_baseline_times_every_core_and_one_core():
    """The oracle's timing on the host: all cores and one core, each on a
    stated row sample of the given workload."""
    import torch
    x = torch.randn(64, 256, generator=torch.Generator().manual_seed(0))
    cb = bench.cpu_baseline(x, 0.05, "test_64x256")
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1
    assert "test_64x256" in cb["sample"]
    one = cb["one_core"]
    assert one["cores"] == 1 and one["value"] > 0 and "1 thread" in one["sample"]


def test_group_mismatch_count():
    """A group counts once whether its code bytes, its scale byte or both
    differ."""
    import numpy as np
    c = np.zeros((4, 16), np.uint8)
    s = np.zeros((4, 2), np.uint8)
    c2, s2 = c.copy(), s.copy()
    c2[0, 3] = 1            # group 0 (codes)
    s2[1, 1] = 0x80         # group 3 (scale)
    c2[2, 0] = 1            # group 4 (codes) ...
    s2[2, 0] = 1            # ... and its scale: still one group
    assert bench._group_mismatches(c2, s2, c, s) == 3
    assert bench._group_mismatches(c, s, c, s) == 0
