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
             "if4_dequantize", "nvfp4_quantize", "if4_decode_f16"]
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
    }
    for k, per_elem in want.items():
        assert t[k]["bytes"] == pytest.approx(per_elem * n, rel=0, abs=0.5), k
        # 1 ms per launch: GB/s is bytes / 1e6
        assert t[k]["gbs"] == pytest.approx(t[k]["bytes"] / 1e6)
