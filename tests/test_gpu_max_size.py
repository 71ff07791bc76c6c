"""GPU parity at the largest tensor the API accepts: rows * cols / 16 groups
just below 2^31 (the kernels index groups with 32-bit integers and address
bytes with 64-bit offsets).  The bf16 input is 68.7 GB and the outputs 19.3
GB, so the check samples rows: the first, the last, and 62 seeded random
rows are compared with the oracle byte for byte under the tensor scale the
GPU computed, and that tensor scale is checked against the exact maximum of
the input (taken on the GPU with torch) through the oracle's scale rule."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

ROWS, COLS = (1 << 23) - 1, 4096          # 2^31 - 256 groups


def _free_bytes():
    free, _ = torch.cuda.mem_get_info()
    return free


@pytest.fixture(scope="module")
def big():
    need = ROWS * COLS * 2 + ROWS * COLS // 2 + ROWS * COLS // 16 + (2 << 30)
    if _free_bytes() < need:
        pytest.skip(f"needs {need / 1e9:.0f} GB of free device memory")
    g = torch.Generator(device="cuda").manual_seed(2024)
    x = torch.empty((ROWS, COLS), dtype=torch.bfloat16, device="cuda")
    step = 1 << 18                           # 2 GB of bf16 per draw
    for r in range(0, ROWS, step):
        n = min(step, ROWS - r)
        x[r:r + n] = torch.randn((n, COLS), generator=g, device="cuda", dtype=torch.bfloat16)
    x[ROWS - 1, COLS - 3] = 123.0            # the tensor max sits in the last group
    yield x
    del x
    torch.cuda.empty_cache()


def _sample_rows():
    rng = np.random.default_rng(5)
    return np.unique(np.concatenate([[0, ROWS - 1], rng.integers(1, ROWS - 1, 62)]))


def B():
    from adaptive_block_scaled_b200 import binding
    return binding


def _check(x, codes, scales, ts):
    # max |x| without a tensor-sized temporary
    amax = max(abs(float(torch.amax(x).item())), abs(float(torch.amin(x).item())))
    assert np.float32(ts) == oracle.tensor_scale(np.float32(amax))
    for r in _sample_rows():
        ref = oracle.quantize(x[r:r + 1].float().cpu().numpy(), np.float32(ts))
        assert np.array_equal(codes[r:r + 1].cpu().numpy(), ref["codes"]), r
        assert np.array_equal(scales[r:r + 1].cpu().numpy(), ref["scales"]), r


def test_quantize_at_the_maximum_group_count(big):
    b = B()
    assert ROWS * (COLS // 16) == (1 << 31) - 256
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, scales, ts = b.quantize(big, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _check(big, codes, scales, ts.item())
    del codes, scales
    torch.cuda.empty_cache()


def test_single_launch_quantizer_at_the_maximum_group_count(big):
    b = B()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, scales, ts = b.quantize_fused(big, with_nvfp4=False, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _check(big, codes, scales, ts.item())
    del codes, scales
    torch.cuda.empty_cache()
