"""GPU parity of IF6 and IF3 through the C ABI against the CPU oracle.

The kernels decide each group by the oracle's own binary64 rule, so codes,
scale bytes and tensor scales must be bit-identical for every mode (adaptive,
FP only, INT only), every input dtype and every workload; dequantized values
are bit-identical too.  The grids are this library's reading of the pages'
IF6 / IF3 (FP6 = E2M3 against INT6 k*15/62, FP3 = E2M0 against INT3 k*4/3).
"""
import numpy as np
import pytest
import torch

import oracle
from adaptive_block_scaled_b200 import workloads

pytestmark = pytest.mark.gpu

MODES = {"adaptive": oracle.W_IF, "fp": oracle.W_FP, "int": oracle.W_INT}


def B():
    from adaptive_block_scaled_b200 import binding
    return binding


def check_w(x_cpu, bits, label, mode="adaptive", ts=None, x_dev=None, dequant=True):
    b = B()
    x_np = x_cpu.float().numpy()
    if ts is None:
        ref = oracle.quantize_tensor_w(x_np, bits, MODES[mode])
        ts_ref = np.float32(ref["ts"])
    else:
        ts_ref = np.float32(ts)
        ref = oracle.quantize_w(x_np, ts_ref, bits, MODES[mode])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = x_cpu.cuda() if x_dev is None else x_dev
    ts_t = None if ts is None else torch.tensor([ts], dtype=torch.float32, device="cuda")
    codes, scales, ts_g = b.quantize_w(x, bits, {"adaptive": b.W_ADAPTIVE, "fp": b.W_FP_ONLY,
                                                 "int": b.W_INT_ONLY}[mode], ts=ts_t, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, label
    assert np.float32(ts_g.item()).view(np.uint32) == ts_ref.view(np.uint32), (label, ts_g, ts_ref)
    c, s = codes.cpu().numpy(), scales.cpu().numpy()
    bad = np.count_nonzero(s != ref["scales"]) + np.count_nonzero(
        (c.reshape(s.size, -1) != ref["codes"].reshape(s.size, -1)).any(axis=1))
    assert bad == 0, f"{label}: {bad} groups differ"
    if dequant:
        y_ref = oracle.dequantize_w(c, s, ts_ref, bits)
        for dt in (torch.float32, torch.bfloat16, torch.float16):
            y = b.dequantize_w(codes, scales, ts_g, bits, dtype=dt).cpu()
            want = torch.from_numpy(y_ref).to(dt)
            assert torch.equal(y.view(torch.int16 if dt != torch.float32 else torch.int32),
                               want.view(torch.int16 if dt != torch.float32 else torch.int32)), \
                (label, dt)
    frac = float(np.mean(s >> 7))
    print(f"[{label} IF{bits} {mode}] groups={s.size} int_frac={frac:.4f} "
          f"near_ties={int(ref['near'].sum())}")
    return ref


@pytest.mark.parametrize("bits", [6, 3])
@pytest.mark.parametrize("name", ["small_fp32_256x1024", "weight_bf16_4096x4096",
                                  "activation_bf16_8192x8192", "gradient_bf16_16384x4096"])
def test_workloads(bits, name):
    x = workloads.WORKLOADS[name].make(0)
    check_w(x, bits, name)


@pytest.mark.parametrize("bits", [6, 3])
@pytest.mark.parametrize("mode", ["fp", "int"])
def test_fixed_modes(bits, mode):
    check_w(workloads.llm_weight(3, rows=512, cols=1024), bits, "weight 512x1024", mode)


@pytest.mark.parametrize("bits", [6, 3])
@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (33, 272), (1000, 16)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_shapes_and_dtypes(bits, shape, dtype):
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(dtype)
    check_w(x, bits, f"{shape} {dtype}")


@pytest.mark.parametrize("bits", [6, 3])
def test_every_bf16_value_both_candidates(bits):
    """Every bf16 value within the FP grid's range goes through both
    candidates' rounding under a unit block scale (v = x)."""
    fpmax = 7.5 if bits == 6 else 4.0
    v = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) <= fpmax)]
    pad = (-v.size) % 15
    v = np.concatenate([v, np.zeros(pad, np.float32)]).reshape(-1, 15)
    x = np.concatenate([np.full((v.shape[0], 1), fpmax, np.float32), v], axis=1).reshape(1, -1)
    x = torch.from_numpy(x).to(torch.bfloat16)
    for mode in ("fp", "int", "adaptive"):
        check_w(x, bits, "every bf16 value", mode, ts=1.0, dequant=mode == "adaptive")


@pytest.mark.parametrize("bits", [6, 3])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_tiny_zero_and_saturated_groups(bits, dtype):
    rng = np.random.default_rng(31)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    x *= np.exp2(-rng.integers(0, 30, (64, 16))).repeat(16, axis=1).astype(np.float32)
    x[0, 0] = 1000.0
    x[1, :16] = -0.0
    x[2, 16:32] = -1e-7
    xt = torch.from_numpy(x).to(dtype)
    ref = check_w(xt, bits, "tiny groups")
    sb = ref["scales"] & 0x7F
    assert (sb == 0).any() and ((sb > 0) & (sb < 8)).any()
    amax = float(xt.float().abs().max())
    fpmax = 7.5 if bits == 6 else 4.0
    check_w(xt, bits, "saturating ts", ts=np.float32(amax / (fpmax * 448) / 64))


@pytest.mark.parametrize("bits", [6, 3])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_scaled_values_overflow(bits, dtype):
    """A given tensor scale (2^-117) far below the data's: every block scale
    saturates and v = x * fl(1/fl(448 ts)) overflows binary32 to +-Inf for
    all but the zero elements.  FP saturates, INT clamps to +-kmax, both
    error sums are infinite, and the rule keeps FP."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((8, 64)) * 1e37).astype(np.float32)
    x[0, :4] = [3e38, -3e38, 0.0, -0.0]
    for mode in ("adaptive", "fp", "int"):
        ref = check_w(torch.from_numpy(x).to(dtype), bits, "overflowing v", mode,
                      ts=np.float32(2.0 ** -117), dequant=mode == "adaptive")
        assert ((ref["scales"] & 0x7F) == 0x7E).all()


@pytest.mark.parametrize("bits", [6, 3])
def test_strided_rows(bits):
    base = workloads.llm_weight(5, rows=128, cols=1024 + 64)
    x_dev = base.cuda()[:, 8:8 + 1024]
    x_cpu = base[:, 8:8 + 1024].contiguous()
    check_w(x_cpu, bits, "strided", x_dev=x_dev)


@pytest.mark.parametrize("bits", [6, 3])
def test_nonfinite_input_sets_flag(bits):
    b = B()
    x = torch.ones((4, 64), dtype=torch.float32, device="cuda")
    x[1, 5] = float("inf")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.quantize_w(x, bits, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & b.DEV_NONFINITE


@pytest.mark.parametrize("bits", [6, 3])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_dequantize_arbitrary_codes(bits, dtype):
    """Random code and scale bytes, every code value of both types (INT6 k =
    -32 and INT3 k = -4 included, which the quantizer never writes; FP
    negative zeros; every magnitude), decoded against the oracle's
    dequantizer and rounded to the output type.  E4M3 NaN scale bytes
    (0x7F, 0xFF) give NaN on both sides, compared as NaN."""
    rng = np.random.default_rng(61 + bits)
    rows, cols = 96, 512
    codes = rng.integers(0, 256, (rows, cols * bits // 8), dtype=np.uint8)
    scales = rng.integers(0, 256, (rows, cols // 16), dtype=np.uint8)
    ts = np.float32(0.37)
    want = torch.from_numpy(oracle.dequantize_w(codes, scales, ts, bits)).to(dtype)
    b = B()
    y = b.dequantize_w(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(),
                       torch.tensor([ts], dtype=torch.float32, device="cuda"), bits,
                       dtype=dtype).cpu()
    nan = torch.isnan(want)
    assert torch.equal(torch.isnan(y), nan)
    iv = torch.int32 if dtype == torch.float32 else torch.int16
    assert torch.equal(y[~nan].view(iv), want[~nan].view(iv))
    assert nan.any() and (~nan).any()

