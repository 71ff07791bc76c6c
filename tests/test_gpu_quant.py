"""GPU parity: the CUDA quantizer, NVFP4 comparator and dequantizer, called
through the C ABI, against the CPU oracle on the same seeded inputs.

Codes, scale bytes and the tensor scale must be bit-identical to the oracle
(the kernels settle every group whose binary32 margin is within rounding with
the oracle's binary64 rule, so no group may differ).  Dequantized outputs
are bit-identical too: every step is one IEEE binary32 rounding shared by
both sides, then one RNE conversion.  Near-tie groups (candidate errors
within 1e-6 relative) are counted and printed.
"""
import numpy as np
import pytest
import torch

import oracle
from adaptive_block_scaled_b200 import workloads

pytestmark = pytest.mark.gpu


def B():
    from adaptive_block_scaled_b200 import binding
    return binding


def gpu_quant(x_cpu, mode="if4", ts=None, x_dev=None):
    b = B()
    x = x_cpu.cuda() if x_dev is None else x_dev
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ts_t = None if ts is None else torch.tensor([ts], dtype=torch.float32, device="cuda")
    codes, scales, ts_out = b.quantize(x, mode, ts=ts_t, err_flag=err)
    torch.cuda.synchronize()
    return (codes.cpu().numpy(), scales.cpu().numpy(), np.float32(ts_out.cpu().item()),
            int(err.item()))


def f32_bits(a):
    return np.asarray(a, np.float32).view(np.uint32)


def check_quant(x_cpu, label, ts=None, check_deq=True):
    """Full bit-parity check of IF4, NVFP4 and the dequantizer on one tensor."""
    x_np = x_cpu.float().numpy()
    if ts is None:
        ref = oracle.quantize_tensor(x_np)
        ts_ref = ref["ts"]
    else:
        ts_ref = np.float32(ts)
        ref = oracle.quantize(x_np, ts_ref)
    codes, scales, ts_g, err = gpu_quant(x_cpu, "if4", ts=ts)
    assert err == 0
    assert f32_bits(ts_g) == f32_bits(ts_ref), (label, ts_g, ts_ref)
    bad_s = np.count_nonzero(scales != ref["scales"])
    bad_c = np.count_nonzero(codes != ref["codes"])
    if bad_s or bad_c:
        idx = np.argwhere(scales != ref["scales"])[:5]
        raise AssertionError(f"{label}: {bad_s} scale bytes / {bad_c} code bytes differ; "
                             f"first groups {idx.tolist()} gpu {scales[tuple(idx.T)] if len(idx) else ''}"
                             f" ref {ref['scales'][tuple(idx.T)] if len(idx) else ''}")
    near = int(ref["near"].sum())
    frac = oracle.group_int4_fraction(scales)
    nv = oracle.quantize(x_np, ts_ref, mode=oracle.MODE_NVFP4)
    ncodes, nscales, nts, nerr = gpu_quant(x_cpu, "nvfp4", ts=float(ts_ref))
    assert nerr == 0 and f32_bits(nts) == f32_bits(ts_ref)
    assert np.array_equal(nscales, nv["scales"]), label
    assert np.array_equal(ncodes, nv["codes"]), label
    print(f"[{label}] groups={scales.size} int4_frac={frac:.4f} near_ties={near}")
    if check_deq:
        check_dequant(codes, scales, ts_ref, label)
    return ref


def check_dequant(codes, scales, ts, label, dtypes=(torch.float32, torch.bfloat16, torch.float16)):
    b = B()
    y_ref = oracle.dequantize(codes, scales, ts)
    c = torch.from_numpy(codes).cuda()
    s = torch.from_numpy(scales).cuda()
    t = torch.tensor([ts], dtype=torch.float32, device="cuda")
    for dt in dtypes:
        y = b.dequantize(c, s, t, dtype=dt).cpu()
        want = torch.from_numpy(y_ref).to(dt)
        if dt == torch.float32:
            same = torch.equal(y.view(torch.int32), want.view(torch.int32))
        else:
            same = torch.equal(y.view(torch.int16), want.view(torch.int16))
        assert same, f"{label}: dequantize to {dt} differs"


# ------------------------------------------------------------- workloads --

def test_small_fp32_workload():
    check_quant(workloads.small_fp32(0), "small_fp32_256x1024")


def test_llm_weight_workload():
    check_quant(workloads.llm_weight(0), "weight_bf16_4096x4096")


def test_activation_workload():
    check_quant(workloads.activation_outliers(0), "activation_bf16_8192x8192")


def test_gradient_workload():
    check_quant(workloads.hadamard_gradient(0), "gradient_bf16_16384x4096")


def test_linear_operands_quantize():
    a, bb = workloads.linear_operands(0, M=1024, N=512, K=4096)
    check_quant(a, "linear_A_1024x4096", check_deq=False)
    check_quant(bb, "linear_B_512x4096", check_deq=False)


# ------------------------------------------------------------ edge cases --

def test_hand_worked_groups():
    import json, os
    from fractions import Fraction
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_groups.json")))
    xs, scales, codes = [], [], []
    for grp in g["groups"]:
        if "x" in grp:
            xs += [float(v) for v in grp["x"]]
        else:
            xs += [float(np.float32(6 * k) / np.float32(7)) for k in grp["k"]]
        scales.append(int(grp["scale"], 16))
        codes += [int(v, 16) for v in grp["codes"].split()]
    x = torch.tensor([xs], dtype=torch.float32)
    c, s, ts, err = gpu_quant(x)
    assert ts == 1.0 and err == 0
    assert s.tolist() == [scales]
    assert c.tolist() == [codes]


@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (7, 80), (2, 1024), (33, 272), (1000, 16)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_small_and_ragged_shapes(shape, dtype):
    g = torch.Generator().manual_seed(shape[0] * 1000 + shape[1])
    x = (torch.randn(shape, generator=g) * 3).to(dtype)
    check_quant(x, f"ragged {shape} {dtype}")


def test_empty_tensor():
    x = torch.zeros((0, 64), dtype=torch.bfloat16)
    c, s, ts, err = gpu_quant(x)
    assert c.shape == (0, 32) and s.shape == (0, 4) and ts == 1.0 and err == 0


def test_all_zero_tensor():
    x = torch.zeros((5, 64), dtype=torch.bfloat16)
    ref = check_quant(x, "zeros")
    assert not ref["scales"].any() and not ref["codes"].any()


def test_signed_zeros_and_tiny_groups():
    """Groups far below the tensor max: E4M3 subnormal and zero block scales,
    negative values that round to FP4 zero (nibble 0x8)."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    x *= np.exp2(-rng.integers(0, 24, (64, 16))).repeat(16, axis=1).astype(np.float32)
    x[0, 0] = 1000.0
    x[1, :16] = -0.0
    x[2, 16:32] = -1e-6
    ref = check_quant(torch.from_numpy(x), "tiny groups")
    sb = ref["scales"] & 0x7F
    assert (sb == 0).any() and ((sb > 0) & (sb < 8)).any()


def test_saturating_given_scale():
    """A caller-given ts smaller than amax/2688 saturates block scales at 448
    and drives the INT4 clamp path."""
    rng = np.random.default_rng(4)
    x = torch.from_numpy(rng.standard_normal((128, 512)).astype(np.float32)).to(torch.bfloat16)
    amax = float(x.abs().max())
    for factor in (0.25, 0.01):
        check_quant(x, f"saturating ts x{factor}", ts=np.float32(amax / 2688.0 * factor))


def test_exact_ties_on_grids():
    """Groups whose values sit on both grids (0 and +-6 only): equal errors,
    so FP4 is kept."""
    rng = np.random.default_rng(5)
    x = rng.choice(np.array([0.0, 6.0, -6.0], np.float32), (32, 128))
    x[:, ::16] = 6.0
    ref = check_quant(torch.from_numpy(x), "grid ties")
    assert not (ref["scales"] & 0x80).any()


def test_every_bf16_value_through_unit_scale():
    """v = x exactly (amax 6 and ts 1 give a block scale of 1): every bf16
    value in [-6, 6] goes through both candidate roundings."""
    bits = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    vals = bits[np.isfinite(bits) & (np.abs(bits) <= 6.0)]
    pad = (-len(vals)) % 15
    vals = np.concatenate([vals, np.zeros(pad, np.float32)]).reshape(-1, 15)
    x = np.concatenate([np.full((vals.shape[0], 1), 6.0, np.float32), vals], axis=1)
    x = x.reshape(1, -1)
    x = torch.from_numpy(x).to(torch.bfloat16)
    check_quant(x, "all bf16 values", ts=1.0)


def test_block_scale_sweep():
    """Group maxima over the whole bf16 range with ts = 1: the E4M3 block scale
    covers zero, subnormal, normal and saturated codes."""
    bits = (np.arange(0x0001, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    rng = np.random.default_rng(6)
    frac = rng.uniform(-1, 1, (bits.size, 15)).astype(np.float32)
    x = np.concatenate([bits[:, None], bits[:, None] * frac], axis=1)      # one group per row
    x = torch.from_numpy(x).to(torch.bfloat16)
    check_quant(x, "block scale sweep", ts=1.0)


def test_random_fp32_groups_fine_grained():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((512, 1024)) * np.exp2(rng.uniform(-20, 20, (512, 1)))).astype(np.float32)
    check_quant(torch.from_numpy(x), "fp32 random scales", ts=None)


def test_strided_rows_and_unaligned_base():
    """ld_x > cols, and a base address that is 16- but not 32-byte aligned
    (the 128-bit load path)."""
    base = workloads.llm_weight(1, rows=256, cols=1024 + 64)
    x_dev = base.cuda()[:, 8:8 + 1024]            # 16 B offset, row stride 1088
    assert x_dev.data_ptr() % 32 == 16
    x_cpu = base[:, 8:8 + 1024].contiguous()
    ref = oracle.quantize_tensor(x_cpu.float().numpy())
    c, s, ts, err = gpu_quant(x_cpu, x_dev=x_dev)
    assert err == 0 and ts == ref["ts"]
    assert np.array_equal(s, ref["scales"]) and np.array_equal(c, ref["codes"])


def test_dequant_strided_output():
    b = B()
    x = workloads.llm_weight(2, rows=64, cols=512)
    c, s, ts = b.quantize(x.cuda())
    y = torch.zeros((64, 512 + 32), dtype=torch.bfloat16, device="cuda")
    b.if4_dequantize(c, s, ts, y[:, :512])
    torch.cuda.synchronize()
    ref = oracle.dequantize(c.cpu().numpy(), s.cpu().numpy(), np.float32(ts.item()))
    assert torch.equal(y[:, :512].cpu().view(torch.int16), torch.from_numpy(ref).to(torch.bfloat16).view(torch.int16))
    assert not y[:, 512:].any()


def test_decode_f16_matches_oracle():
    b = B()
    x = workloads.llm_weight(3, rows=256, cols=2048)
    c, s, ts = b.quantize(x.cuda())
    d = b.decode_f16(c, s).cpu().numpy()
    ref = oracle.decode_f16(c.cpu().numpy(), s.cpu().numpy())
    assert np.array_equal(d.view(np.uint16), ref.view(np.uint16))


def _same_or_both_nan(got, want):
    """Bit equality, except that any two NaNs match (payloads differ between
    the GPU's and the host's invalid operations)."""
    g, w = got.float().numpy(), want.float().numpy()
    gb = got.view(torch.int16 if got.dtype != torch.float32 else torch.int32).numpy()
    wb = want.view(torch.int16 if want.dtype != torch.float32 else torch.int32).numpy()
    return bool(np.all((gb == wb) | (np.isnan(g) & np.isnan(w))))


def _arbitrary_codes(seed, rows=64, cols=4096):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, (rows, cols // 2), dtype=np.uint8)
    scales = np.tile(np.arange(256, dtype=np.uint8), rows * cols // 16 // 256)
    scales = rng.permutation(scales).reshape(rows, cols // 16)
    codes[0, :] = 0x88                  # every nibble 8: INT4 k = -8, FP4 -0
    return codes, scales


@pytest.mark.parametrize("ts", [1.0, 0.3719, 3.0e-3, 211.5, 1.0e38, -0.5, -0.0, 0.0,
                                float("inf"), float("nan")])
def test_dequantize_every_scale_byte_arbitrary_codes(ts):
    """Arbitrary code bytes (INT4 code 8 included, which the encoder never
    emits) under every scale byte and degenerate tensor scales: every output
    of the dequantizer (per-element table decode) equals the oracle's."""
    b = B()
    codes, scales = _arbitrary_codes(int(abs(ts) * 10) % 97 if np.isfinite(ts) else 5)
    ts32 = np.float32(ts)
    y_ref = oracle.dequantize(codes, scales, ts32)
    c, s = torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda()
    t = torch.tensor([ts32], dtype=torch.float32, device="cuda")
    for dt in (torch.float32, torch.bfloat16, torch.float16):
        y = b.dequantize(c, s, t, dtype=dt).cpu()
        assert _same_or_both_nan(y, torch.from_numpy(y_ref).to(dt)), (ts, dt)


def test_decode_f16_arbitrary_codes():
    """As above for the linear's fp16 operand decode, which takes the
    byte-permute decode, and the per-element table for groups holding INT4
    code 8 (scale bytes 0x7F and 0xFF are E4M3 NaN: their groups decode to
    NaN on both sides)."""
    b = B()
    codes, scales = _arbitrary_codes(9)
    d = b.decode_f16(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda()).cpu()
    ref = torch.from_numpy(oracle.decode_f16(codes, scales))
    assert _same_or_both_nan(d, ref)
    finite = np.isfinite(ref.numpy())
    assert np.array_equal(d.numpy().view(np.uint16)[finite], ref.numpy().view(np.uint16)[finite])


def test_tensor_amax_and_scale_entry_points():
    b = B()
    x = workloads.activation_outliers(1, tokens=512, hidden=1024)
    amax = torch.empty(1, dtype=torch.float32, device="cuda")
    ts = torch.empty(1, dtype=torch.float32, device="cuda")
    b.if4_tensor_amax(x.cuda(), amax)
    b.if4_tensor_scale(amax, ts)
    torch.cuda.synchronize()
    ra = oracle.tensor_amax(x.float().numpy())
    assert amax.item() == ra
    assert np.float32(ts.item()) == oracle.tensor_scale(ra)
    for a in (0.0, 1e-40, 2688.0):
        amax.fill_(a)
        b.if4_tensor_scale(amax, ts)
        assert np.float32(ts.item()) == oracle.tensor_scale(np.float32(a))


def test_nonfinite_input_sets_flag():
    x = torch.randn(4, 64).to(torch.bfloat16)
    x[2, 5] = float("inf")
    _, _, _, err = gpu_quant(x)
    assert err & B().DEV_NONFINITE
    x[2, 5] = float("nan")
    _, _, _, err = gpu_quant(x, ts=1.0)
    assert err & B().DEV_NONFINITE


def test_invalid_given_scale_sets_flag():
    x = torch.randn(4, 64).to(torch.bfloat16)
    for bad in (0.0, -1.0, float("inf"), 1e-40):
        _, _, _, err = gpu_quant(x, ts=bad)
        assert err & B().DEV_BAD_SCALE, bad


def test_repeated_calls_are_deterministic():
    b = B()
    x = workloads.llm_weight(4, rows=512, cols=4096).cuda()
    out = [b.quantize(x) for _ in range(3)]
    torch.cuda.synchronize()
    for c, s, t in out[1:]:
        assert torch.equal(c, out[0][0]) and torch.equal(s, out[0][1]) and torch.equal(t, out[0][2])


def _probe_groups(base15, probes):
    """One group per probe value: 15 fixed values (max |x| = 6) and the probe
    in the last slot, float32, ts = 1 so that v = x exactly."""
    base = np.asarray(base15, np.float32)
    x = np.empty((len(probes), 16), np.float32)
    x[:, :15] = base
    x[:, 15] = probes
    return torch.from_numpy(x.reshape(-1, 256) if len(probes) % 16 == 0 else x)


def _bf16_probe_values():
    bits = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    return bits[np.isfinite(bits) & (np.abs(bits) <= 6.0)]


def test_int4_code_of_every_bf16_value():
    """Groups where INT4 must win (15 values on the k*6/7 grid, off the FP4
    grid), so the INT4 nibble of the probe is stored and compared."""
    ks = [7, 6, 5, 4, 3, 2, 1, -1, -2, -3, -4, -5, -6, -7, 0]
    base = [np.float32(6 * k) / np.float32(7) for k in ks]
    probes = _bf16_probe_values()
    x = _probe_groups(base, probes)
    ref = check_quant(x, "int4 code of every bf16 value", ts=1.0)
    assert (ref["scales"] & 0x80).all()


def test_fp4_code_of_every_bf16_value():
    """Groups where FP4 must win (15 values on the E2M1 grid), so the FP4
    nibble of the probe is stored and compared."""
    base = [6, 4, 3, 2, 1.5, 1, 0.5, -6, -4, -3, -2, -1.5, -1, -0.5, 0]
    probes = _bf16_probe_values()
    x = _probe_groups(base, probes)
    ref = check_quant(x, "fp4 code of every bf16 value", ts=1.0)
    assert not (ref["scales"] & 0x80).any()


# ------------------------------------------------------ comparator formats --

_MODES = {"nvint4": oracle.MODE_NVINT4, "4over6": oracle.MODE_4OVER6}


def check_mode(x_cpu, mode, label, ts=None):
    x_np = x_cpu.float().numpy()
    if ts is None:
        ref = oracle.quantize_tensor(x_np, mode=_MODES[mode])
        ts_ref = ref["ts"]
    else:
        ts_ref = np.float32(ts)
        ref = oracle.quantize(x_np, ts_ref, mode=_MODES[mode])
    codes, scales, ts_g, err = gpu_quant(x_cpu, mode, ts=ts)
    assert err == 0
    assert f32_bits(ts_g) == f32_bits(ts_ref)
    bad_s = np.count_nonzero(scales != ref["scales"])
    bad_c = np.count_nonzero(codes != ref["codes"])
    assert bad_s == 0 and bad_c == 0, f"{label} {mode}: {bad_s} scale / {bad_c} code bytes differ"
    y = B().dequantize(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(),
                       torch.tensor([ts_ref], device="cuda"), dtype=torch.float32).cpu().numpy()
    mse = oracle.mse(x_np, y)
    print(f"[{label} {mode}] mse={mse:.6g} near_ties={int(ref['near'].sum())}")
    return ref


@pytest.mark.parametrize("mode", ["nvint4", "4over6"])
def test_comparators_on_workloads(mode):
    check_mode(workloads.small_fp32(0), mode, "small_fp32_256x1024")
    check_mode(workloads.llm_weight(0), mode, "weight_bf16_4096x4096")
    check_mode(workloads.activation_outliers(0), mode, "activation_bf16_8192x8192")
    check_mode(workloads.hadamard_gradient(0), mode, "gradient_bf16_16384x4096")


@pytest.mark.parametrize("mode", ["nvint4", "4over6"])
def test_comparators_edge_cases(mode):
    rng = np.random.default_rng(21)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    x *= np.exp2(-rng.integers(0, 24, (64, 16))).repeat(16, axis=1).astype(np.float32)
    x[0, 0] = 1000.0
    x[1, :16] = -0.0
    check_mode(torch.from_numpy(x), mode, "tiny groups")
    check_mode(torch.zeros((3, 48)), mode, "zeros")
    w = torch.from_numpy(rng.standard_normal((128, 512)).astype(np.float32)).to(torch.bfloat16)
    amax = float(w.abs().max())
    check_mode(w, mode, "saturating ts", ts=np.float32(amax / 2688.0 * 0.05))
    for shape in [(1, 16), (3, 48), (33, 272)]:
        for dt in (torch.float32, torch.bfloat16, torch.float16):
            check_mode((torch.randn(shape) * 2).to(dt), mode, f"ragged {shape} {dt}")
    bits = (np.arange(0x0001, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    frac = rng.uniform(-1, 1, (bits.size, 15)).astype(np.float32)
    sweep = np.concatenate([bits[:, None], bits[:, None] * frac], axis=1)
    check_mode(torch.from_numpy(sweep).to(torch.bfloat16), mode, "block scale sweep", ts=1.0)


def test_mse_ordering_on_workloads():
    """Per-group IF4 error never exceeds NVFP4's or NVINT4's, and 4/6 never
    exceeds NVFP4's (the formats' own guarantees, here on GPU outputs)."""
    x = workloads.llm_weight(5, rows=512, cols=4096)
    xd = x.float().numpy().astype(np.float64)
    errs = {}
    for mode in ("if4", "nvfp4", "nvint4", "4over6"):
        c, s, ts = B().quantize(x.cuda(), mode)
        y = B().dequantize(c, s, ts, dtype=torch.float32).cpu().numpy().astype(np.float64)
        errs[mode] = ((xd - y) ** 2).reshape(x.shape[0], -1, 16).sum(-1)
    slack = 1 + 1e-6
    assert np.all(errs["if4"] <= errs["nvfp4"] * slack + 1e-30)
    assert np.all(errs["4over6"] <= errs["nvfp4"] * slack + 1e-30)
    tot = {k: float(v.sum()) for k, v in errs.items()}
    print("[mse ordering] " + " ".join(f"{k}={v:.4g}" for k, v in tot.items()))
    assert tot["if4"] < tot["nvfp4"] and tot["if4"] < tot["nvint4"]


# -------------------------------------- random-sign Hadamard + quantize --

def check_rht(x_cpu, signs, label, ts=None):
    b = B()
    x_np = x_cpu.float().numpy()
    y = oracle.rht(x_np, signs)
    if ts is None:
        ref = oracle.quantize_tensor(y)
        ts_ref = ref["ts"]
    else:
        ts_ref = np.float32(ts)
        ref = oracle.quantize(y, ts_ref)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ts_t = None if ts is None else torch.tensor([ts], dtype=torch.float32, device="cuda")
    codes, scales, ts_g = b.quantize_rht(x_cpu.cuda(), signs, ts=ts_t, err_flag=err)
    amax = torch.empty(1, dtype=torch.float32, device="cuda")
    b.if4_tensor_amax_rht(x_cpu.cuda(), signs, amax)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert amax.item() == oracle.tensor_amax(y)
    assert f32_bits(np.float32(ts_g.item())) == f32_bits(ts_ref)
    c, s = codes.cpu().numpy(), scales.cpu().numpy()
    assert np.count_nonzero(s != ref["scales"]) == 0 and np.count_nonzero(c != ref["codes"]) == 0, label
    nv = oracle.quantize(y, ts_ref, mode=oracle.MODE_NVFP4)
    yd = y.astype(np.float64)
    e_if4 = oracle.mse(yd, oracle.dequantize(c, s, ts_ref))
    e_nv = oracle.mse(yd, oracle.dequantize(nv["codes"], nv["scales"], ts_ref))
    print(f"[rht {label}] int4_frac={oracle.group_int4_fraction(s):.4f} "
          f"mse if4={e_if4:.4g} nvfp4={e_nv:.4g} near_ties={int(ref['near'].sum())}")


@pytest.mark.parametrize("signs", [0x0000, 0xFFFF, 0x6A3C])
def test_rht_quantize_on_gradient_like_data(signs):
    rng = np.random.default_rng(31)
    x = (rng.standard_normal((2048, 1024)) * 1e-3).astype(np.float32)
    check_rht(torch.from_numpy(x).to(torch.bfloat16), signs, f"normal {signs:#06x}")
    t = (rng.standard_t(3, (1024, 1024)) * 1e-3).astype(np.float32)
    check_rht(torch.from_numpy(t).to(torch.bfloat16), signs, f"student-t {signs:#06x}")


def test_rht_quantize_extreme_magnitudes():
    """The IF4 path with the transform scales v by fl(inv / 4) on H x: groups
    from 2^-110 to 2^121 in magnitude (the largest group's inverse scale
    below 2^-122, where the kernels leave that path; tiny groups whose H x
    elements are subnormal beside a normal amax), and a given tensor scale
    that puts most groups there; codes and scales equal the oracle's."""
    rng = np.random.default_rng(41)
    x = rng.standard_normal((64, 1024)).astype(np.float64)
    x *= np.exp2(rng.integers(-110, 122, (64, 64))).repeat(16, axis=1)
    x[0, :16] = np.ldexp(1.0, 123)          # no sign flips: H x = 2^127 (finite), y = 2^125
    x[1, :16] = np.where(np.arange(16) == 3, np.ldexp(1.0, 20), np.ldexp(1.0, -130))
    x = x.astype(np.float32)
    check_rht(torch.from_numpy(x), 0x0000, "extreme magnitudes")
    check_rht(torch.from_numpy(x), 0x0001, "extreme magnitudes, given ts",
              ts=np.float32(np.ldexp(1.0, 116)))


def test_rht_quantize_dtypes_shapes_and_given_scale():
    rng = np.random.default_rng(32)
    for shape in [(1, 16), (7, 80), (33, 272)]:
        for dt in (torch.float32, torch.bfloat16, torch.float16):
            check_rht((torch.randn(shape) * 3).to(dt), 0x1357, f"{shape} {dt}")
    w = torch.from_numpy(rng.standard_normal((256, 512)).astype(np.float32))
    check_rht(w, 0xBEEF, "given ts", ts=np.float32(float(w.abs().max()) / 2688.0 * 0.1))
    check_rht(torch.zeros((4, 64)), 0xFFFF, "zeros")


@pytest.mark.parametrize("ts", [2.0 ** -117, 2.0 ** -100, 2.0 ** 100, 2.0 ** 117])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_extreme_given_scales(ts, dtype):
    """Valid tensor scales at the ends of the allowed range, on rows whose
    magnitudes run from float32 subnormals to 3e38.  Under a tiny ts most block
    scales saturate at 448 and x * inv overflows the float32 range for large
    rows (the INT4 clamp, the general path, infinite errors in the binary64
    rule), while subnormal rows get ordinary block scales; under a huge ts most
    block scales underflow to zero.  Codes and scale bytes must equal the
    oracle's, for IF4 and for the comparators."""
    rng = np.random.default_rng(int(np.log2(ts)) + 200)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    # row magnitudes from float32 subnormals (2^-140) to near the top of the range
    mags = np.exp2(np.array([-140, -130, -124, -118, -110, -60, 0, 60, 100], np.float64))
    x *= mags[np.arange(64) % mags.size, None].astype(np.float32)
    x[3, :16] = np.float32(3e38)
    xt = torch.from_numpy(x).to(dtype)
    x_np = xt.float().numpy()
    ref = oracle.quantize(x_np, np.float32(ts))
    c, s, t, err = gpu_quant(xt, "if4", ts=np.float32(ts))
    assert err == 0
    assert np.array_equal(s, ref["scales"]), (ts, dtype)
    assert np.array_equal(c, ref["codes"]), (ts, dtype)
    for mode, omode in (("nvfp4", oracle.MODE_NVFP4), ("nvint4", oracle.MODE_NVINT4),
                        ("4over6", oracle.MODE_4OVER6)):
        r2 = oracle.quantize(x_np, np.float32(ts), mode=omode)
        c2, s2, _, e2 = gpu_quant(xt, mode, ts=np.float32(ts))
        assert e2 == 0
        assert np.array_equal(s2, r2["scales"]) and np.array_equal(c2, r2["codes"]), (mode, ts)
