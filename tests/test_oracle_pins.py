"""Pins for the CPU oracle: each check compares it with something other than
itself -- brute force over the format's grids, torch's float8_e4m3fn cast,
exact rational arithmetic, the hand-worked groups in tests/golden, and
invariants the format must satisfy.  No GPU is needed.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_groups.json")

# The E2M1 magnitude set printed for the format (gist.science section 1; the
# NVFP4 element type), indexed by the 3-bit magnitude code.
E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float64)


def all_bf16_as_f32(finite_only=True):
    bits = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    return bits[np.isfinite(bits)] if finite_only else bits


def f32_round(fr: Fraction) -> np.float32:
    """Correctly rounded (RNE) float32 of an exact rational, by bracketing."""
    f = np.float32(float(fr))          # within an ulp; fix up by neighbours
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    best = min(cands, key=lambda c: (abs(Fraction(float(c)) - fr),
                                     int(np.float32(c).view(np.uint32)) & 1))
    return np.float32(best)


# --------------------------------------------------------------- E4M3 -----

def e4m3_table_from_torch():
    """Values of the 127 non-negative finite E4M3 codes, by torch's decoder."""
    codes = torch.arange(0, 127, dtype=torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def brute_e4m3_encode(f):
    """Nearest of the 127 non-negative finite E4M3 values, ties to the even
    code; anything above 448 maps to 448 (saturating, never NaN)."""
    table = e4m3_table_from_torch()
    # above the table every value is nearest to 448; clipping keeps that true
    # while avoiding distances that all round to the same huge float64
    f = np.minimum(np.asarray(f, np.float64), 1e4)
    dist = np.abs(f[:, None] - table[None, :])
    dmin = dist.min(axis=1, keepdims=True)
    is_min = dist == dmin
    even = is_min & ((np.arange(127) % 2) == 0)[None, :]
    pick_even = even.any(axis=1)
    return np.where(pick_even, even.argmax(axis=1), is_min.argmax(axis=1)).astype(np.uint8)


def test_e4m3_value_table_matches_torch_and_anchors():
    table = e4m3_table_from_torch()
    ours = np.array([oracle.e4m3_value(c) for c in range(127)], np.float64)
    assert np.array_equal(ours, table)
    # bit 7 (the IF4 type bit) is ignored by the scale decoder
    assert all(oracle.e4m3_value(c | 0x80) == oracle.e4m3_value(c) for c in range(127))
    assert oracle.e4m3_value(0x38) == 1.0
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x08) == 2.0 ** -6
    assert np.isnan(oracle.e4m3_value(0x7F))
    assert np.all(np.diff(table) > 0)


def e4m3_probe_values():
    table = e4m3_table_from_torch().astype(np.float32)
    mids = ((table[:-1].astype(np.float64) + table[1:]) / 2).astype(np.float32)
    vals = [table, mids]
    for arr in (table, mids):
        up, dn = arr.copy(), arr.copy()
        for _ in range(2):
            up = np.nextafter(up, np.float32(np.inf))
            dn = np.nextafter(dn, np.float32(0))
            vals += [up, dn]
    b = all_bf16_as_f32()
    vals.append(b[(b > 0) & (b < 1e6)])
    rng = np.random.default_rng(1234)
    vals.append(np.exp2(rng.uniform(-24, 12, 400_000)).astype(np.float32))
    vals.append(np.array([0.0, 1e-45, 2.0 ** -126, 2.0 ** -10, 2.0 ** -10 * 1.0000001,
                          448.0, 463.99, 464.0, 464.0001, 1e30, 3.4e38], np.float32))
    v = np.concatenate(vals).astype(np.float32)
    return v[v >= 0]


def test_e4m3_encode_vs_bruteforce():
    v = e4m3_probe_values()
    got = oracle.e4m3_encode_array(v)
    for lo in range(0, v.size, 50_000):
        sl = slice(lo, lo + 50_000)
        assert np.array_equal(got[sl], brute_e4m3_encode(v[sl])), lo


def test_e4m3_encode_vs_torch_cast():
    v = e4m3_probe_values()
    v = v[v < 464.0]                   # torch's cast is non-saturating above
    got = oracle.e4m3_encode_array(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)
    assert np.all(oracle.e4m3_encode_array(np.array([464.0, 465.0, 1e30], np.float32)) == 0x7E)


def test_e4m3_encode_closed_forms():
    assert oracle.e4m3_encode(1.0) == 0x38
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(2.0 ** -9) == 0x01
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00          # tie -> even code 0
    assert oracle.e4m3_encode(1.5 * 2.0 ** -9) == 0x02     # tie between 0x01, 0x02
    assert oracle.e4m3_encode(5.0 / 6.0) == 0x35           # 0.8125
    assert oracle.e4m3_encode(1.0625) == 0x38              # tie 1.0 / 1.125 -> even
    assert oracle.e4m3_encode(1.1875) == 0x3A              # tie 1.125 / 1.25 -> even


# --------------------------------------------------------------- E2M1 -----

def brute_e2m1_nibble(v):
    v = np.asarray(v, np.float32)
    a = np.minimum(np.abs(v.astype(np.float64)), 1e4)   # see brute_e4m3_encode
    dist = np.abs(a[:, None] - E2M1_MAGS[None, :])
    dmin = dist.min(axis=1, keepdims=True)
    is_min = dist == dmin
    even = is_min & ((np.arange(8) % 2) == 0)[None, :]
    code = np.where(even.any(axis=1), even.argmax(axis=1), is_min.argmax(axis=1))
    return (code | (np.signbit(v).astype(np.int64) << 3)).astype(np.uint8)


def grid_probe_values(grid):
    grid = np.asarray(grid, np.float64)
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    vals = [grid.astype(np.float32), mids]
    for arr in (grid.astype(np.float32), mids):
        up, dn = arr.copy(), arr.copy()
        for _ in range(3):
            up = np.nextafter(up, np.float32(np.inf))
            dn = np.nextafter(dn, np.float32(-np.inf))
            vals += [up, dn]
    v = np.concatenate(vals)
    return np.concatenate([v, -v])


def test_e2m1_value_set():
    vals = [oracle.e2m1_value(n) for n in range(16)]
    assert vals[:8] == list(E2M1_MAGS)
    assert vals[8:] == [-m for m in E2M1_MAGS]
    assert np.signbit(oracle.e2m1_value(8))


def test_e2m1_rounding_vs_bruteforce():
    v = np.concatenate([all_bf16_as_f32(), grid_probe_values(list(E2M1_MAGS) + [8.0]),
                        np.random.default_rng(7).uniform(-8, 8, 200_000).astype(np.float32)])
    assert np.array_equal(oracle.e2m1_nibble_array(v), brute_e2m1_nibble(v))


def test_e2m1_named_ties_and_signed_zero():
    # midpoints go to the even code; a negative value rounding to 0 keeps sign
    expect = [(0.25, 0x0), (0.75, 0x2), (1.25, 0x2), (1.75, 0x4), (2.5, 0x4), (3.5, 0x6),
              (5.0, 0x6), (5.0000005, 0x7), (7.0, 0x7), (1e30, 0x7), (-0.1, 0x8),
              (-0.0, 0x8), (0.0, 0x0), (-1.25, 0xA)]
    for v, n in expect:
        assert oracle.e2m1_nibble(v) == n, v


# ------------------------------------------------------- scaled INT4 -----

def exact_int4_grid():
    """fl32(6k/7) for k = -7..7, from exact rationals."""
    return {k: f32_round(Fraction(6 * k, 7)) for k in range(-7, 8)}


def test_int4_value_set():
    grid = exact_int4_grid()
    for nib in range(16):
        if nib == 8:
            continue
        k = nib - 16 if nib & 8 else nib
        assert np.float32(oracle.int4_value(nib)) == grid[k], nib
    assert oracle.int4_value(7) == 6.0 and oracle.int4_value(9) == -6.0
    assert max(abs(oracle.int4_value(n)) for n in range(16) if n != 8) == 6.0


def brute_int4_nibble(v):
    """Nearest integer in [-7, 7] to the exact product v * fl(7/6) (exact in
    float64: 24-bit times 24-bit), ties to even."""
    v = np.asarray(v, np.float32)
    t = v.astype(np.float64) * np.float64(np.float32(7.0) / np.float32(6.0))
    t = np.clip(t, -1e4, 1e4)                             # see brute_e4m3_encode
    ks = np.arange(-7, 8, dtype=np.float64)
    dist = np.abs(t[:, None] - ks[None, :])
    dmin = dist.min(axis=1, keepdims=True)
    is_min = dist == dmin
    even = is_min & ((np.arange(-7, 8) % 2) == 0)[None, :]
    idx = np.where(even.any(axis=1), even.argmax(axis=1), is_min.argmax(axis=1))
    return (ks[idx].astype(np.int64) & 0xF).astype(np.uint8)


def test_int4_rounding_vs_bruteforce():
    grid = np.array([float(g) for g in exact_int4_grid().values()])
    v = np.concatenate([all_bf16_as_f32(), grid_probe_values(grid),
                        grid_probe_values(np.arange(-8, 9) * 6.0 / 7.0 + 3.0 / 7.0),
                        np.random.default_rng(8).uniform(-8, 8, 200_000).astype(np.float32)])
    assert np.array_equal(oracle.int4_nibble_array(v), brute_int4_nibble(v))


def test_int4_rounding_is_nearest_in_exact_arithmetic():
    """Away from a midpoint, k is the integer nearest to v*7/6 computed exactly
    (clamped to +-7): the fp32 pre-scale never moves a value across a
    boundary by more than a couple of ulps."""
    v = np.concatenate([all_bf16_as_f32(), np.random.default_rng(9).uniform(-7, 7, 100_000)
                        .astype(np.float32)])
    v = v[np.abs(v) < 64]
    t = v.astype(np.float64) * 7.0 / 6.0
    frac = np.abs(t - np.floor(t) - 0.5)
    keep = frac > 1e-6
    k = np.clip(np.round(t[keep]), -7, 7).astype(np.int64) & 0xF
    assert np.array_equal(oracle.int4_nibble_array(v[keep]), k.astype(np.uint8))


def test_int4_named_cases():
    # 3 * fl(7/6) = 3.49999988..., just below the midpoint: k = 3 (the value
    # 3 is equidistant from 18/7 and 24/7, so either k has the same error)
    assert oracle.int4_nibble(3.0) == 3
    assert oracle.int4_nibble(-3.0) == 0xD
    assert oracle.int4_nibble(6.0) == 7
    assert oracle.int4_nibble(-6.0) == 9         # -7
    assert oracle.int4_nibble(1e30) == 7 and oracle.int4_nibble(-1e30) == 9
    assert oracle.int4_nibble(-0.1) == 0         # integer zero has no sign


# ------------------------------------------------------- tensor scale -----

def test_tensor_scale_closed_forms():
    assert oracle.tensor_scale(2688.0) == 1.0
    assert oracle.tensor_scale(0.0) == 1.0
    assert oracle.tensor_scale(1.0) == f32_round(Fraction(1, 2688))
    assert oracle.tensor_scale(448.0 * 6 * 2.0 ** 10) == 2.0 ** 10
    assert oracle.tensor_scale(1e-40) == np.float32(2.0 ** -117)
    x = np.zeros((3, 32), np.float32)
    x[2, 17] = -7.25
    assert oracle.tensor_amax(x) == 7.25


# ------------------------------------------------------ hand-worked groups --

def golden_tensor():
    g = json.load(open(GOLDEN))
    xs, scales, codes, deq = [], [], [], []
    for grp in g["groups"]:
        if "x" in grp:
            x = [float(s) if not isinstance(s, str) else float(s) for s in grp["x"]]
        else:
            x = [float(f32_round(Fraction(6 * k, 7))) for k in grp["k"]]
        xs += x
        scales.append(int(grp["scale"], 16))
        codes += [int(b, 16) for b in grp["codes"].split()]
        if "dequant" in grp:
            deq += [float(s) for s in grp["dequant"]]
        else:
            deq += x
    x = np.array([xs], np.float32)
    return g, x, np.array([scales], np.uint8), np.array([codes], np.uint8), np.array([deq], np.float32)


def test_hand_worked_groups():
    g, x, scales, codes, deq = golden_tensor()
    q = oracle.quantize_tensor(x)
    assert q["amax"] == g["amax"] and q["ts"] == g["ts"]
    assert np.array_equal(q["scales"], scales)
    assert np.array_equal(q["codes"], codes)
    y = oracle.dequantize(q["codes"], q["scales"], q["ts"])
    assert np.array_equal(y, deq)
    assert np.array_equal(np.signbit(y), np.signbit(deq))        # H5's signed zeros


# ------------------------------------------ brute force over a group's codes --

def bruteforce_group(x16, ts):
    """For one group: the scale byte by brute-force E4M3 search, then the
    minimum-error nibble of each element over all 16 codes of each type, in
    float64 over the float32 scaled values."""
    x16 = np.asarray(x16, np.float32)
    amax = np.max(np.abs(x16))
    sb_f = (amax / np.float32(6.0)) / np.float32(ts)
    sb = int(brute_e4m3_encode(np.array([sb_f]))[0])
    if sb == 0:
        return sb, None
    e4 = e4m3_table_from_torch()[sb]
    eff = np.float32(np.float32(e4) * np.float32(ts))
    inv = np.float32(np.float32(1.0) / eff)
    v = (x16 * inv).astype(np.float32).astype(np.float64)
    fp_vals = np.array([m if n < 8 else -m for n, m in
                        ((n, E2M1_MAGS[n & 7]) for n in range(16))], np.float64)
    int_vals = np.array([float(f32_round(Fraction(6 * (n - 16 if n & 8 else n), 7)))
                         for n in range(16)], np.float64)
    int_vals[8] = np.inf                 # 0x8 (-8) is not a code
    err_fp = (v[:, None] - fp_vals[None, :]) ** 2
    err_int = (v[:, None] - int_vals[None, :]) ** 2
    return sb, dict(v=v, fp_vals=fp_vals, int_vals=int_vals,
                    min_fp=err_fp.min(axis=1), min_int=err_int.min(axis=1))


def unpack(codes_row):
    c = np.asarray(codes_row, np.uint8)
    out = np.empty(c.size * 2, np.uint8)
    out[0::2] = c & 0xF
    out[1::2] = c >> 4
    return out


@pytest.mark.parametrize("dist", ["normal", "uniform", "student", "outlier", "tiny"])
def test_group_choice_vs_bruteforce(dist):
    rng = np.random.default_rng({"normal": 1, "uniform": 2, "student": 3,
                                 "outlier": 4, "tiny": 5}[dist])
    rows, cols = 64, 256
    if dist == "normal":
        x = rng.standard_normal((rows, cols))
    elif dist == "uniform":
        x = rng.uniform(-1, 1, (rows, cols))
    elif dist == "student":
        x = rng.standard_t(3, (rows, cols))
    elif dist == "outlier":
        x = rng.standard_normal((rows, cols))
        x[:, rng.choice(cols, 5, replace=False)] *= 50
    else:
        x = rng.standard_normal((rows, cols)) * np.exp2(rng.integers(-30, 0, (rows, 1)))
    x = x.astype(np.float32)
    q = oracle.quantize_tensor(x)
    ts = q["ts"]
    n_checked = 0
    for r in range(rows):
        nib = unpack(q["codes"][r])
        for gi in range(cols // 16):
            sb, bf = bruteforce_group(x[r, gi * 16:(gi + 1) * 16], ts)
            byte = int(q["scales"][r, gi])
            assert byte & 0x7F == sb
            nibs = nib[gi * 16:(gi + 1) * 16]
            if sb == 0:
                assert byte == 0 and not nibs.any()
                continue
            is_int = bool(byte & 0x80)
            vals = bf["int_vals"] if is_int else bf["fp_vals"]
            err = (bf["v"] - vals[nibs]) ** 2
            best = bf["min_int"] if is_int else bf["min_fp"]
            # each element takes a minimum-error code of its group's type
            # (INT4 rounds in the 7/6-scaled domain: allow float32 slack)
            assert np.all(err <= best * (1 + 1e-5) + 1e-30)
            e_fp, e_int = bf["min_fp"].sum(), bf["min_int"].sum()
            assert abs(q["e_fp"][r, gi] - e_fp) <= 1e-12 * max(e_fp, 1e-300)
            assert q["e_int"][r, gi] >= e_int * (1 - 1e-12)
            assert q["e_int"][r, gi] <= e_int * (1 + 1e-5) + 1e-30
            if abs(e_fp - e_int) > 1e-4 * max(e_fp, e_int):
                assert is_int == (e_int < e_fp)
            assert min(q["e_fp"][r, gi], q["e_int"][r, gi]) <= q["e_fp"][r, gi]
            n_checked += 1
    assert n_checked > 0


# ------------------------------------------------------------ invariants -----

def _workload_like(seed, rows=128, cols=512):
    rng = np.random.default_rng(seed)
    parts = [rng.standard_normal((rows, cols)),
             rng.standard_t(3, (rows, cols)) * 0.02,
             rng.uniform(-1, 1, (rows, cols))]
    return [p.astype(np.float32) for p in parts]


def test_storage_is_4p5_bits_per_value():
    for x in _workload_like(11):
        q = oracle.quantize_tensor(x)
        assert (q["codes"].nbytes + q["scales"].nbytes) * 8 == 4.5 * x.size


def test_if4_never_worse_than_nvfp4_and_fp4_groups_identical():
    for x in _workload_like(12):
        q = oracle.quantize_tensor(x)
        n = oracle.quantize(x, q["ts"], mode=oracle.MODE_NVFP4)
        assert np.all((n["scales"] & 0x80) == 0)
        assert np.array_equal(n["scales"], q["scales"] & 0x7F)
        fp_groups = (q["scales"] & 0x80) == 0
        cq = q["codes"].reshape(x.shape[0], -1, 8)
        cn = n["codes"].reshape(x.shape[0], -1, 8)
        assert np.array_equal(cq[fp_groups], cn[fp_groups])
        e_if4 = np.where(fp_groups, q["e_fp"], q["e_int"])
        assert np.all(e_if4 <= n["e_fp"])
        # same in the x domain, up to the rounding of the decode
        yq = oracle.dequantize(q["codes"], q["scales"], q["ts"]).astype(np.float64)
        yn = oracle.dequantize(n["codes"], n["scales"], q["ts"]).astype(np.float64)
        xd = x.astype(np.float64)
        gq = ((xd - yq) ** 2).reshape(x.shape[0], -1, 16).sum(-1)
        gn = ((xd - yn) ** 2).reshape(x.shape[0], -1, 16).sum(-1)
        assert np.all(gq <= gn * (1 + 1e-6) + 1e-30)
        assert oracle.mse(x, yq) < oracle.mse(x, yn)


@pytest.mark.parametrize("j", [-5, 3, 20])
def test_power_of_two_scaling_invariance(j):
    for x in _workload_like(13):
        q = oracle.quantize_tensor(x)
        q2 = oracle.quantize_tensor(x * np.float32(2.0 ** j))
        assert q2["ts"] == q["ts"] * np.float32(2.0 ** j)
        assert np.array_equal(q["codes"], q2["codes"])
        assert np.array_equal(q["scales"], q2["scales"])


def test_negation_symmetry():
    for x in _workload_like(14):
        q = oracle.quantize_tensor(x)
        qn = oracle.quantize_tensor(-x)
        assert np.array_equal(q["scales"], qn["scales"])
        rows = x.shape[0]
        n = np.stack([unpack(c) for c in q["codes"]]).reshape(rows, -1, 16)
        nn = np.stack([unpack(c) for c in qn["codes"]]).reshape(rows, -1, 16)
        is_int = ((q["scales"] & 0x80) != 0)[:, :, None]
        zero_scale = (q["scales"] == 0)[:, :, None]
        expect = np.where(is_int, (-(n.astype(np.int64) - 16 * (n >= 8))) & 0xF, n ^ 0x8)
        expect = np.where(zero_scale, 0, expect)
        assert np.array_equal(nn, expect.astype(np.uint8))


def test_permutation_within_group():
    rng = np.random.default_rng(15)
    for x in _workload_like(15):
        perm = rng.permutation(16)
        xp = x.reshape(x.shape[0], -1, 16)[:, :, perm].reshape(x.shape)
        q = oracle.quantize_tensor(x)
        qp = oracle.quantize_tensor(xp)
        rows = x.shape[0]
        n = np.stack([unpack(c) for c in q["codes"]]).reshape(rows, -1, 16)
        npm = np.stack([unpack(c) for c in qp["codes"]]).reshape(rows, -1, 16)
        same = q["scales"] == qp["scales"]
        # the fp64 error sums see another order: only a near tie may flip
        assert np.all(same | (q["near"] == 1))
        assert np.array_equal(n[:, :, perm][same], npm[same])


# ----------------------------------------------------------- dequantize -----

def test_dequant_roundtrip_on_grid():
    """Values built on a group's grid come back exactly."""
    rng = np.random.default_rng(16)
    rows, groups = 32, 16
    x = np.zeros((rows, groups * 16), np.float32)
    want_int = np.zeros((rows, groups), bool)
    int_grid = np.array([float(f32_round(Fraction(6 * k, 7))) for k in range(-7, 8)], np.float32)
    for r in range(rows):
        for g in range(groups):
            e4 = np.float32(e4m3_table_from_torch()[rng.integers(40, 110)])
            if rng.random() < 0.5:
                vals = rng.choice(np.concatenate([E2M1_MAGS, -E2M1_MAGS]).astype(np.float32), 16)
            else:
                vals = rng.choice(int_grid, 16)
                vals[1] = int_grid[9]                    # 6/7*2: off the FP4 grid
                want_int[r, g] = True
            vals[0] = 6.0
            x[r, g * 16:(g + 1) * 16] = (vals * e4).astype(np.float32)
    x[0, 0] = np.float32(6.0 * 448.0)                    # amax 2688 -> ts = 1
    x[0, 1:16] = 0
    want_int[0, 0] = False
    q = oracle.quantize_tensor(x)
    assert q["ts"] == 1.0
    assert np.array_equal((q["scales"] >> 7).astype(bool), want_int)
    y = oracle.dequantize(q["codes"], q["scales"], q["ts"])
    assert np.array_equal(y, x)


def test_dequant_error_bound():
    """|x - xhat| is at most half the widest grid gap (1 for FP4, 3/7 for
    INT4) times the decoded block scale, when the group does not saturate."""
    for x in _workload_like(17):
        q = oracle.quantize_tensor(x)
        y = oracle.dequantize(q["codes"], q["scales"], q["ts"])
        e4 = e4m3_table_from_torch()[(q["scales"] & 0x7F).astype(np.int64)]
        eff = (e4 * np.float64(q["ts"]))[:, :, None]
        amax = np.abs(x).reshape(x.shape[0], -1, 16).max(-1)[:, :, None]
        ok = (amax / eff <= 6.0)[..., 0]
        gap = np.where((q["scales"] & 0x80) != 0, 3.0 / 7.0, 1.0)[:, :, None]
        err = np.abs(x.astype(np.float64) - y).reshape(x.shape[0], -1, 16)
        assert np.all((err <= gap * eff * (1 + 1e-6))[ok])


# --------------------------------------------------------- linear operand --

def test_decode_f16_exact_for_fp4_and_rounded_for_int4():
    x = _workload_like(18, rows=64, cols=256)[0]
    q = oracle.quantize_tensor(x)
    d = oracle.decode_f16(q["codes"], q["scales"])
    e4 = e4m3_table_from_torch()
    for r in range(0, 64, 7):
        nib = unpack(q["codes"][r])
        for g in range(16):
            s = int(q["scales"][r, g])
            for i in range(16):
                n = int(nib[g * 16 + i])
                if s & 0x80:
                    k = n - 16 if n & 8 else n
                    exact = Fraction(float(f32_round(Fraction(6 * k, 7)))) * Fraction(e4[s & 0x7F])
                    got = Fraction(float(d[r, g * 16 + i]))
                    ulp = Fraction(float(np.spacing(np.float16(abs(float(exact)) or 1e-8))))
                    assert abs(got - exact) <= ulp
                else:
                    m = Fraction(E2M1_MAGS[n & 7]) * (-1 if n & 8 else 1)
                    assert Fraction(float(d[r, g * 16 + i])) == m * Fraction(e4[s & 0x7F])


def test_linear_oracle_exact_small():
    rng = np.random.default_rng(19)
    M, N, K = 5, 3, 48
    a = rng.choice(np.concatenate([E2M1_MAGS, -E2M1_MAGS]), (M, K)) * 2.0 ** rng.integers(-4, 4, (M, 1))
    b = rng.choice(np.concatenate([E2M1_MAGS, -E2M1_MAGS]), (N, K)) * 2.0 ** rng.integers(-4, 4, (N, 1))
    c = oracle.linear(a.astype(np.float32), b.astype(np.float32))
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(a[m, k])) * Fraction(float(b[n, k])) for k in range(K))
            assert Fraction(float(c[m, n])) == exact
    sub = oracle.linear(a.astype(np.float32), b.astype(np.float32), rows=[4, 1], cols=[2])
    assert sub.shape == (2, 1) and sub[0, 0] == c[4, 2] and sub[1, 0] == c[1, 2]


# ---------------------------------------- rounding order (readings R2, R4) --
#
# The pages give the block scale as amax/6 over the tensor scale and the
# scaled value as x over the decoded block scale, without an order of
# rounding.  The reading taken (R2) is sb = E4M3(fl(fl(amax/6)/ts)), and
# (R4) v = fl(x * fl(1/eff)) with eff = fl(E4M3(sb) * ts).  Random groups
# almost never land where another order would round differently, so these
# pins search (seeded) for inputs that sit exactly there, and compute the
# expected codes from exact rationals with an explicit float32 rounding at
# each step the reading states.

def _fl(fr):
    return f32_round(Fraction(fr))


def _e4m3_code(f):
    return int(brute_e4m3_encode(np.array([float(f)]))[0])


def _e2m1_nibble_exact(v):
    """Nearest E2M1 value to float v, ties to the even magnitude code."""
    a = abs(Fraction(float(v)))
    dist = [abs(a - Fraction(m)) for m in E2M1_MAGS]
    best = min(range(8), key=lambda c: (dist[c], c & 1))
    if a > 6:
        best = 7
    return (8 if np.signbit(v) else 0) | best


def _int4_nibble_exact(v):
    """k = RNE(v * fl(7/6)) with the product exact, clamped to [-7, 7]."""
    p = Fraction(float(v)) * Fraction(float(np.float32(7.0) / np.float32(6.0)))
    k = round(p)                       # Python rounds Fractions half to even
    k = max(-7, min(7, k))
    return k & 0xF


def _block_scale_cases(n):
    rng = np.random.default_rng(2024)
    table = e4m3_table_from_torch()
    cases = []
    while len(cases) < n:
        c = int(rng.integers(8, 125))
        mid = Fraction(float(table[c])) + (Fraction(float(table[c + 1])) - Fraction(float(table[c]))) / 2
        ts = np.float32(rng.uniform(1.0, 2.0) * 2.0 ** int(rng.integers(-30, 0)))
        a = np.float32(float(mid * 6 * Fraction(float(ts))))
        for _ in range(200):
            r2 = _fl(Fraction(float(_fl(Fraction(float(a)) / 6))) / Fraction(float(ts)))
            alt1 = _fl(Fraction(float(a)) / Fraction(float(_fl(6 * Fraction(float(ts))))))
            alt2 = _fl(Fraction(float(a)) / (6 * Fraction(float(ts))))
            want = _e4m3_code(r2)
            if want != _e4m3_code(alt1) or want != _e4m3_code(alt2):
                cases.append((a, ts, want))
                break
            a = np.nextafter(a, np.float32(np.inf) if rng.integers(2) else np.float32(-np.inf))
    return cases


def test_block_scale_rounding_order():
    """R2: groups whose amax puts fl(fl(amax/6)/ts) next to an E4M3 rounding
    midpoint, where amax/fl(6 ts) or a single rounding of amax/(6 ts) would
    give the neighbouring code."""
    for a, ts, want in _block_scale_cases(12):
        x = np.zeros((1, 16), np.float32)
        x[0, 0] = a
        x[0, 5] = -a * np.float32(0.37)
        q = oracle.quantize(x, ts)
        assert int(q["scales"][0, 0]) & 0x7F == want, (a, ts)


def _scaled_value_cases(n, nibble_fn, mids):
    rng = np.random.default_rng(7)
    table = e4m3_table_from_torch()
    cases = []
    while len(cases) < n:
        sb = int(rng.integers(40, 110))
        e4 = Fraction(float(table[sb]))
        if e4.numerator & (e4.numerator - 1) == 0:
            continue                                   # 1/eff exact: no difference
        ts = np.float32(2.0 ** int(rng.integers(-20, 0)))
        eff = _fl(e4 * Fraction(float(ts)))            # exact here (ts a power of 2)
        inv = _fl(1 / Fraction(float(eff)))
        m = mids[int(rng.integers(len(mids)))]
        x = np.float32(float(Fraction(m) * Fraction(float(eff))))
        for _ in range(64):
            v_r4 = _fl(Fraction(float(x)) * Fraction(float(inv)))
            v_div = _fl(Fraction(float(x)) / Fraction(float(eff)))
            want = nibble_fn(v_r4)
            if want != nibble_fn(v_div) and abs(float(x)) < 6 * float(eff):
                cases.append((sb, ts, eff, x, want))
                break
            x = np.nextafter(x, np.float32(np.inf) if rng.integers(2) else np.float32(-np.inf))
    return cases


@pytest.mark.parametrize("mode", ["fp4", "int4"])
def test_scaled_value_rounding_order(mode):
    """R4: elements x that sit next to an E2M1 (or scaled-INT4) rounding
    boundary, where x / eff would round to the other code than
    x * fl(1/eff).  The group's amax is 6 * eff, so its block scale is the
    chosen code exactly (ts a power of two)."""
    if mode == "fp4":
        fn, mids, omode = _e2m1_nibble_exact, [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], oracle.MODE_NVFP4
    else:
        fn, omode = _int4_nibble_exact, oracle.MODE_NVINT4
        mids = [Fraction(2 * k + 1, 2) * Fraction(6, 7) for k in range(0, 7)]
    for sb, ts, eff, xv, want in _scaled_value_cases(10, fn, mids):
        x = np.zeros((1, 16), np.float32)
        x[0, 0] = np.float32(6.0) * eff              # amax: block scale code sb
        x[0, 3] = xv
        q = oracle.quantize(x, ts, mode=omode)
        assert int(q["scales"][0, 0]) & 0x7F == sb, (sb, ts)
        nib = unpack(q["codes"][0])[3]
        assert int(nib) == want, (mode, sb, float(ts), float(xv), int(nib), want)
