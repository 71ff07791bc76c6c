"""Pins of the oracle's IF6 and IF3 functions, each against something other
than the oracle: the defining properties of the E2M3 and E2M0 grids, exact
rationals for the INT6 and INT3 grids, brute-force nearest-code searches over
every bf16 value, brute force over a group's codes, the bit layout unpacked by
the test's own code, and groups worked by hand.

The pages name IF6 and IF3 and the adaptive choice they share with IF4
(abstract; companion "It Generalizes: IF3 and IF6"; gist.science section 2
"Extensoes") but print no grid for either; the grids pinned here are the
readings the oracle states (FP6 = E2M3 against INT6 k*15/62; FP3 = E2M0
{0, 1, 2, 4} against INT3 k*4/3), not values fixed by the pages.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from test_oracle_pins import (all_bf16_as_f32, brute_e4m3_encode, e4m3_table_from_torch,
                              f32_round)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_groups_widths.json")


def grid_probes(grid, top):
    """Grid points, midpoints, +-3 ulps around both, beyond the top, both signs."""
    g = np.asarray(sorted(set(float(v) for v in grid)), np.float64)
    mids = (g[:-1] + g[1:]) / 2
    pts = [g.astype(np.float32), mids.astype(np.float32)]
    for arr in (g.astype(np.float32), mids.astype(np.float32)):
        up, dn = arr.copy(), arr.copy()
        for _ in range(3):
            up = np.nextafter(up, np.float32(np.inf))
            dn = np.nextafter(dn, np.float32(-np.inf))
            pts += [up, dn]
    pts.append(np.array([top * 1.01, top * 2, 1e30], np.float32))
    v = np.concatenate(pts)
    return np.concatenate([v, -v])


def brute_nearest(values, grid, keys=None):
    """Index of the nearest grid value (float64 distances); a tie goes to the
    entry whose key (its code, or its integer k) is even.  Values beyond the
    grid clip to its ends first."""
    grid = np.asarray(grid, np.float64)
    keys = np.arange(grid.size) if keys is None else np.asarray(keys)
    a = np.clip(np.asarray(values, np.float64), -1e4, 1e4)
    d = np.abs(a[:, None] - grid[None, :])
    is_min = d == d.min(axis=1, keepdims=True)
    even = is_min & ((keys % 2) == 0)[None, :]
    return np.where(even.any(axis=1), even.argmax(axis=1), is_min.argmax(axis=1))


# ---------------------------------------------------------------- E2M3 ----
# A binary float with two exponent bits (bias 1) and three mantissa bits has
# eight values per binade: [1, 2) in steps of 1/8, [2, 4) in steps of 1/4,
# [4, 8) in steps of 1/2, and subnormals [0, 1) in steps of 1/8; with all
# codes finite the largest is 7.5.

E2M3_MAGS = np.concatenate([np.arange(16) / 8.0, 2 + np.arange(8) / 4.0, 4 + np.arange(8) / 2.0])


def test_e2m3_grid():
    assert E2M3_MAGS.size == 32 and E2M3_MAGS.max() == 7.5
    assert np.all(np.diff(E2M3_MAGS) > 0)
    mags = np.array([oracle.e2m3_value(c) for c in range(32)])
    assert np.array_equal(mags, E2M3_MAGS)
    neg = np.array([oracle.e2m3_value(0x20 | c) for c in range(32)])
    assert np.array_equal(neg, -E2M3_MAGS) and np.signbit(oracle.e2m3_value(0x20))


def test_e2m3_rounding_vs_bruteforce():
    rng = np.random.default_rng(61)
    v = np.concatenate([all_bf16_as_f32(), grid_probes(E2M3_MAGS, 7.5),
                        rng.uniform(-9, 9, 200_000).astype(np.float32)])
    mag = brute_nearest(np.abs(v.astype(np.float64)), E2M3_MAGS)
    want = (mag | (np.signbit(v).astype(np.int64) << 5)).astype(np.uint8)
    assert np.array_equal(oracle.e2m3_code_array(v), want)


def test_e2m3_named_cases():
    # midpoints to the even code, across binade edges too; saturation; signed zero
    for v, c in [(0.0625, 0), (1.0625, 8), (1.9375, 16), (2.125, 16), (3.875, 24), (4.25, 24),
                 (7.25, 30), (7.5, 31), (7.75, 31), (1e30, 31), (-0.01, 0x20), (-0.0, 0x20)]:
        assert oracle.e2m3_code(v) == c, v


# ---------------------------------------------------------------- INT6 ----

def exact_int6_grid():
    return {k: f32_round(Fraction(15 * k, 62)) for k in range(-31, 32)}


def test_int6_grid():
    grid = exact_int6_grid()
    for code in range(64):
        if code == 0x20:
            continue                                   # k = -32 is never written
        k = code - 64 if code & 0x20 else code
        assert np.float32(oracle.int6_value(code)) == grid[k], code
    assert oracle.int6_value(31) == 7.5 and oracle.int6_value(33) == -7.5


def test_int6_rounding_vs_bruteforce():
    c = np.float64(np.float32(62.0) / np.float32(15.0))       # fl(62/15)
    grid = [float(g) for g in exact_int6_grid().values()]
    rng = np.random.default_rng(62)
    v = np.concatenate([all_bf16_as_f32(), grid_probes(grid, 7.5),
                        grid_probes(np.arange(-31, 31) * 15 / 62 + 7.5 / 62, 7.5),
                        rng.uniform(-9, 9, 200_000).astype(np.float32)])
    t = v.astype(np.float64) * c                               # exact: 24 x 24 bits
    ks = np.arange(-31, 32)
    k = ks[brute_nearest(t, ks, ks)]
    assert np.array_equal(oracle.int6_code_array(v), (k & 0x3F).astype(np.uint8))


# ---------------------------------------------------------------- E2M0 ----
# Two exponent bits and no mantissa: one value per binade, 1, 2, 4, and zero.

E2M0_MAGS = np.array([0.0, 1.0, 2.0, 4.0])


def test_e2m0_grid_and_rounding():
    assert [oracle.e2m0_value(c) for c in range(4)] == list(E2M0_MAGS)
    assert [oracle.e2m0_value(4 | c) for c in range(4)] == list(-E2M0_MAGS)
    rng = np.random.default_rng(63)
    v = np.concatenate([all_bf16_as_f32(), grid_probes(E2M0_MAGS, 4.0),
                        rng.uniform(-5, 5, 200_000).astype(np.float32)])
    mag = brute_nearest(np.abs(v.astype(np.float64)), E2M0_MAGS)
    want = (mag | (np.signbit(v).astype(np.int64) << 2)).astype(np.uint8)
    assert np.array_equal(oracle.e2m0_code_array(v), want)
    for x, code in [(0.5, 0), (1.5, 2), (3.0, 2), (3.0000002, 3), (-0.0, 4), (9.0, 3)]:
        assert oracle.e2m0_code(x) == code, x


# ---------------------------------------------------------------- INT3 ----

def test_int3_grid_and_rounding():
    for code in range(8):
        if code == 4:
            continue                                   # k = -4 is never written
        k = code - 8 if code & 4 else code
        assert np.float32(oracle.int3_value(code)) == f32_round(Fraction(4 * k, 3)), code
    rng = np.random.default_rng(64)
    grid = [float(f32_round(Fraction(4 * k, 3))) for k in range(-3, 4)]
    v = np.concatenate([all_bf16_as_f32(), grid_probes(grid, 4.0),
                        rng.uniform(-5, 5, 200_000).astype(np.float32)])
    ks = np.arange(-3, 4)
    k = ks[brute_nearest(v.astype(np.float64) * 0.75, ks, ks)]  # exact product
    assert np.array_equal(oracle.int3_code_array(v), (k & 0x7).astype(np.uint8))
    assert oracle.int3_code(2.0) == 2          # 1.5 is a tie: to the even k


# -------------------------------------------------------- tensor scale ----

def test_tensor_scale_w_closed_forms():
    assert oracle.tensor_scale_w(3360.0, 6) == 1.0
    assert oracle.tensor_scale_w(1792.0, 3) == 1.0
    assert oracle.tensor_scale_w(0.0, 6) == 1.0 and oracle.tensor_scale_w(0.0, 3) == 1.0
    assert oracle.tensor_scale_w(1.0, 6) == f32_round(Fraction(1, 3360))
    assert oracle.tensor_scale_w(1e-38, 3) == np.float32(2.0 ** -117)


# -------------------------------------------------------- bit layout ----

def unpack_w(codes_row, bits):
    """Element i's code from bits [bits*i, bits*i + bits) of the little-endian
    bytes, by the test's own bit arithmetic."""
    b = np.unpackbits(np.asarray(codes_row, np.uint8), bitorder="little")
    n = b.size // bits
    w = b[: n * bits].reshape(n, bits).astype(np.int64)
    return (w * (1 << np.arange(bits))[None, :]).sum(axis=1)


@pytest.mark.parametrize("bits", [6, 3])
def test_one_code_lands_at_its_bits(bits):
    # a single nonzero element at position i: its FP code alone, at bit bits*i
    fpmax = 7.5 if bits == 6 else 4.0
    for i in range(16):
        x = np.zeros((1, 16), np.float32)
        x[0, i] = fpmax                         # ts = 1/448, block scale 448
        q = oracle.quantize_tensor_w(x, bits)
        want = np.zeros(16, np.int64)
        want[i] = 31 if bits == 6 else 3
        assert q["codes"].shape == (1, 2 * bits)
        assert np.array_equal(unpack_w(q["codes"][0], bits), want), (bits, i)


@pytest.mark.parametrize("bits", [6, 3])
def test_storage_bits_per_value(bits):
    x = np.random.default_rng(65).standard_normal((8, 256)).astype(np.float32)
    q = oracle.quantize_tensor_w(x, bits)
    total_bits = 8 * (q["codes"].nbytes + q["scales"].nbytes)
    assert total_bits / x.size == bits + 0.5


# ---------------------------------------------------------- hand groups ----

def _golden_value(v):
    if isinstance(v, str):
        num, den = v.split("/")
        a, b = num.split("*")
        return float(f32_round(Fraction(int(a) * int(b), int(den))))
    return float(v)


@pytest.mark.parametrize("fmt,bits", [("if6", 6), ("if3", 3)])
def test_hand_worked_groups(fmt, bits):
    g = json.load(open(GOLDEN))[fmt]
    x = np.array([[_golden_value(v) for v in g["row"]]], np.float32)
    q = oracle.quantize_tensor_w(x, bits)
    assert q["ts"] == np.float32(g["ts"])
    for gi, grp in enumerate(g["groups"]):
        assert int(q["scales"][0, gi]) == grp["scale"], (fmt, gi, grp["what"])
        codes = unpack_w(q["codes"][0, 2 * bits * gi: 2 * bits * (gi + 1)], bits)
        assert list(codes) == grp["codes"], (fmt, gi, grp["what"])


# ------------------------------------------- brute force over a group ----

def _decode_tables(bits):
    n = 1 << bits
    if bits == 6:
        fp = [(-1 if c & 0x20 else 1) * E2M3_MAGS[c & 31] for c in range(n)]
        it = [float(f32_round(Fraction(15 * (c - 64 if c & 0x20 else c), 62))) for c in range(n)]
        it[0x20] = np.inf                                      # not a code
    else:
        fp = [(-1 if c & 4 else 1) * E2M0_MAGS[c & 3] for c in range(n)]
        it = [float(f32_round(Fraction(4 * (c - 8 if c & 4 else c), 3))) for c in range(n)]
        it[4] = np.inf
    return np.array(fp, np.float64), np.array(it, np.float64)


@pytest.mark.parametrize("bits", [6, 3])
@pytest.mark.parametrize("dist", ["normal", "uniform", "outlier", "tiny"])
def test_group_choice_vs_bruteforce(bits, dist):
    rng = np.random.default_rng({"normal": 71, "uniform": 72, "outlier": 73, "tiny": 74}[dist] + bits)
    x = rng.standard_normal((32, 64)).astype(np.float32)
    if dist == "uniform":
        x = rng.uniform(-1, 1, (32, 64)).astype(np.float32)
    elif dist == "outlier":
        x[:, ::16] *= 30
    elif dist == "tiny":
        x *= np.float32(2.0) ** rng.integers(-60, 0, (32, 64)).astype(np.float32)
    fpmax = np.float32(7.5 if bits == 6 else 4.0)
    q = oracle.quantize_tensor_w(x, bits)
    ts = np.float32(q["ts"])
    fp_vals, int_vals = _decode_tables(bits)
    table = e4m3_table_from_torch()
    for r in range(x.shape[0]):
        for g in range(x.shape[1] // 16):
            x16 = x[r, 16 * g: 16 * (g + 1)]
            sb_f = (np.max(np.abs(x16)) / fpmax) / ts
            sb = int(brute_e4m3_encode(np.array([sb_f]))[0])
            byte = int(q["scales"][r, g])
            assert byte & 0x7F == sb
            codes = unpack_w(q["codes"][r, 2 * bits * g: 2 * bits * (g + 1)], bits)
            if sb == 0:
                assert byte == 0 and not codes.any()
                continue
            eff = np.float32(np.float32(table[sb]) * ts)
            v = (x16 * np.float32(np.float32(1.0) / eff)).astype(np.float32).astype(np.float64)
            err_fp = (v[:, None] - fp_vals[None, :]) ** 2
            err_int = (v[:, None] - int_vals[None, :]) ** 2
            e_fp, e_int = err_fp.min(axis=1).sum(), err_int.min(axis=1).sum()
            assert np.isclose(q["e_fp"][r, g], e_fp, rtol=1e-12, atol=0)
            assert np.isclose(q["e_int"][r, g], e_int, rtol=1e-12, atol=0)
            chosen = err_int if byte & 0x80 else err_fp
            # every element's code is a minimum-error code of the chosen type
            assert np.all(chosen[np.arange(16), codes] == chosen.min(axis=1))
            if abs(e_fp - e_int) > 1e-9 * max(e_fp, e_int):
                assert bool(byte & 0x80) == (e_int < e_fp)


@pytest.mark.parametrize("bits", [6, 3])
def test_adaptive_never_worse_than_either_candidate(bits):
    x = np.random.default_rng(75).standard_t(3, (64, 256)).astype(np.float32)
    q = oracle.quantize_tensor_w(x, bits, oracle.W_IF)
    f = oracle.quantize_w(x, q["ts"], bits, oracle.W_FP)
    i = oracle.quantize_w(x, q["ts"], bits, oracle.W_INT)
    e_if = np.where(q["scales"] >> 7, q["e_int"], q["e_fp"])
    assert np.all(e_if <= f["e_fp"]) and np.all(e_if <= i["e_int"])
    fp_groups = (q["scales"] >> 7) == 0
    cb = 2 * bits
    qc = q["codes"].reshape(64, -1, cb)
    assert np.array_equal(qc[fp_groups], f["codes"].reshape(64, -1, cb)[fp_groups])
    assert np.array_equal(qc[~fp_groups], i["codes"].reshape(64, -1, cb)[~fp_groups])
    assert np.all(f["scales"] >> 7 == 0) and np.all(i["scales"][i["scales"] != 0] >> 7 == 1)


@pytest.mark.parametrize("bits", [6, 3])
def test_dequantize_on_grid_round_trip(bits):
    # values q * eff with q on either grid come back exactly
    fp_vals, int_vals = _decode_tables(bits)
    rng = np.random.default_rng(76)
    rows = []
    for _ in range(16):
        vals = fp_vals if rng.random() < 0.5 else int_vals[np.isfinite(int_vals)]
        g = rng.choice(vals, 16).astype(np.float32)
        g[0] = vals.max()                                   # block scale exactly 1
        rows.append(g)
    x = np.stack(rows).reshape(4, 64).astype(np.float32)
    fpmax = 7.5 if bits == 6 else 4.0
    ts = np.float32(1.0)
    q = oracle.quantize_w(x, ts, bits)
    assert np.all(q["scales"] & 0x7F == 0x38) and fpmax == x.max()
    y = oracle.dequantize_w(q["codes"], q["scales"], ts, bits)
    assert np.array_equal(y.view(np.uint32) & 0x7FFFFFFF, x.view(np.uint32) & 0x7FFFFFFF)


# ------------------------------------------------- rounding order, IF6 ----

def _fl(fr):
    return f32_round(Fraction(fr))


def _if6_block_scale_cases(n):
    """(amax, ts) pairs next to an E4M3 midpoint where fl(fl(amax/7.5)/ts)
    and the other orders, amax/fl(7.5 ts) or one rounding of amax/(7.5 ts),
    give different codes.  (For IF3, amax/4 and 4 ts are exact, so every
    order gives the same block scale.)"""
    rng = np.random.default_rng(2025)
    table = e4m3_table_from_torch()
    cases = []
    while len(cases) < n:
        c = int(rng.integers(8, 125))
        lo, hi = Fraction(float(table[c])), Fraction(float(table[c + 1]))
        ts = np.float32(rng.uniform(1.0, 2.0) * 2.0 ** int(rng.integers(-30, 0)))
        a = np.float32(float((lo + (hi - lo) / 2) * Fraction(15, 2) * Fraction(float(ts))))
        for _ in range(200):
            fa = Fraction(float(a))
            r = _fl(Fraction(float(_fl(fa / Fraction(15, 2)))) / Fraction(float(ts)))
            alt1 = _fl(fa / Fraction(float(_fl(Fraction(15, 2) * Fraction(float(ts))))))
            alt2 = _fl(fa / (Fraction(15, 2) * Fraction(float(ts))))
            want = int(brute_e4m3_encode(np.array([float(r)]))[0])
            if want != int(brute_e4m3_encode(np.array([float(alt1)]))[0]) or \
                    want != int(brute_e4m3_encode(np.array([float(alt2)]))[0]):
                cases.append((a, ts, want))
                break
            a = np.nextafter(a, np.float32(np.inf) if rng.integers(2) else np.float32(-np.inf))
    return cases


def test_if6_block_scale_rounding_order():
    for a, ts, want in _if6_block_scale_cases(12):
        x = np.zeros((1, 16), np.float32)
        x[0, 0] = a
        x[0, 7] = -a * np.float32(0.41)
        q = oracle.quantize_w(x, ts, 6)
        assert int(q["scales"][0, 0]) & 0x7F == want, (a, ts)


# ------------------------------------------------------ dequantize ----

@pytest.mark.parametrize("bits", [6, 3])
def test_dequantize_vs_tables(bits):
    """y = fl(q * fl(E4M3 * ts)) with q from the test's own decode tables
    (exact rationals) and the test's own unpacking, under a tensor scale that
    is not a power of two."""
    fp_vals, int_vals = _decode_tables(bits)
    table = e4m3_table_from_torch()
    x = np.random.default_rng(77).standard_t(4, (16, 128)).astype(np.float32)
    q = oracle.quantize_tensor_w(x, bits)
    ts = np.float32(q["ts"])
    assert float(ts).hex().split("p")[0] != "0x1.0000000000000"
    y = oracle.dequantize_w(q["codes"], q["scales"], ts, bits)
    for r in range(16):
        for g in range(8):
            byte = int(q["scales"][r, g])
            eff = np.float32(np.float32(table[byte & 0x7F]) * ts)
            codes = unpack_w(q["codes"][r, 2 * bits * g: 2 * bits * (g + 1)], bits)
            vals = (int_vals if byte & 0x80 else fp_vals)[codes].astype(np.float32)
            want = (vals * eff).astype(np.float32)
            assert np.array_equal(y[r, 16 * g: 16 * (g + 1)].view(np.uint32), want.view(np.uint32))
