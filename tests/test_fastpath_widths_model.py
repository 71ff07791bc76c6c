"""A CPU model of the IF6 / IF3 kernels' binary32 decision, checked against
the binary64 rule on groups built to sit at near ties.

The IF6 and IF3 quantizers decide FP against INT from two squared-error sums
taken in binary32 with fused multiply-adds, in two lanes (even and odd
elements) added at the end, as the IF4 fast path does.  The FP differences
v - qf are exact (qf is v rounded to the FP grid: the two are within a factor
of two, or qf = 0).  Each INT difference is one fused multiply-add,
v - k * fl(c), with c = 15/62 (IF6) or 4/3 (IF3).  The rule's INT value is
the correctly rounded quotient fl(15k/62) or fl(4k/3), so the difference is
off by at most |k| |fl(c) - c| + ulp/2 plus one rounding.  A group whose
binary32 margin |e_fp - e_int| is within the band 2^-16 (S + 1) (S = e_fp +
e_int) is redecided by the binary64 rule.  The claim: outside the band the
binary32 sign is the binary64 rule's.  This models that arithmetic step by
step and checks the claim.  It models the kernels' arithmetic; it does not
run them (the GPU parity tests do)."""
import numpy as np
import pytest

from test_fastpath_model import _fma32_vec, fma32, r32

F32 = np.float32
BAND_EXP = -16
E2M3 = np.array(sorted({m / 8.0 for m in range(16)} | {(8 + m) / 4.0 for m in range(8)}
                       | {(8 + m) / 2.0 for m in range(8)}))     # 0 .. 7.5, 32 values
E2M0 = np.array([0.0, 1.0, 2.0, 4.0])
WIDTHS = {
    6: dict(grid=E2M3, fpmax=7.5, kmax=31, c=float(F32(62.0) / F32(15.0)),
            cq=float(F32(15.0) / F32(62.0)), num=15, den=62),
    3: dict(grid=E2M0, fpmax=4.0, kmax=3, c=0.75, cq=float(F32(4.0) / F32(3.0)), num=4, den=3),
}


def fp_value(v, bits):
    """v rounded to the FP grid, ties to the even code, saturating; the sign
    of v kept (a zero too)."""
    w = WIDTHS[bits]
    grid, a = w["grid"], abs(v)
    if a >= w["fpmax"]:
        q = w["fpmax"]
    else:
        d = np.abs(grid - a)
        best = min(range(len(grid)), key=lambda c: (d[c], c & 1))
        q = grid[best]
    return -q if np.signbit(v) else q


def int_k(v, bits):
    w = WIDTHS[bits]
    return float(np.clip(np.rint(v * w["c"]), -w["kmax"], w["kmax"]))   # RNE of the exact product


def int_value(k, bits):
    w = WIDTHS[bits]
    return r32(w["num"] * k / w["den"])                  # the correctly rounded quotient


def fast_decision(v16, bits, band_exp=BAND_EXP):
    """The kernels' binary32 decision: (int, near, margin d, band)."""
    cq = WIDTHS[bits]["cq"]
    ef = [0.0, 0.0]
    ei = [0.0, 0.0]
    for j in range(8):
        for lane in (0, 1):
            v = v16[2 * j + lane]
            df = r32(fp_value(v, bits) - v)              # exact
            di = fma32(int_k(v, bits), -cq, v)
            ef[lane] = fma32(df, df, ef[lane])
            ei[lane] = fma32(di, di, ei[lane])
    e_fp, e_int = r32(ef[0] + ef[1]), r32(ei[0] + ei[1])
    d = r32(e_fp - e_int)
    S = r32(e_fp + e_int)
    band = r32(r32(S + 1.0) * 2.0 ** band_exp)
    return d > band, (not abs(d) > band) and S != 0.0, d, band


def exact_decision(v16, bits):
    """The binary64 rule: INT iff its error sum, in element order, is lower."""
    e_fp = e_int = 0.0
    for v in v16:
        df = v - fp_value(v, bits)
        di = v - int_value(int_k(v, bits), bits)
        e_fp = e_fp + df * df
        e_int = e_int + di * di
    return e_int < e_fp


def _contribution(v, bits):
    return (v - fp_value(v, bits)) ** 2 - (v - int_value(int_k(v, bits), bits)) ** 2


def near_tie_groups(n, seed, bits):
    """Groups whose last element is chosen, from successively finer scans,
    to bring the two error sums close together."""
    rng = np.random.default_rng(seed)
    top = WIDTHS[bits]["fpmax"] * (1 + 1 / 16)          # |v| reaches fpmax (1 + 2^-4)
    grid = np.array([r32(t) for t in np.linspace(-top, top, 6001)])
    grid_c = np.array([_contribution(t, bits) for t in grid])
    step = float(grid[1] - grid[0])
    out = []
    for _ in range(n):
        v = [r32(t) for t in rng.uniform(-1, 1, 15) * top * rng.uniform(0.2, 1.0)]
        part = sum(_contribution(t, bits) for t in v)
        b = grid[np.argmin(np.abs(part + grid_c))]
        # the last element refined 0 to 3 times, each on a 100x finer scan:
        # groups at every distance from a tie, inside the band and near it
        best, h = float(b), step
        out.append(v + [best])
        for _ in range(3):
            cand = [r32(t) for t in np.linspace(best - h, best + h, 201)]
            best = min(cand, key=lambda t: abs(part + _contribution(t, bits)))
            h /= 100.0
            out.append(v + [best])
    return out


def test_int_value_offsets_are_within_the_stated_bound():
    """|k fl(c) - fl(num k / den)| over every k: the INT difference's offset
    that the band has to cover."""
    for bits, w in WIDTHS.items():
        worst = max(abs(k * w["cq"] - int_value(float(k), bits))
                    for k in range(-w["kmax"], w["kmax"] + 1))
        assert worst <= 2.0 ** -20, (bits, worst)


@pytest.mark.parametrize("bits", [6, 3])
@pytest.mark.parametrize("kind", ["near_ties", "random"])
def test_binary32_decision_outside_the_band_is_the_binary64_rule(bits, kind):
    if kind == "near_ties":
        groups = near_tie_groups(500, 11 + bits, bits)
    else:
        top = WIDTHS[bits]["fpmax"] * (1 + 1 / 16)
        rng = np.random.default_rng(5 + bits)
        groups = [[r32(t) for t in rng.uniform(-top, top, 16) * rng.uniform(0.05, 1.0)]
                  for _ in range(1500)]
    decided = near = close = 0
    for v16 in groups:
        is_int, is_near, d, band = fast_decision(v16, bits)
        if is_near:
            near += 1
            continue
        decided += 1
        close += abs(d) < 10 * band
        assert is_int == exact_decision(v16, bits), (bits, v16)
    assert decided > 0
    if kind == "near_ties":
        assert near > 0 and close > 0


@pytest.mark.parametrize("bits", [6, 3])
def test_a_narrow_band_decides_near_ties_wrongly(bits):
    """Without the band's width the same construction finds groups where
    binary32 and the rule disagree: the band is doing work."""
    wrong = 0
    for v16 in near_tie_groups(500, 11 + bits, bits):
        is_int, is_near, _, _ = fast_decision(v16, bits, band_exp=-40)
        if not is_near and is_int != exact_decision(v16, bits):
            wrong += 1
    assert wrong > 0


def test_fp_grids():
    assert len(E2M3) == 32 and E2M3[-1] == 7.5 and E2M3[1] == 0.125
    assert fp_value(3.0, 3) == 2.0 and fp_value(0.5, 3) == 0.0 and fp_value(3.01, 3) == 4.0
    assert fp_value(0.0625, 6) == 0.0 and fp_value(0.1875, 6) == 0.25 and fp_value(7.9, 6) == 7.5
    assert np.signbit(fp_value(-0.01, 6)) and np.signbit(fp_value(-0.2, 3))


def _e2m0_sets(v):
    """The IF3 kernel's E2M0: three comparisons of a = |v| giving 1 or 0,
    the unordered forms holding for NaN: (value, magnitude code)."""
    a = abs(v)
    s1 = 0.0 if a <= 0.5 else 1.0
    s2 = 0.0 if a < 1.5 else 1.0
    s3 = 0.0 if a <= 3.0 else 1.0
    return s1 + s2 + 2.0 * s3, int(s1 + s2 + s3)


def _codes3(v, clamp=False):
    """(FP code, INT code) of one element as the IF3 kernel forms them."""
    _, mag = _e2m0_sets(v)
    fcode = mag | (4 if np.signbit(v) else 0)
    vc = min(max(v, -2.0 ** 19), 2.0 ** 19) if clamp else v
    k = int(np.rint(vc * 0.75))
    if clamp:
        k = min(max(k, -3), 3)
    return fcode, k & 7


def _coincide_codes(fcodes, icodes):
    """The kernel's test, on 12-bit quads of 3-bit codes."""
    t = 0
    for q in range(4):
        fq = sum(c << (3 * i) for i, c in enumerate(fcodes[4 * q:4 * q + 4]))
        iq = sum(c << (3 * i) for i, c in enumerate(icodes[4 * q:4 * q + 4]))
        t |= (fq ^ (fq >> 1)) | (fq ^ iq)
    return (t & 0x249) == 0


def _v_sweep():
    """Every binary32 value near the comparison and rounding boundaries of
    both grids (1/2, 2/3, 3/2, 2, 3, 10/3), a dense grid over the range,
    zeros of both signs, both infinities and large values."""
    vals = set()
    for b in (0.5, 2 / 3, 1.5, 2.0, 3.0, 10 / 3, 4.0):
        c = np.float32(b)
        for d in range(-40, 41):
            vals.add(float(np.nextafter(c, np.float32(np.inf)) if d > 0 else c) if abs(d) <= 1
                     else float(c + np.float32(d) * np.spacing(c)))
    vals.update(float(t) for t in np.linspace(0, 4.5, 9001, dtype=np.float32))
    vals.update([0.0, 2.0 ** -140, 1e30, 2.0 ** 19, 2.0 ** 25, float("inf")])
    return sorted(vals | {-t for t in vals})


def test_e2m0_by_comparisons_is_the_grid_rounding():
    """The comparisons give the E2M0 rounding with ties to the even code
    (the oracle's grid and tie rule, restated by fp_value), NaN to 4."""
    for v in _v_sweep():
        q, mag = _e2m0_sets(v)
        assert q == abs(fp_value(v, 3)), v
        assert [0.0, 1.0, 2.0, 4.0][mag] == q
    assert _e2m0_sets(float("nan")) == (4.0, 3)


def test_float_packing_of_fp_codes_is_exact():
    """The FP quad as the float 2^23 + sum(code_i 8^i), accumulated as
    2^23 + A w + (4 sign + s3) w per element, reads back the packed codes."""
    rng = np.random.default_rng(41)
    for _ in range(2000):
        codes = rng.integers(0, 8, 4)
        acc = F32(2.0 ** 23)
        for i, c in enumerate(codes):
            mag, sign = int(c) & 3, int(c) >> 2
            s3 = float(mag == 3)
            A = F32(mag - s3)
            w = F32(8 ** i)
            acc = F32(acc + A * w)
            acc = F32(acc + F32(F32(sign * 4.0) + F32(s3)) * w)
        bits = int(np.array([acc], dtype=np.float32).view(np.uint32)[0]) & 0xFFF
        assert bits == sum(int(c) << (3 * i) for i, c in enumerate(codes))


@pytest.mark.parametrize("clamp", [False, True])
def test_code_test_finds_exactly_the_coinciding_elements(clamp):
    """Per element over the sweep, and per group on random groups: the
    kernels' code test holds exactly where the FP value and the rule's INT
    value coincide (both 0, or both +-4), under both the unclamped and the
    clamped integer."""
    sweep = [v for v in _v_sweep() if clamp or abs(v) < 2.0 ** 19]
    for v in sweep:
        f, i = _codes3(v, clamp)
        same = fp_value(v, 3) == int_value(float(np.clip(np.rint(
            (min(max(v, -2.0 ** 19), 2.0 ** 19) if clamp else v) * 0.75), -3, 3)), 3)
        assert _coincide_codes([f] * 16, [i] * 16) == same, v
    rng = np.random.default_rng(23)
    hits = 0
    for _ in range(3000):
        # mostly small elements (both grids 0), the maximum at +-4 (both 4)
        v16 = [r32(t) for t in rng.normal(0, 0.3, 16)]
        v16[rng.integers(16)] = float(rng.choice([-1.0, 1.0]) * 4.0)
        same = all(fp_value(v, 3) == int_value(int_k(v, 3), 3) for v in v16)
        f, i = zip(*(_codes3(v, clamp) for v in v16))
        assert _coincide_codes(list(f), list(i)) == same
        if same:
            hits += 1
            assert not exact_decision(v16, 3)          # a tie keeps FP
    assert 0 < hits < 3000


@pytest.mark.parametrize("bits", [6, 3])
def test_block_scale_second_quotient_equals_the_ieee_division(bits):
    """The kernels' block scale: fl(amax / fpmax) (an IEEE division for IF6,
    the exact amax * 1/4 for IF3), then the quotient by ts by Markstein's
    method, s = fl(a y), s + fl(a - s ts) y with y = fl(1/ts); it equals the
    IEEE division wherever the kernels use it (a >= 2^-100, s < 2^100, a
    normal result), on a million random (amax, ts) pairs and a tenth of
    them exact multiples."""
    rng = np.random.default_rng(31 + bits)
    n = 1_000_000
    amax = (rng.uniform(1, 2, n) * np.exp2(rng.integers(-100, 100, n))).astype(np.float32)
    ts = (rng.uniform(1, 2, n) * np.exp2(rng.integers(-117, 117, n))).astype(np.float32)
    k = n // 10
    fpmax = np.float32(WIDTHS[bits]["fpmax"])
    ts[:k] = np.float32(2.0) ** rng.integers(-60, 60, k).astype(np.float32)
    amax[:k] = (rng.integers(1, 448, k) * float(fpmax) * ts[:k].astype(np.float64)).astype(np.float32)
    with np.errstate(over="ignore", invalid="ignore", under="ignore"):
        a1 = (amax / fpmax) if bits == 6 else (amax * np.float32(0.25))
        a = a1.astype(np.float64)
        t = ts.astype(np.float64)
        y = (np.float32(1.0) / ts).astype(np.float64)
        s = (a * y).astype(np.float32).astype(np.float64)
        got = _fma32_vec(_fma32_vec(-s, t, a), y, s)
        want = (a1 / ts).astype(np.float64)                  # IEEE binary32 division
    valid = (a1 >= np.float32(2.0 ** -100)) & (s < 2.0 ** 100) & (want >= 2.0 ** -126)
    assert valid.sum() > n // 2
    bad = valid & (got != want)
    assert not bad.any(), (amax[bad][:5], ts[bad][:5])


def _markstein_div75(amax):
    """The IF6 kernel's fl(amax / 7.5): q = fl(amax * fl(1/7.5)), then q +
    fl(amax - 7.5 q) * fl(1/7.5) in one fused multiply-add."""
    a = amax.astype(np.float64)
    r = float(np.float32(1.0) / np.float32(7.5))
    q = (a * r).astype(np.float32).astype(np.float64)
    n = a.size
    return _fma32_vec(_fma32_vec(-q, np.full(n, 7.5), a), np.full(n, r), q)


def test_amax_over_7_5_quotient_every_mantissa_and_exponent():
    """IF6's first block-scale quotient by the two-step form equals the IEEE
    division for every one of the 2^23 binary32 values in [1, 2), and for
    4096 mantissas (the 2048 smallest and largest, random ones filling the
    rest) of every binade from 2^-100 (below it the kernel divides) to the
    largest finite float.  Away from under- and overflow both sides scale
    exactly with a power of two, so the first binade covers every mantissa
    of every binade; the sampled binades check the ends."""
    one_binade = (np.arange(1 << 23, dtype=np.uint32) | np.uint32(127 << 23)).view(np.float32)
    got = _markstein_div75(one_binade)
    want = (one_binade / np.float32(7.5)).astype(np.float64)
    assert np.array_equal(got, want)
    rng = np.random.default_rng(37)
    mant = np.concatenate([np.arange(1024), (1 << 23) - 1 - np.arange(1024),
                           rng.integers(0, 1 << 23, 2048)]).astype(np.uint32)
    exps = np.arange(27, 255, dtype=np.uint32)          # 2^-100 .. 2^127
    bits = (exps[:, None] << np.uint32(23)) | mant[None, :]
    amax = bits.ravel().view(np.float32)
    with np.errstate(over="ignore"):
        got = _markstein_div75(amax)
        want = (amax / np.float32(7.5)).astype(np.float64)
    bad = got != want
    assert not bad.any(), amax[bad][:5]
