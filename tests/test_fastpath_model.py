"""A CPU model of the quantizer's binary32 fast-path decision, checked against
the binary64 rule on adversarial groups.

The kernels decide FP4 against INT4 from two squared-error sums taken in
binary32 with fused multiply-adds, in two lanes (even and odd elements) that
are added at the end; a group whose binary32 margin |e_fp - e_int| is within
the band 2^-18 (S + 1) (S = e_fp + e_int) is redecided by the binary64 rule.
The claim is that outside the band the binary32 sign is the binary64 sign.
This models that arithmetic step by step (each fused multiply-add rounded
once, exactly) and checks the claim on groups built to sit at near ties,
where the two sums nearly cancel, and on random groups.  It models the
kernels' arithmetic; it does not run them (the GPU parity tests do)."""
import numpy as np
import pytest

F32 = np.float32
C76 = float(F32(7.0) / F32(6.0))                  # fl(7/6)
C67 = float(F32(6.0) / F32(7.0))                  # fl(6/7)
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def r32(x):
    return float(F32(x))


def fma32(a, b, c):
    """fl32(a*b + c) with one rounding: the product of two binary32 values is
    exact in binary64; the sum is made exact with TwoSum, and the binary32
    rounding of s + e is decided from s unless s sits on a binary32 midpoint."""
    p = a * b
    s = p + c
    bv = s - p
    e = (p - (s - bv)) + (c - bv)
    r = r32(s)
    if e == 0.0 or r == s:
        return r if e == 0.0 else _round_with_tail(s, e)
    return _round_with_tail(s, e)


def _round_with_tail(s, e):
    r = r32(s)
    if r == s:
        # s is a binary32 value and e below its ulp: the sum rounds to s
        # unless e reaches half an ulp (it cannot: |e| <= ulp64(s)/2)
        return r
    other = float(np.nextafter(F32(r), F32(np.inf) if s > r else F32(-np.inf)))
    mid = (r + other) / 2.0
    if s != mid:
        return r
    # s is exactly the midpoint: the tail decides
    return other if (e > 0) == (other > r) else r


def fp4_value(v):
    a = abs(v)
    if a > 6.0:
        q = 6.0
    else:
        d = np.abs(E2M1 - a)
        best = min(range(8), key=lambda c: (d[c], c & 1))
        q = E2M1[best]
    return -q if np.signbit(v) else q


def fast_decision(v16):
    """The kernels' binary32 decision: (int4, near, margin d, band)."""
    ef = [0.0, 0.0]
    ei = [0.0, 0.0]
    for j in range(8):
        for lane in (0, 1):
            v = v16[2 * j + lane]
            df = r32(fp4_value(v) - v)              # exact (mixed-precision subtract)
            k = float(np.rint(v * C76))             # RNE of the exact product
            di = fma32(k, -C67, v)
            ef[lane] = fma32(df, df, ef[lane])
            ei[lane] = fma32(di, di, ei[lane])
    e_fp, e_int = r32(ef[0] + ef[1]), r32(ei[0] + ei[1])
    d = r32(e_fp - e_int)
    S = r32(e_fp + e_int)
    band = r32(r32(S + 1.0) * 2.0 ** -18)
    return d > band, (not abs(d) > band) and S != 0.0, d, band


def exact_decision(v16):
    """The binary64 rule: INT4 iff its error sum, in element order, is lower."""
    e_fp = e_int = 0.0
    for v in v16:
        k = float(np.clip(np.rint(v * C76), -7, 7))
        qi = r32(k * 6.0 / 7.0)                     # fl(6k/7)
        df = v - fp4_value(v)
        di = v - qi
        e_fp = e_fp + df * df
        e_int = e_int + di * di
    return e_int < e_fp


def _contribution(v):
    k = float(np.rint(v * C76))
    qi = r32(k * 6.0 / 7.0)
    return (v - fp4_value(v)) ** 2 - (v - qi) ** 2


def near_tie_groups(n, seed):
    """Groups whose last element is chosen, from a fine grid, to bring the
    two error sums as close together as it can."""
    rng = np.random.default_rng(seed)
    grid = np.array([r32(t) for t in np.linspace(-6.375, 6.375, 4001)])
    grid_c = np.array([_contribution(t) for t in grid])
    out = []
    for _ in range(n):
        scale = 6.0 / max(1e-3, rng.uniform(0.5, 1.0))
        v = [r32(t) for t in rng.uniform(-1, 1, 15) * scale * rng.uniform(0.2, 1.0)]
        v = [min(max(t, -6.375), 6.375) for t in v]
        part = sum(_contribution(t) for t in v)
        best = grid[np.argsort(np.abs(part + grid_c))[:3]]
        for b in best:
            out.append(v + [float(b)])
    return out


@pytest.mark.parametrize("kind", ["near_ties", "random"])
def test_binary32_decision_outside_the_band_is_the_binary64_rule(kind):
    if kind == "near_ties":
        groups = near_tie_groups(700, 3)
    else:
        rng = np.random.default_rng(9)
        groups = [[r32(t) for t in rng.uniform(-6.375, 6.375, 16) * rng.uniform(0.05, 1.0)]
                  for _ in range(2000)]
    decided = near = close = 0
    for v16 in groups:
        int4, is_near, d, band = fast_decision(v16)
        if is_near:
            near += 1
            continue
        decided += 1
        close += abs(d) < 10 * band
        assert int4 == exact_decision(v16), v16
    assert decided > 0
    if kind == "near_ties":
        # the construction reaches the band and decides many groups within ten
        # band widths of it (where a band of 2^-30, or none, decides 3 of them
        # wrongly)
        assert near > 0 and close >= 50


# ---------------------------------------------------------------- 4/6 ----
#
# The 4/6 comparator decides between the block scales of amax/6 and amax/4.
# The kernels sum each candidate's squared differences q - v in the scaled
# domain (exact mixed-precision subtracts, binary32 fused multiply-adds in two
# lanes) and scale each sum by fl(eff^2); the rule compares the x-domain
# sums of (x - fl(q eff))^2.  eff (v - q) differs from x - fl(q eff) by at
# most about 3.1 u X per element (v = fl(x fl(1/eff)), one rounding each),
# which with the sums' roundings stays within 2^-19.3 S + 2^-20.4 X^2.  Groups
# within the band 2^-18 S + 2^-19 X^2 + 2^-126 (X = 6 max(eff6, eff4)), or
# with X above 2^60 (where eff^2 could overflow), are redecided by the
# binary64 rule, and so are groups where exactly one block scale is zero.

def _e4m3_values():
    import torch
    return torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


_E4 = None


def _e4m3(f):
    global _E4
    if _E4 is None:
        _E4 = _e4m3_values()
    f = min(f, 1e4)
    d = np.abs(_E4 - f)
    return min(range(127), key=lambda c: (d[c], c & 1))


def _scales_46(x16, ts):
    amax = max(abs(t) for t in x16)
    sb6 = _e4m3(r32(r32(amax / 6.0) / ts))
    sb4 = _e4m3(r32(r32(amax / 4.0) / ts))
    eff6, eff4 = r32(_E4[sb6] * ts), r32(_E4[sb4] * ts)
    return sb6, sb4, eff6, eff4


def fast_decision_46(x16, ts):
    sb6, sb4, eff6, eff4 = _scales_46(x16, ts)
    inv6, inv4 = r32(1.0 / eff6), r32(1.0 / eff4)
    e6 = [0.0, 0.0]
    e4 = [0.0, 0.0]
    for j in range(8):
        for lane in (0, 1):
            x = x16[2 * j + lane]
            v6, v4 = r32(x * inv6), r32(x * inv4)
            d6 = r32(fp4_value(v6) - v6)          # exact
            d4 = r32(fp4_value(v4) - v4)
            e6[lane] = fma32(d6, d6, e6[lane])
            e4[lane] = fma32(d4, d4, e4[lane])
    s6 = r32(r32(e6[0] + e6[1]) * r32(eff6 * eff6))
    s4 = r32(r32(e4[0] + e4[1]) * r32(eff4 * eff4))
    d = r32(s6 - s4)
    X = r32(6.0 * max(eff6, eff4))
    band = fma32(r32(s6 + s4), 2.0 ** -18, fma32(r32(X * X), 2.0 ** -19, 2.0 ** -126))
    # the rule also decides when one block scale is zero: that candidate's
    # v is 0, so its scaled-domain sum is 0, while its x-domain error is the
    # sum of x^2
    near = not abs(d) > band or X > 2.0 ** 60 or sb6 == 0 or sb4 == 0
    return sb6 != sb4, d > 0.0, near, d, band


def exact_decision_46(x16, ts):
    sb6, sb4, eff6, eff4 = _scales_46(x16, ts)
    inv6, inv4 = r32(1.0 / eff6), r32(1.0 / eff4)
    s6 = s4 = 0.0
    for x in x16:
        xh6 = r32(fp4_value(r32(x * inv6)) * eff6)
        xh4 = r32(fp4_value(r32(x * inv4)) * eff4)
        s6 = s6 + (x - xh6) ** 2
        s4 = s4 + (x - xh4) ** 2
    return s4 < s6


def _fp4_values_vec(v):
    """fp4_value over an array (nearest E2M1 magnitude, ties to the even code,
    saturating at 6, sign of v)."""
    a = np.minimum(np.abs(v), 6.0)
    d = np.abs(E2M1[None, :] - a[:, None])
    dmin = d.min(axis=1, keepdims=True)
    tie_even = (d == dmin) & ((np.arange(8) % 2) == 0)[None, :]
    pick = np.where(tie_even.any(axis=1), tie_even.argmax(axis=1), (d == dmin).argmax(axis=1))
    q = E2M1[pick]
    return np.where(np.signbit(v), -q, q)


def near_tie_groups_46(n, seed):
    """Groups whose 16th element (below the group maximum, so neither block
    scale moves) is chosen from a fine grid to bring the two error sums as
    close together as it can."""
    rng = np.random.default_rng(seed)
    ts = r32(2.0 ** -6)
    out = []
    for _ in range(n):
        amax = r32(rng.uniform(0.5, 3.0))
        base = [amax] + [r32(t) for t in rng.uniform(-1, 1, 14) * amax]
        _, _, eff6, eff4 = _scales_46(base + [0.0], ts)
        inv6, inv4 = r32(1.0 / eff6), r32(1.0 / eff4)
        part = 0.0
        for x in base:
            part += (x - r32(fp4_value(r32(x * inv6)) * eff6)) ** 2
            part -= (x - r32(fp4_value(r32(x * inv4)) * eff4)) ** 2
        t = (np.linspace(-0.999, 0.999, 4001) * amax).astype(np.float32).astype(np.float64)
        xh6 = (_fp4_values_vec((t * inv6).astype(np.float32).astype(np.float64)) * eff6)
        xh4 = (_fp4_values_vec((t * inv4).astype(np.float32).astype(np.float64)) * eff4)
        xh6 = xh6.astype(np.float32).astype(np.float64)
        xh4 = xh4.astype(np.float32).astype(np.float64)
        gaps = part + (t - xh6) ** 2 - (t - xh4) ** 2
        for i in np.argsort(np.abs(gaps))[:3]:
            out.append((base + [float(t[i])], ts))
        # the best point refined three times, each on a 100x finer scan:
        # groups ever closer to a tie, down to the binary32 rounding level
        best, h = float(t[np.argmin(np.abs(gaps))]), float(t[1] - t[0])
        for _ in range(3):
            tt = np.linspace(best - h, best + h, 201).astype(np.float32).astype(np.float64)
            tt = tt[np.abs(tt) < amax]
            if tt.size == 0:
                break
            x6 = (_fp4_values_vec((tt * inv6).astype(np.float32).astype(np.float64)) * eff6)
            x4 = (_fp4_values_vec((tt * inv4).astype(np.float32).astype(np.float64)) * eff4)
            g2 = part + (tt - x6.astype(np.float32).astype(np.float64)) ** 2 - \
                (tt - x4.astype(np.float32).astype(np.float64)) ** 2
            best, h = float(tt[np.argmin(np.abs(g2))]), h / 100.0
            out.append((base + [best], ts))
    return out


def test_46_binary32_decision_outside_the_band_is_the_binary64_rule():
    groups = near_tie_groups_46(100, 5)
    rng = np.random.default_rng(13)
    ts = r32(2.0 ** -6)
    groups += [([r32(t) for t in rng.standard_normal(16) * rng.uniform(0.1, 3.0)], ts)
               for _ in range(300)]
    decided = near = close = 0
    for x16, ts in groups:
        differ, four, is_near, d, band = fast_decision_46(x16, ts)
        if not differ:
            continue                          # identical candidates: kept /6 either way
        if is_near:
            near += 1
            continue
        decided += 1
        close += abs(d) < 10 * band
        assert four == exact_decision_46(x16, ts), (x16, ts)
    # the construction reaches the band and decides groups close to it
    assert near > 0 and close >= 30


def test_46_a_narrow_band_decides_near_ties_wrongly():
    """The refined near ties reach the rounding level: with the band divided
    by 2^20 the binary32 decision and the rule disagree on some of them."""
    wrong = 0
    for x16, ts in near_tie_groups_46(100, 5):
        differ, four, _, d, band = fast_decision_46(x16, ts)
        if differ and abs(d) > band / 2.0 ** 20 and four != exact_decision_46(x16, ts):
            wrong += 1
    assert wrong > 0


# --------------------------------------------------------- block scale ----
#
# The kernels compute the block scale fl(fl(amax/6)/ts) without dividing:
# q = RN(amax * RN(1/6)), q = RN(q + RN(amax - 6q) * RN(1/6)) (two fused
# multiply-adds), then the same with ts and RN(1/ts) (Markstein's method:
# one correction of a quotient from the correctly rounded reciprocal).  The
# claim is that this equals the two IEEE divisions whenever amax >= 2^-100
# and the second quotient stays below 2^100 (outside that, the kernels
# divide).

def _fma32_vec(a, b, c):
    """fl32(a*b + c) elementwise, one rounding (float64 arrays of binary32
    values; the product is exact in binary64, TwoSum makes the sum exact)."""
    p = a * b
    s = p + c
    bv = s - p
    e = (p - (s - bv)) + (c - bv)
    r = s.astype(np.float32).astype(np.float64)
    towards = np.where(s > r, np.inf, -np.inf).astype(np.float32)
    other = np.nextafter(r.astype(np.float32), towards).astype(np.float64)
    mid = (r + other) / 2.0
    fix = (s == mid) & (e != 0) & ((e > 0) == (other > r))
    return np.where(fix, other, r)


def test_block_scale_quotients_equal_the_ieee_divisions():
    rng = np.random.default_rng(17)
    n = 1_000_000
    amax = (rng.uniform(1, 2, n) * np.exp2(rng.integers(-100, 100, n))).astype(np.float32)
    ts = (rng.uniform(1, 2, n) * np.exp2(rng.integers(-117, 117, n))).astype(np.float32)
    # a share of exact cases: amax a multiple of 6 ts
    k = n // 10
    ts[:k] = np.float32(2.0) ** rng.integers(-60, 60, k).astype(np.float32)
    amax[:k] = (rng.integers(1, 448, k) * 6 * ts[:k].astype(np.float64)).astype(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        _check_block_scale(amax, ts, n)


def _markstein_div6(amax):
    """The kernels' first quotient: q = fl(a * fl(1/6)), then one correction
    q + fl(a - 6q) * fl(1/6) by fused multiply-adds (float64 arrays of
    binary32 values)."""
    a = amax.astype(np.float64)
    n = a.size
    r6 = float(np.float32(1.0) / np.float32(6.0))
    q = (a * r6).astype(np.float32).astype(np.float64)
    return _fma32_vec(_fma32_vec(-q, np.full(n, 6.0), a), np.full(n, r6), q)


def test_amax_over_6_quotient_every_mantissa_and_exponent():
    """fl(amax / 6) by the two-step quotient equals the IEEE division for
    every one of the 2^23 binary32 values in [1, 2), and for 4096 mantissas
    (the 2048 smallest and largest, random ones filling the rest to 4096)
    of every binade from 2^-100 (below it the kernels divide) to the largest
    finite float.  Away from under- and overflow, every step of both sides
    scales exactly with a power of two, so the first binade covers every
    mantissa of every binade; the sampled binades check the ends."""
    one_binade = (np.arange(1 << 23, dtype=np.uint32) | np.uint32(127 << 23)).view(np.float32)
    got = _markstein_div6(one_binade)
    want = (one_binade / np.float32(6.0)).astype(np.float64)
    assert np.array_equal(got, want)
    rng = np.random.default_rng(29)
    mant = np.concatenate([np.arange(1024), (1 << 23) - 1 - np.arange(1024),
                           rng.integers(0, 1 << 23, 2048)]).astype(np.uint32)
    exps = np.arange(27, 255, dtype=np.uint32)          # 2^-100 .. 2^127
    bits = (exps[:, None] << np.uint32(23)) | mant[None, :]
    amax = bits.ravel().view(np.float32)
    with np.errstate(over="ignore"):
        got = _markstein_div6(amax)
        want = (amax / np.float32(6.0)).astype(np.float64)
    bad = got != want
    assert not bad.any(), amax[bad][:5]


def _check_block_scale(amax, ts, n):
    a, t = amax.astype(np.float64), ts.astype(np.float64)
    r6 = float(np.float32(1.0) / np.float32(6.0))
    rts = (np.float32(1.0) / ts).astype(np.float64)
    q = (a * r6).astype(np.float32).astype(np.float64)
    q = _fma32_vec(_fma32_vec(-q, np.full(n, 6.0), a), np.full(n, r6), q)
    s = (q * rts).astype(np.float32).astype(np.float64)
    got = _fma32_vec(_fma32_vec(-s, t, q), rts, s)
    want = ((amax / np.float32(6.0)) / ts).astype(np.float64)     # IEEE binary32 divisions
    valid = (amax >= np.float32(2.0 ** -100)) & (s < 2.0 ** 100) & (want >= 2.0 ** -126)
    assert valid.sum() > n // 2
    bad = valid & (got != want)
    assert not bad.any(), (amax[bad][:5], ts[bad][:5])


# ---------------------------------------------------- coinciding candidates --
#
# Before the binary64 rule, the kernels test on the two code words whether
# every element's FP4 and INT4 candidates have the same value (the grids share
# only 0 and +-6), which makes the group an exact tie that keeps FP4.  The bit
# expression below is the kernels' test; it is checked here against the
# decoded values.

def coincide_bits(fp4, int4):
    m = fp4 & 0x77777777
    is6 = m & (m >> 1) & (m >> 2) & 0x11111111
    nz = (m | (m >> 1) | (m >> 2)) & 0x11111111
    sgn = (fp4 >> 3) & 0x11111111
    want = ((is6 * 0xF) & 0xFFFFFFFF) & (0x77777777 ^ ((sgn * 0xE) & 0xFFFFFFFF))
    return (nz & ~is6 & 0xFFFFFFFF) == 0 and int4 == want


def _fp4_nibble_value(n):
    mag = E2M1[n & 7]
    return -mag if n & 8 else mag


def _int4_nibble_value(n):
    k = n - 16 if n & 8 else n
    return r32(k * 6.0 / 7.0)


def test_coinciding_candidates_bit_test_matches_the_values():
    ints = [n for n in range(16) if n != 8]          # 0x8 (k = -8) is never written
    # one element (the others 0 on both grids), at every nibble position
    for pos in range(8):
        for f in range(16):
            for i in ints:
                same = _fp4_nibble_value(f) == _int4_nibble_value(i)
                assert coincide_bits(f << (4 * pos), i << (4 * pos)) == same, (pos, f, i)
    # whole words: coincide iff every element does
    rng = np.random.default_rng(23)
    pairs = [(f, i) for f in range(16) for i in ints]
    equal = [(f, i) for f, i in pairs if _fp4_nibble_value(f) == _int4_nibble_value(i)]
    for trial in range(20000):
        pool = equal if trial % 2 else pairs          # half the words from equal pairs only
        picks = [pool[j] for j in rng.integers(0, len(pool), 8)]
        fw = sum(f << (4 * p) for p, (f, _) in enumerate(picks))
        iw = sum(i << (4 * p) for p, (_, i) in enumerate(picks))
        same = all(_fp4_nibble_value(f) == _int4_nibble_value(i) for f, i in picks)
        assert coincide_bits(fw, iw) == same, (hex(fw), hex(iw))


# ------------------------------------------------------------ INT4 packing --
#
# The kernels get k + 8 in the low bits of the binary32 r = 1.5 * 2^23 + 8 +
# k (one fused multiply-add), combine an element pair as the integer
# bits(r_odd) * 16 + bits(r_even), keep byte 0, and turn the offset-8 nibbles
# into two's complement with XOR 0x88.

def test_int4_nibble_packing_identity():
    m8 = F32(12582912.0 + 8.0)                   # 1.5 * 2^23 + 8
    for ke in range(-7, 8):
        for ko in range(-7, 8):
            re = int(np.array([m8 + F32(ke)], np.float32).view(np.uint32)[0])
            ro = int(np.array([m8 + F32(ko)], np.float32).view(np.uint32)[0])
            byte0 = ((ro * 16 + re) & 0xFFFFFFFF) & 0xFF
            assert byte0 ^ 0x88 == ((ko & 0xF) << 4) | (ke & 0xF), (ke, ko)
