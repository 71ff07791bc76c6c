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
