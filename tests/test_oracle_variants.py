"""Pins for the oracle's comparator formats and the random-sign Hadamard
transform, each against an independent construction: brute force over the
grids and E4M3 codes, the Sylvester matrix built with np.kron and applied in
float64, exact integer arithmetic, invariants."""
import numpy as np
import pytest

import oracle
from test_oracle_pins import (E2M1_MAGS, brute_e4m3_encode, brute_int4_nibble,
                              e4m3_table_from_torch, unpack)


def _data(seed, rows=48, cols=256):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols))
    x[:, rng.choice(cols, 3, replace=False)] *= 12
    x[rows // 2:] = rng.uniform(-1, 1, (rows - rows // 2, cols))
    return x.astype(np.float32)


# -------------------------------------------------------------- NVINT4 -----

def test_nvint4_is_the_int4_candidate_everywhere():
    x = _data(1)
    q = oracle.quantize_tensor(x, mode=oracle.MODE_NVINT4)
    i = oracle.quantize_tensor(x)
    assert np.array_equal(q["scales"] & 0x7F, i["scales"] & 0x7F)
    assert np.all((q["scales"] >> 7) == (q["scales"] != 0))
    # INT4-chosen IF4 groups are byte-identical to NVINT4
    int_groups = (i["scales"] & 0x80) != 0
    assert np.array_equal(q["codes"].reshape(x.shape[0], -1, 8)[int_groups],
                          i["codes"].reshape(x.shape[0], -1, 8)[int_groups])
    # every nibble is the brute-force nearest INT4 code of v = x * inv
    e4 = e4m3_table_from_torch()
    sb = (q["scales"] & 0x7F).astype(np.int64)
    eff = (e4[sb].astype(np.float32) * q["ts"]).astype(np.float32)
    inv = np.where(sb > 0, np.float32(1) / np.where(sb > 0, eff, 1), 0).astype(np.float32)
    v = (x.reshape(x.shape[0], -1, 16) * inv[:, :, None]).astype(np.float32)
    nib = np.stack([unpack(c) for c in q["codes"]]).reshape(v.shape)
    want = brute_int4_nibble(v.reshape(-1)).reshape(v.shape)
    want[sb == 0] = 0
    assert np.array_equal(nib, want)
    # IF4 never worse than NVINT4 (v domain, exact)
    assert np.all(np.where(int_groups, i["e_int"], i["e_fp"]) <= q["e_int"])


# ----------------------------------------------------------- Four over Six --

def test_four_over_six_vs_bruteforce():
    x = _data(2, rows=24, cols=128)
    q = oracle.quantize_tensor(x, mode=oracle.MODE_4OVER6)
    ts = q["ts"]
    e4 = e4m3_table_from_torch()
    mags = np.concatenate([E2M1_MAGS, -E2M1_MAGS])
    n_four = 0
    for r in range(x.shape[0]):
        nib = unpack(q["codes"][r])
        for g in range(x.shape[1] // 16):
            xg = x[r, 16 * g:16 * g + 16]
            amax = np.max(np.abs(xg))
            cands = []
            for div in (6.0, 4.0):
                sb = int(brute_e4m3_encode(np.array([(amax / np.float32(div)) / ts]))[0])
                eff = np.float32(np.float32(e4[sb]) * ts)
                inv = np.float32(1) / eff if sb else np.float32(0)
                v = (xg * inv).astype(np.float32)
                # nearest E2M1 value (brute force), sign from v
                d = np.abs(np.abs(v.astype(np.float64))[:, None] - E2M1_MAGS[None, :])
                code = d.argmin(axis=1)
                tie = (d == d.min(axis=1, keepdims=True)).sum(axis=1) > 1
                code = np.where(tie & (code % 2 == 1), code + 1, code)
                qv = np.where(np.signbit(v), -E2M1_MAGS[code], E2M1_MAGS[code])
                xhat = (qv.astype(np.float32) * eff).astype(np.float32)
                err = float(np.sum((xg.astype(np.float64) - xhat) ** 2))
                cands.append((sb, err))
            (sb6, e6), (sb4, e4_) = cands
            use4 = e4_ < e6
            n_four += use4
            assert q["scales"][r, g] == (sb4 if use4 else sb6)
            assert q["scales"][r, g] & 0x80 == 0
            assert min(e6, e4_) <= e6
    assert n_four > 0


def test_four_over_six_never_worse_than_nvfp4_and_decodes_as_nvfp4():
    x = _data(3)
    q = oracle.quantize_tensor(x, mode=oracle.MODE_4OVER6)
    n = oracle.quantize(x, q["ts"], mode=oracle.MODE_NVFP4)
    xd = x.astype(np.float64)
    yq = oracle.dequantize(q["codes"], q["scales"], q["ts"]).astype(np.float64)
    yn = oracle.dequantize(n["codes"], n["scales"], q["ts"]).astype(np.float64)
    gq = ((xd - yq) ** 2).reshape(x.shape[0], -1, 16).sum(-1)
    gn = ((xd - yn) ** 2).reshape(x.shape[0], -1, 16).sum(-1)
    assert np.all(gq <= gn)
    # the recorded /6 error is NVFP4's reconstruction error
    assert np.allclose(q["e_fp"], gn, rtol=1e-12, atol=0)      # numpy sums in another order


# -------------------------------------------------- random-sign Hadamard ---

def _h16():
    h = np.array([[1.0]])
    for _ in range(4):
        h = np.kron(h, np.array([[1.0, 1.0], [1.0, -1.0]]))
    return h


@pytest.mark.parametrize("signs", [0x0000, 0xFFFF, 0xA5C3, 0x1234])
def test_rht_matches_float64_matrix_product(signs):
    x = _data(4)
    s = np.array([-1.0 if (signs >> j) & 1 else 1.0 for j in range(16)])
    m = _h16() * s[None, :] / 4.0
    xg = x.reshape(-1, 16).astype(np.float64)
    want = xg @ m.T
    got = oracle.rht(x, signs).reshape(-1, 16).astype(np.float64)
    # four levels of binary32 additions: error <= 4 u sum|x| / 4 per output
    bound = 4 * 2.0 ** -24 * np.abs(xg).sum(axis=1, keepdims=True) / 4 * 1.0001
    assert np.all(np.abs(got - want) <= bound)


def test_rht_exact_on_small_integers_and_orthonormal():
    rng = np.random.default_rng(5)
    x = rng.integers(-1000, 1000, (64, 64)).astype(np.float32)
    signs = 0x3C5A
    s = np.array([-1.0 if (signs >> j) & 1 else 1.0 for j in range(16)])
    m = _h16() * s[None, :] / 4.0
    got = oracle.rht(x, signs).reshape(-1, 16)
    assert np.array_equal(got.astype(np.float64), x.reshape(-1, 16).astype(np.float64) @ m.T)
    # orthonormal: the transform preserves the sum of squares, and applying
    # H16 again and undoing the signs returns the input
    assert np.allclose((got.astype(np.float64) ** 2).sum(1), (x.reshape(-1, 16).astype(np.float64) ** 2).sum(1))
    back = (got.astype(np.float64) @ _h16().T / 4.0) * s[None, :]
    assert np.array_equal(back, x.reshape(-1, 16))


def test_rht_then_quantize_is_quantize_of_the_transform():
    x = _data(6)
    q = oracle.quantize_tensor_rht(x, 0x5A5A)
    r = oracle.quantize_tensor(oracle.rht(x, 0x5A5A))
    assert q["ts"] == r["ts"]
    assert np.array_equal(q["codes"], r["codes"]) and np.array_equal(q["scales"], r["scales"])


def test_four_over_six_equal_errors_keep_six():
    """Equal errors keep the amax/6 scale (reading R22).  ts = 1 and
    x = [6, 3, -6, 0, ...] are exact under both candidate scales: E4M3 1.0
    from amax/6 puts them on the grid as 6, 3, -6, and E4M3 1.5 from amax/4
    scales them to 4, 2, -4, which decode back to 6, 3, -6.  Both errors are
    zero, so the /6 scale (code 0x38) and its codes must be kept."""
    x = np.zeros((1, 16), np.float32)
    x[0, :3] = [6.0, 3.0, -6.0]
    q = oracle.quantize(x, np.float32(1.0), mode=oracle.MODE_4OVER6)
    assert q["e_fp"][0, 0] == 0.0 and q["e_int"][0, 0] == 0.0
    assert int(q["scales"][0, 0]) == 0x38           # E4M3 1.0, not 1.5 (0x3C)
    assert list(unpack(q["codes"][0])[:3]) == [0x7, 0x5, 0xF]


def _rht_f32(x16, signs, order):
    y = np.array([-v if (signs >> j) & 1 else v for j, v in enumerate(x16)], np.float32)
    for h in order:
        for i in range(16):
            if not i & h:
                a, b = y[i], y[i + h]
                y[i], y[i + h] = np.float32(a + b), np.float32(a - b)
    return (y * np.float32(0.25)).astype(np.float32)


def test_rht_butterfly_stage_order():
    """Reading R23 fixes the butterfly stages h = 1, 2, 4, 8 in that order.
    The opposite order is the same transform in exact arithmetic but rounds
    differently in binary32.  On seeded groups where the two orders give
    different binary32 results, the oracle must give the stated order's."""
    rng = np.random.default_rng(11)
    signs = 0x6A1D
    found = 0
    for _ in range(2000):
        x = (rng.standard_normal(16) * np.exp2(rng.integers(-3, 4, 16))).astype(np.float32)
        fwd = _rht_f32(x, signs, (1, 2, 4, 8))
        if np.array_equal(fwd, _rht_f32(x, signs, (8, 4, 2, 1))):
            continue
        got = oracle.rht(x[None, :], signs)[0]
        assert np.array_equal(got.view(np.uint32), fwd.view(np.uint32)), x
        found += 1
        if found == 20:
            break
    assert found == 20
