"""IF4 CPU oracle -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct statement of what the IF4 quantizer computes,
written from the pages on "Adaptive Block-Scaled Data Types", and of the same
adaptive choice at 6 and 3 bits (IF6, IF3; their grids are readings, not fixed
by the pages).  The scalar
arithmetic lives in ``if4_oracle.c`` (binary32 values, binary64 error sums);
this module only marshals numpy arrays and adds the reductions that are plain
library calls (means, the float64 matrix product for the linear).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It never imports the CUDA package and
the CUDA package never imports it.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")

MODE_IF4 = 0
MODE_NVFP4 = 1
MODE_NVINT4 = 2
MODE_4OVER6 = 3


def lib():
    """Load (building on first use) the oracle's shared library."""
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_value.restype = ctypes.c_float
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e2m1_nibble.argtypes = [ctypes.c_float]
        L.orc_e2m1_nibble.restype = ctypes.c_uint8
        L.orc_e2m1_value.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_value.restype = ctypes.c_float
        L.orc_int4_nibble.argtypes = [ctypes.c_float]
        L.orc_int4_nibble.restype = ctypes.c_uint8
        L.orc_int4_value.argtypes = [ctypes.c_uint8]
        L.orc_int4_value.restype = ctypes.c_float
        L.orc_tensor_amax.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
        L.orc_tensor_amax.restype = ctypes.c_float
        L.orc_tensor_scale.argtypes = [ctypes.c_float]
        L.orc_tensor_scale.restype = ctypes.c_float
        L.orc_quantize.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_float, ctypes.c_int, _u8p, _u8p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_int]
        L.orc_quantize.restype = None
        L.orc_dequantize.argtypes = [_u8p, _u8p, ctypes.c_float, ctypes.c_int64,
                                     ctypes.c_int64, _f32p, ctypes.c_int]
        L.orc_dequantize.restype = None
        for name in ("orc_e4m3_encode_array", "orc_e2m1_nibble_array", "orc_int4_nibble_array"):
            fn = getattr(L, name)
            fn.argtypes = [_f32p, ctypes.c_int64, _u8p]
            fn.restype = None
        L.orc_rht16.argtypes = [_f32p, ctypes.c_uint32, _f32p]
        L.orc_rht16.restype = None
        L.orc_rht.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                              ctypes.c_uint32, _f32p, ctypes.c_int]
        L.orc_rht.restype = None
        for name in ("orc_e2m3_code", "orc_int6_code", "orc_e2m0_code", "orc_int3_code"):
            fn = getattr(L, name)
            fn.argtypes = [ctypes.c_float]
            fn.restype = ctypes.c_uint8
        for name in ("orc_e2m3_value", "orc_int6_value", "orc_e2m0_value", "orc_int3_value"):
            fn = getattr(L, name)
            fn.argtypes = [ctypes.c_uint8]
            fn.restype = ctypes.c_float
        for name in ("orc_e2m3_code_array", "orc_int6_code_array", "orc_e2m0_code_array",
                     "orc_int3_code_array"):
            fn = getattr(L, name)
            fn.argtypes = [_f32p, ctypes.c_int64, _u8p]
            fn.restype = None
        L.orc_tensor_scale_w.argtypes = [ctypes.c_float, ctypes.c_int]
        L.orc_tensor_scale_w.restype = ctypes.c_float
        L.orc_quantize_w.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_float, ctypes.c_int, ctypes.c_int, _u8p, _u8p,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_int]
        L.orc_quantize_w.restype = None
        L.orc_dequantize_w.argtypes = [_u8p, _u8p, ctypes.c_float, ctypes.c_int64,
                                       ctypes.c_int64, ctypes.c_int, _f32p, ctypes.c_int]
        L.orc_dequantize_w.restype = None
        L.orc_max_threads.argtypes = []
        L.orc_max_threads.restype = ctypes.c_int
        _LIB = L
    return _LIB


def max_threads() -> int:
    return int(lib().orc_max_threads())


# ----------------------------------------------------------- element level --

def e4m3_value(b: int) -> float:
    return float(lib().orc_e4m3_value(int(b) & 0xFF))


def e4m3_encode(f: float) -> int:
    return int(lib().orc_e4m3_encode(float(np.float32(f))))


def e2m1_nibble(v: float) -> int:
    return int(lib().orc_e2m1_nibble(float(np.float32(v))))


def e2m1_value(n: int) -> float:
    return float(lib().orc_e2m1_value(int(n)))


def int4_nibble(v: float) -> int:
    return int(lib().orc_int4_nibble(float(np.float32(v))))


def int4_value(n: int) -> float:
    return float(lib().orc_int4_value(int(n)))


def _array_fn(name, values):
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float32).ravel())
    out = np.zeros(v.shape, np.uint8)
    getattr(lib(), name)(v, v.size, out)
    return out


def e4m3_encode_array(values):
    return _array_fn("orc_e4m3_encode_array", values)


def e2m1_nibble_array(values):
    return _array_fn("orc_e2m1_nibble_array", values)


def int4_nibble_array(values):
    return _array_fn("orc_int4_nibble_array", values)


# ------------------------------------------------------------ tensor level --

def _as_f32_2d(x):
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    if x.ndim != 2 or x.shape[1] % 16:
        raise ValueError("oracle expects a 2-D float32 array with cols % 16 == 0")
    return x


def tensor_amax(x) -> np.float32:
    x = _as_f32_2d(x)
    return np.float32(lib().orc_tensor_amax(x, x.shape[0], x.shape[1], x.shape[1]))


def tensor_scale(amax) -> np.float32:
    """ts = amax/(6*448); 1 for amax == 0; floored at 2^-117."""
    return np.float32(lib().orc_tensor_scale(float(np.float32(amax))))


def quantize(x, ts, mode: int = MODE_IF4, threads: int = 0):
    """Quantize a [rows, cols] float32 array.

    Returns dict(codes uint8 [rows, cols/2], scales uint8 [rows, cols/16],
    e_fp, e_int float64 [rows, cols/16] (scaled-domain squared errors of the
    two candidates; for MODE_4OVER6 the x-domain errors of the /6 and the /4
    candidates), near uint8 [rows, cols/16] (1 = the two errors are within
    1e-6 relative, or the group's block scale is zero)).
    """
    x = _as_f32_2d(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    e_fp = np.zeros((rows, cols // 16), np.float64)
    e_int = np.zeros((rows, cols // 16), np.float64)
    near = np.zeros((rows, cols // 16), np.uint8)
    lib().orc_quantize(x, rows, cols, cols, float(np.float32(ts)), int(mode), codes, scales,
                       e_fp.ctypes.data, e_int.ctypes.data, near.ctypes.data,
                       int(threads) if threads else max_threads())
    return dict(codes=codes, scales=scales, e_fp=e_fp, e_int=e_int, near=near)


def quantize_tensor(x, mode: int = MODE_IF4, threads: int = 0):
    """Tensor amax, tensor scale, then the per-group quantizer."""
    amax = tensor_amax(x)
    ts = tensor_scale(amax)
    out = quantize(x, ts, mode, threads)
    out["amax"] = amax
    out["ts"] = ts
    return out


def rht(x, signs: int, threads: int = 0):
    """y = H16 diag(s) x_g / 4 for every 16-group (see orc_rht16)."""
    x = _as_f32_2d(x)
    y = np.zeros_like(x)
    lib().orc_rht(x, x.shape[0], x.shape[1], x.shape[1], int(signs) & 0xFFFF, y,
                  int(threads) if threads else max_threads())
    return y


def quantize_tensor_rht(x, signs: int, mode: int = MODE_IF4, threads: int = 0):
    """The transform, then amax, tensor scale and quantizer on its output."""
    out = quantize_tensor(rht(x, signs, threads), mode, threads)
    return out


def dequantize(codes, scales, ts, threads: int = 0):
    """Dequantize: float32 [rows, cols] = fl(q * fl(E4(scale) * ts))."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    if scales.shape != (rows, cols // 16):
        raise ValueError("scales must be [rows, cols/16]")
    y = np.zeros((rows, cols), np.float32)
    lib().orc_dequantize(codes, scales, float(np.float32(ts)), rows, cols, y,
                         int(threads) if threads else max_threads())
    return y


def decode_f16(codes, scales, threads: int = 0):
    """Decoded operand of the IF4 linear: fp16 RNE of fl(q * E4(scale)),
    i.e. the dequantized value with the tensor scale factored out."""
    return dequantize(codes, scales, np.float32(1.0), threads).astype(np.float16)


def linear(a_hat, b_hat, rows=None, cols=None):
    """float64 C[m, n] = sum_k A_hat[m, k] * B_hat[n, k] over the dequantized
    operands (B stored [N, K]); optionally only the given rows of A / B."""
    a = np.asarray(a_hat, dtype=np.float64)
    b = np.asarray(b_hat, dtype=np.float64)
    if rows is not None:
        a = a[np.asarray(rows)]
    if cols is not None:
        b = b[np.asarray(cols)]
    return a @ b.T


# --------------------------------------------------- other widths: IF6, IF3 --
#
# The same adaptive choice at 6 and 3 bits.  The pages name IF6 and IF3 but
# fix neither grid; see if4_oracle.c for the readings (FP6 = E2M3 against a
# 31-level INT6 reaching 7.5; FP3 = E2M0 {0, 1, 2, 4} against a 3-level INT3
# reaching 4).  Codes: element i at bits [w*i, w*i + w) of the group's
# little-endian bytes (12 per group for IF6, 6 for IF3).

W_IF, W_FP, W_INT = 0, 1, 2


def e2m3_code(v: float) -> int:
    return int(lib().orc_e2m3_code(float(np.float32(v))))


def e2m3_value(c: int) -> float:
    return float(lib().orc_e2m3_value(int(c) & 0x3F))


def int6_code(v: float) -> int:
    return int(lib().orc_int6_code(float(np.float32(v))))


def int6_value(c: int) -> float:
    return float(lib().orc_int6_value(int(c) & 0x3F))


def e2m0_code(v: float) -> int:
    return int(lib().orc_e2m0_code(float(np.float32(v))))


def e2m0_value(c: int) -> float:
    return float(lib().orc_e2m0_value(int(c) & 0x7))


def int3_code(v: float) -> int:
    return int(lib().orc_int3_code(float(np.float32(v))))


def int3_value(c: int) -> float:
    return float(lib().orc_int3_value(int(c) & 0x7))


def e2m3_code_array(values):
    return _array_fn("orc_e2m3_code_array", values)


def int6_code_array(values):
    return _array_fn("orc_int6_code_array", values)


def e2m0_code_array(values):
    return _array_fn("orc_e2m0_code_array", values)


def int3_code_array(values):
    return _array_fn("orc_int3_code_array", values)


def tensor_scale_w(amax, bits: int) -> np.float32:
    """ts = amax/(fpmax*448) (fpmax 7.5 for 6 bits, 4 for 3); 1 for amax 0."""
    return np.float32(lib().orc_tensor_scale_w(float(np.float32(amax)), int(bits)))


def quantize_w(x, ts, bits: int, mode: int = W_IF, threads: int = 0):
    """Quantize a [rows, cols] float32 array to IF6 / IF3 (bits 6 or 3), or to
    the FP-only or INT-only candidate (mode W_FP / W_INT).  Returns dict(codes
    uint8 [rows, cols*bits/8], scales uint8 [rows, cols/16], e_fp, e_int,
    near) as quantize()."""
    if bits not in (3, 6):
        raise ValueError("bits must be 3 or 6")
    x = _as_f32_2d(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols * bits // 8), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    e_fp = np.zeros((rows, cols // 16), np.float64)
    e_int = np.zeros((rows, cols // 16), np.float64)
    near = np.zeros((rows, cols // 16), np.uint8)
    lib().orc_quantize_w(x, rows, cols, cols, float(np.float32(ts)), int(bits), int(mode), codes,
                         scales, e_fp.ctypes.data, e_int.ctypes.data, near.ctypes.data,
                         int(threads) if threads else max_threads())
    return dict(codes=codes, scales=scales, e_fp=e_fp, e_int=e_int, near=near)


def quantize_tensor_w(x, bits: int, mode: int = W_IF, threads: int = 0):
    """Tensor amax, the width's tensor scale, then quantize_w."""
    amax = tensor_amax(x)
    ts = tensor_scale_w(amax, bits)
    out = quantize_w(x, ts, bits, mode, threads)
    out["amax"] = amax
    out["ts"] = ts
    return out


def dequantize_w(codes, scales, ts, bits: int, threads: int = 0):
    """float32 [rows, cols] = fl(q * fl(E4(scale) * ts)) at width bits."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, cols = scales.shape[0], scales.shape[1] * 16
    if codes.shape != (rows, cols * bits // 8):
        raise ValueError("codes must be [rows, cols*bits/8]")
    y = np.zeros((rows, cols), np.float32)
    lib().orc_dequantize_w(codes, scales, float(np.float32(ts)), rows, cols, int(bits), y,
                           int(threads) if threads else max_threads())
    return y


def mse(x, xhat) -> float:
    d = np.asarray(x, np.float64) - np.asarray(xhat, np.float64)
    return float(np.mean(d * d))


def group_int4_fraction(scales) -> float:
    s = np.asarray(scales, np.uint8)
    return float(np.mean((s >> 7) & 1)) if s.size else 0.0
