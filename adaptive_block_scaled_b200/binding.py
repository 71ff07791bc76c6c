"""ctypes binding of libif4.so.

The functions named like the C entry points take torch tensors, check that
their dtypes and strides describe what the C call expects, and pass raw
device pointers, sizes and the current CUDA stream.  Every step of the IF4
path runs in the library's kernels; torch only owns memory and streams.  The
helpers at the bottom (``quantize``, ``dequantize`` ...) allocate outputs with
torch and call the entry points.

There is no fallback: if libif4.so is missing or a call fails, an exception
is raised.
"""
import ctypes
import os

import torch

from . import build as _build

LIB_PATH = _build.LIB

IF4_OK = 0
TS_COMPUTE = 0
TS_GIVEN = 1
DEV_NONFINITE = 1
DEV_BAD_SCALE = 2
DEV_TIMEOUT = 4

_DTYPES = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int


class IF4Error(RuntimeError):
    pass


def _load():
    if not os.path.exists(LIB_PATH):
        raise IF4Error(f"{LIB_PATH} is not built; run `python -m adaptive_block_scaled_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "if4_tensor_amax": [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp],
        "if4_tensor_scale": [_vp, _vp, _vp],
        "if4_quantize": [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _int, _vp, _vp],
        "nvfp4_quantize": [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _int, _vp, _vp],
        "nvint4_quantize": [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _int, _vp, _vp],
        "nvfp4_4over6_quantize": [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _int, _vp, _vp],
        "if4_dequantize": [_vp, _vp, _vp, _i64, _i64, _vp, _int, _i64, _vp],
        "if4_tensor_amax_rht": [_vp, _int, _i64, _i64, _i64, ctypes.c_uint32, _vp, _vp, _vp],
        "if4_quantize_rht": [_vp, _int, _i64, _i64, _i64, ctypes.c_uint32, _vp, _vp, _vp, _int,
                             _vp, _vp],
        "if4_quantize_fused": [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                               _vp],
        "if4_quantize_fused_rht": [_vp, _int, _i64, _i64, _i64, ctypes.c_uint32, _vp, _vp, _vp,
                                   _vp, _vp, _vp, _vp, _vp],
        "if4_quantize_fused_shared": [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp,
                                      _int, _vp, _vp],
        "if4_quantize_fused_rht_shared": [_vp, _int, _i64, _i64, _i64, ctypes.c_uint32, _vp, _vp,
                                          _vp, _vp, _vp, _vp, _int, _vp, _vp],
        "if4_quantize_fused_dequant": [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp,
                                       _vp, _vp, _vp, _vp],
        "if4_quantize_fused_dequant_shared": [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp,
                                              _vp, _vp, _vp, _int, _vp, _vp],
        "if4_decode_f16": [_vp, _vp, _i64, _i64, _vp, _vp],
        "if4_gemm_f16": [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp],
        "if4_linear_workspace_bytes": [_i64, _i64, _i64],
        "if4_linear": [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, ctypes.c_size_t,
                       _vp, _vp, _vp],
        "if4_linear_noalloc": [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp],
        "if4_linear_fused": [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp],
        "if4_linear_quantized": [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp,
                                 ctypes.c_size_t, _vp, _vp, _vp, _vp, _vp, _vp],
        "if6_quantize": [_vp, _int, _i64, _i64, _i64, _int, _vp, _vp, _vp, _int, _vp, _vp],
        "if3_quantize": [_vp, _int, _i64, _i64, _i64, _int, _vp, _vp, _vp, _int, _vp, _vp],
        "if6_dequantize": [_vp, _vp, _vp, _i64, _i64, _vp, _int, _i64, _vp],
        "if3_dequantize": [_vp, _vp, _vp, _i64, _i64, _vp, _int, _i64, _vp],
        "if4_status_str": [_int],
        "if4_version": [],
    }
    for name, args in sig.items():
        fn = getattr(lib, name, None)
        if fn is None:
            continue
        fn.argtypes = args
        fn.restype = _int
    lib.if4_status_str.restype = ctypes.c_char_p
    if hasattr(lib, "if4_linear_workspace_bytes"):
        lib.if4_linear_workspace_bytes.restype = ctypes.c_size_t
    return lib


lib = _load()


def _check(rc: int, name: str):
    if rc != IF4_OK:
        raise IF4Error(f"{name}: {lib.if4_status_str(rc).decode()} (status {rc})")


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return _vp(s.cuda_stream)


def _ptr(t):
    return _vp(t.data_ptr()) if t is not None else _vp(0)


def _matrix(t, name):
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D")
    if t.shape[1] > 1 and t.stride(1) != 1:
        raise ValueError(f"{name} must be contiguous along its last dimension")
    return t.shape[0], t.shape[1], max(t.stride(0), t.shape[1])


def _dtype(t, name):
    if t.dtype not in _DTYPES:
        raise ValueError(f"{name}: unsupported dtype {t.dtype}")
    return _DTYPES[t.dtype]


def _u8(t, name, shape):
    if t.dtype != torch.uint8 or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous uint8 tensor of shape {tuple(shape)}")


# ------------------------------------------------------- C entry points ---

def if4_tensor_amax(x, amax, err_flag=None, stream=None):
    rows, cols, ld = _matrix(x, "x")
    _check(lib.if4_tensor_amax(_ptr(x), _dtype(x, "x"), rows, cols, ld, _ptr(amax),
                               _ptr(err_flag), _stream(stream)), "if4_tensor_amax")


def if4_tensor_scale(amax, ts, stream=None):
    _check(lib.if4_tensor_scale(_ptr(amax), _ptr(ts), _stream(stream)), "if4_tensor_scale")


def _quantize_call(fn, name, x, codes, scales, ts, ts_mode, err_flag, stream):
    rows, cols, ld = _matrix(x, "x")
    _u8(codes, "codes", (rows, cols // 2))
    _u8(scales, "scales", (rows, cols // 16))
    if ts.dtype != torch.float32 or ts.numel() < 1:
        raise ValueError("ts must be a float32 device tensor")
    _check(fn(_ptr(x), _dtype(x, "x"), rows, cols, ld, _ptr(codes), _ptr(scales), _ptr(ts),
              int(ts_mode), _ptr(err_flag), _stream(stream)), name)


def if4_quantize(x, codes, scales, ts, ts_mode=TS_COMPUTE, err_flag=None, stream=None):
    _quantize_call(lib.if4_quantize, "if4_quantize", x, codes, scales, ts, ts_mode, err_flag, stream)


def nvfp4_quantize(x, codes, scales, ts, ts_mode=TS_COMPUTE, err_flag=None, stream=None):
    _quantize_call(lib.nvfp4_quantize, "nvfp4_quantize", x, codes, scales, ts, ts_mode, err_flag,
                   stream)


def if4_tensor_amax_rht(x, signs, amax, err_flag=None, stream=None):
    rows, cols, ld = _matrix(x, "x")
    _check(lib.if4_tensor_amax_rht(_ptr(x), _dtype(x, "x"), rows, cols, ld, int(signs) & 0xFFFF,
                                   _ptr(amax), _ptr(err_flag), _stream(stream)),
           "if4_tensor_amax_rht")


def if4_quantize_rht(x, signs, codes, scales, ts, ts_mode=TS_COMPUTE, err_flag=None, stream=None):
    rows, cols, ld = _matrix(x, "x")
    _u8(codes, "codes", (rows, cols // 2))
    _u8(scales, "scales", (rows, cols // 16))
    _check(lib.if4_quantize_rht(_ptr(x), _dtype(x, "x"), rows, cols, ld, int(signs) & 0xFFFF,
                                _ptr(codes), _ptr(scales), _ptr(ts), int(ts_mode), _ptr(err_flag),
                                _stream(stream)), "if4_quantize_rht")


def _fused_args(x, codes, scales, nv_codes, nv_scales, sync_words):
    rows, cols, ld = _matrix(x, "x")
    _u8(codes, "codes", (rows, cols // 2))
    _u8(scales, "scales", (rows, cols // 16))
    if (nv_codes is None) != (nv_scales is None):
        raise ValueError("nv_codes and nv_scales go together")
    if nv_codes is not None:
        _u8(nv_codes, "nv_codes", (rows, cols // 2))
        _u8(nv_scales, "nv_scales", (rows, cols // 16))
    if sync_words.dtype != torch.int32 or sync_words.numel() < FUSED_SYNC_WORDS:
        raise ValueError(f"sync_words must be an int32 device tensor of at least "
                         f"{FUSED_SYNC_WORDS} elements")
    return rows, cols, ld


def if4_quantize_fused_shared(x, codes, scales, nv_codes, nv_scales, ts, sync_words, share,
                              err_flag=None, stream=None, signs=None):
    """The single-launch quantizer (signs=None) or its transform form on
    1/share of the device's resident blocks (if4_quantize_fused_shared /
    if4_quantize_fused_rht_shared); outputs byte-identical to the plain
    call."""
    rows, cols, ld = _fused_args(x, codes, scales, nv_codes, nv_scales, sync_words)
    if signs is None:
        _check(lib.if4_quantize_fused_shared(_ptr(x), _dtype(x, "x"), rows, cols, ld,
                                             _ptr(codes), _ptr(scales), _ptr(nv_codes),
                                             _ptr(nv_scales), _ptr(ts), _ptr(sync_words),
                                             int(share), _ptr(err_flag), _stream(stream)),
               "if4_quantize_fused_shared")
    else:
        _check(lib.if4_quantize_fused_rht_shared(_ptr(x), _dtype(x, "x"), rows, cols, ld,
                                                 int(signs) & 0xFFFF, _ptr(codes), _ptr(scales),
                                                 _ptr(nv_codes), _ptr(nv_scales), _ptr(ts),
                                                 _ptr(sync_words), int(share), _ptr(err_flag),
                                                 _stream(stream)),
               "if4_quantize_fused_rht_shared")


def if4_quantize_fused(x, codes, scales, nv_codes, nv_scales, ts, sync_words, err_flag=None,
                       stream=None, signs=None):
    """signs=None: the plain single-launch quantizer; an int: the same on the
    random-sign Hadamard transform of x (if4_quantize_fused_rht)."""
    rows, cols, ld = _fused_args(x, codes, scales, nv_codes, nv_scales, sync_words)
    if signs is None:
        _check(lib.if4_quantize_fused(_ptr(x), _dtype(x, "x"), rows, cols, ld, _ptr(codes),
                                      _ptr(scales), _ptr(nv_codes), _ptr(nv_scales), _ptr(ts),
                                      _ptr(sync_words), _ptr(err_flag), _stream(stream)),
               "if4_quantize_fused")
    else:
        _check(lib.if4_quantize_fused_rht(_ptr(x), _dtype(x, "x"), rows, cols, ld,
                                          int(signs) & 0xFFFF, _ptr(codes), _ptr(scales),
                                          _ptr(nv_codes), _ptr(nv_scales), _ptr(ts),
                                          _ptr(sync_words), _ptr(err_flag), _stream(stream)),
               "if4_quantize_fused_rht")


def nvint4_quantize(x, codes, scales, ts, ts_mode=TS_COMPUTE, err_flag=None, stream=None):
    _quantize_call(lib.nvint4_quantize, "nvint4_quantize", x, codes, scales, ts, ts_mode,
                   err_flag, stream)


def nvfp4_4over6_quantize(x, codes, scales, ts, ts_mode=TS_COMPUTE, err_flag=None, stream=None):
    _quantize_call(lib.nvfp4_4over6_quantize, "nvfp4_4over6_quantize", x, codes, scales, ts,
                   ts_mode, err_flag, stream)


def if4_dequantize(codes, scales, ts, y, stream=None):
    rows, cols, ld = _matrix(y, "y")
    _u8(codes, "codes", (rows, cols // 2))
    _u8(scales, "scales", (rows, cols // 16))
    _check(lib.if4_dequantize(_ptr(codes), _ptr(scales), _ptr(ts), rows, cols, _ptr(y),
                              _dtype(y, "y"), ld, _stream(stream)), "if4_dequantize")


def if4_decode_f16(codes, scales, y, stream=None):
    rows, cols = y.shape
    if y.dtype != torch.float16 or not y.is_contiguous():
        raise ValueError("y must be a contiguous float16 tensor")
    _u8(codes, "codes", (rows, cols // 2))
    _u8(scales, "scales", (rows, cols // 16))
    _check(lib.if4_decode_f16(_ptr(codes), _ptr(scales), rows, cols, _ptr(y), _stream(stream)),
           "if4_decode_f16")


def if4_gemm_f16(a, b, a_ts, b_ts, c, err_flag, stream=None):
    M, K = a.shape
    N = b.shape[0]
    for t, n in ((a, "a"), (b, "b")):
        if t.dtype != torch.float16 or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous float16 tensor")
    if b.shape[1] != K or tuple(c.shape) != (M, N) or c.dtype != torch.bfloat16:
        raise ValueError("shapes: a [M,K], b [N,K], c bf16 [M,N]")
    _check(lib.if4_gemm_f16(_ptr(a), _ptr(b), _ptr(a_ts), _ptr(b_ts), M, N, K, _ptr(c),
                            _ptr(err_flag), _stream(stream)), "if4_gemm_f16")


def if4_linear_workspace_bytes(M, N, K):
    return int(lib.if4_linear_workspace_bytes(int(M), int(N), int(K)))


def if4_linear(a_codes, a_scales, a_ts, b_codes, b_scales, b_ts, workspace, c, err_flag,
               stream=None):
    M, N = c.shape
    K = a_codes.shape[1] * 2
    _u8(a_codes, "a_codes", (M, K // 2))
    _u8(a_scales, "a_scales", (M, K // 16))
    _u8(b_codes, "b_codes", (N, K // 2))
    _u8(b_scales, "b_scales", (N, K // 16))
    if c.dtype != torch.bfloat16 or not c.is_contiguous():
        raise ValueError("c must be a contiguous bf16 tensor")
    _check(lib.if4_linear(_ptr(a_codes), _ptr(a_scales), _ptr(a_ts), _ptr(b_codes),
                          _ptr(b_scales), _ptr(b_ts), M, N, K, _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _ptr(c),
                          _ptr(err_flag), _stream(stream)), "if4_linear")


def if4_linear_fused(a_codes, a_scales, a_ts, b_codes, b_scales, b_ts, c, err_flag,
                     stream=None):
    """The IF4 x IF4 linear with the operand decode inside the GEMM (no
    workspace); the same C as if4_linear, bit for bit."""
    M, N = c.shape
    K = a_codes.shape[1] * 2
    _u8(a_codes, "a_codes", (M, K // 2))
    _u8(a_scales, "a_scales", (M, K // 16))
    _u8(b_codes, "b_codes", (N, K // 2))
    _u8(b_scales, "b_scales", (N, K // 16))
    if c.dtype != torch.bfloat16 or not c.is_contiguous():
        raise ValueError("c must be a contiguous bf16 tensor")
    _check(lib.if4_linear_fused(_ptr(a_codes), _ptr(a_scales), _ptr(a_ts), _ptr(b_codes),
                                _ptr(b_scales), _ptr(b_ts), M, N, K, _ptr(c), _ptr(err_flag),
                                _stream(stream)), "if4_linear_fused")


def if4_linear_noalloc(a_codes, a_scales, a_ts, b_codes, b_scales, b_ts, c, err_flag,
                       stream=None):
    """if4_linear with the library's fixed device scratch instead of a
    caller workspace (problems up to IF4_LINEAR_NOALLOC_MAX_BYTES)."""
    M, N = c.shape
    K = a_codes.shape[1] * 2
    _u8(a_codes, "a_codes", (M, K // 2))
    _u8(a_scales, "a_scales", (M, K // 16))
    _u8(b_codes, "b_codes", (N, K // 2))
    _u8(b_scales, "b_scales", (N, K // 16))
    if c.dtype != torch.bfloat16 or not c.is_contiguous():
        raise ValueError("c must be a contiguous bf16 tensor")
    _check(lib.if4_linear_noalloc(_ptr(a_codes), _ptr(a_scales), _ptr(a_ts), _ptr(b_codes),
                                  _ptr(b_scales), _ptr(b_ts), M, N, K, _ptr(c),
                                  _ptr(err_flag), _stream(stream)), "if4_linear_noalloc")


def if4_linear_quantized(a_codes, a_scales, a_ts, b_codes, b_scales, b_ts, workspace, c_codes,
                         c_scales, c_ts, c=None, err_flag=None, stream=None):
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    _u8(a_codes, "a_codes", (M, K // 2))
    _u8(a_scales, "a_scales", (M, K // 16))
    _u8(b_codes, "b_codes", (N, K // 2))
    _u8(b_scales, "b_scales", (N, K // 16))
    _u8(c_codes, "c_codes", (M, N // 2))
    _u8(c_scales, "c_scales", (M, N // 16))
    if c is not None and (c.dtype != torch.bfloat16 or not c.is_contiguous()):
        raise ValueError("c must be a contiguous bf16 tensor")
    _check(lib.if4_linear_quantized(_ptr(a_codes), _ptr(a_scales), _ptr(a_ts), _ptr(b_codes),
                                    _ptr(b_scales), _ptr(b_ts), M, N, K, _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _ptr(c),
                                    _ptr(c_codes), _ptr(c_scales), _ptr(c_ts), _ptr(err_flag),
                                    _stream(stream)), "if4_linear_quantized")


# ------------------------------------------------------- IF6 and IF3 ---

W_ADAPTIVE, W_FP_ONLY, W_INT_ONLY = 0, 1, 2


def _width_fns(bits):
    if bits == 6:
        return lib.if6_quantize, lib.if6_dequantize, "if6"
    if bits == 3:
        return lib.if3_quantize, lib.if3_dequantize, "if3"
    raise ValueError("bits must be 6 or 3")


def ifw_quantize(x, bits, mode, codes, scales, ts, ts_mode=TS_COMPUTE, err_flag=None,
                 stream=None):
    """if6_quantize / if3_quantize: codes uint8 [rows, cols*bits/8]."""
    qfn, _, name = _width_fns(bits)
    rows, cols, ld = _matrix(x, "x")
    _u8(codes, "codes", (rows, cols * bits // 8))
    _u8(scales, "scales", (rows, cols // 16))
    if ts.dtype != torch.float32 or ts.numel() < 1:
        raise ValueError("ts must be a float32 device tensor")
    _check(qfn(_ptr(x), _dtype(x, "x"), rows, cols, ld, int(mode), _ptr(codes), _ptr(scales),
               _ptr(ts), int(ts_mode), _ptr(err_flag), _stream(stream)), name + "_quantize")


def ifw_dequantize(codes, scales, ts, bits, y, stream=None):
    """if6_dequantize / if3_dequantize into y [rows, cols] (f32, bf16 or f16)."""
    _, dfn, name = _width_fns(bits)
    rows, cols, ld = _matrix(y, "y")
    _u8(codes, "codes", (rows, cols * bits // 8))
    _u8(scales, "scales", (rows, cols // 16))
    _check(dfn(_ptr(codes), _ptr(scales), _ptr(ts), rows, cols, _ptr(y), _dtype(y, "y"), ld,
               _stream(stream)), name + "_dequantize")


def quantize_w(x, bits, mode=W_ADAPTIVE, ts=None, err_flag=None, stream=None):
    """IF6 (bits=6) or IF3 (bits=3) of a 2-D tensor, or the FP-only / INT-only
    candidate (mode).  Returns (codes, scales, ts); ts=None computes it."""
    rows, cols, _ = _matrix(x, "x")
    dev = x.device
    codes = torch.empty((rows, cols * bits // 8), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    if ts is None:
        ts_t, ts_mode = torch.empty(1, dtype=torch.float32, device=dev), TS_COMPUTE
    else:
        ts_t, ts_mode = ts, TS_GIVEN
    ifw_quantize(x, bits, mode, codes, scales, ts_t, ts_mode, err_flag, stream)
    return codes, scales, ts_t


def dequantize_w(codes, scales, ts, bits, dtype=torch.bfloat16, stream=None):
    rows, cols = scales.shape[0], scales.shape[1] * 16
    y = torch.empty((rows, cols), dtype=dtype, device=codes.device)
    ifw_dequantize(codes, scales, ts, bits, y, stream)
    return y


LINEAR_NOALLOC_MAX_BYTES = 32 * 1024 * 1024
FUSED_SYNC_WORDS = 64


# ---------------------------------------------------- allocating helpers ---

def quantize(x, mode="if4", ts=None, err_flag=None, stream=None):
    """Quantize a 2-D tensor on its device with mode "if4", "nvfp4", "nvint4"
    or "4over6".  Returns (codes, scales, ts).  ts=None computes the tensor
    scale; a float32 tensor is used as given."""
    rows, cols, _ = _matrix(x, "x")
    dev = x.device
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    if ts is None:
        ts_t, ts_mode = torch.empty(1, dtype=torch.float32, device=dev), TS_COMPUTE
    else:
        ts_t, ts_mode = ts, TS_GIVEN
    fn = {"if4": if4_quantize, "nvfp4": nvfp4_quantize, "nvint4": nvint4_quantize,
          "4over6": nvfp4_4over6_quantize}[mode]
    fn(x, codes, scales, ts_t, ts_mode, err_flag, stream)
    return codes, scales, ts_t


def quantize_rht(x, signs, ts=None, err_flag=None, stream=None):
    """Random-sign Hadamard transform + IF4 quantize.  Returns (codes, scales, ts)."""
    rows, cols, _ = _matrix(x, "x")
    dev = x.device
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    if ts is None:
        ts_t, ts_mode = torch.empty(1, dtype=torch.float32, device=dev), TS_COMPUTE
    else:
        ts_t, ts_mode = ts, TS_GIVEN
    if4_quantize_rht(x, signs, codes, scales, ts_t, ts_mode, err_flag, stream)
    return codes, scales, ts_t


def if4_quantize_fused_dequant(x, codes, scales, nv_codes, nv_scales, ts, sync_words, y,
                               err_flag=None, stream=None):
    """The single launch that also writes y, the bf16 decode of its IF4 codes
    (dense, 32-byte aligned)."""
    rows, cols, ld = _fused_dequant_args(x, codes, scales, nv_codes, nv_scales, sync_words, y)
    _check(lib.if4_quantize_fused_dequant(_ptr(x), _dtype(x, "x"), rows, cols, ld, _ptr(codes),
                                          _ptr(scales), _ptr(nv_codes), _ptr(nv_scales),
                                          _ptr(ts), _ptr(sync_words), _ptr(y), _ptr(err_flag),
                                          _stream(stream)),
           "if4_quantize_fused_dequant")


def if4_quantize_fused_dequant_shared(x, codes, scales, nv_codes, nv_scales, ts, sync_words, y,
                                      share, err_flag=None, stream=None):
    """The same launch on 1/share of the device's resident blocks, for
    `share` calls at once on different streams (each with its own
    sync_words); outputs byte-identical to if4_quantize_fused_dequant."""
    rows, cols, ld = _fused_dequant_args(x, codes, scales, nv_codes, nv_scales, sync_words, y)
    _check(lib.if4_quantize_fused_dequant_shared(_ptr(x), _dtype(x, "x"), rows, cols, ld,
                                                 _ptr(codes), _ptr(scales), _ptr(nv_codes),
                                                 _ptr(nv_scales), _ptr(ts), _ptr(sync_words),
                                                 _ptr(y), int(share), _ptr(err_flag),
                                                 _stream(stream)),
           "if4_quantize_fused_dequant_shared")


def _fused_dequant_args(x, codes, scales, nv_codes, nv_scales, sync_words, y):
    rows, cols, ld = _matrix(x, "x")
    _u8(codes, "codes", (rows, cols // 2))
    _u8(scales, "scales", (rows, cols // 16))
    if (nv_codes is None) != (nv_scales is None):
        raise ValueError("nv_codes and nv_scales go together")
    if nv_codes is not None:
        _u8(nv_codes, "nv_codes", (rows, cols // 2))
        _u8(nv_scales, "nv_scales", (rows, cols // 16))
    if sync_words.dtype != torch.int32 or sync_words.numel() < FUSED_SYNC_WORDS:
        raise ValueError(f"sync_words must be an int32 device tensor of at least "
                         f"{FUSED_SYNC_WORDS} elements")
    if y.dtype != torch.bfloat16 or tuple(y.shape) != (rows, cols) or not y.is_contiguous():
        raise ValueError("y must be a dense bf16 tensor of the shape of x")
    return rows, cols, ld


def quantize_fused_dequant(x, with_nvfp4=True, sync_words=None, err_flag=None, stream=None):
    """The quantize-then-dequantize round trip in one launch.  Returns
    (codes, scales, ts, y) or (codes, scales, ts, nv_codes, nv_scales, y)."""
    rows, cols, _ = _matrix(x, "x")
    dev = x.device
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    nv_codes = torch.empty_like(codes) if with_nvfp4 else None
    nv_scales = torch.empty_like(scales) if with_nvfp4 else None
    ts = torch.empty(1, dtype=torch.float32, device=dev)
    y = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev)
    if sync_words is None:
        sync_words = torch.zeros(FUSED_SYNC_WORDS, dtype=torch.int32, device=dev)
    if4_quantize_fused_dequant(x, codes, scales, nv_codes, nv_scales, ts, sync_words, y,
                               err_flag, stream)
    if with_nvfp4:
        return codes, scales, ts, nv_codes, nv_scales, y
    return codes, scales, ts, y


def quantize_fused(x, with_nvfp4=True, sync_words=None, err_flag=None, stream=None, signs=None):
    """amax, tensor scale, IF4 quantize (and NVFP4) in one launch, of x or,
    with signs, of its random-sign Hadamard transform.  Returns (codes,
    scales, ts) or (codes, scales, ts, nv_codes, nv_scales)."""
    rows, cols, _ = _matrix(x, "x")
    dev = x.device
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    nv_codes = torch.empty_like(codes) if with_nvfp4 else None
    nv_scales = torch.empty_like(scales) if with_nvfp4 else None
    ts = torch.empty(1, dtype=torch.float32, device=dev)
    if sync_words is None:
        sync_words = torch.zeros(FUSED_SYNC_WORDS, dtype=torch.int32, device=dev)
    if4_quantize_fused(x, codes, scales, nv_codes, nv_scales, ts, sync_words, err_flag, stream,
                       signs)
    return (codes, scales, ts, nv_codes, nv_scales) if with_nvfp4 else (codes, scales, ts)


def dequantize(codes, scales, ts, dtype=torch.bfloat16, stream=None):
    rows, cols = codes.shape[0], codes.shape[1] * 2
    y = torch.empty((rows, cols), dtype=dtype, device=codes.device)
    if4_dequantize(codes, scales, ts, y, stream)
    return y


def decode_f16(codes, scales, stream=None):
    rows, cols = codes.shape[0], codes.shape[1] * 2
    y = torch.empty((rows, cols), dtype=torch.float16, device=codes.device)
    if4_decode_f16(codes, scales, y, stream)
    return y
