"""The C ABI on a host without a GPU: libif4.so builds for sm_100a, loads,
exports every function include/*.h declares, and rejects invalid arguments
with the documented status before touching the device.  No kernel runs and
no pointer passed here is dereferenced."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from adaptive_block_scaled_b200 import build
    path = build.build()
    L = ctypes.CDLL(path)
    vp, i64, i = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.if4_quantize.argtypes = [vp, i, i64, i64, i64, vp, vp, vp, i, vp, vp]
    L.nvfp4_quantize.argtypes = L.if4_quantize.argtypes
    L.if4_dequantize.argtypes = [vp, vp, vp, i64, i64, vp, i, i64, vp]
    L.if4_tensor_amax.argtypes = [vp, i, i64, i64, i64, vp, vp, vp]
    L.if4_tensor_scale.argtypes = [vp, vp, vp]
    L.if4_decode_f16.argtypes = [vp, vp, i64, i64, vp, vp]
    L.if4_quantize_fused.argtypes = [vp, i, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp]
    L.if4_quantize_fused_rht.argtypes = [vp, i, i64, i64, i64, ctypes.c_uint32, vp, vp, vp, vp,
                                         vp, vp, vp, vp]
    L.if4_quantize_fused_dequant.argtypes = [vp, i, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp,
                                             vp, vp]
    L.if4_quantize_fused_dequant_shared.argtypes = [vp, i, i64, i64, i64, vp, vp, vp, vp, vp, vp,
                                                    vp, i, vp, vp]
    L.if4_quantize_fused_shared.argtypes = [vp, i, i64, i64, i64, vp, vp, vp, vp, vp, vp, i, vp,
                                            vp]
    L.if4_quantize_fused_rht_shared.argtypes = [vp, i, i64, i64, i64, ctypes.c_uint32, vp, vp,
                                                vp, vp, vp, vp, i, vp, vp]
    L.if4_linear_quantized.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, ctypes.c_size_t,
                                       vp, vp, vp, vp, vp, vp]
    L.if4_linear_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, vp, vp]
    for w in ("if6", "if3"):
        getattr(L, w + "_quantize").argtypes = [vp, i, i64, i64, i64, i, vp, vp, vp, i, vp, vp]
        getattr(L, w + "_dequantize").argtypes = [vp, vp, vp, i64, i64, vp, i, i64, vp]
    L.if4_status_str.restype = ctypes.c_char_p
    return L


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(",
                             text, flags=re.M):
            if not m.group(0).lstrip().startswith(("typedef", "enum", "struct", "#")):
                names.append(m.group(1))
    return sorted(set(names))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("if4_quantize", "nvfp4_quantize", "if4_dequantize", "if4_tensor_amax",
              "if4_tensor_scale", "if4_decode_f16", "if4_status_str", "if4_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from adaptive_block_scaled_b200 import build
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in declared_functions():
        assert n in exported, n
        assert hasattr(lib, n)
    # nothing but the C ABI leaks out (the static CUDA runtime stays local)
    assert all(n.startswith(("if4_", "if6_", "if3_", "nvfp4_", "nvint4_")) for n in exported), \
        sorted(exported)[:10]


def test_status_strings(lib):
    assert lib.if4_version() >= 100
    for s in range(9):
        assert lib.if4_status_str(s)
    assert b"unknown" in lib.if4_status_str(99)


A = 0x100000          # a 256-byte aligned address; never dereferenced here


@pytest.mark.parametrize("fn", ["if4_quantize", "nvfp4_quantize"])
def test_quantize_host_validation(lib, fn):
    f = getattr(lib, fn)
    # null input, codes, ts
    assert f(None, 1, 4, 32, 32, A, A, A, 0, None, None) == 1
    assert f(A, 1, 4, 32, 32, None, A, A, 0, None, None) == 1
    assert f(A, 1, 4, 32, 32, A, A, None, 0, None, None) == 1
    # shapes: cols % 16, negative sizes, ld < cols, too many groups
    assert f(A, 1, 4, 24, 24, A, A, A, 0, None, None) == 2
    assert f(A, 1, -1, 32, 32, A, A, A, 0, None, None) == 2
    assert f(A, 1, 4, 32, 16, A, A, A, 0, None, None) == 2
    assert f(A, 1, 1 << 31, 32, 32, A, A, A, 0, None, None) == 2
    # dtype, mode
    assert f(A, 7, 4, 32, 32, A, A, A, 0, None, None) == 3
    assert f(A, 1, 4, 32, 32, A, A, A, 9, None, None) == 5
    # alignment: x, ld, codes, ts
    assert f(A + 8, 1, 4, 32, 32, A, A, A, 0, None, None) == 4
    assert f(A, 1, 4, 32, 36, A, A, A, 0, None, None) == 4
    assert f(A, 1, 4, 32, 32, A + 8, A, A, 0, None, None) == 4
    assert f(A, 1, 4, 32, 32, A, A, A + 2, 0, None, None) == 4


def test_fused_quantize_host_validation(lib):
    f = lib.if4_quantize_fused
    # null x / codes / ts / sync words, half of the NVFP4 pair
    assert f(None, 1, 4, 32, 32, A, A, None, None, A, A, None, None) == 1
    assert f(A, 1, 4, 32, 32, None, A, None, None, A, A, None, None) == 1
    assert f(A, 1, 4, 32, 32, A, A, None, None, None, A, None, None) == 1
    assert f(A, 1, 4, 32, 32, A, A, None, None, A, None, None, None) == 1
    assert f(A, 1, 4, 32, 32, A, A, A, None, A, A, None, None) == 1
    # shape, dtype, alignment of x, codes, nv_codes, ts, sync words
    assert f(A, 1, 4, 24, 24, A, A, None, None, A, A, None, None) == 2
    assert f(A, 9, 4, 32, 32, A, A, None, None, A, A, None, None) == 3
    assert f(A + 8, 1, 4, 32, 32, A, A, None, None, A, A, None, None) == 4
    assert f(A, 1, 4, 32, 32, A + 8, A, None, None, A, A, None, None) == 4
    assert f(A, 1, 4, 32, 32, A, A, A + 8, A, A, A, None, None) == 4
    assert f(A, 1, 4, 32, 32, A, A, None, None, A + 2, A, None, None) == 4
    assert f(A, 1, 4, 32, 32, A, A, None, None, A, A + 4, None, None) == 4
    assert f(A, 1, 4, 32, 32, A, A, None, None, A, A + 128, None, None) == 4
    h = lib.if4_quantize_fused_dequant
    # null y of a non-empty tensor; y not 32-byte aligned; the rest as above
    assert h(A, 1, 4, 32, 32, A, A, None, None, A, A, None, None, None) == 1
    assert h(A, 1, 4, 32, 32, A, A, None, None, A, A, A + 16, None, None) == 4
    assert h(A, 1, 4, 32, 32, A, A, None, None, None, A, A, None, None) == 1
    assert h(A, 1, 4, 24, 24, A, A, None, None, A, A, A, None, None) == 2
    assert h(A, 1, 4, 32, 32, A, A, None, None, A, A + 64, A, None, None) == 4
    k = lib.if4_quantize_fused_dequant_shared
    # the share of the device: 1..64; then the rules of the plain call
    assert k(A, 1, 4, 32, 32, A, A, None, None, A, A, A, 0, None, None) == 2
    assert k(A, 1, 4, 32, 32, A, A, None, None, A, A, A, 65, None, None) == 2
    assert k(A, 1, 4, 32, 32, A, A, None, None, A, A, None, 2, None, None) == 1
    assert k(A, 1, 4, 32, 32, A, A, None, None, A, A, A + 16, 2, None, None) == 4
    assert k(A, 1, 4, 24, 24, A, A, None, None, A, A, A, 2, None, None) == 2
    assert k(A, 1, 4, 32, 32, A, A, None, None, A, A + 64, A, 2, None, None) == 4
    m = lib.if4_quantize_fused_shared
    assert m(A, 1, 4, 32, 32, A, A, None, None, A, A, 0, None, None) == 2
    assert m(A, 1, 4, 32, 32, A, A, None, None, None, A, 2, None, None) == 1
    assert m(A, 1, 4, 32, 32, A, A, None, None, A, A + 64, 2, None, None) == 4
    n = lib.if4_quantize_fused_rht_shared
    assert n(A, 1, 4, 32, 32, 0x1234, A, A, None, None, A, A, 65, None, None) == 2
    assert n(A, 1, 4, 32, 32, 0x1234, A, A, None, None, None, A, 2, None, None) == 1
    g = lib.if4_quantize_fused_rht
    assert g(A, 1, 4, 32, 32, 0x1234, A, A, None, None, None, A, None, None) == 1
    assert g(A, 1, 4, 24, 24, 0x1234, A, A, None, None, A, A, None, None) == 2
    assert g(A, 1, 4, 32, 32, 0x1234, A, A, None, None, A, A + 64, None, None) == 4


def test_linear_quantized_host_validation(lib):
    f = lib.if4_linear_quantized
    W = 1 << 30
    # null output codes / scales / tensor scale
    assert f(A, A, A, A, A, A, 128, 256, 64, A, W, None, None, A, A, A, None) == 1
    assert f(A, A, A, A, A, A, 128, 256, 64, A, W, None, A, None, A, A, None) == 1
    assert f(A, A, A, A, A, A, 128, 256, 64, A, W, None, A, A, None, A, None) == 1
    # N % 16, misaligned codes / ts, too small a workspace
    assert f(A, A, A, A, A, A, 128, 264, 64, A, W, None, A, A, A, A, None) == 2
    assert f(A, A, A, A, A, A, 128, 256, 64, A, W, None, A + 8, A, A, A, None) == 4
    assert f(A, A, A, A, A, A, 128, 256, 64, A, W, None, A, A, A + 2, A, None) == 4
    assert f(A, A, A, A, A, A, 128, 256, 64, A, 16, None, A, A, A, A, None) == 6


def test_linear_noalloc_error_order(lib):
    """The allocation-free linear reports errors in if4_linear's order: a
    problem too large for its scratch array is refused with
    IF4_ERR_WORKSPACE only when every other argument is valid."""
    f = lib.if4_linear_noalloc
    big = (4096, 4096, 4096)        # 64 MiB of decoded operands > the 32 MiB array
    assert f(A, A, A, A, A, A, *big, A, A, None) == 6
    assert f(None, A, A, A, A, A, *big, A, A, None) == 1
    assert f(A, A, A, A, A, A, *big, A, None, None) == 1      # err_flag
    assert f(A, A, A, A, A, A, 4096, 4096, 4104, A, A, None) == 2
    assert f(A, A, A, A, A, A, *big, A + 8, A, None) == 4     # c misaligned
    assert f(A, A, A, A, A, A, 0, 4096, 4096, A, A, None) == 2


@pytest.mark.parametrize("w", ["if6", "if3"])
def test_other_widths_host_validation(lib, w):
    """IF6 / IF3 entry points reject invalid arguments before any launch."""
    q = getattr(lib, w + "_quantize")
    assert q(A, 1, 4, 24, 24, 0, A, A, A, 0, None, None) == 2          # cols % 16
    assert q(A, 9, 4, 32, 32, 0, A, A, A, 0, None, None) == 3          # dtype
    assert q(A, 1, 4, 32, 32, 3, A, A, A, 0, None, None) == 5          # mode
    assert q(A, 1, 4, 32, 32, 0, A, A, A, 7, None, None) == 5          # ts_mode
    assert q(A, 1, 4, 32, 32, 0, A, A, None, 0, None, None) == 1       # ts
    assert q(A, 1, 4, 32, 32, 0, None, A, A, 0, None, None) == 1       # codes
    assert q(A + 8, 1, 4, 32, 32, 0, A, A, A, 0, None, None) == 4      # x alignment
    assert q(A, 1, 4, 32, 32, 0, A + 2, A, A, 0, None, None) == 4      # codes alignment
    d = getattr(lib, w + "_dequantize")
    assert d(None, A, A, 4, 32, A, 1, 32, None) == 1
    assert d(A, A, A, 4, 40, A, 1, 40, None) == 2
    assert d(A, A, A, 4, 32, A, 5, 32, None) == 3
    assert d(A + 2, A, A, 4, 32, A, 1, 32, None) == 4


def test_linear_fused_host_validation(lib):
    f = lib.if4_linear_fused
    f.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int64] * 3 + [ctypes.c_void_p] * 3
    assert f(None, A, A, A, A, A, 128, 256, 64, A, A, None) == 1
    assert f(A, A, A, A, A, A, 128, 256, 80, A, A, None) == 2      # K % 64
    assert f(A + 16, A, A, A, A, A, 128, 256, 64, A, A, None) == 4  # codes not 32-byte aligned
    assert f(A, A + 2, A, A, A, A, 128, 256, 64, A, A, None) == 4   # scales not 4-byte aligned
    assert f(A, A, A, A, A, A, 128, 252, 64, A, A, None) == 2      # N % 8


def test_dequantize_and_decode_host_validation(lib):
    f = lib.if4_dequantize
    assert f(None, A, A, 4, 32, A, 1, 32, None) == 1
    assert f(A, A, None, 4, 32, A, 1, 32, None) == 1
    assert f(A, A, A, 4, 40, A, 1, 40, None) == 2
    assert f(A, A, A, 4, 32, A, 5, 32, None) == 3
    assert f(A, A, A, 4, 32, A + 4, 1, 32, None) == 4
    assert f(A + 1, A, A, 4, 32, A, 1, 32, None) == 4
    g = lib.if4_decode_f16
    assert g(None, A, 4, 32, A, None) == 1
    assert g(A, A, 4, 33, A, None) == 2
    assert g(A, A, 4, 32, A + 2, None) == 4


def test_amax_and_scale_host_validation(lib):
    assert lib.if4_tensor_amax(A, 1, 4, 32, 32, None, None, None) == 1
    assert lib.if4_tensor_amax(A, 3, 4, 32, 32, A, None, None) == 3
    assert lib.if4_tensor_amax(A, 0, 4, 32, 30, A, None, None) == 2
    assert lib.if4_tensor_scale(None, A, None) == 1
    assert lib.if4_tensor_scale(A + 1, A, None) == 4


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    """The Python binding has no fallback: a missing library is an error."""
    import importlib
    import sys
    import adaptive_block_scaled_b200.build as b
    saved = sys.modules.pop("adaptive_block_scaled_b200.binding", None)
    monkeypatch.setattr(b, "LIB", str(tmp_path / "missing.so"))
    try:
        with pytest.raises(RuntimeError, match="not built"):
            importlib.import_module("adaptive_block_scaled_b200.binding")
    finally:
        monkeypatch.undo()
        sys.modules.pop("adaptive_block_scaled_b200.binding", None)
        if saved is not None:
            sys.modules["adaptive_block_scaled_b200.binding"] = saved


def test_round_trip_binding_checks_y(lib):
    """The binding of if4_quantize_fused_dequant rejects a y that is not a
    dense bf16 tensor of the shape of x before calling the library."""
    import torch
    from adaptive_block_scaled_b200 import binding as b
    x = torch.zeros((4, 32), dtype=torch.bfloat16)
    codes = torch.zeros((4, 16), dtype=torch.uint8)
    scales = torch.zeros((4, 2), dtype=torch.uint8)
    ts = torch.zeros(1)
    sync = torch.zeros(b.FUSED_SYNC_WORDS, dtype=torch.int32)
    for y in (torch.zeros((4, 32)),                                  # float32
              torch.zeros((4, 16), dtype=torch.bfloat16),            # wrong shape
              torch.zeros((4, 64), dtype=torch.bfloat16)[:, ::2]):   # not dense
        with pytest.raises(ValueError):
            b.if4_quantize_fused_dequant(x, codes, scales, None, None, ts, sync, y)
