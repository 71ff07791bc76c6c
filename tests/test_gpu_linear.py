"""GPU tests of the IF4 x IF4 linear, through the C ABI.

The GEMM stage alone (if4_gemm_f16) is compared with a float64 product of
its fp16 operands on small and ragged shapes.  The whole linear is compared
with the oracle's float64 product of the dequantized IF4 operands:
max |C - R| / max |R| <= 1e-2 (the stated tolerance), on sampled full rows
and columns at 8192 x 4096 x 4096 and on every entry at 512 x 512 x 4096.
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


def gemm(a, b, a_ts=1.0, b_ts=1.0):
    bb = B()
    M, N = a.shape[0], b.shape[0]
    c = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ta = torch.tensor([a_ts], dtype=torch.float32, device="cuda")
    tb = torch.tensor([b_ts], dtype=torch.float32, device="cuda")
    bb.if4_gemm_f16(a, b, ta, tb, c, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return c


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 264, 80), (1, 8, 16), (300, 520, 4096),
                                   (1024, 1024, 4096), (129, 257 + 7, 1008), (2048, 4096, 512)])
def test_gemm_f16_against_float64(M, N, K):
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    a = torch.randn((M, K), generator=g).to(torch.float16)
    b = (torch.randn((N, K), generator=g) * 0.1).to(torch.float16)
    s_a, s_b = 0.75, 1.25
    c = gemm(a.cuda(), b.cuda(), s_a, s_b).float().cpu().numpy()
    a64, b64 = a.double().numpy(), b.double().numpy()
    ref = (a64 @ b64.T) * (np.float32(s_a) * np.float32(s_b))
    mag = (np.abs(a64) @ np.abs(b64).T) * s_a * s_b
    assert np.all(np.isfinite(c))
    err = np.abs(c - ref)
    tol = 2.0 ** -8 * np.abs(ref) + 1e-5 * mag + 1e-30
    assert np.all(err <= tol), (float(err.max()), int((err > tol).sum()))


def test_gemm_does_not_write_outside_c():
    bb = B()
    M, N, K = 130, 264, 96
    a = torch.randn((M, K)).to(torch.float16).cuda()
    b = torch.randn((N, K)).to(torch.float16).cuda()
    big = torch.full((M + 2, N), 7.0, dtype=torch.bfloat16, device="cuda")
    c = big[1:M + 1]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    bb.if4_gemm_f16(a, b, one, one, c, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.all(big[0] == 7.0) and torch.all(big[M + 1] == 7.0)


def _quantized(x):
    codes, scales, ts = B().quantize(x.cuda())
    return codes, scales, ts


def _linear(aq, bq, M, N, K):
    bb = B()
    ws = torch.empty(bb.if4_linear_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    c = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bb.if4_linear(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], ws, c, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return c


def _dequant_ref(q):
    return oracle.dequantize(q[0].cpu().numpy(), q[1].cpu().numpy(), np.float32(q[2].item()))


def _rel(c, ref):
    return float(np.max(np.abs(c - ref)) / np.max(np.abs(ref)))


def test_linear_full_check_512():
    a, b = workloads.linear_operands(0, M=512, N=512, K=4096)
    aq, bq = _quantized(a), _quantized(b)
    c = _linear(aq, bq, 512, 512, 4096).float().cpu().numpy()
    ref = oracle.linear(_dequant_ref(aq), _dequant_ref(bq))
    rel = _rel(c, ref)
    med = float(np.median(np.abs(c - ref) / np.maximum(np.abs(ref), 1e-30)))
    print(f"[linear 512x512x4096] max|C-R|/max|R| = {rel:.3e}, median rel = {med:.3e}")
    assert rel <= 1e-2


def test_linear_workload_sampled_rows_and_columns():
    M, N, K = 8192, 4096, 4096
    a, b = workloads.linear_operands(0, M=M, N=N, K=K)
    aq, bq = _quantized(a), _quantized(b)
    c = _linear(aq, bq, M, N, K).float().cpu().numpy()
    ah, bh = _dequant_ref(aq), _dequant_ref(bq)
    rng = np.random.default_rng(11)
    rows = np.sort(rng.choice(M, 128, replace=False))
    cols = np.sort(rng.choice(N, 128, replace=False))
    r_ref = oracle.linear(ah, bh, rows=rows)
    c_ref = oracle.linear(ah, bh, cols=cols)
    rel_r = _rel(c[rows], r_ref)
    rel_c = _rel(c[:, cols], c_ref)
    print(f"[linear 8192x4096x4096] rows {rel_r:.3e} cols {rel_c:.3e}")
    assert rel_r <= 1e-2 and rel_c <= 1e-2


def test_linear_ragged_shapes():
    for (M, N, K) in [(100, 264, 48), (257, 136, 1040)]:
        a, b = workloads.linear_operands(1, M=M, N=N, K=K)
        aq, bq = _quantized(a), _quantized(b)
        c = _linear(aq, bq, M, N, K).float().cpu().numpy()
        ref = oracle.linear(_dequant_ref(aq), _dequant_ref(bq))
        assert _rel(c, ref) <= 1e-2


def test_linear_workspace_and_shape_errors():
    bb = B()
    assert bb.if4_linear_workspace_bytes(128, 256, 64) >= (128 + 256) * 64 * 2
    assert bb.if4_linear_workspace_bytes(128, 256, 24) == 0
    a, b = workloads.linear_operands(2, M=64, N=64, K=64)
    aq, bq = _quantized(a), _quantized(b)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    c = torch.empty((64, 64), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(bb.IF4Error, match="workspace"):
        bb.if4_linear(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], small, c, err)


def test_pair_and_single_cta_paths_agree():
    """M, N >= 256 runs the CTA-pair kernel; 128-row slices of the same A run
    the one-CTA kernel.  Both accumulate each output over K in the same order
    (16-wide MMA steps, 64-wide slabs), so the results are identical."""
    M, N, K = 512, 768, 2048
    g = torch.Generator().manual_seed(77)
    a = torch.randn((M, K), generator=g).to(torch.float16).cuda()
    b = (torch.randn((N, K), generator=g) * 0.05).to(torch.float16).cuda()
    full = gemm(a, b, 0.5, 2.0)
    parts = torch.cat([gemm(a[i:i + 128].contiguous(), b, 0.5, 2.0) for i in range(0, M, 128)])
    assert torch.equal(full, parts)


@pytest.mark.parametrize("M,N,K", [(512, 512, 1024), (300, 528, 256), (128, 256, 64)])
def test_linear_quantized_output_equals_separate_quantize(M, N, K):
    """The IF4 output of the epilogue equals if4_quantize of the bf16 C of
    if4_linear under the same given tensor scale, byte for byte, on both GEMM
    kernels (M >= 256 uses CTA pairs), with a ragged last 32-column chunk
    (N % 32 == 16), with and without the bf16 C written beside it, and with a
    small given scale that saturates block scales (the epilogue's rare path)."""
    bb = B()
    a, b = workloads.linear_operands(4, M=M, N=N, K=K)
    aq, bq = _quantized(a), _quantized(b)
    c_ref = _linear(aq, bq, M, N, K)
    c_np = c_ref.float().cpu().numpy()
    ts_data = oracle.tensor_scale(np.float32(np.max(np.abs(c_np))))
    ws = torch.empty(bb.if4_linear_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    for factor, write_c in ((1.0, True), (1.0, False), (0.05, False)):
        c_ts = np.float32(ts_data * factor)
        t = torch.tensor([c_ts], dtype=torch.float32, device="cuda")
        codes = torch.empty((M, N // 2), dtype=torch.uint8, device="cuda")
        scales = torch.empty((M, N // 16), dtype=torch.uint8, device="cuda")
        c = torch.empty((M, N), dtype=torch.bfloat16, device="cuda") if write_c else None
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        bb.if4_linear_quantized(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], ws, codes, scales, t,
                                c=c, err_flag=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        if write_c:
            assert torch.equal(c, c_ref)
        ref = oracle.quantize(c_np, c_ts)
        assert np.array_equal(scales.cpu().numpy(), ref["scales"]), (M, N, K, factor)
        assert np.array_equal(codes.cpu().numpy(), ref["codes"]), (M, N, K, factor)
        if factor < 1.0:
            assert np.any((ref["scales"] & 0x7F) == 0x7E)     # saturated block scales


def test_linear_quantized_output_flags_invalid_scale():
    bb = B()
    M, N, K = 128, 256, 64
    a, b = workloads.linear_operands(5, M=M, N=N, K=K)
    aq, bq = _quantized(a), _quantized(b)
    ws = torch.empty(bb.if4_linear_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    codes = torch.empty((M, N // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, N // 16), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    t = torch.tensor([0.0], dtype=torch.float32, device="cuda")
    bb.if4_linear_quantized(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], ws, codes, scales, t,
                            err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & bb.DEV_BAD_SCALE


def test_linear_quantized_output_full_workload():
    """The IF4 output of the 8192 x 4096 x 4096 linear, every group, against
    the oracle's quantization of the same bf16 C under the same scale."""
    bb = B()
    M, N, K = 8192, 4096, 4096
    a, b = workloads.linear_operands(0, M=M, N=N, K=K)
    aq, bq = _quantized(a), _quantized(b)
    c = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    codes = torch.empty((M, N // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, N // 16), dtype=torch.uint8, device="cuda")
    ws = torch.empty(bb.if4_linear_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    c_ts = torch.ones(1, dtype=torch.float32, device="cuda")
    bb.if4_linear(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], ws, c, err)
    bb.if4_tensor_amax(c, c_ts, err)
    bb.if4_tensor_scale(c_ts, c_ts)
    bb.if4_linear_quantized(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], ws, codes, scales, c_ts,
                            err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = oracle.quantize(c.float().cpu().numpy(), np.float32(c_ts.item()))
    assert np.array_equal(scales.cpu().numpy(), ref["scales"])
    assert np.array_equal(codes.cpu().numpy(), ref["codes"])


# ------------------------------------------------ fused-decode linear ----

def _linear_fused(aq, bq, M, N):
    bb = B()
    c = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bb.if4_linear_fused(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], c, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return c


@pytest.mark.parametrize("M,N,K", [(512, 512, 4096), (256, 256, 64), (200, 264, 1024),
                                   (1, 8, 64), (777, 520, 2048), (1024, 1536, 512)])
def test_fused_linear_equals_linear(M, N, K):
    """The decoders inside the GEMM produce the same fp16 operands as
    if4_decode_f16 and the MMAs accumulate in the same order, so C equals
    if4_linear's bit for bit (and so is within the linear's 1e-2 of the
    float64 product); shapes include partial tiles on both sides."""
    a, b = workloads.linear_operands(4, M=M, N=N, K=K)
    aq, bq = _quantized(a), _quantized(b)
    want = _linear(aq, bq, M, N, K)
    got = _linear_fused(aq, bq, M, N)
    assert torch.equal(got.view(torch.int16), want.view(torch.int16)), (M, N, K)
    if M * N <= 512 * 512:
        ref = oracle.linear(_dequant_ref(aq), _dequant_ref(bq))
        assert _rel(got.float().cpu().numpy(), ref) <= 1e-2


def test_fused_linear_full_workload():
    M, N, K = 8192, 4096, 4096
    a, b = workloads.linear_operands(0, M=M, N=N, K=K)
    aq, bq = _quantized(a), _quantized(b)
    want = _linear(aq, bq, M, N, K)
    got = _linear_fused(aq, bq, M, N)
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_fused_linear_arbitrary_code_bytes():
    """Random code and scale bytes (INT4 code 8 included, which the encoder
    never emits and the byte-permute decode hands to the per-element table):
    the fused-decode linear still equals if4_linear bit for bit."""
    M, N, K = 384, 520, 1024
    rng = np.random.default_rng(11)

    def operand(rows):
        c = torch.from_numpy(rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)).cuda()
        s = torch.from_numpy(rng.integers(0, 256, (rows, K // 16), dtype=np.uint8)).cuda()
        s[0, :] |= 0x80
        c[0, :] = 0x88                  # a row of INT4 groups holding code 8 only
        return c, s, torch.tensor([0.0125], dtype=torch.float32, device="cuda")

    aq, bq = operand(M), operand(N)
    want = _linear(aq, bq, M, N, K)
    got = _linear_fused(aq, bq, M, N)
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_fused_linear_rejects_k_not_multiple_of_64():
    bb = B()
    a, b = workloads.linear_operands(5, M=64, N=64, K=80)
    aq, bq = _quantized(a), _quantized(b)
    c = torch.empty((64, 64), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(bb.IF4Error, match="shape"):
        bb.if4_linear_fused(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], c, err)
