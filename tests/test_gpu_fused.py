"""GPU parity of the single-launch quantizer (if4_quantize_fused): tensor
amax, tensor scale, IF4 codes and the NVFP4 comparator from one cooperative
launch must equal the oracle byte for byte, and equal the separate calls.
Words 0 (arrivals) and 1 (amax) of the synchronisation words must come back
zero after every call; word 32 counts barrier generations, word 33 keeps ts."""
import numpy as np
import pytest
import torch

import oracle
from adaptive_block_scaled_b200 import workloads

pytestmark = pytest.mark.gpu


def B():
    from adaptive_block_scaled_b200 import binding
    return binding


def fused(x_dev, sync=None, with_nvfp4=True):
    b = B()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    if sync is None:
        sync = torch.zeros(b.FUSED_SYNC_WORDS, dtype=torch.int32, device="cuda")
    out = b.quantize_fused(x_dev, with_nvfp4=with_nvfp4, sync_words=sync, err_flag=err)
    torch.cuda.synchronize()
    w = sync.tolist()
    assert w[0] == 0 and w[1] == 0, w[:2]
    return [o.cpu().numpy() for o in out], int(err.item())


def check(x_cpu, label, x_dev=None):
    x_np = x_cpu.float().numpy()
    ref = oracle.quantize_tensor(x_np)
    nv = oracle.quantize(x_np, ref["ts"], mode=oracle.MODE_NVFP4)
    (codes, scales, ts, ncodes, nscales), err = fused(x_cpu.cuda() if x_dev is None else x_dev)
    assert err == 0
    assert np.float32(ts[0]).view(np.uint32) == np.float32(ref["ts"]).view(np.uint32), label
    assert np.array_equal(scales, ref["scales"]), label
    assert np.array_equal(codes, ref["codes"]), label
    assert np.array_equal(nscales, nv["scales"]), label
    assert np.array_equal(ncodes, nv["codes"]), label
    print(f"[fused {label}] groups={scales.size} ok")


def test_fused_on_small_and_weight_workloads():
    check(workloads.small_fp32(0), "small_fp32_256x1024")
    check(workloads.llm_weight(0), "weight_bf16_4096x4096")


def test_fused_on_activation_and_gradient_like_rows():
    check(workloads.activation_outliers(0, tokens=1024, hidden=8192), "activation rows")
    check(workloads.hadamard_gradient(0, rows=1024, cols=4096), "gradient rows")


@pytest.mark.parametrize("shape", [(1, 16), (7, 80), (33, 272), (1000, 16), (300, 4096)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_fused_ragged_shapes_and_dtypes(shape, dtype):
    g = torch.Generator().manual_seed(shape[0] * 31 + shape[1])
    x = (torch.randn(shape, generator=g) * 5).to(dtype)
    check(x, f"{shape} {dtype}")


def test_fused_tiny_groups_and_zeros():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    x *= np.exp2(-rng.integers(0, 24, (64, 16))).repeat(16, axis=1).astype(np.float32)
    x[0, 0] = 1000.0
    x[1, :16] = -0.0
    x[3] = 0.0
    check(torch.from_numpy(x), "tiny groups")


def test_fused_all_zero_and_empty():
    (codes, scales, ts, nc, ns), err = fused(torch.zeros((5, 64), dtype=torch.bfloat16,
                                                         device="cuda"))
    assert err == 0 and ts[0] == 1.0 and not codes.any() and not scales.any() and not nc.any()
    (codes, scales, ts, nc, ns), err = fused(torch.zeros((0, 64), dtype=torch.bfloat16,
                                                         device="cuda"))
    assert err == 0 and ts[0] == 1.0 and codes.shape == (0, 32)


def test_fused_strided_rows_and_unaligned_base():
    base = workloads.llm_weight(1, rows=256, cols=1024 + 64)
    x_dev = base.cuda()[:, 8:8 + 1024]
    assert x_dev.data_ptr() % 32 == 16
    check(base[:, 8:8 + 1024].contiguous(), "strided", x_dev=x_dev)


def test_fused_equals_separate_calls_and_reuses_sync_words():
    b = B()
    sync = torch.zeros(b.FUSED_SYNC_WORDS, dtype=torch.int32, device="cuda")
    for seed in range(3):
        x = workloads.llm_weight(seed, rows=512, cols=2048).cuda()
        (codes, scales, ts, nc, ns), err = fused(x, sync=sync)
        c2, s2, t2 = b.quantize(x)
        n2, m2, _ = b.quantize(x, "nvfp4", ts=t2)
        torch.cuda.synchronize()
        assert err == 0 and ts[0] == t2.item()
        assert np.array_equal(codes, c2.cpu().numpy()) and np.array_equal(scales, s2.cpu().numpy())
        assert np.array_equal(nc, n2.cpu().numpy()) and np.array_equal(ns, m2.cpu().numpy())


def test_fused_if4_only():
    x = workloads.llm_weight(5, rows=128, cols=1024)
    ref = oracle.quantize_tensor(x.float().numpy())
    (codes, scales, ts), err = fused(x.cuda(), with_nvfp4=False)
    assert err == 0 and np.array_equal(codes, ref["codes"]) and np.array_equal(scales, ref["scales"])


def test_fused_nonfinite_sets_flag_and_leaves_sync_zero():
    x = torch.randn(64, 256).to(torch.bfloat16)
    x[7, 9] = float("inf")
    _, err = fused(x.cuda())
    assert err & B().DEV_NONFINITE


@pytest.mark.parametrize("signs", [0x0000, 0xA5C3])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_fused_rht_matches_oracle_and_separate_calls(signs, dtype):
    """The single launch on the random-sign Hadamard transform: ts, IF4 and
    NVFP4 of the transformed tensor, against the oracle (transform, then
    quantize) and against if4_quantize_rht + nvfp4 of the transform."""
    b = B()
    g = torch.Generator().manual_seed(signs + 17)
    x = (torch.randn((96, 1024), generator=g) * 3).to(dtype)
    x[:, 5] *= 40                                   # an outlier channel
    x_np = x.float().numpy()
    ref = oracle.quantize_tensor_rht(x_np, signs)
    y = oracle.rht(x_np, signs)
    nv = oracle.quantize(y, ref["ts"], mode=oracle.MODE_NVFP4)
    sync = torch.zeros(b.FUSED_SYNC_WORDS, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, scales, ts, nc, ns = b.quantize_fused(x.cuda(), sync_words=sync, err_flag=err,
                                                 signs=signs)
    c2, s2, t2 = b.quantize_rht(x.cuda(), signs)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and sync[0].item() == 0 and sync[1].item() == 0
    assert np.float32(ts.item()) == ref["ts"] and ts.item() == t2.item()
    assert np.array_equal(scales.cpu().numpy(), ref["scales"])
    assert np.array_equal(codes.cpu().numpy(), ref["codes"])
    assert torch.equal(codes, c2) and torch.equal(scales, s2)
    assert np.array_equal(ns.cpu().numpy(), nv["scales"])
    assert np.array_equal(nc.cpu().numpy(), nv["codes"])


def test_fused_grid_barrier_times_out_cleanly():
    """Failure detection without a fault: an arrival counter preset so that
    no block is ever the last to arrive means nobody releases the grid
    barrier.  Every block's wait is bounded (1 s of the global timer); the
    kernel must end with IF4_DEV_TIMEOUT in the error word, write no codes,
    and leave the context usable: with the words zeroed again, the next call
    is correct."""
    import time
    b = B()
    x = workloads.llm_weight(6, rows=256, cols=1024).cuda()
    sync = torch.zeros(b.FUSED_SYNC_WORDS, dtype=torch.int32, device="cuda")
    sync[0] = 1 << 30                      # arrivals never reach gridDim - 1
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes = torch.full((256, 512), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((256, 64), 0xAB, dtype=torch.uint8, device="cuda")
    ts = torch.zeros(1, dtype=torch.float32, device="cuda")
    t0 = time.time()
    b.if4_quantize_fused(x, codes, scales, None, None, ts, sync, err)
    torch.cuda.synchronize()
    waited = time.time() - t0
    assert int(err.item()) & b.DEV_TIMEOUT
    assert 0.5 < waited < 30, waited
    assert torch.all(codes == 0xAB) and torch.all(scales == 0xAB)
    # the context still works
    sync.zero_()
    err.zero_()
    (c2, s2, t2), e2 = fused(x, sync=sync, with_nvfp4=False)
    ref = oracle.quantize_tensor(x.float().cpu().numpy())
    assert e2 == 0 and np.array_equal(c2, ref["codes"]) and np.array_equal(s2, ref["scales"])


@pytest.mark.parametrize("name", ["activation_bf16_8192x8192", "gradient_bf16_16384x4096"])
def test_fused_full_size_workloads(name):
    """The single launch at the full sizes of the large workloads (one
    134 MB bf16 tensor each): every code, scale byte and the tensor scale
    against the oracle, and the NVFP4 output too."""
    x = (workloads.activation_outliers(0) if name.startswith("activation")
         else workloads.hadamard_gradient(0))
    check(x, name)


def test_fused_then_dequantize_in_stream_order():
    """The step's sequence: the dequantizer (launched with programmatic
    dependent launch) right after the single launch on the same stream must
    read the finished codes, scales and tensor scale: bit-identical to the
    oracle's dequantization, repeated on several tensors back to back."""
    b = B()
    sync = torch.zeros(b.FUSED_SYNC_WORDS, dtype=torch.int32, device="cuda")
    outs = []
    xs = [workloads.llm_weight(s, rows=1024, cols=4096) for s in range(3)]
    for x in xs:
        codes, scales, ts, nc, ns = b.quantize_fused(x.cuda(), sync_words=sync)
        y = b.dequantize(codes, scales, ts, dtype=torch.float32)
        outs.append((y, ts))
    torch.cuda.synchronize()
    for x, (y, ts) in zip(xs, outs):
        ref = oracle.quantize_tensor(x.float().numpy())
        want = oracle.dequantize(ref["codes"], ref["scales"], ref["ts"])
        assert np.float32(ts.item()) == ref["ts"]
        assert np.array_equal(y.cpu().numpy().view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("shape,dtype", [((4096, 4096), torch.bfloat16),
                                         ((4096, 4192), torch.bfloat16),
                                         ((4096, 4256), torch.bfloat16),
                                         ((4096, 4096), torch.float16),
                                         ((4096, 2048), torch.float32),
                                         ((4096, 2112), torch.float32),
                                         ((333, 4096), torch.bfloat16)])
def test_fused_weight_sized_shapes(shape, dtype):
    """Contiguous tensors of 1.4-17.4 M elements in each input type, around
    the size of the weight workload, with an outlier channel and a row count
    (333) that leaves a ragged last round of the grid: every code, scale byte
    and the tensor scale against the oracle."""
    g = torch.Generator().manual_seed(shape[0] + shape[1])
    x = (torch.randn(shape, generator=g) * 0.02).to(dtype)
    x[:, 7] *= 30                                   # an outlier channel
    check(x, f"{shape} {dtype}")


def test_fused_contiguous_and_strided_agree():
    """The same weight tensor as a contiguous tensor and as a strided view
    of a padded buffer (the two addressing paths of the kernel):
    byte-identical outputs."""
    b = B()
    x = workloads.llm_weight(3)
    pad = torch.zeros((4096, 4096 + 64), dtype=torch.bfloat16)
    pad[:, :4096] = x
    outs = []
    for xd in (x.cuda(), pad.cuda()[:, :4096]):
        sync = torch.zeros(b.FUSED_SYNC_WORDS, dtype=torch.int32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        outs.append(b.quantize_fused(xd, sync_words=sync, err_flag=err))
        torch.cuda.synchronize()
        assert int(err.item()) == 0
    for a, c in zip(*outs):
        assert torch.equal(a, c)


@pytest.mark.parametrize("case", ["weight", "f32_ragged", "f16_small", "strided", "activation"])
def test_fused_round_trip(case):
    """if4_quantize_fused_dequant: codes, scales, ts and the NVFP4 output
    byte-identical to if4_quantize_fused; y bit-identical to if4_dequantize
    of those codes (bf16) and to the oracle's dequantization rounded to bf16."""
    b = B()
    g = torch.Generator().manual_seed(41)
    if case == "weight":
        x = workloads.llm_weight(2)
        xd = x.cuda()
    elif case == "f32_ragged":
        x = torch.randn((333, 4096), generator=g) * 3
        xd = x.cuda()
    elif case == "f16_small":
        x = torch.randn((7, 80), generator=g).half()
        xd = x.cuda()
    elif case == "strided":
        base = workloads.llm_weight(1, rows=256, cols=1024 + 64)
        xd = base.cuda()[:, 8:8 + 1024]
        x = base[:, 8:8 + 1024].contiguous()
    else:
        x = workloads.activation_outliers(0)
        xd = x.cuda()
    sync = torch.zeros(b.FUSED_SYNC_WORDS, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, scales, ts, nc, ns, y = b.quantize_fused_dequant(xd, sync_words=sync, err_flag=err)
    c2, s2, t2, n2, m2 = b.quantize_fused(xd)
    y2 = b.dequantize(c2, s2, t2)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and sync[0].item() == 0 and sync[1].item() == 0
    assert torch.equal(codes, c2) and torch.equal(scales, s2) and ts.item() == t2.item()
    assert torch.equal(nc, n2) and torch.equal(ns, m2)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    ref = oracle.quantize_tensor(x.float().numpy())
    assert np.float32(ts.item()) == ref["ts"]
    assert np.array_equal(codes.cpu().numpy(), ref["codes"])
    want = torch.from_numpy(oracle.dequantize(ref["codes"], ref["scales"], ref["ts"]))
    assert torch.equal(y.cpu().view(torch.int16), want.to(torch.bfloat16).view(torch.int16))


def _round_trip_buffers(x):
    rows, cols = x.shape
    dev = x.device
    return dict(codes=torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
                scales=torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev),
                nc=torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
                ns=torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev),
                ts=torch.empty(1, dtype=torch.float32, device=dev),
                y=torch.empty((rows, cols), dtype=torch.bfloat16, device=dev),
                sync=torch.zeros(B().FUSED_SYNC_WORDS, dtype=torch.int32, device=dev))


def _same(o, ref):
    return (torch.equal(o["codes"], ref[0]) and torch.equal(o["scales"], ref[1])
            and o["ts"].item() == ref[2].item() and torch.equal(o["nc"], ref[3])
            and torch.equal(o["ns"], ref[4])
            and torch.equal(o["y"].view(torch.int16), ref[5].view(torch.int16)))


@pytest.mark.parametrize("share", [1, 2, 3, 4, 64])
def test_shared_round_trip_is_byte_identical(share):
    """if4_quantize_fused_dequant_shared: the grid shrinks to 1/share of the
    resident blocks (64: one block per SM), the outputs do not change."""
    b = B()
    x = workloads.activation_outliers(1, tokens=2048, hidden=8192).cuda()
    ref = b.quantize_fused_dequant(x)
    o = _round_trip_buffers(x)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.if4_quantize_fused_dequant_shared(x, o["codes"], o["scales"], o["nc"], o["ns"], o["ts"],
                                        o["sync"], o["y"], share, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and o["sync"][0].item() == 0 and o["sync"][1].item() == 0
    assert _same(o, ref)


def test_shared_launches_on_two_streams_at_once():
    """Two tensors quantized by shared launches (share 2) on two streams, six
    calls each, each stream with its own buffers and synchronisation words:
    every result equals the plain single-stream call on the same tensor."""
    b = B()
    xs = [workloads.activation_outliers(s, tokens=4096, hidden=8192).cuda() for s in (2, 3)]
    refs = [b.quantize_fused_dequant(x) for x in xs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    bufs = [_round_trip_buffers(x) for x in xs]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cur = torch.cuda.current_stream()
    for s in streams:
        s.wait_stream(cur)
    for rep in range(6):
        for k in (0, 1):
            o = bufs[k]
            with torch.cuda.stream(streams[k]):
                b.if4_quantize_fused_dequant_shared(xs[k], o["codes"], o["scales"], o["nc"],
                                                    o["ns"], o["ts"], o["sync"], o["y"], 2,
                                                    err_flag=err)
    for s in streams:
        cur.wait_stream(s)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for k in (0, 1):
        assert bufs[k]["sync"][0].item() == 0 and bufs[k]["sync"][1].item() == 0
        assert _same(bufs[k], refs[k])


@pytest.mark.parametrize("signs", [None, 0xA5C3])
@pytest.mark.parametrize("share", [2, 64])
def test_shared_single_launch_is_byte_identical(signs, share):
    """if4_quantize_fused_shared and if4_quantize_fused_rht_shared: the same
    codes, scales, ts and NVFP4 output as the plain single launch."""
    b = B()
    x = workloads.hadamard_gradient(1, rows=2048, cols=4096).cuda()
    rows, cols = x.shape
    ref = [torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda"),
           torch.empty((rows, cols // 16), dtype=torch.uint8, device="cuda"),
           torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda"),
           torch.empty((rows, cols // 16), dtype=torch.uint8, device="cuda"),
           torch.empty(1, dtype=torch.float32, device="cuda")]
    got = [torch.empty_like(t) for t in ref]
    s0 = torch.zeros(b.FUSED_SYNC_WORDS, dtype=torch.int32, device="cuda")
    s1 = torch.zeros(b.FUSED_SYNC_WORDS, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.if4_quantize_fused(x, ref[0], ref[1], ref[2], ref[3], ref[4], s0, err_flag=err, signs=signs)
    b.if4_quantize_fused_shared(x, got[0], got[1], got[2], got[3], got[4], s1, share,
                                err_flag=err, signs=signs)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and s1[0].item() == 0 and s1[1].item() == 0
    for a, c in zip(ref, got):
        assert torch.equal(a, c)

