"""The allocation-free linear, if4_linear_noalloc, through the C ABI.

It is meant for callers that cannot hand the library device memory at the
call (a plugin inside a framework that owns all device memory, or a path that
must not risk cudaMalloc's synchronisation); it keeps the decoded operands in
a fixed 32 MiB device array instead.  This file is collected last, so a run
that stops at the first failure has already run every other test.

Two calls in a row, with different operands and the second smaller than the
first, must each equal the existing if4_linear (same kernels, so bit for bit,
and therefore within the linear's tolerance of 1e-2); further calls leave the
device's free memory exactly as it was (nothing allocated, nothing leaked); a
problem larger than the array is refused before anything runs.
"""
import numpy as np
import pytest
import torch

from adaptive_block_scaled_b200 import workloads

pytestmark = pytest.mark.gpu


def _operands(seed, M, N, K):
    from adaptive_block_scaled_b200 import binding as b
    a, w = workloads.linear_operands(seed, M=M, N=N, K=K)
    return b.quantize(a.cuda()), b.quantize(w.cuda())


def _with_workspace(aq, bq, M, N, K):
    from adaptive_block_scaled_b200 import binding as b
    ws = torch.empty(b.if4_linear_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    c = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.if4_linear(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], ws, c, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return c


def _no_alloc(aq, bq, M, N):
    from adaptive_block_scaled_b200 import binding as b
    c = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.if4_linear_noalloc(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], c, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return c


def test_no_alloc_linear_matches_workspace_linear_twice():
    for seed, (M, N, K) in ((0, (512, 1024, 4096)), (1, (200, 264, 2048))):
        aq, bq = _operands(seed, M, N, K)
        want = _with_workspace(aq, bq, M, N, K).float()
        got = _no_alloc(aq, bq, M, N).float()
        rel = float((got - want).abs().max() / want.abs().max())
        assert rel <= 1e-2, (M, N, K, rel)
        assert torch.equal(got, want), (M, N, K)


def test_no_alloc_linear_allocates_nothing():
    """With every buffer allocated beforehand and torch's caching allocator
    idle, calls of if4_linear_noalloc leave the device's free memory
    unchanged.  The first call on a device may load the library's device
    code, which holds the scratch array; it is made before the count
    starts."""
    from adaptive_block_scaled_b200 import binding as b
    M, N, K = 512, 1024, 4096
    aq, bq = _operands(2, M, N, K)
    want = _with_workspace(aq, bq, M, N, K)
    c = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.if4_linear_noalloc(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], c, err)   # first call
    # the comparison below, once, so that any block torch needs for it is
    # already in its cache when the count starts
    assert torch.equal(c, want)
    c.fill_(float("nan"))
    torch.cuda.synchronize()
    reserved = torch.cuda.memory_reserved()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        c.fill_(float("nan"))
        b.if4_linear_noalloc(aq[0], aq[1], aq[2], bq[0], bq[1], bq[2], c, err)
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert free1 == free0, (free0, free1)
        assert torch.equal(c, want)
    assert torch.cuda.memory_reserved() == reserved
    assert int(err.item()) == 0


def test_no_alloc_linear_refuses_problems_beyond_its_scratch():
    from adaptive_block_scaled_b200 import binding as b
    M, N, K = 4096, 4096, 4096          # needs 64 MiB of scratch
    assert b.if4_linear_workspace_bytes(M, N, K) > b.LINEAR_NOALLOC_MAX_BYTES
    dev = "cuda"
    codes_a = torch.zeros((M, K // 2), dtype=torch.uint8, device=dev)
    scales_a = torch.zeros((M, K // 16), dtype=torch.uint8, device=dev)
    ts = torch.ones(1, dtype=torch.float32, device=dev)
    c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    with pytest.raises(b.IF4Error, match="workspace"):
        b.if4_linear_noalloc(codes_a, scales_a, ts, codes_a, scales_a, ts, c, err)
    assert int(err.item()) == 0
