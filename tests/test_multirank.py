"""The multi-rank host path on CPU with two gloo ranks: row sharding, the
MAX all-reduce of the tensor amax, and the timing reduction of bench.py.
The per-rank quantization here is the oracle (this is a CPU test of the host
logic); the result must equal the single-process quantization byte for
byte."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from adaptive_block_scaled_b200.sharding import shard_rows


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, rows, cols, out_dir):
    import datetime
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle
    from adaptive_block_scaled_b200 import workloads
    from adaptive_block_scaled_b200.sharding import allreduce_amax, shard_rows
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    x = workloads.activation_outliers(0, tokens=rows, hidden=cols).float().numpy()
    r0, r1 = shard_rows(rows, world, rank)
    mine = np.ascontiguousarray(x[r0:r1])
    amax = torch.tensor([float(oracle.tensor_amax(mine))], dtype=torch.float32)
    allreduce_amax(amax)
    ts = oracle.tensor_scale(np.float32(amax.item()))
    q = oracle.quantize(mine, ts)
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), codes=q["codes"], scales=q["scales"],
             ts=np.float32(ts), r0=r0, r1=r1)
    import bench
    worst = bench.max_over_ranks(float(rank + 1) * 1.5, world)
    assert worst == 1.5 * world
    bench.barrier(world)
    dist.destroy_process_group()


def test_shard_rows_cover_everything():
    for rows in (0, 1, 7, 8192, 8193):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(rows, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


def test_two_gloo_ranks_match_single_process(tmp_path):
    import oracle
    from adaptive_block_scaled_b200 import workloads
    rows, cols = 96, 512
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, rows, cols, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    x = workloads.activation_outliers(0, tokens=rows, hidden=cols).float().numpy()
    full = oracle.quantize_tensor(x)
    parts = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    assert all(p["ts"] == full["ts"] for p in parts)
    assert np.array_equal(np.concatenate([p["codes"] for p in parts]), full["codes"])
    assert np.array_equal(np.concatenate([p["scales"] for p in parts]), full["scales"])
