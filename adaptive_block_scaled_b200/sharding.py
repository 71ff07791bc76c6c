"""Host-side plumbing for quantizing one tensor split across ranks.

Groups of 16 are independent, so rows shard with no exchange except one: the
tensor scale ts = amax/2688 needs the amax of the whole tensor.  Each rank
runs if4_tensor_amax on its rows, the ranks take the MAX of that one float
(``allreduce_amax``, NCCL on GPUs), and every rank then runs
if4_tensor_scale and quantizes its rows with IF4_TS_GIVEN.  The result is
byte-identical to quantizing the whole tensor on one GPU.
"""
import torch


def shard_rows(rows: int, world: int, rank: int):
    """Contiguous, balanced [start, stop) row range of ``rank``."""
    if world < 1 or not 0 <= rank < world or rows < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_amax(amax: torch.Tensor, group=None) -> torch.Tensor:
    """In-place MAX over ranks of a one-element float32 amax tensor."""
    import torch.distributed as dist
    if amax.numel() != 1 or amax.dtype != torch.float32:
        raise ValueError("amax must be a one-element float32 tensor")
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax
