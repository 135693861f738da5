"""Data-parallel plumbing for the layer across GPUs (one process per GPU).

Rows of the activation matrix (tokens) are independent through every step
of the layer -- per-token quantization, the GEMM against a replicated weight,
the per-row epilogue -- so the layer shards over token rows with no
collective on the data path.  torch.distributed is used only for barriers
and for taking the max of per-rank timings.
"""
from __future__ import annotations


def shard_rows(M: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous, balanced [start, stop) of M token rows for `rank`; the
    first M % world ranks take one extra row."""
    if world < 1 or not 0 <= rank < world or M < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar (e.g. a kernel time) over the default group;
    the value itself when torch.distributed is not initialised."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def forward_sharded(layer, x, rank: int, world: int, out=None, stream=None):
    """Run `layer` (an Int8DynamicLinear) on this rank's rows of x [M, K];
    returns (start, stop, out_shard)."""
    start, stop = shard_rows(x.shape[0], world, rank)
    return start, stop, layer(x[start:stop], out=out, stream=stream)
