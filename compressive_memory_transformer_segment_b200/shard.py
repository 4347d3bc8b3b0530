"""Host-side data parallelism for the layer: independent (batch, KV head) chains.

Each KV head's memory (and the query heads that read it) is independent of
every other head and batch row: the method keeps one compressive memory per
head ("Leave No Context Behind" explainer, section "メモリ構造").  So the work
splits across ranks with no data-path exchange: a rank takes a contiguous
range of batch rows (whole rows keep every GQA group and every segment chain
together), runs the forward on its own GPU, and results are assembled by
concatenation.  The only collectives are for timing (max over ranks) and,
when a caller wants the full result on one rank, a gather.
"""

import torch
import torch.distributed as dist


def batch_range(B, world, rank):
    """Contiguous batch rows [b0, b1) for `rank` of `world` (near-equal split)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(B, world)
    b0 = rank * base + min(rank, extra)
    return b0, b0 + base + (1 if rank < extra else 0)


def shard_batch(t, world, rank, dim=0):
    """The rank's slice of a [B, ...] tensor along `dim` (a view)."""
    b0, b1 = batch_range(t.shape[dim], world, rank)
    return t.narrow(dim, b0, b1 - b0)


def gather_batch(local, B, world, group=None):
    """All-gather per-rank batch slices (possibly unequal) into the full tensor."""
    sizes = [batch_range(B, world, r)[1] - batch_range(B, world, r)[0] for r in range(world)]
    width = max(sizes)
    pad = torch.zeros((width,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[: local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:n] for p, n in zip(parts, sizes)], dim=0)


def max_over_ranks(value, device=None, group=None):
    """Max of a per-rank float (e.g. elapsed ms), identical on every rank."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
