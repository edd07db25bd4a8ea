"""Head sharding of one attention problem over the ranks of a process group.

The (batch, head) slices of the Longformer attention are independent (every
row attends within its own batch and head), so one problem splits over ranks
by heads with no exchange on the data path: rank r computes heads
[h0_r, h1_r) of every batch, and the output is the heads laid side by side
again.  The masks are shared by all heads; the dilation list is sliced with
the heads.  This module holds only the host bookkeeping: ranges, slicing and
the gather of the results.
"""
from __future__ import annotations


def head_ranges(H: int, world: int) -> list[tuple[int, int]]:
    """Contiguous head ranges, one per rank, sizes differing by at most one
    (the first H % world ranks take one head more).  A rank may get none when
    world > H."""
    if H < 1 or world < 1:
        raise ValueError("need H >= 1 and world >= 1")
    base, extra = divmod(H, world)
    out, h = [], 0
    for r in range(world):
        size = base + (1 if r < extra else 0)
        out.append((h, h + size))
        h += size
    return out


def shard_inputs(x: dict, h0: int, h1: int) -> dict:
    """The inputs of heads [h0, h1): the six projections sliced on dim 1
    (contiguous copies), the dilation list sliced, masks and scalars kept."""
    out = dict(x)
    for key in ("q", "k", "v", "qg", "kg", "vg"):
        out[key] = x[key][:, h0:h1].contiguous()
    out["dilation"] = list(x["dilation"])[h0:h1]
    return out


def gather_heads(local, ranges, group=None):
    """All-gathers each rank's [B, h1-h0, n, d] output and returns the full
    [B, H, n, d] tensor on every rank (tensors are padded to the largest
    range for the collective and trimmed after)."""
    import torch
    import torch.distributed as dist
    widest = max(h1 - h0 for h0, h1 in ranges)
    B, _, n, d = local.shape
    buf = torch.zeros((B, widest, n, d), dtype=local.dtype, device=local.device)
    buf[:, :local.shape[1]] = local
    bufs = [torch.empty_like(buf) for _ in ranges]
    dist.all_gather(bufs, buf, group=group)
    return torch.cat([bufs[r][:, :h1 - h0] for r, (h0, h1) in enumerate(ranges)], dim=1)
