"""Host bookkeeping for multi-GPU expert parallelism (one process per GPU).

Each rank holds T/R tokens and E/R experts.  The ranks exchange their
routing (topk_idx, T/R x k int64 each) with one all-gather, and every rank
runs the same layout over the gathered [T, k] ids, so slots are global.
Owner rank o's receive buffers hold the global rows
[expert_offset[o*E/R], expert_offset[(o+1)*E/R]).  The *_peers calls of the
C ABI then move this rank's tokens into, or out of, the owners' buffers
(include/ep.h, "Multi-GPU expert parallelism").  Only plumbing lives here:
the collective is torch.distributed's, and every step of the data path runs
in the CUDA library.
"""

from __future__ import annotations


def token_range(T: int, R: int, rank: int) -> tuple[int, int]:
    """[begin, end) of rank's tokens."""
    if T % R:
        raise ValueError("T must be a multiple of R")
    per = T // R
    return rank * per, (rank + 1) * per


def gather_routing(topk_idx_local, group=None):
    """All ranks' topk_idx, in rank order: [T, k] from each rank's [T/R, k]
    (one all-gather of T*k int64)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = [torch.empty_like(topk_idx_local) for _ in range(world)]
    dist.all_gather(parts, topk_idx_local.contiguous(), group=group)
    return torch.cat(parts, dim=0)


def owner_rows(expert_offset, E: int, R: int) -> list[tuple[int, int]]:
    """(first global row, row count) of every owner rank's receive buffers,
    from the layout's expert_offset [E + 1] (host values)."""
    if E % R:
        raise ValueError("E must be a multiple of R")
    er = E // R
    off = [int(v) for v in expert_offset]
    return [(off[o * er], off[(o + 1) * er] - off[o * er]) for o in range(R)]
