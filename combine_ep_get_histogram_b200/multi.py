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


class PeerBuffers:
    """Every rank's copy of a set of named device buffers, for the peer
    tables of the *_peers calls: this rank's own tensors, and the other
    ranks' buffers opened through CUDA IPC (ep_ipc_export / ep_ipc_open of
    the C ABI).

    Collective over `group` (a torch.distributed group, gloo is enough): every
    rank passes buffers under the same names.  The buffers must live in
    cudaMalloc allocations (torch's default caching allocator; not its
    expandable segments, whose memory CUDA IPC cannot export: the export
    raises).  One all-gather of the
    80-byte export records, then each rank maps the others' buffers.
    ``table(name)`` lists the device addresses in rank order, this rank's own
    entry being its local pointer.  ``close()`` unmaps every buffer this rank
    opened and then waits for the other ranks at a barrier, so that once it
    returns no rank maps anyone's buffers any more and each rank may free its
    own.  Until then every rank keeps its local tensors alive."""

    def __init__(self, local: dict, group=None):
        import torch.distributed as dist
        from . import ep
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        mine = {n: (ep.ep_ipc_export(t), t.numel() * t.element_size()) for n, t in local.items()}
        everyone = [None] * self.world
        dist.all_gather_object(everyone, mine, group=group)
        self._bases = []
        self.ptrs = {}
        try:
            for name, t in local.items():
                row = []
                for r in range(self.world):
                    if r == self.rank:
                        row.append(t.data_ptr())
                        continue
                    record, nbytes = everyone[r][name]
                    if ep.ipc_record_bytes(record) < nbytes:
                        raise ValueError(f"rank {r}'s {name}: the exported allocation is smaller than the buffer")
                    base, ptr = ep.ep_ipc_open(record)
                    self._bases.append(base)
                    row.append(ptr)
                self.ptrs[name] = row
        except Exception:
            self._unmap()
            raise

    def table(self, name: str) -> list:
        return self.ptrs[name]

    def _unmap(self):
        from . import ep
        while self._bases:
            ep.ep_ipc_close(self._bases.pop())

    def close(self):
        import torch.distributed as dist
        self._unmap()
        self.ptrs = {}
        dist.barrier(group=self.group)
