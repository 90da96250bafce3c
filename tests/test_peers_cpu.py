"""Host bookkeeping of multi-GPU expert parallelism, on CPU with two gloo ranks.

Each rank draws its own tokens' routing; one all-gather gives every rank all
ranks' ids in rank order, so every rank computes the same global layout (here
the oracle's); owner rank o's receive rows are one contiguous range of that
layout, the ranges tile [0, pairs) in rank order, and each range holds
exactly the pairs routed to o's experts."""

import datetime
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
T, K, E, R = 64, 4, 16, 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _local_routing(rank: int) -> np.ndarray:
    rng = np.random.default_rng(100 + rank)
    idx = np.argsort(rng.random((T // R, E)), axis=1)[:, :K]
    idx[rng.random(idx.shape) < 0.1] = -1  # some masked pairs
    return np.ascontiguousarray(idx.astype(np.int64))


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import oracle
    from combine_ep_get_histogram_b200 import multi
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = _local_routing(rank)
        everyone = multi.gather_routing(torch.from_numpy(mine)).numpy()
        lay = oracle.layout(everyone, E, R)
        rows = multi.owner_rows(lay["expert_offset"], E, R)
        b, e = multi.token_range(T, R, rank)
        q.put((rank, everyone.tobytes(), rows, (b, e), lay["slot_of_pair"].tobytes()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ranks_agree_on_the_global_layout_and_the_owner_rows():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, R, port, q)) for r in range(R)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(R))
    expect = np.concatenate([_local_routing(r) for r in range(R)])
    for rank, ids, rows, rng, slots in res:
        assert np.array_equal(np.frombuffer(ids, np.int64).reshape(T, K), expect)
        assert rng == (rank * T // R, (rank + 1) * T // R)
    assert len({r[4] for r in res}) == 1 and len({tuple(r[2]) for r in res}) == 1  # same layout everywhere
    rows = res[0][2]
    assert rows[0][0] == 0
    for o in range(R - 1):
        assert rows[o][0] + rows[o][1] == rows[o + 1][0]
    assert rows[-1][0] + rows[-1][1] == int((expect >= 0).sum())
    slots = np.frombuffer(res[0][4], np.int32).reshape(T, K)
    for o, (r0, n) in enumerate(rows):  # the pairs routed to o's experts are exactly o's rows
        mine = (expect >= 0) & (expect // (E // R) == o)
        assert sorted(slots[mine].tolist()) == list(range(r0, r0 + n))


def test_token_range_and_owner_rows_reject_uneven_splits():
    sys.path.insert(0, ROOT)
    import pytest
    from combine_ep_get_histogram_b200 import multi
    with pytest.raises(ValueError):
        multi.token_range(10, 4, 0)
    with pytest.raises(ValueError):
        multi.owner_rows([0] * 11, 10, 4)


class _FakeBuf:
    """Stands in for a device tensor: an address and a size, nothing else."""

    def __init__(self, ptr, n):
        self.ptr, self.n = ptr, n

    def data_ptr(self):
        return self.ptr

    def numel(self):
        return self.n

    def element_size(self):
        return 4


def _peer_buffers_main(rank, world, port, q, short):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from combine_ep_get_histogram_b200 import ep, multi
    opened, closed = [], []

    # host-side fakes of the C ABI's IPC calls: a record names the exporter's
    # address and the bytes its allocation holds from there
    def export(t):
        nbytes = t.numel() * t.element_size()
        if short and rank == 1 and t.ptr % 1000 == 2:
            nbytes -= 4  # rank 1 claims an allocation too small for its "b" buffer
        return f"{t.data_ptr()}:{nbytes}".encode()

    def record_bytes(rec):
        return int(rec.decode().split(":")[1])

    def open_(rec):
        ptr = int(rec.decode().split(":")[0])
        opened.append(ptr + 5)
        return ptr + 5, ptr + 7

    ep.ep_ipc_export, ep.ipc_record_bytes, ep.ep_ipc_open = export, record_bytes, open_
    ep.ep_ipc_close = closed.append
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local = {"a": _FakeBuf(10_000 * (rank + 1) + 1, 16), "b": _FakeBuf(10_000 * (rank + 1) + 2, 8)}
        try:
            pb = multi.PeerBuffers(local)
        except ValueError as e:
            q.put((rank, "refused", str(e), sorted(opened), sorted(closed)))
            dist.barrier()
            return
        tables = {n: pb.table(n) for n in local}
        pb.close()
        q.put((rank, "ok", tables, sorted(opened), sorted(closed)))
    finally:
        dist.destroy_process_group()


def _run_peer_buffers(short):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 3
    procs = [ctx.Process(target=_peer_buffers_main, args=(r, world, port, q, short)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return sorted(q.get(timeout=10) for _ in range(world))


def test_peer_buffers_tables_and_close():
    """Each rank's table lists every rank's buffer in rank order: its own
    local address, the others' through the opened mappings; close() unmaps
    every mapping it opened."""
    res = _run_peer_buffers(short=False)
    for rank, status, tables, opened, closed in res:
        assert status == "ok"
        for name, off in (("a", 1), ("b", 2)):
            expect = [10_000 * (r + 1) + off + (0 if r == rank else 7) for r in range(3)]
            assert tables[name] == expect
        assert len(opened) == 2 * 2 and opened == closed


def test_peer_buffers_refuse_a_short_allocation():
    """A peer whose exported allocation cannot hold the buffer is refused,
    and whatever was already mapped is unmapped."""
    res = _run_peer_buffers(short=True)
    for rank, status, msg, opened, closed in res:
        if rank == 1:
            assert status == "ok" or status == "refused"
        else:
            assert status == "refused" and "rank 1" in msg
            assert opened == closed
