"""Two processes, one rank each, on one GPU: the peer calls on buffers that
another process owns, reached through CUDA IPC (multi.PeerBuffers over the
C ABI's ep_ipc_export / ep_ipc_open).

Each rank holds its own tokens and its own experts' receive buffers
(payload, scales, weights, expert outputs, their gradients).  The ranks
all-gather their routing over gloo, build the same global layout, exchange
their buffers' IPC records, and run, with a stream synchronisation and a
host barrier between a buffer's writers and its readers:

    dispatch_peers -> barrier -> combine_peers, combine_backward_peers
    -> barrier -> dispatch_backward_peers -> barrier

Every rank then compares what it holds with the CPU oracle: its receive rows
(owner side), and its tokens' combined output, grad_w and grad_x (token
side).  The ranks leave only after every IPC mapping is closed.  No kernel
waits on another rank: the ordering is all on the host."""

import datetime
import os
import socket
import sys
import traceback

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = {
    # H = 7168 with FP8: dispatch writes the peers' rows with TMA bulk copies
    "fp8-bulk-H7168": dict(T=2 * 256, H=7168, k=8, E=64, use_fp8=True, mask=0.0),
    # ragged H, BF16 and masked pairs: the warp-per-chunk dispatch and ragged gathers
    "bf16-ragged-masked": dict(T=2 * 200, H=640, k=6, E=32, use_fp8=False, mask=0.15),
}


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    try:
        import numpy as np
        import torch
        import torch.distributed as dist

        import combine_ep_get_histogram_b200 as ep
        import oracle
        from combine_ep_get_histogram_b200 import multi
        from combine_ep_get_histogram_b200 import workloads as wl
        from gpu_util import assert_bits_equal, bf16_host, grad_w_close, to_dev

        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
        dev = torch.device("cuda:0")
        torch.cuda.set_device(dev)
        c = CASES[case]
        w = wl.Workload("ipc", T=c["T"], H=c["H"], k=c["k"], E=c["E"], R=world, use_fp8=c["use_fp8"],
                        routing="group", n_groups=4, topk_groups=2)
        # every rank draws the same global inputs and keeps its own share
        d = wl.make_inputs(w, parts=("routing", "x", "g"))
        idx_all = d["topk_idx"]
        if c["mask"]:
            rng = np.random.default_rng(7)
            idx_all = np.ascontiguousarray(np.where(rng.random(idx_all.shape) < c["mask"], -1, idx_all))
        P = w.T * w.k
        y_all = wl.normal_bf16(P, w.H, w.seed, 2)
        b, e = multi.token_range(w.T, world, rank)

        # routing exchange and the global layout, the same on every rank
        ids = multi.gather_routing(torch.from_numpy(np.ascontiguousarray(idx_all[b:e]))).numpy()
        assert np.array_equal(ids, idx_all)
        shape = ep.make_shape(w.T, w.H, w.k, w.E, world, w.use_fp8)
        idx_dev = torch.from_numpy(ids).to(dev)
        h = ep.Handle(shape, dev)
        ep.ep_get_dispatch_layout(shape, idx_dev, h, ep.workspace(shape, dev))
        eoff = h.expert_offset.cpu().numpy()
        r0, n = multi.owner_rows(eoff, w.E, world)[rank]

        # this rank's receive buffers (its experts' rows)
        rows = max(n, 1)
        own = {
            "rx": torch.zeros((rows, w.H), dtype=torch.uint8 if w.use_fp8 else torch.int16, device=dev),
            "rs": torch.zeros((rows, w.G if w.use_fp8 else 1), dtype=torch.float32, device=dev),
            "rw": torch.zeros(rows, dtype=torch.float32, device=dev),
            "y": to_dev(y_all[r0:r0 + rows] if n else np.zeros((1, w.H), np.uint16), dev),
            "gy": torch.zeros((rows, w.H), dtype=torch.int16, device=dev),
        }
        peers = multi.PeerBuffers(own)
        tab = peers.table
        x_r = to_dev(d["x"][b:e], dev)
        w_r = to_dev(d["topk_weights"][b:e].astype(np.float32), dev)
        g_r = to_dev(d["g"][b:e], dev)

        def sync():
            torch.cuda.synchronize()
            dist.barrier()

        ep.ep_dispatch_peers(shape, rank, idx_dev, h, x_r, w_r, tab("rx"), tab("rs") if w.use_fp8 else None,
                             tab("rw"))
        sync()
        out = torch.empty((e - b, w.H), dtype=torch.int16, device=dev)
        gw = torch.full((e - b, w.k), -7.0, dtype=torch.float32, device=dev)
        ep.ep_combine_peers(shape, rank, idx_dev, h, tab("y"), w_r, out)
        ep.ep_combine_backward_peers(shape, rank, idx_dev, h, g_r, tab("y"), w_r, tab("gy"), gw)
        sync()
        gx = torch.empty((e - b, w.H), dtype=torch.int16, device=dev)
        ep.ep_dispatch_backward_peers(shape, rank, idx_dev, h, tab("gy"), gx)
        sync()
        assert ep.ep_get_error(h) == 0
        got = {k_: v.cpu().numpy() for k_, v in own.items()}
        out_h, gw_h, gx_h = bf16_host(out), gw.cpu().numpy(), bf16_host(gx)
        peers.close()  # every mapping closed on every rank before anyone frees
        del own

        # the oracle over the global problem; this rank's share of it
        lay = oracle.layout(ids, w.E, world)
        assert np.array_equal(lay["expert_offset"], eoff)
        slots = lay["slot_of_pair"]
        orx, ors, orw = oracle.dispatch(d["x"], d["topk_weights"], slots, w.use_fp8)
        sl = slice(r0, r0 + n)
        assert_bits_equal(f"rank {rank} recv_x", got["rx"][:n] if w.use_fp8 else got["rx"][:n].view(np.uint16),
                          orx[sl])
        assert_bits_equal(f"rank {rank} recv_weight", got["rw"][:n].view(np.uint32), orw[sl].view(np.uint32))
        if w.use_fp8:
            assert_bits_equal(f"rank {rank} recv_scale", got["rs"][:n].view(np.uint32), ors[sl].view(np.uint32))
        assert_bits_equal(f"rank {rank} combine", out_h, oracle.combine(y_all, d["topk_weights"], slots)[b:e])
        rgy, rgw = oracle.combine_backward(d["g"], y_all, d["topk_weights"], slots)
        assert_bits_equal(f"rank {rank} grad_y", got["gy"][:n].view(np.uint16), rgy[sl])
        ok, worst = grad_w_close(gw_h, rgw[b:e])
        assert ok, worst
        assert_bits_equal(f"rank {rank} grad_x", gx_h, oracle.dispatch_backward(rgy, slots, w.T, w.k)[b:e])
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, "ok", n))
    except Exception:
        q.put((rank, traceback.format_exc(), -1))
        raise


@pytest.mark.parametrize("case", list(CASES))
def test_two_processes_through_ipc(cuda_device, case):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    results = []
    while not q.empty():
        results.append(q.get(timeout=5))
    for p in procs:
        if p.is_alive():
            p.kill()
    msgs = {r: m for r, m, _ in results}
    assert all(p.exitcode == 0 for p in procs), msgs
    assert sorted(msgs) == [0, 1] and all(m == "ok" for m in msgs.values()), msgs
    assert sum(n for _, _, n in results) > 0
