"""Multi-GPU expert parallelism, R ranks emulated on one GPU.

Every owner rank's receive buffers (dispatch payload, scales, weights, expert
outputs, their gradients) are separate allocations.  Each rank calls the
*_peers entry points for its own tokens only, with peer tables that point at
all owners' buffers, exactly as it would with other GPUs' memory.

Every output is compared with the CPU oracle directly: the concatenation of
the owners' buffers with the oracle's receive buffer (payload, scales,
weights, grad_y), every rank's combined tokens and grad_x with the oracle's
combine and dispatch backward, grad_w within its tolerance.  The outputs are
also bit-identical to the single-GPU path's (the same arithmetic, element for
element, in the same order)."""

import numpy as np
import pytest
import torch

import combine_ep_get_histogram_b200 as ep
import oracle
from combine_ep_get_histogram_b200 import multi
from combine_ep_get_histogram_b200 import workloads as wl
from gpu_util import GpuPath, assert_bits_equal, bf16_host, grad_w_close, to_dev

pytestmark = pytest.mark.gpu


def masked(idx, frac, seed):
    rng = np.random.default_rng(seed)
    return np.ascontiguousarray(np.where(rng.random(idx.shape) < frac, -1, idx))


CASES = {
    "tiny-bf16": (wl.CONFIGS["tiny"], 0.0),
    "tiny-fp8-outliers": (wl.CONFIGS["tiny"].with_(use_fp8=True, outlier_frac=0.02, outlier_gain=50.0), 0.0),
    "decode-shape-fp8-8ranks": (wl.CONFIGS["decode"].with_(T=8 * 32), 0.0),
    "masked-pairs-ragged-H": (wl.Workload("ragged", T=96, H=640, k=4, E=32, R=4, use_fp8=False,
                                          routing="group", n_groups=4, topk_groups=2), 0.2),
    # 4 to 16 chunks: dispatch by TMA bulk copies into the owners' buffers
    "bulk-bf16-masked": (wl.Workload("bulk", T=256, H=2560, k=8, E=64, R=8, use_fp8=False,
                                     routing="group", n_groups=8, topk_groups=4), 0.1),
    "bulk-fp8-ragged-H": (wl.Workload("bulk", T=512, H=2176, k=6, E=48, R=4, use_fp8=True,
                                      routing="group", n_groups=4, topk_groups=2), 0.15),
    # k, E and the owner count at their maxima (k = 32, E = 1024, R = 64): the shared-memory tables full
    "maxima-bulk-fp8": (wl.Workload("maxima", T=64 * 8, H=2048, k=32, E=1024, R=64, use_fp8=True,
                                    routing="group", n_groups=8, topk_groups=4), 0.05),
    "maxima-warp-bf16": (wl.Workload("maxima", T=64 * 4, H=256, k=32, E=1024, R=64, use_fp8=False,
                                     routing="group", n_groups=8, topk_groups=4), 0.0),
    # 2560 tokens per rank, past 16 per SM: the bulk-copy dispatch on an oversubscribed grid
    "bulk-fp8-large-batch": (wl.Workload("bulk", T=4 * 2560, H=2176, k=4, E=32, R=4, use_fp8=True,
                                         routing="group", n_groups=4, topk_groups=2), 0.0),
}


@pytest.mark.parametrize("name", list(CASES))
def test_ranks_reproduce_the_single_gpu_path(cuda_device, name):
    w, mask = CASES[name]
    d = wl.make_inputs(w, parts=("routing", "x", "g"))
    idx = masked(d["topk_idx"], mask, seed=7) if mask else d["topk_idx"]
    wts = d["topk_weights"]
    P = w.T * w.k
    y = wl.normal_bf16(P, w.H, w.seed, 2)

    # the single-GPU path (itself checked against the oracle elsewhere)
    one = GpuPath(w, idx, wts, cuda_device).layout()
    rx1, rs1, rw1 = one.dispatch(to_dev(d["x"], cuda_device))
    yd = to_dev(y, cuda_device)
    out1 = bf16_host(one.combine(yd))
    gy1, gw1 = one.combine_backward(to_dev(d["g"], cuda_device), yd)
    gx1 = bf16_host(one.dispatch_backward(gy1))
    torch.cuda.synchronize()
    eoff = one.handle.tensors["expert_offset"].cpu().numpy()
    rows = multi.owner_rows(eoff, w.E, w.R)
    n_valid = int(eoff[-1])

    # owners' buffers: payload, scales, weights, expert outputs, their gradients
    pay = torch.uint8 if w.use_fp8 else torch.int16
    rx = [torch.full((max(n, 1), w.H), 0, dtype=pay, device=cuda_device) for _, n in rows]
    rs = [torch.zeros((max(n, 1), w.G), dtype=torch.float32, device=cuda_device) for _, n in rows]
    rw = [torch.zeros(max(n, 1), dtype=torch.float32, device=cuda_device) for _, n in rows]
    ys = [yd[r0:r0 + n].clone() if n else torch.zeros((1, w.H), dtype=torch.int16, device=cuda_device)
          for r0, n in rows]
    gys = [torch.zeros((max(n, 1), w.H), dtype=torch.int16, device=cuda_device) for _, n in rows]

    shape = one.shape
    idx_all = to_dev(idx, cuda_device)
    outs, gws, gxs = [], [], []
    for r in range(w.R):  # every rank's calls; each one sees all owners' buffers
        b, e = multi.token_range(w.T, w.R, r)
        x_r = to_dev(d["x"][b:e], cuda_device)
        w_r = to_dev(wts[b:e].astype(np.float32), cuda_device)
        ep.ep_dispatch_peers(shape, r, idx_all, one.handle, x_r, w_r, rx, rs if w.use_fp8 else None, rw)
    for r in range(w.R):
        b, e = multi.token_range(w.T, w.R, r)
        w_r = to_dev(wts[b:e].astype(np.float32), cuda_device)
        out_r = torch.empty((e - b, w.H), dtype=torch.int16, device=cuda_device)
        ep.ep_combine_peers(shape, r, idx_all, one.handle, ys, w_r, out_r)
        gw_r = torch.full((e - b, w.k), -7.0, dtype=torch.float32, device=cuda_device)
        ep.ep_combine_backward_peers(shape, r, idx_all, one.handle, to_dev(d["g"][b:e], cuda_device), ys, w_r,
                                     gys, gw_r)
        outs.append(out_r)
        gws.append(gw_r)
    for r in range(w.R):  # after every rank's combine backward wrote grad_y
        b, e = multi.token_range(w.T, w.R, r)
        gx_r = torch.empty((e - b, w.H), dtype=torch.int16, device=cuda_device)
        ep.ep_dispatch_backward_peers(shape, r, idx_all, one.handle, gys, gx_r)
        gxs.append(gx_r)
    torch.cuda.synchronize()

    def cat(bufs):
        return np.concatenate([t.cpu().numpy()[:n] for t, (_, n) in zip(bufs, rows)])

    assert np.array_equal(cat(rx), rx1.cpu().numpy()[:n_valid])
    assert np.array_equal(cat(rw).view(np.uint32), rw1.cpu().numpy()[:n_valid].view(np.uint32))
    if w.use_fp8:
        assert np.array_equal(cat(rs).view(np.uint32), rs1.cpu().numpy()[:n_valid].view(np.uint32))
    assert np.array_equal(np.concatenate([bf16_host(o) for o in outs]), out1[:w.T])
    assert np.array_equal(cat(gys).view(np.uint16), bf16_host(gy1)[:n_valid])
    assert np.array_equal(np.concatenate([bf16_host(g) for g in gxs]), gx1[:w.T])
    got_gw = np.concatenate([g.cpu().numpy() for g in gws])
    # the same partial sums in the same order as the single-GPU kernel: bit-identical
    assert np.array_equal(got_gw.view(np.uint32), gw1.cpu().numpy()[:w.T].reshape(got_gw.shape).view(np.uint32))

    # every output against the oracle
    lay = oracle.layout(idx, w.E, w.R)
    assert np.array_equal(lay["expert_offset"], eoff)
    slots = lay["slot_of_pair"]
    orx, ors, orw = oracle.dispatch(d["x"], wts, slots, w.use_fp8)
    got_rx = cat(rx)
    assert_bits_equal("peer recv_x", got_rx if w.use_fp8 else got_rx.view(np.uint16), orx[:n_valid])
    assert_bits_equal("peer recv_weight", cat(rw).view(np.uint32), orw[:n_valid].view(np.uint32))
    if w.use_fp8:
        assert_bits_equal("peer recv_scale", cat(rs).view(np.uint32), ors[:n_valid].view(np.uint32))
    assert_bits_equal("peer combine out", np.concatenate([bf16_host(o) for o in outs]), oracle.combine(y, wts, slots))
    rgy, rgw = oracle.combine_backward(d["g"], y, wts, slots)
    assert_bits_equal("peer grad_y", cat(gys).view(np.uint16), rgy[:n_valid])
    ok, worst = grad_w_close(got_gw, rgw)
    assert ok, worst
    assert_bits_equal("peer grad_x", np.concatenate([bf16_host(g) for g in gxs]),
                      oracle.dispatch_backward(rgy, slots, w.T, w.k))


def test_one_rank_is_the_single_gpu_path(cuda_device):
    """R = 1: the owner table has one entry, the whole receive buffer."""
    w = wl.CONFIGS["tiny"].with_(R=1)
    d = wl.make_inputs(w, parts=("routing", "x"))
    one = GpuPath(w, d["topk_idx"], d["topk_weights"], cuda_device).layout()
    rx1, _, rw1 = one.dispatch(to_dev(d["x"], cuda_device))
    rx = torch.zeros_like(rx1)
    rw = torch.zeros_like(rw1)
    ep.ep_dispatch_peers(one.shape, 0, one.idx, one.handle, to_dev(d["x"], cuda_device), one.wts, [rx], None, [rw])
    torch.cuda.synchronize()
    assert torch.equal(rx, rx1) and torch.equal(rw, rw1)
    orx, _, orw = oracle.dispatch(d["x"], d["topk_weights"], oracle.layout(d["topk_idx"], w.E, w.R)["slot_of_pair"],
                                  False)
    assert_bits_equal("R=1 recv_x", bf16_host(rx), orx)
    assert_bits_equal("R=1 recv_weight", rw.cpu().numpy().view(np.uint32), orw.view(np.uint32))
