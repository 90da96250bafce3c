"""Ordering under programmatic dependent launch.

Small batches launch every kernel with programmatic stream serialization:
a kernel may become resident while the previous one on the stream still
runs, and waits for it (griddepcontrol.wait) before its first global load or
store.  These tests chain calls whose buffers overlap, so that a kernel that
read before the wait would see its predecessor's half-written output, and a
kernel that wrote before it would overwrite data its predecessor still
reads:

* layout A -> dispatch -> layout B (overwrites the slots dispatch read) ->
  dispatch into the same buffers, and torch writing x between the two;
* combine -> combine backward -> dispatch backward, each reading what the
  previous one wrote, and the same calls replayed from a CUDA graph.

Every result is compared with the oracle."""

import numpy as np
import pytest
import torch

import combine_ep_get_histogram_b200 as ep
import oracle
from combine_ep_get_histogram_b200 import workloads as wl
from gpu_util import assert_bits_equal, bf16_host, grad_w_close, to_dev

pytestmark = pytest.mark.gpu


def _routing(T, k, E, seed):
    rng = np.random.default_rng(seed)
    return np.ascontiguousarray(np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int64))


def test_layouts_and_dispatches_back_to_back(cuda_device):
    T, H, k, E, R = 1024, 7168, 8, 256, 8  # the decode shape: below 16 tokens per SM
    shape = ep.make_shape(T, H, k, E, R, use_fp8=True)
    idx_a, idx_b = _routing(T, k, E, 1), _routing(T, k, E, 2)
    wts = np.random.default_rng(3).uniform(0.1, 1.0, (T, k)).astype(np.float32)
    x_a, x_b = wl.normal_bf16(T, H, 4, 1), wl.normal_bf16(T, H, 5, 1)
    h = ep.Handle(shape, cuda_device)
    ws = ep.workspace(shape, cuda_device)
    ia, ib = to_dev(idx_a, cuda_device), to_dev(idx_b, cuda_device)
    wd = to_dev(wts, cuda_device)
    x = to_dev(x_a, cuda_device)
    xb = to_dev(x_b, cuda_device)
    P = T * k
    rx = torch.empty((P, H), dtype=torch.uint8, device=cuda_device)
    rs = torch.empty((P, H // 128), dtype=torch.float32, device=cuda_device)
    rw = torch.empty(P, dtype=torch.float32, device=cuda_device)
    rx_a = torch.empty_like(rx)
    torch.cuda.synchronize()
    # all on one stream, no host synchronisation in between
    ep.ep_get_dispatch_layout(shape, ia, h, ws)
    ep.ep_dispatch(shape, x, wd, h, rx, rs, rw)
    ep.ep_get_dispatch_layout(shape, ib, h, ws)  # overwrites the slots the dispatch right before it reads
    rx_a.copy_(rx)                               # torch reads what the first dispatch wrote
    x.copy_(xb)                                  # torch overwrites the x the first dispatch read
    ep.ep_dispatch(shape, x, wd, h, rx, rs, rw)
    torch.cuda.synchronize()
    ref_a = oracle.dispatch(x_a, wts, oracle.layout(idx_a, E, R)["slot_of_pair"], True)
    ref_b = oracle.dispatch(x_b, wts, oracle.layout(idx_b, E, R)["slot_of_pair"], True)
    assert_bits_equal("first dispatch", rx_a.cpu().numpy(), ref_a[0])
    assert_bits_equal("second dispatch", rx.cpu().numpy(), ref_b[0])
    assert_bits_equal("second scales", rs.cpu().numpy().view(np.uint32), ref_b[1].view(np.uint32))
    assert_bits_equal("second weights", rw.cpu().numpy().view(np.uint32), ref_b[2].view(np.uint32))
    assert ep.ep_get_error(h) == 0


@pytest.mark.parametrize("graph", [False, True])
def test_backward_chain(cuda_device, graph):
    """combine -> combine backward (reads y, writes grad_y) -> dispatch
    backward (reads grad_y) -> combine again over grad_y (reads what dispatch
    backward's predecessor wrote), eagerly or from a CUDA graph."""
    w = wl.CONFIGS["decode"]
    d = wl.make_inputs(w, parts=("routing", "y", "g"))
    shape = ep.make_shape(w.T, w.H, w.k, w.E, w.R, w.use_fp8)
    h = ep.Handle(shape, cuda_device)
    ws = ep.workspace(shape, cuda_device)
    idx = to_dev(d["topk_idx"], cuda_device)
    wts = to_dev(d["topk_weights"], cuda_device)
    y, g = to_dev(d["y"], cuda_device), to_dev(d["g"], cuda_device)
    P = w.T * w.k
    out = torch.empty((w.T, w.H), dtype=torch.int16, device=cuda_device)
    gy = torch.empty((P, w.H), dtype=torch.int16, device=cuda_device)
    gw = torch.empty((w.T, w.k), dtype=torch.float32, device=cuda_device)
    gx = torch.empty((w.T, w.H), dtype=torch.int16, device=cuda_device)
    out2 = torch.empty_like(out)

    def chain():
        ep.ep_get_dispatch_layout(shape, idx, h, ws)
        ep.ep_combine(shape, y, wts, h, out)
        ep.ep_combine_backward(shape, g, y, wts, h, gy, gw)
        ep.ep_dispatch_backward(shape, gy, h, gx)
        ep.ep_combine(shape, gy, wts, h, out2)

    torch.cuda.synchronize()
    if graph:
        ep.ep_get_dispatch_layout(shape, idx, h, ws)  # first call outside the capture
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(gr, stream=s):
                chain()
        gr.replay()
        gr.replay()
    else:
        chain()
    torch.cuda.synchronize()
    slots = oracle.layout(d["topk_idx"], w.E, w.R)["slot_of_pair"]
    assert_bits_equal("combine", bf16_host(out), oracle.combine(d["y"], d["topk_weights"], slots))
    rgy, rgw = oracle.combine_backward(d["g"], d["y"], d["topk_weights"], slots)
    assert_bits_equal("grad_y", bf16_host(gy), rgy)
    ok, worst = grad_w_close(gw.cpu().numpy(), rgw)
    assert ok, worst
    assert_bits_equal("grad_x", bf16_host(gx), oracle.dispatch_backward(rgy, slots, w.T, w.k))
    assert_bits_equal("combine of grad_y", bf16_host(out2), oracle.combine(rgy, d["topk_weights"], slots))
