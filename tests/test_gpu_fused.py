"""ep_dispatch_with_layout: the layout and the dispatch in one call.

Below 16 tokens per SM, with the bulk-store dispatch, the call's dispatch
kernel loads and quantises x before it waits for the layout; the layout lets
it be scheduled only once everything before the call has completed.  These
tests compare the call with the oracle (layout, then dispatch) on the shapes
that take each path: the one-cluster, tiled and padded layouts before the
early dispatch, CTAs with more tokens than row stages, the plain dispatch
(large batch, other H), and orderings in which the kernel right before the
call writes x."""

import numpy as np
import pytest
import torch

import combine_ep_get_histogram_b200 as ep
import oracle
from combine_ep_get_histogram_b200 import workloads as wl
from gpu_util import assert_bits_equal, assert_layout_equal, bf16_host, to_dev, LAYOUT_FIELDS

pytestmark = pytest.mark.gpu


def _routing(T, k, E, seed, masked=0.0):
    rng = np.random.default_rng(seed)
    idx = np.argsort(rng.random((T, E)), axis=1)[:, :k]
    if masked:
        idx = np.where(rng.random((T, k)) < masked, -1, idx)
    return np.ascontiguousarray(idx.astype(np.int64))


class Fused:
    def __init__(self, device, T, H, k, E, R, use_fp8, num_sms=0, M=0):
        self.T, self.H, self.k, self.E, self.R, self.M = T, H, k, E, R, M
        self.use_fp8 = use_fp8
        self.device = device
        self.shape = ep.make_shape(T, H, k, E, R, use_fp8, num_sms, M)
        self.rows = ep.ep.receive_rows(self.shape)
        self.handle = ep.Handle(self.shape, device)
        self.ws = ep.workspace(self.shape, device)
        P = max(self.rows, 1)
        dt = torch.uint8 if use_fp8 else torch.int16
        self.rx = torch.zeros((P, H), dtype=dt, device=device)
        self.rs = torch.zeros((P, H // 128), dtype=torch.float32, device=device) if use_fp8 else None
        self.rw = torch.zeros(P, dtype=torch.float32, device=device)

    def call(self, idx_dev, x_dev, w_dev):
        ep.ep_dispatch_with_layout(self.shape, idx_dev, x_dev, w_dev, self.handle, self.ws, self.rx, self.rs,
                                   self.rw)

    def check(self, idx, x, wts):
        torch.cuda.synchronize()
        ref = oracle.layout_padded(idx, self.E, self.R, self.M) if self.M else oracle.layout(idx, self.E, self.R)
        counts = ep.handle_sizes(self.shape)
        got = {n: self.handle.tensors[n].cpu().numpy()[: counts[n]] for n in LAYOUT_FIELDS}
        assert_layout_equal(got, ref)
        slots = ref["slot_of_pair"]
        used = np.sort(slots[slots >= 0])
        rx, rs, rw = oracle.dispatch(x, wts, slots, self.use_fp8, P=self.rows)
        gx = self.rx.cpu().numpy()
        if self.use_fp8:
            assert_bits_equal("recv_x", gx[used], rx[used])
            assert_bits_equal("recv_scale", self.rs.cpu().numpy()[used].view(np.uint32), rs[used].view(np.uint32))
        else:
            assert_bits_equal("recv_x", gx[used].view(np.uint16), rx[used])
        assert_bits_equal("recv_weight", self.rw.cpu().numpy()[used].view(np.uint32), rw[used].view(np.uint32))
        assert ep.ep_get_error(self.handle) == 0


@pytest.mark.parametrize("T,H,k,E,R,use_fp8,num_sms,M", [
    (1024, 7168, 8, 256, 8, True, 0, 0),     # decode: one-cluster layout, early FP8 dispatch
    (1024, 2048, 8, 64, 8, False, 0, 0),     # early BF16 dispatch
    (2056, 2048, 8, 256, 8, True, 0, 0),     # tiled layout (three kernels) before the early dispatch
    (1024, 7168, 8, 256, 8, True, 8, 0),     # 8-SM budget: 24 CTAs, tokens past the row stages
    (1024, 7168, 8, 256, 8, True, 0, 128),   # padded layout (one cluster) before the early dispatch
    (512, 2048, 4, 64, 16, True, 0, 40),     # padded layout with 16 ranks (atomics)
    (8, 4096, 4, 16, 4, True, 0, 0),         # fewer tokens than CTAs
    (512, 8192, 4, 64, 8, False, 8, 0),      # BF16 at H = 8192: two row stages, then the loop (8-SM budget)
    (512, 8192, 32, 64, 8, True, 0, 0),      # k = 32: every lane of a staging warp reads a slot
    (6144, 4096, 8, 128, 8, False, 0, 0),    # 41 tokens per SM: no programmatic launch, plain dispatch
    (256, 256, 4, 16, 4, True, 0, 0),        # H = 256: the warp-per-chunk dispatch
])
def test_fused_matches_the_oracle(cuda_device, T, H, k, E, R, use_fp8, num_sms, M):
    idx = _routing(T, k, E, seed=T + H, masked=0.05)
    wts = np.random.default_rng(1).uniform(0.05, 1.0, (T, k)).astype(np.float32)
    x = wl.normal_bf16(T, H, 7, 1)
    f = Fused(cuda_device, T, H, k, E, R, use_fp8, num_sms, M)
    f.call(to_dev(idx, cuda_device), to_dev(x, cuda_device), to_dev(wts, cuda_device))
    f.check(idx, x, wts)


def test_fused_empty(cuda_device):
    f = Fused(cuda_device, 0, 2048, 8, 64, 8, True)
    idx = torch.zeros((1, 8), dtype=torch.int64, device=cuda_device)
    x = torch.zeros((1, 2048), dtype=torch.int16, device=cuda_device)
    w = torch.zeros((1, 8), dtype=torch.float32, device=cuda_device)
    f.call(idx, x, w)
    torch.cuda.synchronize()
    assert int(f.handle.tensors["expert_offset"].cpu()[-1]) == 0
    assert ep.ep_get_error(f.handle) == 0


@pytest.mark.parametrize("graph", [False, True])
def test_x_written_right_before_the_call(cuda_device, graph):
    """The kernel right before the call writes x: combine writes out, which
    the next layer dispatches (decode shape, stacked MoE layers), and torch
    overwrites the other x right before the second call.  Every call is
    compared with the oracle on the x the stream order defines."""
    T, H, k, E, R = 1024, 7168, 8, 256, 8
    idx_a, idx_b = _routing(T, k, E, 3), _routing(T, k, E, 4)
    wts = np.random.default_rng(5).uniform(0.05, 1.0, (T, k)).astype(np.float32)
    x0 = wl.normal_bf16(T, H, 8, 1)
    x1 = wl.normal_bf16(T, H, 9, 1)
    y = wl.normal_bf16(T * k, H, 10, 2)
    dev = cuda_device
    ia, ib, wd = to_dev(idx_a, dev), to_dev(idx_b, dev), to_dev(wts, dev)
    x_dev, x_new, yd = to_dev(x0, dev), to_dev(x1, dev), to_dev(y, dev)
    # the first layer's layout and combine produce out
    shape_c = ep.make_shape(T, H, k, E, R, True)
    hc, wsc = ep.Handle(shape_c, dev), ep.workspace(shape_c, dev)
    out = torch.empty((T, H), dtype=torch.int16, device=dev)
    ep.ep_get_dispatch_layout(shape_c, ia, hc, wsc)
    f1 = Fused(dev, T, H, k, E, R, True)
    f2 = Fused(dev, T, H, k, E, R, True)
    torch.cuda.synchronize()

    def seq():
        ep.ep_combine(shape_c, yd, wd, hc, out)   # writes out ...
        f1.call(ib, out, wd)                      # ... which this call dispatches
        x_dev.copy_(x_new)                        # torch overwrites x ...
        f2.call(ia, x_dev, wd)                    # ... right before this call reads it

    if graph:
        f1.call(ib, out, wd)  # first calls outside the capture
        f2.call(ia, x_dev, wd)
        torch.cuda.synchronize()
        x_dev.copy_(to_dev(x0, dev))
        out.zero_()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                seq()
        g.replay()
    else:
        seq()
    torch.cuda.synchronize()
    out_ref = oracle.combine(y, wts, oracle.layout(idx_a, E, R)["slot_of_pair"])
    assert_bits_equal("combine", bf16_host(out), out_ref)
    f1.check(idx_b, out_ref, wts)
    f2.check(idx_a, x1, wts)


def test_fused_equals_the_two_calls(cuda_device):
    """Same handle, receive rows, scales and weights as the layout call
    followed by the dispatch call, bit for bit (decode shape)."""
    T, H, k, E, R = 1024, 7168, 8, 256, 8
    idx = _routing(T, k, E, 12, masked=0.02)
    wts = np.random.default_rng(13).uniform(0.05, 1.0, (T, k)).astype(np.float32)
    x = to_dev(wl.normal_bf16(T, H, 14, 1), cuda_device)
    idx_d, w_d = to_dev(idx, cuda_device), to_dev(wts, cuda_device)
    a = Fused(cuda_device, T, H, k, E, R, True)
    b = Fused(cuda_device, T, H, k, E, R, True)
    a.call(idx_d, x, w_d)
    ep.ep_get_dispatch_layout(b.shape, idx_d, b.handle, b.ws)
    ep.ep_dispatch(b.shape, x, w_d, b.handle, b.rx, b.rs, b.rw)
    torch.cuda.synchronize()
    for n in LAYOUT_FIELDS:
        assert torch.equal(a.handle.tensors[n], b.handle.tensors[n]), n
    assert torch.equal(a.rx, b.rx) and torch.equal(a.rs, b.rs) and torch.equal(a.rw, b.rw)


def test_fused_bad_index(cuda_device):
    """An out-of-range expert id through the fused call: the pair is masked
    and the error word reports it, as with the two separate calls."""
    T, H, k, E, R = 256, 2048, 4, 16, 4
    idx = _routing(T, k, E, seed=21)
    idx[7, 2] = E + 5
    wts = np.random.default_rng(22).uniform(0.05, 1.0, (T, k)).astype(np.float32)
    x = wl.normal_bf16(T, H, 23, 1)
    f = Fused(cuda_device, T, H, k, E, R, True)
    f.call(to_dev(idx, cuda_device), to_dev(x, cuda_device), to_dev(wts, cuda_device))
    torch.cuda.synchronize()
    ref = oracle.layout(idx, E, R)
    assert ref["slot_of_pair"][7 * k + 2] == -1
    counts = ep.handle_sizes(f.shape)
    got = {n: f.handle.tensors[n].cpu().numpy()[: counts[n]] for n in LAYOUT_FIELDS}
    assert_layout_equal(got, ref)
    slots = ref["slot_of_pair"]
    used = np.sort(slots[slots >= 0])
    rx, rs, rw = oracle.dispatch(x, wts, slots, True)
    assert_bits_equal("recv_x", f.rx.cpu().numpy()[used], rx[used])
    assert_bits_equal("recv_scale", f.rs.cpu().numpy()[used].view(np.uint32), rs[used].view(np.uint32))
    assert ep.ep_get_error(f.handle) == ep.ep.EP_ERR_BAD_INDEX
