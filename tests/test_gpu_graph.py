"""The whole hot path can be captured in a CUDA graph and replayed.

The C ABI never allocates or synchronises and its grids depend only on the
shape, not on the routing, so one captured step (layout, dispatch, combine,
both backward passes) serves any routing of that shape.  Replaying it on two
different routings must give exactly the outputs of eager calls."""

import numpy as np
import pytest
import torch

import combine_ep_get_histogram_b200 as ep
from combine_ep_get_histogram_b200 import workloads as wl
from gpu_util import to_dev

pytestmark = pytest.mark.gpu


class Step:
    def __init__(self, w, device, max_tokens_per_rank=0):
        self.w = w
        self.shape = ep.make_shape(w.T, w.H, w.k, w.E, w.R, w.use_fp8, 0, max_tokens_per_rank)
        P = ep.ep.receive_rows(self.shape)
        self.h = ep.Handle(self.shape, device)
        self.ws = ep.workspace(self.shape, device)
        self.idx = torch.empty((w.T, w.k), dtype=torch.int64, device=device)
        self.wts = torch.empty((w.T, w.k), dtype=torch.float32, device=device)
        self.x = torch.empty((w.T, w.H), dtype=torch.int16, device=device)
        self.y = torch.empty((P, w.H), dtype=torch.int16, device=device)
        self.g = torch.empty((w.T, w.H), dtype=torch.int16, device=device)
        self.rx = torch.empty((P, w.H), dtype=torch.uint8 if w.use_fp8 else torch.int16, device=device)
        self.rs = torch.empty((P, w.G), dtype=torch.float32, device=device) if w.use_fp8 else None
        self.rw = torch.empty(P, dtype=torch.float32, device=device)
        self.out = torch.empty((w.T, w.H), dtype=torch.int16, device=device)
        self.gy = torch.empty((P, w.H), dtype=torch.int16, device=device)
        self.gw = torch.empty((w.T, w.k), dtype=torch.float32, device=device)
        self.gx = torch.empty((w.T, w.H), dtype=torch.int16, device=device)

    def load(self, d):
        self.idx.copy_(torch.from_numpy(d["topk_idx"]))
        self.wts.copy_(torch.from_numpy(d["topk_weights"]))
        for n in ("x", "y", "g"):
            getattr(self, n).copy_(to_dev(d[n], "cpu"))

    def run(self):
        ep.ep_get_dispatch_layout(self.shape, self.idx, self.h, self.ws)
        ep.ep_dispatch(self.shape, self.x, self.wts, self.h, self.rx, self.rs, self.rw)
        ep.ep_combine(self.shape, self.y, self.wts, self.h, self.out)
        ep.ep_combine_backward(self.shape, self.g, self.y, self.wts, self.h, self.gy, self.gw)
        ep.ep_dispatch_backward(self.shape, self.gy, self.h, self.gx)

    def outputs(self):
        """Handle arrays, and the receive rows that hold a pair (padded
        layouts leave the other rows unwritten)."""
        torch.cuda.synchronize()
        if self.shape.max_tokens_per_rank:
            rows = torch.nonzero(self.h.src_of_slot >= 0).squeeze(1)
        else:
            rows = torch.arange(int(self.h.expert_offset[-1].item()), device=self.rx.device)
        res = [self.h.tensors[f].clone() for f in ("slot_of_pair", "src_of_slot", "expert_offset",
                                                    "num_tokens_per_rank", "is_token_in_rank")]
        res += [self.rx[rows].clone(), self.rw[rows].clone(), self.out.clone(), self.gy[rows].clone(),
                self.gw.clone(), self.gx.clone()]
        if self.rs is not None:
            res.append(self.rs[rows].clone())
        return res


@pytest.mark.parametrize("name,padded", [("decode", False), ("tiny", False), ("tiny", True)])
def test_step_replays_from_a_cuda_graph(cuda_device, name, padded):
    w = wl.CONFIGS[name]
    M = w.T // w.R if padded else 0
    inputs = [wl.make_inputs(w.with_(seed=s), parts=("routing", "x", "y", "g")) for s in (0, 1)]
    if padded:  # expert outputs live in the padded receive rows
        for s, d in enumerate(inputs):
            d["y"] = wl.normal_bf16(w.E * w.R * M, w.H, s, 2)
    assert not np.array_equal(inputs[0]["topk_idx"], inputs[1]["topk_idx"])

    eager = Step(w, cuda_device, M)
    expected = []
    for d in inputs:
        eager.load(d)
        eager.run()
        expected.append(eager.outputs())

    step = Step(w, cuda_device, M)
    step.load(inputs[0])
    step.run()  # first use on the device happens outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step.run()
    for d, exp in zip(inputs, expected):
        step.load(d)
        graph.replay()
        got = step.outputs()
        for a, b in zip(got, exp):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    del graph
