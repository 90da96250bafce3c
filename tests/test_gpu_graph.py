"""The whole hot path can be captured in a CUDA graph and replayed.

The C ABI never allocates or synchronises and its grids depend only on the
shape, not on the routing, so one captured step (layout, dispatch, combine,
both backward passes) serves any routing of that shape.  Replaying it on two
different routings must give exactly the outputs of eager calls."""

import numpy as np
import pytest
import torch

from combine_ep_get_histogram_b200 import workloads as wl
from gpu_util import StepBuffers as Step

pytestmark = pytest.mark.gpu


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
